// Split-KV decode over a KQV cache ([TQ] "Quantization Schemes": rotated keys and
// values by scalar MSE codes of their direction, values with a one-bit QJL sketch of the
// residual; "Key Contributions": the sketch estimate of a residual is unbiased).
//
// Keys and values live in the Walsh-Hadamard basis (H orthonormal, its own inverse):
//   q . k^_t      = n_t (H q) . C[code_t]
//   sum_t p_t v^_t = H ( sum_t p_t n_t C[code_t]  +  kappa S^T sum_t p_t rn_t s_t ),
// kappa = sqrt(pi / 2) / D.  So a split accumulates, per query head, the rotated-basis
// value sum o and the sketch-coordinate sum u (both D floats), with the usual online
// softmax; the combine merges (o, u) over the splits, applies S^T once per query head and
// transforms back.  The raw sink + residual split works in the original basis and
// rotates its o at the end so that every split's state is in the same basis.
//
// Work split and partial-state workspace as the generic kernel (split = a run of token
// groups of one KV head, or the raw tokens; four warps); a warp takes 32-token chunks
// k = warp, warp + 4, ... staged through its own two-stage cp.async ring, lane l owning
// channels (and sketch coordinates) 4 l .. 4 l + 3; four tokens' scores are reduced
// together, then one softmax update per head.  The workspace also carries a copy
// of S (written by the first CTA), so the combine needs nothing but the workspace.
#include <cmath>

#include "decode_common.cuh"
#include "wht.cuh"

namespace kvq {

namespace {

constexpr int kW = 4;
constexpr int kB = 2;   // tokens per score reduction
constexpr int kD = 128;
constexpr int kRec = 2 * kD + 4;     // per warp and head: o[128], u[128], m, l, padding
// A warp's 32-token chunk staged in shared memory: key rows, value rows (at most 16 words
// each), then the fp32 key norms, value norms and residual norms.
constexpr int kChunk = 32;
constexpr int kStK = 0, kStV = kChunk * 64, kStKn = 2 * kChunk * 64, kStVn = kStKn + 4 * kChunk,
              kStVr = kStVn + 4 * kChunk, kStBytes = kStVr + 4 * kChunk;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kKappa = 0.009791516697777345f;   // sqrt(pi / 2) / 128

struct KqvDec {
  Layout L;
  const void* q;
  int q_dtype, Hq;
  int64_t t_quant;
  int t_res;
  float qscale;
  int S, split_groups, n_packed, raw_slot;
  float* ws_m;
  float* ws_l;
  float* ws_o;    // [rows][2 D]: o then u
  float* ws_sk;   // [D][D] copy of the sketch matrix
  int32_t* status;
};

struct KqvComb {
  int Hq, S;
  const float* m;
  const float* l;
  const float* o;
  const float* sk;
  void* out;
  int out_dtype;
  float* lse;
  float rot_scale;
};

__device__ __forceinline__ void ld4f(const void* p, int64_t i, int dtype, float (&x)[4]) {
  if (dtype == KVQ_F32) {
    const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    return;
  }
  const uint2 w = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(p) + i);
  if (dtype == KVQ_F16) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    x[0] = __uint_as_float(w.x << 16);
    x[1] = __uint_as_float(w.x & 0xffff0000u);
    x[2] = __uint_as_float(w.y << 16);
    x[3] = __uint_as_float(w.y & 0xffff0000u);
  }
}

// The lane's four codes of a packed row (b = 3: low-bit plane then high-bit plane; else the
// row layout), as centroid values looked up in the lane-held codebook (lane i: C[i mod 2^b]).
__device__ __forceinline__ void row_centroids(const uint32_t* row, int b, int lane, float clane, float (&x)[4]) {
  int code[4];
  if (b == 3) {
    const uint32_t lo = row[lane >> 2] >> (8 * (lane & 3));
    const uint32_t hi = row[kD / 16 + (lane >> 3)] >> (4 * (lane & 7));
#pragma unroll
    for (int j = 0; j < 4; ++j) code[j] = (int)(((lo >> (2 * j)) & 3u) | (((hi >> j) & 1u) << 2));
  } else {
    const int lpw = 8 / b;
    const uint32_t f = row[lane / lpw] >> (4 * b * (lane % lpw));
#pragma unroll
    for (int j = 0; j < 4; ++j) code[j] = (int)((f >> (b * j)) & ((1u << b) - 1));
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = __shfl_sync(0xffffffffu, clane, code[j]);
}

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void stage_bytes(uint8_t* dst, const void* src, int bytes, int lane) {
  for (int o = 16 * lane; o < bytes; o += 512) cp16(dst + o, reinterpret_cast<const uint8_t*>(src) + o);
}

template <int GM>
struct KqvState {
  float q[GM][4], o[GM][4], u[GM][4];
  float m[GM], l[GM];
};

template <int GM>
__global__ void __launch_bounds__(kW * 32, GM <= 4 ? 4 : 2) decode_kqv_kernel(KqvDec a) {
  extern __shared__ __align__(16) float smem[];   // [kW][GM][kRec] records, [GM][D] tile, [kW][2] stages
  const Layout& L = a.L;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / L.Hkv;
  const int64_t sl = (int64_t)b * L.Hkv + h;
  if (split == 0 && h == 0 && b == 0) {   // the combine reads S from the workspace
    const float4* src = reinterpret_cast<const float4*>(L.sketch);
    float4* dst = reinterpret_cast<float4*>(a.ws_sk);
    for (int i = threadIdx.x; i < kD * kD / 4; i += blockDim.x) dst[i] = src[i];
  }
  const bool packed = split < a.n_packed;
  KqvState<GM> st;
  int bad = 0;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    st.m[hh] = -INFINITY;
    st.l[hh] = 0.0f;
    float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (hh < G) ld4f(a.q, ((int64_t)b * a.Hq + h * G + hh) * kD + 4 * lane, a.q_dtype, x);
#pragma unroll
    for (int j = 0; j < 4; ++j) bad |= !isfinite(x[j]);
    if (packed) {   // the packed keys are in the rotated basis: so is the query
      wht128_quad_unscaled(x, lane);
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] *= L.rot_scale;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      st.q[hh][j] = x[j] * a.qscale;
      st.o[hh][j] = 0.0f;
      st.u[hh][j] = 0.0f;
    }
  }

  if (packed) {
    const Side& SK = L.side[0];
    const Side& SV = L.side[1];
    const int kb = SK.bits, vb = SV.bits - 1;
    const int kw = kb * kD / 32, vw = SV.bits * kD / 32;
    const float klane = SK.lutf[lane & ((1 << kb) - 1)];
    const float vlane = SV.lutf[lane & ((1 << vb) - 1)];
    const uint32_t* kbase = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(SK.codes) +
                                                              sl * SK.code_slab_bytes);
    const uint32_t* vbase = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(SV.codes) +
                                                              sl * SV.code_slab_bytes);
    const float* kn = reinterpret_cast<const float*>(SK.scale) + sl * L.C;
    const float* vn = reinterpret_cast<const float*>(SV.scale) + sl * L.C;
    const float* vr = reinterpret_cast<const float*>(SV.zero) + sl * L.C;
    const int64_t ngv = (a.t_quant + L.g - 1) / L.g;
    const int64_t g0 = (int64_t)split * a.split_groups;
    const int64_t tb = g0 * L.g;
    const int64_t te = min(a.t_quant, min(ngv, g0 + a.split_groups) * L.g);
    // the warp's 32-token chunks k = warp, warp + kW, ... through a two-stage cp.async ring
    // (a chunk's rows past te stay inside the capacity, a multiple of g)
    uint8_t* ring = reinterpret_cast<uint8_t*>(smem + (size_t)kW * GM * kRec + (size_t)GM * kD) +
                    (size_t)warp * 2 * kStBytes;
    const int64_t nchunk = (te - tb + kChunk - 1) / kChunk;
    auto issue = [&](int64_t k, int bufi) {
      if (k < nchunk) {
        uint8_t* stg = ring + bufi * kStBytes;
        const int64_t t0 = tb + kChunk * k;
        stage_bytes(stg + kStK, kbase + t0 * kw, kChunk * kw * 4, lane);
        stage_bytes(stg + kStV, vbase + t0 * vw, kChunk * vw * 4, lane);
        stage_bytes(stg + kStKn, kn + t0, 4 * kChunk, lane);
        stage_bytes(stg + kStVn, vn + t0, 4 * kChunk, lane);
        stage_bytes(stg + kStVr, vr + t0, 4 * kChunk, lane);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    issue(warp, 0);
    int bufi = 0;
    for (int64_t k = warp; k < nchunk; k += kW) {
      issue(k + kW, bufi ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
      __syncwarp();
      const uint8_t* stg = ring + bufi * kStBytes;
      const uint32_t* krows = reinterpret_cast<const uint32_t*>(stg + kStK);
      const uint32_t* vrows = reinterpret_cast<const uint32_t*>(stg + kStV);
      const float* skn = reinterpret_cast<const float*>(stg + kStKn);
      const float* svn = reinterpret_cast<const float*>(stg + kStVn);
      const float* svr = reinterpret_cast<const float*>(stg + kStVr);
      const int nt = (int)min((int64_t)kChunk, te - (tb + kChunk * k));
    for (int r0 = 0; r0 < nt; r0 += kB) {
      float kf[kB][4], vf[kB][4], nk[kB], nv[kB], rv[kB], sgf[kB][4];
      uint32_t sg[kB];
      bool ok[kB];
#pragma unroll
      for (int e = 0; e < kB; ++e) {
        const int r = r0 + e;
        ok[e] = r < nt;
        const int rr = ok[e] ? r : 0;   // a valid row for the reads of unused slots
        row_centroids(krows + rr * kw, kb, lane, klane, kf[e]);
        const uint32_t* vrow = vrows + rr * vw;
        row_centroids(vrow, vb, lane, vlane, vf[e]);
        sg[e] = vrow[vb * kD / 32 + (lane >> 3)] >> (4 * (lane & 7));
#pragma unroll
        for (int j = 0; j < 4; ++j)   // sketch bit j as +1.0f (set) or -1.0f
          sgf[e][j] = __uint_as_float(0xBF800000u ^ ((sg[e] << (31 - j)) & 0x80000000u));
        nk[e] = skn[rr];
        nv[e] = svn[rr];
        rv[e] = svr[rr];
      }
      float sc[kB][GM];
#pragma unroll
      for (int e = 0; e < kB; ++e)
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) {
          float part = 0.0f;
#pragma unroll
          for (int j = 0; j < 4; ++j) part = fmaf(st.q[hh][j], kf[e][j], part);
          sc[e][hh] = part;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int e = 0; e < kB; ++e)
#pragma unroll
          for (int hh = 0; hh < GM; ++hh) sc[e][hh] += __shfl_xor_sync(0xffffffffu, sc[e][hh], o);
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        if (hh < G) {
          float mn = st.m[hh];
#pragma unroll
          for (int e = 0; e < kB; ++e) {
            sc[e][hh] *= nk[e];
            if (ok[e]) mn = fmaxf(mn, sc[e][hh]);
          }
          if (mn > st.m[hh]) {   // uniform over the warp (reduced scores); a factor 1 changes nothing
            const float corr = exp2f(st.m[hh] - mn);   // 0 when m = -inf
            st.l[hh] *= corr;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              st.o[hh][j] *= corr;
              st.u[hh][j] *= corr;
            }
          }
#pragma unroll
          for (int e = 0; e < kB; ++e) {
            if (ok[e]) {
              const float p = exp2f(sc[e][hh] - mn);
              st.l[hh] += p;
              const float pv = p * nv[e], pr = p * rv[e];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                st.o[hh][j] = fmaf(pv, vf[e][j], st.o[hh][j]);
                st.u[hh][j] = fmaf(pr, sgf[e][j], st.u[hh][j]);   // u + (+-pr), one rounding
              }
            }
          }
          st.m[hh] = mn;
        }
      }
    }
      __syncwarp();   // the stage's reads are done before it is refilled
      bufi ^= 1;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  } else if (split == a.raw_slot) {
    const int nraw = L.n_sink + a.t_res;
    for (int r = warp; r < nraw; r += kW) {
      const bool sink = r < L.n_sink;
      const int64_t row = sink ? r : r - L.n_sink;
      const int64_t rows = sink ? L.n_sink : L.res_cap;
      const int64_t i = (sl * rows + row) * kD + 4 * lane;
      float kh[4], vh[4];
      ld4f(sink ? L.sink[0] : L.res[0], i, L.src_dtype, kh);
      ld4f(sink ? L.sink[1] : L.res[1], i, L.src_dtype, vh);
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        if (hh < G) {
          float s = 0.0f;
#pragma unroll
          for (int j = 0; j < 4; ++j) s = fmaf(st.q[hh][j], kh[j], s);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          const float mn = fmaxf(st.m[hh], s);
          const float corr = exp2f(st.m[hh] - mn), p = exp2f(s - mn);
          st.l[hh] = fmaf(st.l[hh], corr, p);
#pragma unroll
          for (int j = 0; j < 4; ++j) st.o[hh][j] = fmaf(st.o[hh][j], corr, p * vh[j]);
          st.m[hh] = mn;
        }
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);

  // merge the warps' states; the raw split's o goes to the rotated basis first
  float* rec = smem + (size_t)warp * GM * kRec;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        rec[hh * kRec + 4 * lane + j] = st.o[hh][j];
        rec[hh * kRec + kD + 4 * lane + j] = st.u[hh][j];
      }
      if (lane == 0) {
        rec[hh * kRec + 2 * kD] = st.m[hh];
        rec[hh * kRec + 2 * kD + 1] = st.l[hh];
      }
    }
  }
  __syncthreads();
  float* tile = smem + (size_t)kW * GM * kRec;
  const int c = threadIdx.x;   // blockDim.x = D
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) M = fmaxf(M, smem[((size_t)w * GM + hh) * kRec + 2 * kD]);
    float lsum = 0.0f, oc = 0.0f, uc = 0.0f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      const float* p = smem + ((size_t)w * GM + hh) * kRec;
      const float f = p[2 * kD] == -INFINITY ? 0.0f : exp2f(p[2 * kD] - M);
      lsum = fmaf(p[2 * kD + 1], f, lsum);
      oc = fmaf(p[c], f, oc);
      uc = fmaf(p[kD + c], f, uc);
    }
    const int64_t slot = ((int64_t)b * a.Hq + h * G + hh) * a.S + split;
    a.ws_o[slot * 2 * kD + kD + c] = uc;
    if (packed) a.ws_o[slot * 2 * kD + c] = oc;
    else tile[hh * kD + c] = oc;
    if (c == 0) {
      a.ws_m[slot] = M;
      a.ws_l[slot] = lsum;
    }
  }
  if (!packed) {   // uniform over the CTA
    __syncthreads();
    wht_tile_rows(tile, G, kD, L.rot_scale);
    __syncthreads();
    for (int hh = 0; hh < G; ++hh) {
      const int64_t slot = ((int64_t)b * a.Hq + h * G + hh) * a.S + split;
      a.ws_o[slot * 2 * kD + c] = tile[hh * kD + c];
    }
  }
}

// One CTA (D threads) per query-head row: merge (o, u) over the splits, add kappa S^T u,
// transform back to the original basis, normalise.
__global__ void __launch_bounds__(kD) combine_kqv_kernel(KqvComb a) {
  __shared__ __align__(16) float U[kD];
  __shared__ __align__(16) float V[kD];
  const int hq = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const int64_t row = (int64_t)b * a.Hq + hq;
  const float* m = a.m + row * a.S;
  const float* l = a.l + row * a.S;
  float M = -INFINITY;
  for (int s = 0; s < a.S; ++s) M = fmaxf(M, m[s]);
  float lsum = 0.0f, oc = 0.0f, uc = 0.0f;
  for (int s = 0; s < a.S; ++s) {
    const float f = m[s] == -INFINITY ? 0.0f : exp2f(m[s] - M);
    const float* o = a.o + (row * a.S + s) * 2 * kD;
    lsum = fmaf(l[s], f, lsum);
    oc = fmaf(o[c], f, oc);
    uc = fmaf(o[kD + c], f, uc);
  }
  U[c] = uc;
  __syncthreads();
  float acc = 0.0f;
#pragma unroll 8
  for (int i = 0; i < kD; ++i) acc = fmaf(a.sk[i * kD + c], U[i], acc);
  V[c] = fmaf(kKappa, acc, oc);
  __syncthreads();
  wht_tile_rows(V, 1, kD, a.rot_scale);
  __syncthreads();
  const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
  store_elem(a.out, row * kD + c, a.out_dtype, V[c] * inv);
  if (a.lse && c == 0) a.lse[row] = lsum > 0.0f ? (M + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
}

size_t a16(size_t x) { return (x + 15) & ~(size_t)15; }

template <int GM>
cudaError_t launch_g(const KqvDec& a, cudaStream_t s) {
  const size_t smem = ((size_t)kW * GM * kRec + (size_t)GM * kD) * sizeof(float) + (size_t)kW * 2 * kStBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_kqv_kernel<GM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.L.Hkv, a.L.B);
  decode_kqv_kernel<GM><<<grid, kW * 32, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

// Workspace: m [rows], l [rows], (o, u) [rows][2 D], S [D][D]  (rows = B Hq S).
size_t kqv_workspace_bytes(const Layout& L, int Hq, const DecodePlan& p) {
  const size_t rows = (size_t)L.B * Hq * p.S;
  return a16(rows * 4) * 2 + a16(rows * 2 * kD * 4) + (size_t)kD * kD * 4;
}

cudaError_t launch_decode_kqv(const Layout& L, const DecodePlan& p, const void* q, int q_dtype, int Hq,
                              int64_t t_quant, int t_res, float scale, void* ws, int32_t* d_status,
                              cudaStream_t s) {
  const size_t rows = (size_t)L.B * Hq * p.S;
  char* w = reinterpret_cast<char*>(ws);
  KqvDec a;
  a.L = L;
  a.q = q;
  a.q_dtype = q_dtype;
  a.Hq = Hq;
  a.t_quant = t_quant;
  a.t_res = t_res;
  a.qscale = scale * kLog2e;
  a.S = p.S;
  a.split_groups = p.split_groups;
  a.n_packed = p.n_packed_splits;
  a.raw_slot = p.raw_slot;
  a.ws_m = reinterpret_cast<float*>(w);
  a.ws_l = reinterpret_cast<float*>(w + a16(rows * 4));
  a.ws_o = reinterpret_cast<float*>(w + 2 * a16(rows * 4));
  a.ws_sk = reinterpret_cast<float*>(w + 2 * a16(rows * 4) + a16(rows * 2 * kD * 4));
  a.status = d_status;
  const int G = Hq / L.Hkv;
  if (G <= 1) return launch_g<1>(a, s);
  if (G <= 2) return launch_g<2>(a, s);
  if (G <= 4) return launch_g<4>(a, s);
  if (G <= 8) return launch_g<8>(a, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine_kqv(const Layout& L, int Hq, const DecodePlan& p, const void* ws, void* out,
                               int out_dtype, float* lse, cudaStream_t s) {
  const size_t rows = (size_t)L.B * Hq * p.S;
  const char* w = reinterpret_cast<const char*>(ws);
  KqvComb c;
  c.Hq = Hq;
  c.S = p.S;
  c.m = reinterpret_cast<const float*>(w);
  c.l = reinterpret_cast<const float*>(w + a16(rows * 4));
  c.o = reinterpret_cast<const float*>(w + 2 * a16(rows * 4));
  c.sk = reinterpret_cast<const float*>(w + 2 * a16(rows * 4) + a16(rows * 2 * kD * 4));
  c.out = out;
  c.out_dtype = out_dtype;
  c.lse = lse;
  c.rot_scale = (float)(1.0 / std::sqrt((double)kD));
  dim3 grid(Hq, L.B);
  combine_kqv_kernel<<<grid, kD, 0, s>>>(c);
  return cudaGetLastError();
}

}  // namespace kvq
