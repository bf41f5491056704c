// Split-KV decode attention: the generic path (any format, CUDA cores, fp32), the
// cross-split combine, planning and dispatch.
//
//   out[h] = sum_t softmax_t(scale * q[h] . k^_t) v^_t      [AXES] "Separate the two
//   error paths"; over sink + packed + residual tokens ([KVQ] "Approach", [MIX] Fig. 4).
//
// Partial softmax states are kept in the log2 domain (the query is pre-multiplied by
// scale * log2(e)): per split and query head, m = max score, l = sum 2^(s - m),
// o[d] = sum 2^(s - m) v[d].  The combine merges the splits with the usual
// log-sum-exp rescaling.  Splits never wait on one another.
#include <cmath>

#include "decode_common.cuh"
#include "wht.cuh"

namespace kvq {

// Fast tensor-core path (decode_mma.cu)
bool mma_path_ok(const Layout& L, int Hq);
void plan_mma(const Layout& L, int64_t t_quant, int t_res, int max_ctas, DecodePlan& p);
cudaError_t launch_combine_mma(const Layout& L, const DecodePlan& p, int Hq, const float* ws_m,
                               const float* ws_l, const float* ws_o, void* out, int out_dtype,
                               float* lse, cudaStream_t s);
cudaError_t launch_decode_mma(const Layout& L, const DecodePlan& p, const void* q, int q_dtype,
                              int Hq, int64_t t_quant, int t_res, float scale, float* ws_m,
                              float* ws_l, float* ws_o, int32_t* d_status, cudaStream_t s);

// CUDA-core path with four consecutive channels per lane (decode_cc.cu)
bool cc_path_ok(const Layout& L, int Hq);
cudaError_t launch_decode_cc(const Layout& L, const DecodePlan& p, const void* q, int q_dtype, int Hq,
                             int64_t t_quant, int t_res, float scale, float* ws_m, float* ws_l,
                             float* ws_o, int32_t* d_status, cudaStream_t s);

// KQV caches (decode_kqv.cu)
size_t kqv_workspace_bytes(const Layout& L, int Hq, const DecodePlan& p);
cudaError_t launch_decode_kqv(const Layout& L, const DecodePlan& p, const void* q, int q_dtype, int Hq,
                              int64_t t_quant, int t_res, float scale, void* ws, int32_t* d_status,
                              cudaStream_t s);
cudaError_t launch_combine_kqv(const Layout& L, int Hq, const DecodePlan& p, const void* ws, void* out,
                               int out_dtype, float* lse, cudaStream_t s);

namespace {

constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct DecArgs {
  Layout L;
  const void* q;
  int q_dtype, Hq;
  int64_t t_quant;
  int t_res;
  float qscale;          // softmax scale * log2(e)
  int S, split_groups, n_packed, raw_slot;
  float* ws_m;
  float* ws_l;
  float* ws_o;
  int32_t* status;
};

template <int NC, int GM_>
struct WarpState {
  // query and accumulators of up to GM heads, NC channels per lane (c = lane + 32 j)
  static constexpr int GM = GM_;
  float q[GM][NC];
  float o[GM][NC];
  float m[GM], l[GM];
};

// Process one token of the current KV head: kh / vh are the lane's key / value
// channels (already reconstructed and, for keys, rotated).
template <int NC, int GM>
__device__ __forceinline__ void consume_token(WarpState<NC, GM>& st, int G, const float* kh,
                                              const float* vh) {
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
      float part = 0.0f;
#pragma unroll
      for (int j = 0; j < NC; ++j) part = fmaf(st.q[hh][j], kh[j], part);
      const float s = warp_sum(part);
      if (s > st.m[hh]) {
        const float corr = exp2f(st.m[hh] - s);   // 0 when m = -inf
        st.l[hh] = st.l[hh] * corr + 1.0f;
#pragma unroll
        for (int j = 0; j < NC; ++j) st.o[hh][j] = fmaf(st.o[hh][j], corr, vh[j]);
        st.m[hh] = s;
      } else {
        const float p = exp2f(s - st.m[hh]);
        st.l[hh] += p;
#pragma unroll
        for (int j = 0; j < NC; ++j) st.o[hh][j] = fmaf(p, vh[j], st.o[hh][j]);
      }
    }
  }
}

// Process up to kBatch tokens at once (ok[e] marks the valid ones): the score
// reductions of all tokens and heads run together, then one softmax update per head.
constexpr int kBatch = 4;
template <int NC, int GM>
__device__ __forceinline__ void consume_batch(WarpState<NC, GM>& st, int G, const float (&kh)[kBatch][NC],
                                              const float (&vh)[kBatch][NC], const bool (&ok)[kBatch]) {
  float sc[kBatch][GM];
#pragma unroll
  for (int e = 0; e < kBatch; ++e)
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) {
      float part = 0.0f;
#pragma unroll
      for (int j = 0; j < NC; ++j) part = fmaf(st.q[hh][j], kh[e][j], part);
      sc[e][hh] = part;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int e = 0; e < kBatch; ++e)
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) sc[e][hh] += __shfl_xor_sync(0xffffffffu, sc[e][hh], o);
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
      float mn = st.m[hh];
#pragma unroll
      for (int e = 0; e < kBatch; ++e)
        if (ok[e]) mn = fmaxf(mn, sc[e][hh]);
      const float corr = exp2f(st.m[hh] - mn);   // 0 when m = -inf
      st.l[hh] *= corr;
#pragma unroll
      for (int j = 0; j < NC; ++j) st.o[hh][j] *= corr;
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        if (ok[e]) {
          const float p = exp2f(sc[e][hh] - mn);
          st.l[hh] += p;
#pragma unroll
          for (int j = 0; j < NC; ++j) st.o[hh][j] = fmaf(p, vh[e][j], st.o[hh][j]);
        }
      }
      st.m[hh] = mn;
    }
  }
}

// Rotate-half RoPE of the lane's key channels at absolute position pos: channel pairs
// (c, c + D/2) are both owned by the lane (j and j + NC/2).
template <int NC>
__device__ __forceinline__ void rope(float* kh, const double* theta, int64_t pos) {
#pragma unroll
  for (int j = 0; j < NC / 2; ++j) {
    float s, c;
    angle_sincos((double)pos, theta[j], &s, &c);
    const float x1 = kh[j], x2 = kh[j + NC / 2];
    kh[j] = x1 * c - x2 * s;
    kh[j + NC / 2] = x2 * c + x1 * s;
  }
}

// The same rotation from a running (cos, sin) per channel pair, which then advances by
// the per-step rotation (cst, snt): exact anchors in fp64 at every group, fp32 steps
// within it.
template <int NC>
__device__ __forceinline__ void rope_step(float* kh, float* cs, float* sn, const float* cst,
                                          const float* snt) {
#pragma unroll
  for (int j = 0; j < NC / 2; ++j) {
    const float x1 = kh[j], x2 = kh[j + NC / 2];
    kh[j] = x1 * cs[j] - x2 * sn[j];
    kh[j + NC / 2] = x2 * cs[j] + x1 * sn[j];
    const float c2 = cs[j] * cst[j] - sn[j] * snt[j];
    sn[j] = sn[j] * cst[j] + cs[j] * snt[j];
    cs[j] = c2;
  }
}

template <int NC, int GM>
__global__ void __launch_bounds__(kWarps * 32) decode_generic_kernel(DecArgs a) {
  extern __shared__ __align__(16) float smem[];
  const Layout& L = a.L;
  const int D = L.D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / L.Hkv;
  const int64_t sl = (int64_t)b * L.Hkv + h;
  int* inv = reinterpret_cast<int*>(smem);                 // [D] channel -> slot (MIXED)
  float* wst = smem + 256;                                  // [kWarps][G][D + 2]

  WarpState<NC, GM> st;
  int bad = 0;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    st.m[hh] = -INFINITY;
    st.l[hh] = 0.0f;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      st.o[hh][j] = 0.0f;
      float x = 0.0f;
      if (hh < G) {
        x = load_elem(a.q, ((int64_t)b * a.Hq + h * G + hh) * D + lane + 32 * j, a.q_dtype);
        bad |= !isfinite(x);
      }
      st.q[hh][j] = x * a.qscale;
    }
    // packed keys of a rotating format are in the Walsh-Hadamard basis: so is the query
    if (L.k_rotate && split < a.n_packed) wht_strided<NC>(st.q[hh], lane, L.rot_scale);
  }
  double theta[NC / 2 > 0 ? NC / 2 : 1];
  if (L.rope) {
#pragma unroll
    for (int j = 0; j < NC / 2; ++j)
      theta[j] = pow((double)L.rope_base, -2.0 * (double)(lane + 32 * j) / (double)D);
  }
  float kh[NC], vh[NC];

  if (split < a.n_packed) {
    const int64_t ngv = (a.t_quant + L.g - 1) / L.g;
    const int64_t g0 = (int64_t)split * a.split_groups;
    const int64_t g1 = min(ngv, g0 + a.split_groups);
    const Side& SK = L.side[0];
    const Side& SV = L.side[1];
    // fast element paths: keys per channel (ASYM b < 8, NUQ), values per token (ASYM b < 8, NUQ)
    const bool k_fast = (SK.scheme == KVQ_ASYM && SK.bits < 8 && SK.axis == KVQ_AXIS_CHANNEL) ||
                        (SK.scheme == KVQ_NUQ && SK.axis == KVQ_AXIS_CHANNEL);
    const bool v_fast = (SV.scheme == KVQ_ASYM && SV.bits < 8 && SV.axis == KVQ_AXIS_TOKEN) ||
                        (SV.scheme == KVQ_NUQ && SV.axis == KVQ_AXIS_TOKEN);
    // nuq codebooks: lane i holds entry i & 7
    const float klut = SK.scheme == KVQ_NUQ ? __half2float(SK.lut[lane & 7]) : 0.0f;
    const float vlut = SV.scheme == KVQ_NUQ ? __half2float(SV.lut[lane & 7]) : 0.0f;
    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(SK.codes) + sl * SK.code_slab_bytes;
    const uint8_t* vbase = reinterpret_cast<const uint8_t*>(SV.codes) + sl * SV.code_slab_bytes;
    float cst[NC / 2 > 0 ? NC / 2 : 1], snt[NC / 2 > 0 ? NC / 2 : 1];
    if (L.rope) {
#pragma unroll
      for (int j = 0; j < NC / 2; ++j) {
        angle_sincos((double)kWarps, theta[j], &snt[j], &cst[j]);
      }
    }
    for (int64_t gi = g0; gi < g1; ++gi) {
      if (SK.scheme == KVQ_MIXED) {
        __syncthreads();
        for (int j = threadIdx.x; j < D; j += blockDim.x) inv[L.k_order[(sl * L.ng + gi) * D + j]] = j;
        __syncthreads();
      }
      const int64_t tb = gi * L.g, te = min(a.t_quant, tb + L.g);
      // this group's per-channel key metadata for the lane's channels
      float ks[NC], kz[NC];
      if (k_fast) {
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int64_t mi = (sl * L.ng + gi) * D + lane + 32 * j;
          ks[j] = meta_f16(SK.scale, mi);
          kz[j] = meta_f16(SK.zero, mi);
        }
      }
      // RoPE anchor at this warp's first token of the group
      float cs[NC / 2 > 0 ? NC / 2 : 1], sn[NC / 2 > 0 ? NC / 2 : 1];
      if (L.rope) {
#pragma unroll
        for (int j = 0; j < NC / 2; ++j) {
          angle_sincos((double)(L.n_sink + tb + warp), theta[j], &sn[j], &cs[j]);
        }
      }
      for (int64_t t0 = tb + warp; t0 < te; t0 += kWarps * kBatch) {
        float kb[kBatch][NC], vb[kBatch][NC];
        bool ok[kBatch];
#pragma unroll
        for (int e = 0; e < kBatch; ++e) {
          const int64_t t = t0 + (int64_t)e * kWarps;
          ok[e] = t < te;
          const int64_t tt = ok[e] ? t : tb;   // a valid row for the loads of unused slots
#pragma unroll
          for (int j = 0; j < NC; ++j) {
            const int c = lane + 32 * j;
            float kv;
            if (k_fast) {
              uint32_t code;
              if (SK.scheme == KVQ_NUQ) {
                const uint32_t* w = reinterpret_cast<const uint32_t*>(kbase) + tt * (3 * D / 32);
                code = ((w[c / 16] >> (2 * (c % 16))) & 3u) | (((w[D / 16 + c / 32] >> (c % 32)) & 1u) << 2);
                kv = __fmaf_rn(__shfl_sync(0xffffffffu, klut, (int)code), ks[j], kz[j]);
              } else {
                const int b = SK.bits, per = 32 / b;
                const uint32_t w = reinterpret_cast<const uint32_t*>(kbase)[tt * (D / per) + c / per];
                code = (w >> (b * (c % per))) & ((1u << b) - 1);
                kv = __fmaf_rn((float)code, ks[j], kz[j]);
              }
            } else {
              kv = SK.scheme == KVQ_MIXED ? mixed_slot_value(L, sl, tt, inv[c]) : deq_dense(L, 0, sl, tt, c);
            }
            kb[e][j] = kv;
          }
          if (v_fast) {
            const float vs = meta_f16(SV.scale, sl * L.C + tt), vz = meta_f16(SV.zero, sl * L.C + tt);
#pragma unroll
            for (int j = 0; j < NC; ++j) {
              const int c = lane + 32 * j;
              if (SV.scheme == KVQ_NUQ) {
                const uint32_t* w = reinterpret_cast<const uint32_t*>(vbase) + tt * (3 * D / 32);
                const uint32_t code = ((w[c / 16] >> (2 * (c % 16))) & 3u) | (((w[D / 16 + c / 32] >> (c % 32)) & 1u) << 2);
                vb[e][j] = __fmaf_rn(__shfl_sync(0xffffffffu, vlut, (int)code), vs, vz);
              } else {
                const int b = SV.bits, per = 16 / b;
                const uint32_t w = reinterpret_cast<const uint32_t*>(vbase)[(tt >> 1) * (D / per) + c / per];
                const uint32_t code = (w >> (16 * (int)(tt & 1) + b * (c % per))) & ((1u << b) - 1);
                vb[e][j] = __fmaf_rn((float)code, vs, vz);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < NC; ++j) vb[e][j] = deq_dense(L, 1, sl, tt, lane + 32 * j);
          }
          if (SK.nout > 0 && ok[e]) {
            const int rr = (int)(t - tb);
            const int32_t* rp = L.k_out_rowptr + (sl * L.ng + gi) * (L.g + 1);
            const int64_t e0 = (sl * L.ng + gi) * (int64_t)D * SK.nout;
            for (int x = rp[rr]; x < rp[rr + 1]; ++x) {
              const int c = L.k_out_col[e0 + x];
              const float v = __half2float(L.k_out_val[e0 + x]);
#pragma unroll
              for (int j = 0; j < NC; ++j)
                if (c == lane + 32 * j) kb[e][j] = v;
            }
          }
          if (SV.nout > 0 && ok[e]) {
            for (int x = 0; x < SV.nout; ++x) {
              const int64_t idx = (sl * L.C + t) * SV.nout + x;
              const int c = L.v_out_col[idx];
              const float v = __half2float(L.v_out_val[idx]);
#pragma unroll
              for (int j = 0; j < NC; ++j)
                if (c == lane + 32 * j) vb[e][j] = v;
            }
          }
          if (L.rope) rope_step<NC>(kb[e], cs, sn, cst, snt);
        }
        consume_batch<NC, GM>(st, G, kb, vb, ok);
      }
    }
  } else if (split == a.raw_slot) {
    const int nraw = L.n_sink + a.t_res;
    for (int r = warp; r < nraw; r += kWarps) {
      const bool sink = r < L.n_sink;
      const int64_t row = sink ? r : r - L.n_sink;
      const void* kb = sink ? L.sink[0] : L.res[0];
      const void* vb = sink ? L.sink[1] : L.res[1];
      const int64_t rows = sink ? L.n_sink : L.res_cap;
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const int64_t i = (sl * rows + row) * D + lane + 32 * j;
        kh[j] = load_elem(kb, i, L.src_dtype);
        vh[j] = load_elem(vb, i, L.src_dtype);
      }
      const int64_t pos = sink ? r : L.n_sink + a.t_quant + row;
      if (L.rope) rope<NC>(kh, theta, pos);
      consume_token<NC, GM>(st, G, kh, vh);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);

  // merge the warps' states and write this split's partial state
  float* mine = wst + (size_t)warp * G * (D + 2);
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
#pragma unroll
      for (int j = 0; j < NC; ++j) mine[hh * (D + 2) + lane + 32 * j] = st.o[hh][j];
      if (lane == 0) {
        mine[hh * (D + 2) + D] = st.m[hh];
        mine[hh * (D + 2) + D + 1] = st.l[hh];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int hh = i / D, d = i % D;
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wst[((size_t)w * G + hh) * (D + 2) + D]);
    float l = 0.0f, o = 0.0f;
    for (int w = 0; w < kWarps; ++w) {
      const float* p = wst + ((size_t)w * G + hh) * (D + 2);
      const float f = p[D] == -INFINITY ? 0.0f : exp2f(p[D] - M);
      l = fmaf(p[D + 1], f, l);
      o = fmaf(p[d], f, o);
    }
    const int64_t slot = ((int64_t)b * a.Hq + h * G + hh) * a.S + split;
    a.ws_o[slot * D + d] = o;
    if (d == 0) {
      a.ws_m[slot] = M;
      a.ws_l[slot] = l;
    }
  }
}

struct CombArgs {
  int D, Hq, S;
  const float* m;
  const float* l;
  const float* o;
  void* out;
  int out_dtype;
  float* lse;   // nullable
};

__global__ void __launch_bounds__(256) combine_kernel(CombArgs a) {
  const int hq = blockIdx.x, b = blockIdx.y;
  const int64_t row = (int64_t)b * a.Hq + hq;
  const float* m = a.m + row * a.S;
  const float* l = a.l + row * a.S;
  float M = -INFINITY;
  for (int s = 0; s < a.S; ++s) M = fmaxf(M, m[s]);
  for (int d = threadIdx.x; d < a.D; d += blockDim.x) {
    float L = 0.0f, o = 0.0f;
    for (int s = 0; s < a.S; ++s) {
      const float f = m[s] == -INFINITY ? 0.0f : exp2f(m[s] - M);
      L = fmaf(l[s], f, L);
      o = fmaf(a.o[(row * a.S + s) * a.D + d], f, o);
    }
    store_elem(a.out, row * a.D + d, a.out_dtype, o / L);
    if (a.lse && d == 0) a.lse[row] = (M + log2f(L)) * 0.6931471805599453f;   // natural log
  }
}

template <int NC, int GM>
cudaError_t launch_generic_g(const DecArgs& a, int grid_x, cudaStream_t s) {
  const int G = a.Hq / a.L.Hkv;
  const size_t smem = 256 * sizeof(float) + (size_t)kWarps * G * (a.L.D + 2) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(decode_generic_kernel<NC, GM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(grid_x, a.L.Hkv, a.L.B);
  decode_generic_kernel<NC, GM><<<grid, kWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

// G (query heads per KV head) is at most 16 and G * D at most 2048.
template <int NC>
cudaError_t launch_generic(const DecArgs& a, int grid_x, cudaStream_t s) {
  const int G = a.Hq / a.L.Hkv;
  if (G <= 1) return launch_generic_g<NC, 1>(a, grid_x, s);
  if (G <= 2) return launch_generic_g<NC, 2>(a, grid_x, s);
  if (G <= 4) return launch_generic_g<NC, 4>(a, grid_x, s);
  if (G <= 8) return launch_generic_g<NC, 8>(a, grid_x, s);
  if constexpr (NC <= 4) {
    if (G <= 16) return launch_generic_g<NC, 16>(a, grid_x, s);
  }
  return cudaErrorInvalidValue;
}

size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

}  // namespace

bool fast_path_ok(const Layout& L, int Hq) { return mma_path_ok(L, Hq); }

DecodePlan plan_decode(const Layout& L, int Hq, int64_t t_quant, int t_res, int num_splits) {
  DecodePlan p;
  const int64_t ngv = (t_quant + L.g - 1) / L.g;
  const bool raw = L.n_sink + t_res > 0;
  const int64_t heads = (int64_t)L.B * L.Hkv;
  p.fast = (ngv > 0 && fast_path_ok(L, Hq)) ? 1 : 0;
  p.raw_pieces = 0;
  if (p.fast) {
    // persistent partition over (head, group) units; num_splits caps the CTA count
    plan_mma(L, t_quant, t_res, num_splits, p);
    return p;
  }
  int sp = 0, sg = 1;
  if (ngv > 0) {
    int64_t want;
    if (num_splits > 0) {
      want = num_splits;
    } else {
      const int64_t target = (int64_t)device_sm_count() * 8;
      want = (target + heads - 1) / heads;
    }
    want = std::max<int64_t>(1, std::min<int64_t>(want, ngv));
    sg = (int)((ngv + want - 1) / want);
    sp = (int)((ngv + sg - 1) / sg);
  }
  p.n_packed_splits = sp;
  p.split_groups = sg;
  p.raw_slot = raw ? sp : -1;
  p.S = sp + (raw ? 1 : 0);
  p.grid_ctas = (int)(p.S * heads);
  return p;
}

// m [rows], l [rows], o [rows][D] (rows = B * Hq * S).
size_t workspace_bytes(const Layout& L, int Hq, const DecodePlan& p) {
  if (L.side[0].scheme == KVQ_KQV) return kqv_workspace_bytes(L, Hq, p);
  const size_t rows = (size_t)L.B * Hq * p.S;
  // the fast path keeps 32 flags per KV head after the partial states (fused append)
  const size_t flags = p.fast ? align16((size_t)L.B * L.Hkv * 32 * 4) : 0;
  return align16(rows * 4) * 2 + align16(rows * L.D * 4) + flags;
}

cudaError_t launch_decode_partial(const Layout& L, const DecodePlan& p, const void* q, int q_dtype,
                                  int Hq, int64_t t_quant, int t_res, float scale, void* ws,
                                  int32_t* d_status, cudaStream_t s) {
  if (L.side[0].scheme == KVQ_KQV)
    return launch_decode_kqv(L, p, q, q_dtype, Hq, t_quant, t_res, scale, ws, d_status, s);
  const size_t rows = (size_t)L.B * Hq * p.S;
  float* ws_m = reinterpret_cast<float*>(ws);
  float* ws_l = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + align16(rows * 4));
  float* ws_o = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + 2 * align16(rows * 4));
  if (p.fast) {
    DecodePlan pf = p;
    pf.flags = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 2 * align16(rows * 4) +
                                           align16(rows * L.D * 4));
    return launch_decode_mma(L, pf, q, q_dtype, Hq, t_quant, t_res, scale, ws_m, ws_l, ws_o, d_status, s);
  }
  if (cc_path_ok(L, Hq))
    return launch_decode_cc(L, p, q, q_dtype, Hq, t_quant, t_res, scale, ws_m, ws_l, ws_o, d_status, s);
  DecArgs a;
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
  a.ws_m = ws_m;
  a.ws_l = ws_l;
  a.ws_o = ws_o;
  a.status = d_status;
  switch (L.D) {
    case 32: return launch_generic<1>(a, p.S, s);
    case 64: return launch_generic<2>(a, p.S, s);
    case 128: return launch_generic<4>(a, p.S, s);
    default: return launch_generic<8>(a, p.S, s);
  }
}

cudaError_t launch_combine(const Layout& L, int Hq, const DecodePlan& p, const void* ws, void* out,
                           int out_dtype, float* lse, cudaStream_t s) {
  if (L.side[0].scheme == KVQ_KQV) return launch_combine_kqv(L, Hq, p, ws, out, out_dtype, lse, s);
  const size_t rows = (size_t)L.B * Hq * p.S;
  const float* m = reinterpret_cast<const float*>(ws);
  const float* l = reinterpret_cast<const float*>(reinterpret_cast<const char*>(ws) + align16(rows * 4));
  const float* o = reinterpret_cast<const float*>(reinterpret_cast<const char*>(ws) + 2 * align16(rows * 4));
  if (p.fast) return launch_combine_mma(L, p, Hq, m, l, o, out, out_dtype, lse, s);
  CombArgs c;
  c.D = L.D;
  c.Hq = Hq;
  c.S = p.S;
  c.m = m;
  c.l = l;
  c.o = o;
  c.out = out;
  c.out_dtype = out_dtype;
  c.lse = lse;
  dim3 grid(Hq, L.B);
  combine_kernel<<<grid, L.D < 256 ? L.D : 256, 0, s>>>(c);
  return cudaGetLastError();
}

}  // namespace kvq
