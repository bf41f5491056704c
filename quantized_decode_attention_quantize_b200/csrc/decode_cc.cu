// Split-KV decode on CUDA cores for D = 128 packed formats that the tensor-core kernel
// does not take: nuq3 keys and values with sparse outliers and RoPE on the keys
// ([KVQ] "Approach", "Dense-and-Sparse"), MixKVQ salience-ordered keys ([MIX] Fig. 4),
// asymmetric 2/4-bit keys with RoPE, G <= 8 query heads per KV head.
//
// Same work split, partial states and combine as the generic kernel (split = a run of
// token groups of one KV head, or the raw sink + residual tokens; four warps, token t
// to warp t mod 4).  What differs is the lane layout: lane l owns the four consecutive
// channels 4 l .. 4 l + 3, so one 32-bit word of a packed row holds all of its codes,
// one load per plane and token; the group's per-channel key scale / zero-point sit in
// registers.  MIXED keys are walked in storage-slot order (lane l: slots 4 l .. 4 l + 3)
// against the query gathered into slot order once per group.  RoPE pairs (c, c + 64)
// live in lanes l and l ^ 16 and meet through one shuffle; the rotation is anchored
// exactly (fp64) at each group and advanced in fp32 from token to token.  Scores of
// four tokens are reduced together, then one softmax update per head.
#include <cmath>

#include "decode_common.cuh"
#include "wht.cuh"

namespace kvq {

namespace {

constexpr int kW = 4;        // warps per CTA
constexpr int kB = 4;        // tokens per batch
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRS = 132;     // merge record stride (floats): o[128], m, l, padding to 16 bytes

// Byte offsets of the regions of a chunk stage (32 tokens of one group, with the
// group's metadata), each 16-byte aligned; computed on the host for the layout.
struct CcStage {
  int k, k_mid, k_lo;       // key rows (MIXED: raw, 4-bit and 2-bit planes)
  int v, vs, vz;            // value rows, value scale / zero-point
  int voc, vov;             // value outliers: columns, values
  int ks, kz, ord;          // group key scale / zero-point, MIXED slot order
  int rp, kc, kv;           // key outliers: 33 row pointers, the group's columns and values
  int bytes;
};

struct CcArgs {
  CcStage st;
  Layout L;
  const void* q;
  int q_dtype, Hq;
  int64_t t_quant;
  int t_res;
  float qscale;
  int S, split_groups, n_packed, raw_slot;
  float* ws_m;
  float* ws_l;
  float* ws_o;
  int32_t* status;
};

// Four consecutive elements of a raw row (16-bit or fp32 source).
__device__ __forceinline__ float4 ld4(const void* p, int64_t i, int dtype) {
  if (dtype == KVQ_F32) return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
  const uint2 x = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(p) + i);
  if (dtype == KVQ_F16) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&x.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&x.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
  return make_float4(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xffff0000u),
                     __uint_as_float(x.y << 16), __uint_as_float(x.y & 0xffff0000u));
}

// Rotate-half RoPE of the lane's four channels: lanes l < 16 hold x1 of pairs
// i = 4 l + j, lanes l + 16 the partner x2.
__device__ __forceinline__ void rope4(float* x, const float* cs, const float* sn, int lane) {
  const bool first = lane < 16;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float other = __shfl_xor_sync(0xffffffffu, x[j], 16);
    x[j] = first ? fmaf(x[j], cs[j], -other * sn[j]) : fmaf(x[j], cs[j], other * sn[j]);
  }
}

// nuq3 codes of channels 4 l .. 4 l + 3 of a row (2-bit plane then 1-bit plane).
__device__ __forceinline__ void nuq_codes(const uint32_t* row, int lane, uint32_t* code) {
  const uint32_t w2 = row[lane >> 2] >> (8 * (lane & 3));
  const uint32_t w1 = row[8 + (lane >> 3)] >> (4 * (lane & 7));
#pragma unroll
  for (int j = 0; j < 4; ++j) code[j] = ((w2 >> (2 * j)) & 3u) | (((w1 >> j) & 1u) << 2);
}

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// bytes (a multiple of 16) from src to dst, all lanes of the warp
__device__ __forceinline__ void cp_range(uint8_t* dst, const void* src, int bytes, int lane) {
  for (int o = 16 * lane; o < bytes; o += 512) cp16(dst + o, reinterpret_cast<const uint8_t*>(src) + o);
}

// KF: key format (kNuq, kAsym, kMixed); VF: value format (kNuq, kAsym); ROPE on keys.
constexpr int kNuq = 0, kAsym = 1, kMixed = 2;

template <int GM, int KF, int VF, bool ROPE>
__global__ void __launch_bounds__(kW * 32, GM <= 4 ? 4 : 2) decode_cc_kernel(CcArgs a) {
  extern __shared__ __align__(16) float smem[];
  const Layout& L = a.L;
  constexpr int D = 128;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / L.Hkv;
  const int64_t sl = (int64_t)b * L.Hkv + h;
  const Side& SK = L.side[0];
  const Side& SV = L.side[1];
  constexpr bool mixed = KF == kMixed;
  const CcStage& SG = a.st;
  uint8_t* ring = reinterpret_cast<uint8_t*>(smem) + (size_t)warp * 2 * SG.bytes;   // [kW][2] stages
  float* qsm = smem + (size_t)kW * 2 * SG.bytes / 4;  // [GM][128] pre-scaled queries (MIXED)
  float* wst = qsm + GM * D;                          // [kW][G][kRS] merge records

  float q[GM][4], o[GM][4], m[GM], l[GM];
  int bad = 0;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.0f;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (hh < G) {
      x = ld4(a.q, ((int64_t)b * a.Hq + h * G + hh) * D + 4 * lane, a.q_dtype);
      bad |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
    }
    float sc = a.qscale;
    if (L.k_rotate && split < a.n_packed) {   // packed keys in the Walsh-Hadamard basis
      float v[4] = {x.x, x.y, x.z, x.w};
      wht128_quad_unscaled(v, lane);
      x = make_float4(v[0], v[1], v[2], v[3]);
      sc *= L.rot_scale;
    }
    q[hh][0] = x.x * sc; q[hh][1] = x.y * sc;
    q[hh][2] = x.z * sc; q[hh][3] = x.w * sc;
#pragma unroll
    for (int j = 0; j < 4; ++j) o[hh][j] = 0.0f;
    if (mixed && warp == 0)
      *reinterpret_cast<float4*>(qsm + hh * D + 4 * lane) = make_float4(q[hh][0], q[hh][1], q[hh][2], q[hh][3]);
  }
  // RoPE frequencies of this lane's pairs i = 4 (l & 15) + j
  double theta[4];
  if (ROPE) {
#pragma unroll
    for (int j = 0; j < 4; ++j) theta[j] = pow((double)L.rope_base, -2.0 * (double)(4 * (lane & 15) + j) / (double)D);
  }

  // Scores of kB tokens x GM heads: value i = e GM + hh, N = kB GM values (a power of two
  // <= 32).  A reduce-scatter over the warp (each level halves the values a lane keeps)
  // leaves lane l with the full score of value l >> (5 - log2 N); the softmax of a head
  // over the batch then takes two shuffle levels, and every lane gets each probability by
  // one broadcast for the value accumulation.
  auto consume = [&](const float (&kb)[kB][4], const float (&vb)[kB][4], const float (&qk)[GM][4],
                     const bool (&ok)[kB]) {
    constexpr int N = kB * GM;
    constexpr int LN = N == 4 ? 2 : N == 8 ? 3 : N == 16 ? 4 : 5;
    float v[N];
#pragma unroll
    for (int e = 0; e < kB; ++e)
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        float part = qk[hh][0] * kb[e][0];
        part = fmaf(qk[hh][1], kb[e][1], part);
        part = fmaf(qk[hh][2], kb[e][2], part);
        part = fmaf(qk[hh][3], kb[e][3], part);
        v[e * GM + hh] = part;
      }
    // reduce-scatter: level with offset o = 16, 8, ... keeps the half selected by that lane bit
#pragma unroll
    for (int lev = 0; lev < LN; ++lev) {
      const int off = 16 >> lev;
      const int half = N >> (lev + 1);
      const bool upper = lane & off;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
#pragma unroll
    for (int off = 16 >> LN; off > 0; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    const int idx = lane >> (5 - LN);
    const int my_e = idx / GM, my_h = idx % GM;
    const bool my_ok = ok[0] && (my_e == 0) || ok[1] && (my_e == 1) || ok[2] && (my_e == 2) || ok[3] && (my_e == 3);
    const float s_mine = my_ok ? v[0] : -INFINITY;
    // batch max of my head over the tokens (lane bits 4 and 3 carry the token)
    float bm = fmaxf(s_mine, __shfl_xor_sync(0xffffffffu, s_mine, 16));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
    float mh_old = m[0];
#pragma unroll
    for (int hh = 1; hh < GM; ++hh)
      if (my_h == hh) mh_old = m[hh];
    const float mnew = fmaxf(mh_old, bm);
    const float p_mine = my_ok ? exp2f(s_mine - mnew) : 0.0f;
    float psum = p_mine + __shfl_xor_sync(0xffffffffu, p_mine, 16);
    psum += __shfl_xor_sync(0xffffffffu, psum, 8);
    const float corr_mine = exp2f(mh_old - mnew);   // 0 when m = -inf
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) {
      const int src = hh << (5 - LN);   // lane of (token 0, head hh)
      const float corr = __shfl_sync(0xffffffffu, corr_mine, src);
      const float mn = __shfl_sync(0xffffffffu, mnew, src);
      const float ps = __shfl_sync(0xffffffffu, psum, src);
      if (hh < G) {
        l[hh] = fmaf(l[hh], corr, ps);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[hh][j] *= corr;
#pragma unroll
        for (int e = 0; e < kB; ++e) {
          const float p = __shfl_sync(0xffffffffu, p_mine, (e * GM + hh) << (5 - LN));
#pragma unroll
          for (int j = 0; j < 4; ++j) o[hh][j] = fmaf(p, vb[e][j], o[hh][j]);
        }
        m[hh] = mn;
      }
    }
  };

  if (split < a.n_packed) {
    if (mixed) __syncthreads();   // qsm written
    const int64_t ngv = (a.t_quant + L.g - 1) / L.g;
    const int64_t g0 = (int64_t)split * a.split_groups;
    const int64_t g1 = min(ngv, g0 + a.split_groups);
    const int cpg = L.g / 32;                         // chunks per group
    const int64_t nchunk = (g1 - g0) * cpg;
    const float klut = KF == kNuq ? __half2float(SK.lut[lane & 7]) : 0.0f;
    const float vlut = VF == kNuq ? __half2float(SV.lut[lane & 7]) : 0.0f;
    const int hi = L.mixed_hi, mid = L.mixed_mid, lo = L.mixed_lo;
    const int krow = SK.code_row_bytes, vrow = SV.code_row_bytes;
    const int nmeta = mixed ? D - hi : D;
    float cst[4], snt[4];
    if (ROPE) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        angle_sincos(1.0, theta[j], &snt[j], &cst[j]);   // one position
      }
    }
    // the warp's chunks: k = warp, warp + kW, ...; a chunk past t_quant is skipped
    auto chunk_t0 = [&](int64_t k) { return (g0 + k / cpg) * L.g + 32 * (k % cpg); };
    int64_t lk = warp;   // load cursor
    int issued = 0;
    auto issue_next = [&]() {
      while (lk < nchunk && chunk_t0(lk) >= a.t_quant) lk += kW;
      if (lk < nchunk) {
        uint8_t* st = ring + (issued & 1) * SG.bytes;
        const int64_t gi = g0 + lk / cpg, sub = lk % cpg, t0 = chunk_t0(lk);
        const int64_t grp = sl * L.ng + gi;
        if constexpr (mixed) {
          const uint8_t* gb = reinterpret_cast<const uint8_t*>(SK.codes) + grp * (int64_t)L.mixed_group_bytes;
          cp_range(st + SG.k, gb + sub * 32 * hi * 2, 32 * hi * 2, lane);
          cp_range(st + SG.k_mid, gb + (int64_t)L.g * hi * 2 + sub * 32 * mid / 2, 32 * mid / 2, lane);
          cp_range(st + SG.k_lo, gb + (int64_t)L.g * hi * 2 + (int64_t)L.g * mid / 2 + sub * 32 * lo / 4, 32 * lo / 4, lane);
          cp_range(st + SG.ord, L.k_order + grp * D, D, lane);
        } else {
          cp_range(st + SG.k, reinterpret_cast<const uint8_t*>(SK.codes) + sl * SK.code_slab_bytes + t0 * krow,
                   32 * krow, lane);
        }
        cp_range(st + SG.ks, reinterpret_cast<const __half*>(SK.scale) + grp * nmeta, nmeta * 2, lane);
        cp_range(st + SG.kz, reinterpret_cast<const __half*>(SK.zero) + grp * nmeta, nmeta * 2, lane);
        cp_range(st + SG.v, reinterpret_cast<const uint8_t*>(SV.codes) + sl * SV.code_slab_bytes + t0 * vrow,
                 32 * vrow, lane);
        cp_range(st + SG.vs, reinterpret_cast<const __half*>(SV.scale) + sl * L.C + t0, 64, lane);
        cp_range(st + SG.vz, reinterpret_cast<const __half*>(SV.zero) + sl * L.C + t0, 64, lane);
        if (SV.nout > 0) {
          cp_range(st + SG.voc, L.v_out_col + (sl * L.C + t0) * SV.nout, 32 * SV.nout, lane);
          cp_range(st + SG.vov, L.v_out_val + (sl * L.C + t0) * SV.nout, 64 * SV.nout, lane);
        }
        if (SK.nout > 0) {
          const int32_t* rp = L.k_out_rowptr + grp * (L.g + 1) + 32 * sub;
          cp4(st + SG.rp + 4 * lane, rp + lane);
          if (lane == 0) cp4(st + SG.rp + 128, rp + 32);
          cp_range(st + SG.kc, L.k_out_col + grp * D * SK.nout, D * SK.nout, lane);
          cp_range(st + SG.kv, L.k_out_val + grp * D * SK.nout, D * SK.nout * 2, lane);
        }
        lk += kW;
      }
      cp_commit();
      ++issued;
    };
    issue_next();
    int consumed = 0;
    for (int64_t k = warp; k < nchunk; k += kW) {
      const int64_t t0 = chunk_t0(k);
      if (t0 >= a.t_quant) continue;
      issue_next();
      cp_wait<1>();
      __syncwarp();
      const uint8_t* st = ring + (consumed & 1) * SG.bytes;
      const int nt = (int)min((int64_t)32, a.t_quant - t0);
      // group metadata of the lane's channels (slots for MIXED); MIXED: query in slot order
      float ks[4] = {0.f, 0.f, 0.f, 0.f}, kz[4] = {0.f, 0.f, 0.f, 0.f};
      float qk[GM][4];
#pragma unroll
      for (int hh = 0; hh < GM; ++hh)
#pragma unroll
        for (int j = 0; j < 4; ++j) qk[hh][j] = q[hh][j];
      const __half* kss = reinterpret_cast<const __half*>(st + SG.ks);
      const __half* kzs = reinterpret_cast<const __half*>(st + SG.kz);
      if constexpr (mixed) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int slot = 4 * lane + j;
          const int ch = st[SG.ord + slot];
#pragma unroll
          for (int hh = 0; hh < GM; ++hh) qk[hh][j] = qsm[hh * D + ch];
          if (slot >= hi) {
            ks[j] = __half2float(kss[slot - hi]);
            kz[j] = __half2float(kzs[slot - hi]);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ks[j] = __half2float(kss[4 * lane + j]);
          kz[j] = __half2float(kzs[4 * lane + j]);
        }
      }
      // MIXED: the lane's plane (raw 16-bit, 4-bit or 2-bit slots), its word offset in a row,
      // the row stride, and the first code's shift
      int m_base = 0, m_stride = 0, m_shift = 0, m_bw = 0;
      uint32_t m_mask = 0u;
      bool m_raw = false;
      if constexpr (mixed) {
        const int s0 = 4 * lane;
        if (s0 < hi) {
          m_raw = true;   // m_bw = 0: the code formula is not used (and shifts stay < 32)
          m_base = SG.k + 2 * s0;
          m_stride = 2 * hi;
        } else if (s0 < hi + mid) {
          const int e0 = s0 - hi;
          m_base = SG.k_mid + 4 * (e0 / 8);
          m_stride = mid / 2;
          m_shift = 4 * (e0 % 8);
          m_bw = 4;
        } else {
          const int e0 = s0 - hi - mid;
          m_base = SG.k_lo + 4 * (e0 / 16);
          m_stride = lo / 4;
          m_shift = 2 * (e0 % 16);
          m_bw = 2;
        }
        m_mask = m_raw ? 0u : (1u << m_bw) - 1u;
      }
      float cs[4], sn[4];
      if (ROPE) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          angle_sincos((double)(L.n_sink + t0), theta[j], &sn[j], &cs[j]);
        }
      }
      for (int r0 = 0; r0 < nt; r0 += kB) {
        float kb[kB][4], vb[kB][4];
        bool ok[kB];
#pragma unroll
        for (int e = 0; e < kB; ++e) {
          const int r = r0 + e;
          ok[e] = r < nt;
          const int rr = ok[e] ? r : 0;
          // keys
          if constexpr (mixed) {
            // one word (two for raw slots) at the lane's plane position; no divergent paths
            const uint8_t* wp = st + m_base + rr * m_stride;
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(wp);
            uint32_t w1 = 0u;
            if (m_raw) w1 = *reinterpret_cast<const uint32_t*>(wp + 4);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t hbits = ((j < 2 ? w0 : w1) >> (16 * (j & 1))) & 0xffffu;
              const float raw = L.src_dtype == KVQ_F16 ? half_bits_to_float((uint16_t)hbits)
                                                       : __uint_as_float(hbits << 16);
              const float dq = __fmaf_rn((float)((w0 >> (m_shift + m_bw * j)) & m_mask), ks[j], kz[j]);
              kb[e][j] = m_raw ? raw : dq;
            }
          } else if constexpr (KF == kNuq) {
            uint32_t code[4];
            nuq_codes(reinterpret_cast<const uint32_t*>(st + SG.k + rr * krow), lane, code);
#pragma unroll
            for (int j = 0; j < 4; ++j) kb[e][j] = __fmaf_rn(__shfl_sync(0xffffffffu, klut, (int)code[j]), ks[j], kz[j]);
          } else {   // ASYM 2 / 4 bits, row layout
            const int bb = SK.bits;
            const int bitoff = 4 * lane * bb;
            const uint32_t w = reinterpret_cast<const uint32_t*>(st + SG.k + rr * krow)[bitoff / 32] >> (bitoff % 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) kb[e][j] = __fmaf_rn((float)((w >> (bb * j)) & ((1u << bb) - 1)), ks[j], kz[j]);
          }
          // values
          const float vs = __half2float(reinterpret_cast<const __half*>(st + SG.vs)[rr]);
          const float vz = __half2float(reinterpret_cast<const __half*>(st + SG.vz)[rr]);
          if constexpr (VF == kNuq) {
            uint32_t code[4];
            nuq_codes(reinterpret_cast<const uint32_t*>(st + SG.v + rr * vrow), lane, code);
#pragma unroll
            for (int j = 0; j < 4; ++j) vb[e][j] = __fmaf_rn(__shfl_sync(0xffffffffu, vlut, (int)code[j]), vs, vz);
          } else {   // ASYM 2 / 4 bits, pair layout (t0 even)
            const int bb = SV.bits, per = 16 / bb;
            const int c0 = 4 * lane;
            const uint32_t w = reinterpret_cast<const uint32_t*>(st + SG.v)[(rr >> 1) * (D / per) + c0 / per] >>
                               (16 * (rr & 1) + bb * (c0 % per));
#pragma unroll
            for (int j = 0; j < 4; ++j) vb[e][j] = __fmaf_rn((float)((w >> (bb * j)) & ((1u << bb) - 1)), vs, vz);
          }
          // sparse outliers overwrite (before RoPE)
          if (SK.nout > 0 && ok[e]) {
            const int32_t* rp = reinterpret_cast<const int32_t*>(st + SG.rp);
            const int x0 = rp[rr], x1 = rp[rr + 1];
            for (int x = x0; x < x1; ++x) {
              const int c = st[SG.kc + x];
              const float v = __half2float(reinterpret_cast<const __half*>(st + SG.kv)[x]);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                if (c == 4 * lane + j) kb[e][j] = v;
            }
          }
          if (SV.nout == 2 && ok[e]) {   // both entries in two loads
            const uint32_t cols = *reinterpret_cast<const uint16_t*>(st + SG.voc + rr * 2);
            const uint32_t vals = *reinterpret_cast<const uint32_t*>(st + SG.vov + rr * 4);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const int c = (int)((cols >> (8 * x)) & 0xffu);
              const float v = half_bits_to_float((uint16_t)(vals >> (16 * x)));
#pragma unroll
              for (int j = 0; j < 4; ++j)
                if (c == 4 * lane + j) vb[e][j] = v;
            }
          } else if (SV.nout > 0 && ok[e]) {
            for (int x = 0; x < SV.nout; ++x) {
              const int c = st[SG.voc + rr * SV.nout + x];
              const float v = __half2float(reinterpret_cast<const __half*>(st + SG.vov)[rr * SV.nout + x]);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                if (c == 4 * lane + j) vb[e][j] = v;
            }
          }
          if (ROPE) {
            rope4(kb[e], cs, sn, lane);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float c2 = cs[j] * cst[j] - sn[j] * snt[j];
              sn[j] = sn[j] * cst[j] + cs[j] * snt[j];
              cs[j] = c2;
            }
          }
        }
        consume(kb, vb, qk, ok);
      }
      __syncwarp();
      ++consumed;
    }
    cp_wait<0>();
    __syncwarp();
  } else if (split == a.raw_slot) {
    const int nraw = L.n_sink + a.t_res;
    for (int r0 = warp; r0 < nraw; r0 += kW * kB) {
      float kb[kB][4], vb[kB][4];
      bool ok[kB];
#pragma unroll
      for (int e = 0; e < kB; ++e) {
        const int r = r0 + e * kW;
        ok[e] = r < nraw;
        const int rr = ok[e] ? r : r0;
        const bool sink = rr < L.n_sink;
        const int64_t row = sink ? rr : rr - L.n_sink;
        const int64_t rows = sink ? L.n_sink : L.res_cap;
        const int64_t i = (sl * rows + row) * D + 4 * lane;
        const float4 kf = ld4(sink ? L.sink[0] : L.res[0], i, L.src_dtype);
        const float4 vf = ld4(sink ? L.sink[1] : L.res[1], i, L.src_dtype);
        kb[e][0] = kf.x; kb[e][1] = kf.y; kb[e][2] = kf.z; kb[e][3] = kf.w;
        vb[e][0] = vf.x; vb[e][1] = vf.y; vb[e][2] = vf.z; vb[e][3] = vf.w;
        if (ROPE) {
          const int64_t pos = sink ? rr : L.n_sink + a.t_quant + row;
          float cs[4], sn[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            angle_sincos((double)pos, theta[j], &sn[j], &cs[j]);
          }
          rope4(kb[e], cs, sn, lane);
        }
      }
      consume(kb, vb, q, ok);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);

  // merge the warps' states and write this split's partial state
  float* mine = wst + (size_t)warp * G * kRS;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
      *reinterpret_cast<float4*>(mine + hh * kRS + 4 * lane) = make_float4(o[hh][0], o[hh][1], o[hh][2], o[hh][3]);
      if (lane == 0) {
        mine[hh * kRS + D] = m[hh];
        mine[hh * kRS + D + 1] = l[hh];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int hh = i / D, d = i % D;
    float M = -INFINITY;
    for (int w = 0; w < kW; ++w) M = fmaxf(M, wst[((size_t)w * G + hh) * kRS + D]);
    float lsum = 0.0f, osum = 0.0f;
    for (int w = 0; w < kW; ++w) {
      const float* pw = wst + ((size_t)w * G + hh) * kRS;
      const float f = pw[D] == -INFINITY ? 0.0f : exp2f(pw[D] - M);
      lsum = fmaf(pw[D + 1], f, lsum);
      osum = fmaf(pw[d], f, osum);
    }
    const int64_t slot = ((int64_t)b * a.Hq + h * G + hh) * a.S + split;
    a.ws_o[slot * D + d] = osum;
    if (d == 0) {
      a.ws_m[slot] = M;
      a.ws_l[slot] = lsum;
    }
  }
}

template <int GM, int KF, int VF, bool ROPE>
cudaError_t launch_cc_k(const CcArgs& a, int grid_x, cudaStream_t s) {
  const int G = a.Hq / a.L.Hkv;
  // stage rings, queries (GM x 128), merge records; every part 16-byte aligned
  const size_t smem = (size_t)kW * 2 * a.st.bytes + ((size_t)GM * 128 + (size_t)kW * G * kRS) * sizeof(float);
  auto kern = decode_cc_kernel<GM, KF, VF, ROPE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(grid_x, a.L.Hkv, a.L.B);
  kern<<<grid, kW * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <int GM, int KF>
cudaError_t launch_cc_v(const CcArgs& a, int grid_x, cudaStream_t s) {
  const bool vnuq = a.L.side[1].scheme == KVQ_NUQ;
  if constexpr (KF == kMixed) {   // MIXED keys take no RoPE
    return vnuq ? launch_cc_k<GM, KF, kNuq, false>(a, grid_x, s) : launch_cc_k<GM, KF, kAsym, false>(a, grid_x, s);
  } else {
    if (a.L.rope)
      return vnuq ? launch_cc_k<GM, KF, kNuq, true>(a, grid_x, s) : launch_cc_k<GM, KF, kAsym, true>(a, grid_x, s);
    return vnuq ? launch_cc_k<GM, KF, kNuq, false>(a, grid_x, s) : launch_cc_k<GM, KF, kAsym, false>(a, grid_x, s);
  }
}

template <int GM>
cudaError_t launch_cc_g(const CcArgs& a, int grid_x, cudaStream_t s) {
  const int ks = a.L.side[0].scheme;
  if (ks == KVQ_NUQ) return launch_cc_v<GM, kNuq>(a, grid_x, s);
  if (ks == KVQ_MIXED) return launch_cc_v<GM, kMixed>(a, grid_x, s);
  return launch_cc_v<GM, kAsym>(a, grid_x, s);
}

}  // namespace

constexpr int kStageMax = 8192;

int up16(int x) { return (x + 15) & ~15; }

CcStage stage_layout(const Layout& L) {
  const Side& K = L.side[0];
  const Side& V = L.side[1];
  const bool mixed = K.scheme == KVQ_MIXED;
  CcStage g;
  int o = 0;
  g.k = o;
  if (mixed) {
    g.k_mid = g.k + 32 * L.mixed_hi * 2;
    g.k_lo = g.k_mid + 32 * L.mixed_mid / 2;
    o = g.k_lo + 32 * L.mixed_lo / 4;
  } else {
    g.k_mid = g.k_lo = 0;
    o += 32 * K.code_row_bytes;
  }
  o = up16(o);
  g.v = o;  o = up16(o + 32 * V.code_row_bytes);
  g.vs = o; o += 64;
  g.vz = o; o += 64;
  g.voc = o; o = up16(o + 32 * V.nout);
  g.vov = o; o = up16(o + 64 * V.nout);
  const int nmeta = mixed ? L.D - L.mixed_hi : L.D;
  g.ks = o; o = up16(o + nmeta * 2);
  g.kz = o; o = up16(o + nmeta * 2);
  g.ord = o; o += mixed ? L.D : 0;
  g.rp = o; o += K.nout > 0 ? 144 : 0;
  g.kc = o; o = up16(o + L.D * K.nout);
  g.kv = o; o = up16(o + L.D * K.nout * 2);
  g.bytes = o;
  return g;
}

bool cc_path_ok(const Layout& L, int Hq) {
  const Side& K = L.side[0];
  const Side& V = L.side[1];
  const int G = Hq / L.Hkv;
  if (L.D != 128 || G < 1 || G > 8 || L.g % 32) return false;
  if (stage_layout(L).bytes > kStageMax) return false;
  const bool k_ok = (K.scheme == KVQ_NUQ && K.axis == KVQ_AXIS_CHANNEL) ||
                    (K.scheme == KVQ_ASYM && K.axis == KVQ_AXIS_CHANNEL && (K.bits == 2 || K.bits == 4)) ||
                    (K.scheme == KVQ_MIXED && !L.rope);
  const bool v_ok = (V.scheme == KVQ_NUQ && V.axis == KVQ_AXIS_TOKEN) ||
                    (V.scheme == KVQ_ASYM && V.axis == KVQ_AXIS_TOKEN && (V.bits == 2 || V.bits == 4));
  return k_ok && v_ok;
}

cudaError_t launch_decode_cc(const Layout& L, const DecodePlan& p, const void* q, int q_dtype, int Hq,
                             int64_t t_quant, int t_res, float scale, float* ws_m, float* ws_l,
                             float* ws_o, int32_t* d_status, cudaStream_t s) {
  CcArgs a;
  a.st = stage_layout(L);
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
  const int G = Hq / L.Hkv;
  if (G <= 1) return launch_cc_g<1>(a, p.S, s);
  if (G <= 2) return launch_cc_g<2>(a, p.S, s);
  if (G <= 4) return launch_cc_g<4>(a, p.S, s);
  return launch_cc_g<8>(a, p.S, s);
}

}  // namespace kvq
