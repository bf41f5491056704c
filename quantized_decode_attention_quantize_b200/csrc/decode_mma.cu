// Tensor-core split-KV decode over a packed cache of 4-bit per-channel keys and 2-bit
// per-token values (the K4V2 allocation of [K4V2]; grouping of [KVQ] "Approach"),
// D = 128, token groups of 128, 2 <= G <= 8 query heads per KV head.
//
// Work.  Units are the packed token groups of every KV head plus a few pieces of
// each head's raw (sink + residual) tokens, in head-major order.  One CTA per SM
// takes a contiguous range of units; its twelve warps take the range's
// units round-robin.  A warp keeps one online-softmax state per (head, unit kind)
// and writes it to its own partial slot when it moves on; the combine kernel finds
// the slots of a head from the same partition.  No warp ever waits for another.
//
// Memory.  Every warp streams its own units through a ring of two half-group
// stages in shared memory with 16-byte cp.async copies (all 32 lanes, coalesced): per
// 64 tokens the key codes (4 KiB), value codes (2 KiB), value scale / zero-point
// (256 B) and, with the first half, the group's key scale / zero-point (512 B).
// Every byte of the format is read once; the next half group is in flight while the
// warp computes on the current one (twelve warps per SM).
//
// Math.  A 4-bit or 2-bit code masked into the low mantissa bits of an fp16 half with
// a zero exponent field is the subnormal number c * 2^-24 * f, exact, where f = 2^p
// for a field starting at bit p of the half.  Scores are a tensor-core product with
// tokens as M and query heads as N (m16n8k16, fp16 in, fp32 accumulate):
//   A[t][d] = c[t][d] 2^-24 f_d,   B[d][h] = fp16(q~[h][d] s[d] 2^(24 - e) / f_d)
//   score   = 2^e (A.B) + sum_d q~[h][d] z[d]        (q~ = q * scale * log2 e)
// (e: one exponent per group so that B fits fp16).  B is split into an fp16 high part
// and an fp16 remainder so that the key product carries ~22 bits: with G <= 4 the two
// parts ride in the otherwise empty columns 4..7 of the same product (hi in column h,
// remainder in column h + 4, summed with one shuffle); with G > 4 they take two
// products.  The probabilities become the B
// operand of the value product through an in-register 8x8 transpose (movmatrix) and
// the value codes (pair layout) are the A operand with channels as M:
//   A[d][t] = c[t][d] 2^-24 f_d,   B[t][h] = fp16(p[t][h] s[t])
//   o[h][d] = 2^24 / f_d (A.B)[d][h] + sum_t p[t][h] z[t].
// Online softmax is kept in the log2 domain.
//
// Waits.  A warp only waits for its own copies (cp.async.wait_group); no warp waits for
// another.
#include <algorithm>
#include <cstdint>

#include "kvq_internal.cuh"

namespace kvq {

namespace {

constexpr int kCW = 12;                       // warps per CTA (one CTA per SM)
constexpr int kBuffers = 2;                   // per-warp ring of half-group stages
constexpr int kThreads = kCW * 32;
// a stage holds 64 tokens: key codes, value codes, value scale / zero-point, and (first
// half only) the group's key scale / zero-point
constexpr int kHalfK = 64 * 64, kHalfV = 32 * 64, kHalfVM = 2 * 64 * 2, kHalfKM = 2 * 128 * 2;
constexpr int kStageBytes = kHalfK + kHalfV + kHalfVM + kHalfKM;
constexpr int kScratchBytes = 2 * 32 * 16 * 4;  // per warp: hi and lo B fragments
constexpr int kRawPieces = 12;                // raw-token units per head (<= kCW)
constexpr float kLog2e = 1.4426950408889634f;

struct MmaArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const __half* k_scale;
  const __half* k_zero;
  const __half* v_scale;
  const __half* v_zero;
  int64_t k_slab_bytes, v_slab_bytes;
  int64_t C;
  int ng;
  int B, Hkv, Hq, G;
  int64_t t_quant;
  int t_res, n_sink, res_cap, src_dtype;
  const void* sink_k;
  const void* sink_v;
  const void* res_k;
  const void* res_v;
  const void* q;
  int q_dtype;
  float qscale;
  int ngv;        // valid groups per head
  int rw;         // raw pieces per head
  int uph;        // units per head (rw + ngv)
  int64_t N;      // total units
  int grid;
  int S;          // partial slots per query head
  float* ws_m;
  float* ws_l;
  float* ws_o;
  int32_t* status;
};

// ---- PTX helpers ------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float pow2(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// byte 1 -> byte 0 and byte 3 -> byte 2 (other bytes zero)
__device__ __forceinline__ uint32_t odd_bytes_down(uint32_t w) { return __byte_perm(w, 0u, 0x4341u); }

// ---- unit partition (shared with the combine kernel) -----------------------------
__host__ __device__ __forceinline__ int64_t unit_start(int64_t c, int64_t N, int grid) {
  return c * N / grid;
}
__host__ __device__ __forceinline__ int cta_of_unit(int64_t u, int64_t N, int grid) {
  return (int)(((u + 1) * grid - 1) / N);
}
// slot of (CTA c, warp w, kind) within the head whose first CTA is c0
__host__ __device__ __forceinline__ int slot_of(int c, int c0, int w, int kind) {
  return ((c - c0) * kCW + w) * 2 + kind;
}

// ---- raw tokens (sink + residual) on CUDA cores ----------------------------------------
// Four consecutive elements at element offset i (i a multiple of 4).
__device__ __forceinline__ float4 load4(const void* p, int64_t i, int dtype) {
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

// Lane owns channels 4 lane .. 4 lane + 3; fp32, log2 domain.  Tokens go four at a
// time: their loads are issued together, the 4 x G score reductions of a chunk are
// independent, then one softmax update per chunk.  Writes the piece's slot.
template <int GM>
__device__ void raw_piece(const MmaArgs& a, int head, int piece, int slot) {
  constexpr int kBatch = 4;
  const int lane = threadIdx.x & 31;
  const int b = head / a.Hkv, h = head % a.Hkv;
  const int G = a.G;
  const int nraw = a.n_sink + a.t_res;
  const int r0 = piece * nraw / a.rw, r1 = (piece + 1) * nraw / a.rw;
  float q[GM][4], o[GM][4], m[GM], l[GM];
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.0f;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (hh < G) x = load4(a.q, ((int64_t)b * a.Hq + h * G + hh) * 128 + 4 * lane, a.q_dtype);
    q[hh][0] = x.x * a.qscale; q[hh][1] = x.y * a.qscale;
    q[hh][2] = x.z * a.qscale; q[hh][3] = x.w * a.qscale;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[hh][k] = 0.0f;
  }
  auto fetch = [&](int rb, float4 (&kt)[kBatch], float4 (&vt)[kBatch]) {
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      const int r = rb + e;
      kt[e] = vt[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < r1) {
        const bool sink = r < a.n_sink;
        const int64_t row = sink ? r : r - a.n_sink;
        const int64_t rows = sink ? a.n_sink : a.res_cap;
        const int64_t i = ((int64_t)head * rows + row) * 128 + 4 * lane;
        kt[e] = load4(sink ? a.sink_k : a.res_k, i, a.src_dtype);
        vt[e] = load4(sink ? a.sink_v : a.res_v, i, a.src_dtype);
      }
    }
  };
  float4 kt[kBatch], vt[kBatch];
  for (int rb = r0; rb < r1; rb += kBatch) {
    fetch(rb, kt, vt);
    float sc[kBatch][GM];
#pragma unroll
    for (int e = 0; e < kBatch; ++e)
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        float part = q[hh][0] * kt[e].x;
        part = fmaf(q[hh][1], kt[e].y, part);
        part = fmaf(q[hh][2], kt[e].z, part);
        part = fmaf(q[hh][3], kt[e].w, part);
        sc[e][hh] = part;
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int e = 0; e < kBatch; ++e)
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) sc[e][hh] += __shfl_xor_sync(0xffffffffu, sc[e][hh], off);
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) {
      float cm = m[hh];
#pragma unroll
      for (int e = 0; e < kBatch; ++e)
        if (rb + e < r1) cm = fmaxf(cm, sc[e][hh]);
      const float corr = ex2(m[hh] - cm);
      l[hh] *= corr;
#pragma unroll
      for (int k = 0; k < 4; ++k) o[hh][k] *= corr;
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const float p = rb + e < r1 ? ex2(sc[e][hh] - cm) : 0.0f;
        l[hh] += p;
        o[hh][0] = fmaf(p, vt[e].x, o[hh][0]);
        o[hh][1] = fmaf(p, vt[e].y, o[hh][1]);
        o[hh][2] = fmaf(p, vt[e].z, o[hh][2]);
        o[hh][3] = fmaf(p, vt[e].w, o[hh][3]);
      }
      m[hh] = cm;
    }
  }
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
      const int64_t sl = ((int64_t)b * a.Hq + h * G + hh) * a.S + slot;
      *reinterpret_cast<float4*>(a.ws_o + sl * 128 + 4 * lane) = make_float4(o[hh][0], o[hh][1], o[hh][2], o[hh][3]);
      if (lane == 0) {
        a.ws_m[sl] = m[hh];
        a.ws_l[sl] = l[hh];
      }
    }
  }
}

// ---- packed groups: per-warp state of the tensor-core path ------------------------------
struct MmaState {
  float O[8][4];     // O^T tiles: (channel rows of tile cm) x (heads 2j, 2j+1)
  float m[2], l[2], W[2];
};

__device__ __forceinline__ void state_reset(MmaState& st) {
#pragma unroll
  for (int cm = 0; cm < 8; ++cm) st.O[cm][0] = st.O[cm][1] = st.O[cm][2] = st.O[cm][3] = 0.0f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = st.W[0] = st.W[1] = 0.0f;
}

// Write a warp's tensor-core state for `head` into its slot.  Lane (g, j) holds heads
// 2j, 2j + 1 (with DUAL, lanes j >= 2 hold copies of lanes j - 2 and write nothing).
template <bool DUAL>
__device__ void state_flush(const MmaArgs& a, MmaState& st, int head, int slot) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const int b = head / a.Hkv, h = head % a.Hkv, G = a.G;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    st.l[0] += __shfl_xor_sync(0xffffffffu, st.l[0], o);
    st.l[1] += __shfl_xor_sync(0xffffffffu, st.l[1], o);
    st.W[0] += __shfl_xor_sync(0xffffffffu, st.W[0], o);
    st.W[1] += __shfl_xor_sync(0xffffffffu, st.W[1], o);
  }
  // rows of tile cm: g -> field 2 (cm % 4) (factor 1, 16, 1, 16), g + 8 -> next field
  // (factor 4, 64, 4, 64); 2^24 / f undoes the subnormal encoding
  const float inv_lo[2] = {16777216.0f, 1048576.0f};   // 2^24, 2^20
  const float inv_hi[2] = {4194304.0f, 262144.0f};     // 2^22, 2^18
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int hh = 2 * j + e;
    if (hh < G && (!DUAL || j < 2)) {
      const int64_t sl = ((int64_t)b * a.Hq + h * G + hh) * a.S + slot;
      float* dst = a.ws_o + sl * 128;
#pragma unroll
      for (int cm = 0; cm < 8; ++cm) {
        const int d0 = 16 * g + 8 * (cm >> 2) + 2 * (cm & 3);
        const float v0 = fmaf(st.O[cm][e], inv_lo[cm & 1], st.W[e]);
        const float v1 = fmaf(st.O[cm][2 + e], inv_hi[cm & 1], st.W[e]);
        *reinterpret_cast<float2*>(dst + d0) = make_float2(v0, v1);
      }
      if (g == 0) {
        a.ws_m[sl] = st.m[e];
        a.ws_l[sl] = st.l[e];
      }
    }
  }
}

// The key-product B operand of one group (per lane), its exponent and bias.
struct KeyOp {
  uint32_t bh[8][2], bl[8][2];
  float mult, bias0, bias1;
};

// Build the key-product B operand of a group from its per-channel scale / zero-point
// (ks, kz in shared memory) and the head's pre-scaled queries.  DUAL: G <= 4, the
// remainder rides in columns 4..7.
template <bool DUAL, int GM>
__device__ __forceinline__ void key_operand(const MmaArgs& a, const __half* ks, const __half* kz,
                                            uint32_t* scratch, const float (&qv)[GM][4], KeyOp& ko) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const int G = a.G;
  // lane owns channels 4 lane .. 4 lane + 3 of every head
  const uint2 sv = *reinterpret_cast<const uint2*>(ks + 4 * lane);
  const uint2 zv = *reinterpret_cast<const uint2*>(kz + 4 * lane);
  const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
  const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
  const float2 z01 = __half22float2(*reinterpret_cast<const __half2*>(&zv.x));
  const float2 z23 = __half22float2(*reinterpret_cast<const __half2*>(&zv.y));
  const float s[4] = {s01.x, s01.y, s23.x, s23.y};
  const float z[4] = {z01.x, z01.y, z23.x, z23.y};
  float av[GM][4], dz[GM];
  float amax = 0.0f;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    dz[hh] = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      av[hh][k] = qv[hh][k] * s[k];
      dz[hh] = fmaf(qv[hh][k], z[k], dz[hh]);
      amax = fmaxf(amax, fabsf(av[hh][k]));
    }
  }
  amax = warp_max(amax);
  // one exponent for the group: max |a 2^(24 - e)| < 2^15
  int ex = 0;
  if (amax > 0.0f) ex = (int)((__float_as_uint(amax) >> 23) & 0xff) - 127 + 10;
  ex = max(-100, min(127, ex));
  ko.mult = pow2(ex);
  const float sc = __uint_as_float((uint32_t)max(1, min(254, 127 + 24 - ex)) << 23);
  const float sc16 = sc * 0.0625f;
  // scatter into the fragment layout: channel c = 4 lane + k -> consumer lane
  // 4 hh + lane / 8, k-step 2 ((lane & 7) / 2) + k / 2, register k & 1, half lane & 1
  uint16_t* sh = reinterpret_cast<uint16_t*>(scratch);
  uint16_t* sl = sh + 32 * 16 * 2;
  const int kkbase = 2 * ((lane & 7) >> 1), half = lane & 1;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
      const int dl = 4 * hh + (lane >> 3);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x = av[hh][k] * ((k & 1) ? sc16 : sc);
        const __half hi = __float2half_rn(x);
        const int idx = ((dl * 8 + kkbase + (k >> 1)) * 2 + (k & 1)) * 2 + half;
        const uint16_t lo = __half_as_ushort(__float2half_rn(x - __half2float(hi)));
        sh[idx] = __half_as_ushort(hi);
        if (DUAL) sh[idx + 4 * 4 * 8 * 2 * 2] = lo;   // consumer lane + 16: column hh + 4
        else sl[idx] = lo;
      }
    }
  }
  // butterfly reduction of the per-head sums q~ . z over the warp
  const int h0 = DUAL ? 2 * (j & 1) : 2 * j, h1 = h0 + 1;
  const bool u4 = lane & 16, u3 = lane & 8, u2 = lane & 4;
  if constexpr (GM == 4) {
    // four heads: the lane ends with head 2 b4 + b3 (b_k = bit k of the lane)
    float v2[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float send = u4 ? dz[k] : dz[k + 2];
      const float keep = u4 ? dz[k + 2] : dz[k];
      v2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float v3 = (u3 ? v2[1] : v2[0]) + __shfl_xor_sync(0xffffffffu, u3 ? v2[0] : v2[1], 8);
    v3 += __shfl_xor_sync(0xffffffffu, v3, 4);
    v3 += __shfl_xor_sync(0xffffffffu, v3, 2);
    v3 += __shfl_xor_sync(0xffffffffu, v3, 1);
    ko.bias0 = __shfl_sync(0xffffffffu, v3, 16 * ((h0 >> 1) & 1) + 8 * (h0 & 1));
    ko.bias1 = __shfl_sync(0xffffffffu, v3, 16 * ((h1 >> 1) & 1) + 8 * (h1 & 1));
  } else {
    // eight heads: the lane ends with head 4 b4 + 2 b3 + b2
    float v2[4], v3[2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float send = u4 ? dz[k] : dz[k + 4];
      const float keep = u4 ? dz[k + 4] : dz[k];
      v2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float send = u3 ? v2[k] : v2[k + 2];
      const float keep = u3 ? v2[k + 2] : v2[k];
      v3[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float v4 = (u2 ? v3[1] : v3[0]) + __shfl_xor_sync(0xffffffffu, u2 ? v3[0] : v3[1], 4);
    v4 += __shfl_xor_sync(0xffffffffu, v4, 2);
    v4 += __shfl_xor_sync(0xffffffffu, v4, 1);
    ko.bias0 = __shfl_sync(0xffffffffu, v4, ((h0 >> 2) & 1) * 16 + ((h0 >> 1) & 1) * 8 + (h0 & 1) * 4);
    ko.bias1 = __shfl_sync(0xffffffffu, v4, ((h1 >> 2) & 1) * 16 + ((h1 >> 1) & 1) * 8 + (h1 & 1) * 4);
  }
  __syncwarp();
  if ((DUAL ? (g & 3) : g) < G) {
    const uint4* src = reinterpret_cast<const uint4*>(scratch) + lane * 4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 x = src[u];
      ko.bh[2 * u][0] = x.x; ko.bh[2 * u][1] = x.y; ko.bh[2 * u + 1][0] = x.z; ko.bh[2 * u + 1][1] = x.w;
    }
    if (!DUAL) {
      const uint4* srl = reinterpret_cast<const uint4*>(scratch) + 32 * 4 + lane * 4;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 x = srl[u];
        ko.bl[2 * u][0] = x.x; ko.bl[2 * u][1] = x.y; ko.bl[2 * u + 1][0] = x.z; ko.bl[2 * u + 1][1] = x.w;
      }
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) ko.bh[kk][0] = ko.bh[kk][1] = ko.bl[kk][0] = ko.bl[kk][1] = 0u;
  }
  __syncwarp();
}

// 64 tokens (one half of a group) held in a ring stage: key codes [64][16] words,
// value codes [32 pairs][16] words, value scale / zero-point [64] each.
template <bool DUAL>
__device__ __forceinline__ void mma_half(MmaState& st, const uint8_t* stage, const KeyOp& ko,
                                         int tvalid) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const uint32_t* kc = reinterpret_cast<const uint32_t*>(stage);
  const uint32_t* vc = reinterpret_cast<const uint32_t*>(stage + kHalfK);
  const __half* vs = reinterpret_cast<const __half*>(stage + kHalfK + kHalfV);
  const __half* vz = vs + 64;

  // ---- scores of the 64 tokens (4 tiles of 16) ----
  float S[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    S[mt][0] = S[mt][1] = S[mt][2] = S[mt][3] = 0.0f;
    const uint4 w0 = *reinterpret_cast<const uint4*>(kc + (16 * mt + g) * 16 + 4 * j);
    const uint4 w1 = *reinterpret_cast<const uint4*>(kc + (16 * mt + g + 8) * 16 + 4 * j);
    const uint32_t x0[4] = {w0.x, w0.y, w0.z, w0.w};
    const uint32_t x1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t p0 = odd_bytes_down(x0[w]), p1 = odd_bytes_down(x1[w]);
      // k-step 2w: nibbles 0 (f 1) and 1 (f 16) of each half
      const uint32_t a00 = x0[w] & 0x000F000Fu, a01 = x1[w] & 0x000F000Fu;
      const uint32_t a02 = x0[w] & 0x00F000F0u, a03 = x1[w] & 0x00F000F0u;
      // k-step 2w + 1: nibbles 2 (f 1) and 3 (f 16)
      const uint32_t a10 = p0 & 0x000F000Fu, a11 = p1 & 0x000F000Fu;
      const uint32_t a12 = p0 & 0x00F000F0u, a13 = p1 & 0x00F000F0u;
      mma16816(S[mt], a00, a01, a02, a03, ko.bh[2 * w][0], ko.bh[2 * w][1]);
      mma16816(S[mt], a10, a11, a12, a13, ko.bh[2 * w + 1][0], ko.bh[2 * w + 1][1]);
      if (!DUAL) {
        mma16816(S[mt], a00, a01, a02, a03, ko.bl[2 * w][0], ko.bl[2 * w][1]);
        mma16816(S[mt], a10, a11, a12, a13, ko.bl[2 * w + 1][0], ko.bl[2 * w + 1][1]);
      }
    }
  }
  // ---- online softmax (log2 domain) ----
  if (DUAL) {   // add the remainder columns (lane j ^ 2) to the high-part columns
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) S[mt][e] += __shfl_xor_sync(0xffffffffu, S[mt][e], 2);
  }
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    S[mt][0] = fmaf(S[mt][0], ko.mult, ko.bias0);
    S[mt][1] = fmaf(S[mt][1], ko.mult, ko.bias1);
    S[mt][2] = fmaf(S[mt][2], ko.mult, ko.bias0);
    S[mt][3] = fmaf(S[mt][3], ko.mult, ko.bias1);
  }
  const bool partial = tvalid < 64;
  if (partial) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      if (16 * mt + g >= tvalid) S[mt][0] = S[mt][1] = -INFINITY;
      if (16 * mt + g + 8 >= tvalid) S[mt][2] = S[mt][3] = -INFINITY;
    }
  }
  float gm0 = -INFINITY, gm1 = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    gm0 = fmaxf(gm0, fmaxf(S[mt][0], S[mt][2]));
    gm1 = fmaxf(gm1, fmaxf(S[mt][1], S[mt][3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    gm0 = fmaxf(gm0, __shfl_xor_sync(0xffffffffu, gm0, o));
    gm1 = fmaxf(gm1, __shfl_xor_sync(0xffffffffu, gm1, o));
  }
  const float mn0 = fmaxf(st.m[0], gm0), mn1 = fmaxf(st.m[1], gm1);
  if (__any_sync(0xffffffffu, mn0 != st.m[0] || mn1 != st.m[1])) {
    const float c0 = ex2(st.m[0] - mn0), c1 = ex2(st.m[1] - mn1);
#pragma unroll
    for (int cm = 0; cm < 8; ++cm) {
      st.O[cm][0] *= c0;
      st.O[cm][1] *= c1;
      st.O[cm][2] *= c0;
      st.O[cm][3] *= c1;
    }
    st.l[0] *= c0;
    st.l[1] *= c1;
    st.W[0] *= c0;
    st.W[1] *= c1;
    st.m[0] = mn0;
    st.m[1] = mn1;
  }
  // ---- value product: one 16-token k-step per score tile ----
  // with DUAL, columns 4..7 (lanes j >= 2) of the probability operand are zero
  const float keep = (!DUAL || j < 2) ? 1.0f : 0.0f;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int t0 = 16 * mt + g, t1 = t0 + 8;
    float s0 = __half2float(vs[t0]), s1 = __half2float(vs[t1]);
    float z0 = __half2float(vz[t0]), z1 = __half2float(vz[t1]);
    if (partial) {
      if (t0 >= tvalid) s0 = z0 = 0.0f;
      if (t1 >= tvalid) s1 = z1 = 0.0f;
    }
    const float p00 = ex2(S[mt][0] - mn0), p01 = ex2(S[mt][1] - mn1);
    const float p10 = ex2(S[mt][2] - mn0), p11 = ex2(S[mt][3] - mn1);
    st.l[0] += p00 + p10;
    st.l[1] += p01 + p11;
    st.W[0] = fmaf(p00, z0, fmaf(p10, z1, st.W[0]));
    st.W[1] = fmaf(p01, z0, fmaf(p11, z1, st.W[1]));
    const float sk0 = s0 * keep, sk1 = s1 * keep;
    const uint32_t pb0 = movtrans(pack_half2(p00 * sk0, p01 * sk0));
    const uint32_t pb1 = movtrans(pack_half2(p10 * sk1, p11 * sk1));
    const uint2 va = *reinterpret_cast<const uint2*>(vc + (8 * mt + j) * 16 + 2 * g);
    const uint2 vb = *reinterpret_cast<const uint2*>(vc + (8 * mt + j + 4) * 16 + 2 * g);
    const uint32_t ya = odd_bytes_down(va.x), yb = odd_bytes_down(vb.x);
    const uint32_t za = odd_bytes_down(va.y), zb = odd_bytes_down(vb.y);
    // fields at bits 0, 2, 4, 6 of each half: factors 1, 4, 16, 64
    mma16816(st.O[0], va.x & 0x00030003u, va.x & 0x000C000Cu, vb.x & 0x00030003u, vb.x & 0x000C000Cu, pb0, pb1);
    mma16816(st.O[1], va.x & 0x00300030u, va.x & 0x00C000C0u, vb.x & 0x00300030u, vb.x & 0x00C000C0u, pb0, pb1);
    mma16816(st.O[2], ya & 0x00030003u, ya & 0x000C000Cu, yb & 0x00030003u, yb & 0x000C000Cu, pb0, pb1);
    mma16816(st.O[3], ya & 0x00300030u, ya & 0x00C000C0u, yb & 0x00300030u, yb & 0x00C000C0u, pb0, pb1);
    mma16816(st.O[4], va.y & 0x00030003u, va.y & 0x000C000Cu, vb.y & 0x00030003u, vb.y & 0x000C000Cu, pb0, pb1);
    mma16816(st.O[5], va.y & 0x00300030u, va.y & 0x00C000C0u, vb.y & 0x00300030u, vb.y & 0x00C000C0u, pb0, pb1);
    mma16816(st.O[6], za & 0x00030003u, za & 0x000C000Cu, zb & 0x00030003u, zb & 0x000C000Cu, pb0, pb1);
    mma16816(st.O[7], za & 0x00300030u, za & 0x00C000C0u, zb & 0x00300030u, zb & 0x00C000C0u, pb0, pb1);
  }
}

// ---- per-warp staging with cp.async ----------------------------------------------------
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copy one half group (64 rows) of head `head`, group `gi` into a stage buffer: every
// lane moves 16-byte chunks, coalesced.
__device__ __forceinline__ void load_half(const MmaArgs& a, uint8_t* buf, int head, int gi, int hf) {
  const int lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)gi * 128 + 64 * hf;
  const uint8_t* kc = a.k_codes + (int64_t)head * a.k_slab_bytes + t0 * 64;
  const uint8_t* vc = a.v_codes + (int64_t)head * a.v_slab_bytes + t0 * 32;
#pragma unroll
  for (int e = 0; e < kHalfK / 512; ++e) cp_async16(buf + 16 * (lane + 32 * e), kc + 16 * (lane + 32 * e));
#pragma unroll
  for (int e = 0; e < kHalfV / 512; ++e)
    cp_async16(buf + kHalfK + 16 * (lane + 32 * e), vc + 16 * (lane + 32 * e));
  if (lane < 16) {   // value scale (lanes 0..7) and zero-point (lanes 8..15), 64 rows each
    const __half* src = (lane < 8 ? a.v_scale : a.v_zero) + (int64_t)head * a.C + t0 + 8 * (lane & 7);
    cp_async16(buf + kHalfK + kHalfV + 16 * lane, src);
  }
  if (hf == 0) {     // the group's key scale (lanes 0..15) and zero-point (16..31)
    const __half* src = (lane < 16 ? a.k_scale : a.k_zero) + ((int64_t)head * a.ng + gi) * 128 + 8 * (lane & 15);
    cp_async16(buf + kHalfK + kHalfV + kHalfVM + 16 * lane, src);
  }
}

// Walks a warp's units (u = U0 + warp + i * kCW) without division.
struct UnitCursor {
  int64_t u;
  int head, r;
  __device__ __forceinline__ void init(int64_t u0, int uph) {
    u = u0;
    head = (int)(u0 / uph);
    r = (int)(u0 % uph);
  }
  __device__ __forceinline__ void next(int uph) {
    u += kCW;
    r += kCW;
    while (r >= uph) {
      r -= uph;
      ++head;
    }
  }
};

// ---- the kernel --------------------------------------------------------------------------
template <bool DUAL>
__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(MmaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int GM = DUAL ? 4 : 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int64_t U0 = unit_start(c, a.N, a.grid), U1 = unit_start(c + 1, a.N, a.grid);
  uint8_t* ring = smem + (size_t)warp * (kBuffers * kStageBytes);
  uint32_t* my_scratch = reinterpret_cast<uint32_t*>(smem + (size_t)kCW * kBuffers * kStageBytes) +
                         warp * (kScratchBytes / 4);

  // load cursor: runs kBuffers - 1 half groups ahead of the compute cursor
  UnitCursor lc;
  lc.init(U0 + warp, a.uph);
  int lhf = 0;
  auto skip_raw = [&]() {
    while (lc.u < U1 && lc.r < a.rw) lc.next(a.uph);
  };
  skip_raw();
  int issued = 0;
  auto issue_next = [&]() {
    if (lc.u < U1) {
      load_half(a, ring + (issued % kBuffers) * kStageBytes, lc.head, lc.r - a.rw, lhf);
      if (++lhf == 2) {
        lhf = 0;
        lc.next(a.uph);
        skip_raw();
      }
    }
    cp_async_commit();   // an empty group keeps the group count uniform
    ++issued;
  };
#pragma unroll 1
  for (int e = 0; e < kBuffers - 1; ++e) issue_next();

  MmaState st;
  state_reset(st);
  float qv[GM][4];
  int cur_head = -1, cur_c0 = 0;
  bool qbad = false;
  int consumed = 0;
  UnitCursor cc;
  cc.init(U0 + warp, a.uph);
  for (; cc.u < U1; cc.next(a.uph)) {
    const int head = cc.head, r = cc.r;
    if (r < a.rw) {
      if (cur_head >= 0) {
        state_flush<DUAL>(a, st, cur_head, slot_of(c, cur_c0, warp, 1));
        state_reset(st);
        cur_head = -1;
      }
      raw_piece<GM>(a, head, r, slot_of(c, cta_of_unit((int64_t)head * a.uph, a.N, a.grid), warp, 0));
      continue;
    }
    if (head != cur_head) {
      if (cur_head >= 0) {
        state_flush<DUAL>(a, st, cur_head, slot_of(c, cur_c0, warp, 1));
        state_reset(st);
      }
      cur_head = head;
      cur_c0 = cta_of_unit((int64_t)head * a.uph, a.N, a.grid);
      // this head's queries, pre-scaled, for channels 4 lane .. 4 lane + 3
      const int b = head / a.Hkv, h = head % a.Hkv;
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (hh < a.G) x = load4(a.q, ((int64_t)b * a.Hq + h * a.G + hh) * 128 + 4 * lane, a.q_dtype);
        qbad |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
        qv[hh][0] = x.x * a.qscale; qv[hh][1] = x.y * a.qscale;
        qv[hh][2] = x.z * a.qscale; qv[hh][3] = x.w * a.qscale;
      }
    }
    const int gi = r - a.rw;
    const int tvalid = (int)min((int64_t)128, a.t_quant - (int64_t)gi * 128);
    KeyOp ko;
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
      cp_async_wait<kBuffers - 2>();
      __syncwarp();
      const uint8_t* stg = ring + (consumed % kBuffers) * kStageBytes;
      if (hf == 0) {
        const __half* ks = reinterpret_cast<const __half*>(stg + kHalfK + kHalfV + kHalfVM);
        key_operand<DUAL, GM>(a, ks, ks + 128, my_scratch, qv, ko);
      }
      if (tvalid > 64 * hf) mma_half<DUAL>(st, stg, ko, tvalid - 64 * hf);
      __syncwarp();
      ++consumed;
      issue_next();
    }
  }
  cp_async_wait<0>();
  if (cur_head >= 0) state_flush<DUAL>(a, st, cur_head, slot_of(c, cur_c0, warp, 1));
  if (__any_sync(0xffffffffu, qbad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);
}

// ---- combine for this path: finds the slots of a head from the partition --------------
struct CombArgsMma {
  int Hkv, Hq, G, uph, rw, grid, S;
  int64_t N;
  const float* m;
  const float* l;
  const float* o;
  void* out;
  int out_dtype;
};

__global__ void __launch_bounds__(128) combine_mma_kernel(CombArgsMma a) {
  extern __shared__ float sh[];           // [S] m, [S] weight, [S] (int) slot of valid entries
  float* sm_m = sh;
  float* sm_w = sh + a.S;
  int* sm_slot = reinterpret_cast<int*>(sh + 2 * a.S);
  __shared__ int warp_cnt[4];
  __shared__ float red[4];
  __shared__ float sM, sL;
  const int hq = blockIdx.x, b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int head = b * a.Hkv + hq / a.G;
  const int64_t Hs = (int64_t)head * a.uph, He = Hs + a.uph;
  const int c0 = cta_of_unit(Hs, a.N, a.grid), c1 = cta_of_unit(He - 1, a.N, a.grid);
  const int nslots = (c1 - c0 + 1) * kCW * 2;
  const int64_t row = (int64_t)b * a.Hq + hq;
  // 1. compact the valid slots in slot order: slot (c, w, kind) holds data iff warp w of
  //    CTA c owns a unit of this head and kind
  int base = 0;
  for (int s0 = 0; s0 < nslots; s0 += blockDim.x) {
    const int s = s0 + threadIdx.x;
    bool valid = false;
    if (s < nslots) {
      const int kind = s & 1, w = (s >> 1) % kCW, c = c0 + (s >> 1) / kCW;
      const int64_t U0 = unit_start(c, a.N, a.grid), U1 = unit_start(c + 1, a.N, a.grid);
      const int64_t lo0 = kind ? Hs + a.rw : Hs, hi0 = kind ? He : Hs + a.rw;
      const int64_t lo = U0 > lo0 ? U0 : lo0, hi = U1 < hi0 ? U1 : hi0;
      if (lo < hi) valid = lo + (((w - (lo - U0)) % kCW) + kCW) % kCW < hi;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, valid);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += warp_cnt[w];
    if (valid) {
      const int idx = off + __popc(bal & ((1u << lane) - 1));
      sm_slot[idx] = s;
      sm_m[idx] = a.m[row * a.S + s];
    }
    for (int w = 0; w < 4; ++w) base += warp_cnt[w];
    __syncthreads();
  }
  const int nv = base;
  // 2. max and weights
  float M = -INFINITY;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) M = fmaxf(M, sm_m[i]);
  M = warp_max(M);
  if (lane == 0) red[warp] = M;
  __syncthreads();
  if (threadIdx.x == 0) sM = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  M = sM;
  float L = 0.0f;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const float f = sm_m[i] == -INFINITY ? 0.0f : exp2f(sm_m[i] - M);
    sm_w[i] = f;
    L = fmaf(a.l[row * a.S + sm_slot[i]], f, L);
  }
  L = warp_sum(L);
  __syncthreads();
  if (lane == 0) red[warp] = L;
  __syncthreads();
  if (threadIdx.x == 0) sL = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();
  const float invL = 1.0f / sL;
  // 3. weighted sum of the partial outputs
  const int d = threadIdx.x;
  float o0 = 0.0f, o1 = 0.0f;
  int i = 0;
  for (; i + 1 < nv; i += 2) {
    o0 = fmaf(a.o[(row * a.S + sm_slot[i]) * 128 + d], sm_w[i], o0);
    o1 = fmaf(a.o[(row * a.S + sm_slot[i + 1]) * 128 + d], sm_w[i + 1], o1);
  }
  if (i < nv) o0 = fmaf(a.o[(row * a.S + sm_slot[i]) * 128 + d], sm_w[i], o0);
  store_elem(a.out, row * 128 + d, a.out_dtype, (o0 + o1) * invL);
}

// per-warp rings of half-group stages, then per-warp scratch
static_assert(kStageBytes % 128 == 0, "stage alignment");
size_t mma_smem() { return (size_t)kCW * kBuffers * kStageBytes + (size_t)kCW * kScratchBytes; }

}  // namespace

bool mma_path_ok(const Layout& L, int Hq) {
  const Side& K = L.side[0];
  const Side& V = L.side[1];
  const int G = Hq / L.Hkv;
  return L.D == 128 && L.g == 128 && K.scheme == KVQ_ASYM && K.bits == 4 &&
         K.axis == KVQ_AXIS_CHANNEL && V.scheme == KVQ_ASYM && V.bits == 2 &&
         V.axis == KVQ_AXIS_TOKEN && L.rope == 0 && G >= 2 && G <= 8;
}

// Partition of the fast path: fills the plan's slot count and grid.
void plan_mma(const Layout& L, int64_t t_quant, int t_res, int max_ctas, DecodePlan& p) {
  const int64_t heads = (int64_t)L.B * L.Hkv;
  const int ngv = (int)((t_quant + 127) / 128);
  const int nraw = L.n_sink + t_res;
  const int rw = nraw > 0 ? std::min(kRawPieces, nraw) : 0;
  const int uph = ngv + rw;
  const int64_t N = heads * uph;
  int64_t cap = device_sm_count();
  if (max_ctas > 0) cap = std::min<int64_t>(cap, max_ctas);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cap, N));
  int span = 1;
  for (int64_t h = 0; h < heads; ++h) {
    const int c0 = cta_of_unit(h * uph, N, grid), c1 = cta_of_unit(h * uph + uph - 1, N, grid);
    span = std::max(span, c1 - c0 + 1);
  }
  p.S = span * kCW * 2;
  p.grid_ctas = grid;
  p.raw_slot = -1;
  p.raw_pieces = rw;
  p.n_packed_splits = ngv;
  p.split_groups = 1;
}

cudaError_t launch_decode_mma(const Layout& L, const DecodePlan& p, const void* q, int q_dtype, int Hq,
                              int64_t t_quant, int t_res, float scale, float* ws_m, float* ws_l,
                              float* ws_o, int32_t* d_status, cudaStream_t s) {
  MmaArgs a;
  a.k_codes = reinterpret_cast<const uint8_t*>(L.side[0].codes);
  a.v_codes = reinterpret_cast<const uint8_t*>(L.side[1].codes);
  a.k_scale = reinterpret_cast<const __half*>(L.side[0].scale);
  a.k_zero = reinterpret_cast<const __half*>(L.side[0].zero);
  a.v_scale = reinterpret_cast<const __half*>(L.side[1].scale);
  a.v_zero = reinterpret_cast<const __half*>(L.side[1].zero);
  a.k_slab_bytes = L.side[0].code_slab_bytes;
  a.v_slab_bytes = L.side[1].code_slab_bytes;
  a.C = L.C;
  a.ng = L.ng;
  a.B = L.B;
  a.Hkv = L.Hkv;
  a.Hq = Hq;
  a.G = Hq / L.Hkv;
  a.t_quant = t_quant;
  a.t_res = t_res;
  a.n_sink = L.n_sink;
  a.res_cap = L.res_cap;
  a.src_dtype = L.src_dtype;
  a.sink_k = L.sink[0];
  a.sink_v = L.sink[1];
  a.res_k = L.res[0];
  a.res_v = L.res[1];
  a.q = q;
  a.q_dtype = q_dtype;
  a.qscale = scale * kLog2e;
  a.ngv = p.n_packed_splits;
  a.rw = p.raw_pieces;
  a.uph = a.ngv + a.rw;
  a.N = (int64_t)L.B * L.Hkv * a.uph;
  a.grid = p.grid_ctas;
  a.S = p.S;
  a.ws_m = ws_m;
  a.ws_l = ws_l;
  a.ws_o = ws_o;
  a.status = d_status;
  const size_t smem = mma_smem();
  auto kern = a.G <= 4 ? decode_mma_kernel<true> : decode_mma_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<a.grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine_mma(const Layout& L, const DecodePlan& p, int Hq, const float* ws_m,
                               const float* ws_l, const float* ws_o, void* out, int out_dtype,
                               cudaStream_t s) {
  CombArgsMma c;
  c.Hkv = L.Hkv;
  c.Hq = Hq;
  c.G = Hq / L.Hkv;
  c.rw = p.raw_pieces;
  c.uph = p.n_packed_splits + c.rw;
  c.grid = p.grid_ctas;
  c.S = p.S;
  c.N = (int64_t)L.B * L.Hkv * c.uph;
  c.m = ws_m;
  c.l = ws_l;
  c.o = ws_o;
  c.out = out;
  c.out_dtype = out_dtype;
  dim3 grid(Hq, L.B);
  combine_mma_kernel<<<grid, 128, (size_t)p.S * 3 * sizeof(float), s>>>(c);
  return cudaGetLastError();
}

}  // namespace kvq
