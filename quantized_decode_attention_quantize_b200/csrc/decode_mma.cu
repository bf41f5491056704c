// Tensor-core split-KV decode over a packed cache of 4-bit per-channel keys and 2-bit
// per-token values (the K4V2 allocation of [K4V2]; grouping of [KVQ] "Approach"),
// D = 128, token groups of 128, 1 <= G <= 8 query heads per KV head.
//
// Work.  Each KV head is a row of U items: first its raw (sink + residual) tokens in
// items of up to 8 tokens (4 for fp32 sources), each weighted as two positions of
// the row (the second carries no work: a raw item costs about two half groups), then
// its packed tokens in half groups of 64.  The rows of all heads, end to end, are cut
// into one contiguous range of positions per warp, as equal as integers allow; the
// twelve warps of a CTA hold consecutive ranges.  Warp ranges never exceed U
// positions, so a warp touches at most two heads.  A warp keeps one online-softmax state; when its range crosses from one
// head into the next, the state of the first goes straight to that head's partial
// slot 0.  At the end the warps of a CTA merge, per head, the states they hold in
// shared memory, and the CTA writes one partial state per head into slot
// 1 + (CTA - first CTA holding the head).  The combine kernel derives every valid
// slot of a head from the same partition.  No warp ever waits for another warp except
// at the one CTA barrier before the merge.
//
// Memory.  Every warp streams its items through a ring of two stages in shared
// memory with 16-byte cp.async copies (all 32 lanes, coalesced): per half group the
// key codes (4 KiB), value codes (2 KiB), value scale / zero-point (256 B) and, when
// the half opens the group for this warp, the group's key scale / zero-point (512 B);
// per raw item its key and value rows.  The copy of the next item is issued before
// the math on the current one, so every warp keeps one item in flight while it
// computes; every byte of the format is read once.
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
// products.  The probabilities become the B operand of the value product through an
// in-register 8x8 transpose (movmatrix) and the value codes (pair layout) are the A
// operand with channels as M:
//   A[d][t] = c[t][d] 2^-24 f_d,   B[t][h] = fp16(p[t][h] s[t])
//   o[h][d] = 2^24 / f_d (A.B)[d][h] + sum_t p[t][h] z[t].
// Raw tokens are scored in fp32 on CUDA cores and accumulated in fp32 into the same
// accumulator tiles (scaled by the tile's f_d / 2^24).  Online softmax is kept in the
// log2 domain.
//
// Waits.  A warp only waits for its own copies (cp.async.wait_group) and, once, at
// the CTA barrier before the merge, which every warp reaches.
#include <algorithm>
#include <cstring>
#include <cstdint>

#include "kvq_internal.cuh"
#include "wht.cuh"

namespace kvq {

namespace {

constexpr int kCW = 12;                       // warps per CTA (one CTA per SM)
constexpr int kBuffers = 2;                   // per-warp ring of item stages
constexpr int kThreads = kCW * 32;
// a half-group stage holds 64 tokens: key codes, value codes, value scale / zero-point,
// and (when the half opens the group for the warp) the group's key scale / zero-point
constexpr int kHalfK = 64 * 64, kHalfV = 32 * 64, kHalfVM = 2 * 64 * 2, kHalfKM = 2 * 128 * 2;
constexpr int kStageBytes = kHalfK + kHalfV + kHalfVM + kHalfKM;
constexpr int kRawBytes = 2048;               // raw item: key rows, then value rows at +kRawBytes
// per warp: hi and lo B fragments (4 KiB); with MixKVQ keys the slot products [GM][kAv]
// (rows padded to kAv floats so that the lanes of a fragment read spread over the banks) and,
// for G <= 4, the queries [4][128] in the last 2 KiB
constexpr int kScratchBytes = 2 * 32 * 16 * 4 + 512;
constexpr int kAv = 132;
constexpr int kRecordFloats = 8 * 130;        // merge record: o[G][128], m[G], l[G]
constexpr float kLog2e = 1.4426950408889634f;
// MIXED keys (8 raw bf16 / 24 4-bit / 96 2-bit slots per token) in the key region of a
// half stage: raw plane [64][8] bf16, 4-bit plane [64][3] words, 2-bit plane [64][6]
// words, then the group's slot order [128]; slot scale / zero-point [120] each in the
// key-metadata region (zero-points at +256 bytes).
constexpr int kMixRaw = 0, kMixMid = 64 * 16, kMixLo = kMixMid + 64 * 12, kMixOrd = kMixLo + 64 * 24;
static_assert(kMixOrd + 128 <= kHalfK, "mixed key planes fit the key region");
static_assert(2 * kRawBytes <= kStageBytes, "raw item fits a stage");
static_assert(kRecordFloats * 4 <= kBuffers * kStageBytes, "record fits the warp's ring");

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
  int Hkv, Hq, G;
  int64_t t_quant;
  int t_res, n_sink, res_cap, src_dtype;
  const void* sink_k;
  const void* sink_v;
  const void* res_k;
  const void* res_v;
  const uint8_t* k_order;   // MIXED keys: slot -> channel per group
  int64_t k_group_bytes;    // MIXED keys: bytes of one group's three planes
  const void* q;
  int q_dtype;
  float qscale;
  int k_rotate;   // packed keys in the Walsh-Hadamard basis: their queries are rotated
  float rot_scale;
  int nrp;        // raw positions per head (two per raw item)
  int rt;         // raw tokens per raw item
  int U;          // positions per head (nrp + packed halves)
  int64_t I;      // positions in all
  int64_t W;      // warps in all (grid * kCW)
  int S;          // partial slots per query head
  float* ws_m;
  float* ws_l;
  float* ws_o;
  int32_t* status;
  // defer = 1: the kernel before this one on the stream writes packed rows [dep_lo, dep_hi)
  // (an append) and nothing else that this kernel reads; a warp waits for it only before
  // it first copies a group meeting those rows, and every thread waits before it exits.
  int defer;
  int64_t dep_lo, dep_hi;
  // fuse = 1 (contiguous cache, K4 per channel / V2 per token, 16-bit sources): this
  // kernel writes packed rows [dep_lo, dep_lo + app_n) of one group of every head itself,
  // before its decode, in warp-sized units (fused_append); each unit then sets its flag to
  // `epoch`, and a warp waits for a head's 32 flags before it first copies that group.
  int fuse;
  int app_n;
  const void* app_k;
  const void* app_v;
  int64_t app_sb, app_sh, app_st;
  uint32_t* flags;   // [heads][32]
  uint32_t epoch;
  int64_t heads;
};

// ---- partition of the items over the warps (shared with the combine kernel) ------------
// Warp gw holds items [item_start(gw), item_start(gw + 1)).
__host__ __device__ __forceinline__ int64_t item_start(int64_t gw, int64_t I, int64_t W) {
  return gw * I / W;
}
// The warp holding item x.
__host__ __device__ __forceinline__ int64_t warp_of_item(int64_t x, int64_t I, int64_t W) {
  return ((x + 1) * W - 1) / I;
}
// Warps whose range ends inside head h (including empty warps placed there): the
// first is the least gw with item_start(gw + 1) >= h U + 1, the last the greatest gw
// with item_start(gw + 1) <= (h + 1) U.
__host__ __device__ __forceinline__ int64_t first_ending_warp(int64_t h, int64_t U, int64_t I, int64_t W) {
  const int64_t x = h * U + 1;
  return (x * W + I - 1) / I - 1;
}
__host__ __device__ __forceinline__ int64_t last_ending_warp(int64_t h, int64_t U, int64_t I, int64_t W) {
  const int64_t y = (h + 1) * U + 1;
  const int64_t w = (y * W + I - 1) / I - 2;
  return w < W - 1 ? w : W - 1;
}
// Head h's state that a warp carries out of h into h + 1 (slot 0) exists iff the warp
// holding the head's last item runs past it.
__host__ __device__ __forceinline__ bool has_crossing(int64_t h, int64_t U, int64_t I, int64_t W) {
  const int64_t last = (h + 1) * U - 1;
  return item_start(warp_of_item(last, I, W) + 1, I, W) > last + 1;
}
// The valid slots of head h: s_lo (0 with a crossing state, else 1) .. s_hi.
__host__ __device__ __forceinline__ void head_slots(int64_t h, int64_t U, int64_t I, int64_t W, int cw,
                                                    int* s_lo, int* s_hi) {
  const int64_t ca = first_ending_warp(h, U, I, W) / cw, cb = last_ending_warp(h, U, I, W) / cw;
  *s_lo = has_crossing(h, U, I, W) ? 0 : 1;
  *s_hi = 1 + (int)(cb - ca);
}

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
__device__ __forceinline__ void mma16816_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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

// Four consecutive elements at element offset i (i a multiple of 4) of a raw row
// (global or shared memory).
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

// ---- per-warp online-softmax state of the tensor-core path ------------------------------
// Lane (g, j) holds the accumulator tiles O[cm] of the value product: rows g and g + 8
// of tile cm are channels d0 = 16 g + 8 (cm >> 2) + 2 (cm & 3) and d0 + 1 (fields with
// factors f = 1, 16, 1, 16 ... and 4, 64, 4, 64 ...), columns 2j, 2j + 1 are query
// heads; m, l, W are the running max, sum and sum of p * z of heads 2j, 2j + 1 (l and
// W summed over the lanes of a column at the end).  With DUAL (G <= 4) lanes j >= 2
// track heads 2 (j - 2), 2 (j - 2) + 1 with zero tiles and are never written out.
struct MmaState {
  float O[8][4];
  float m[2], l[2], W[2];
};

__device__ __forceinline__ void state_reset(MmaState& st) {
#pragma unroll
  for (int cm = 0; cm < 8; ++cm) st.O[cm][0] = st.O[cm][1] = st.O[cm][2] = st.O[cm][3] = 0.0f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = st.W[0] = st.W[1] = 0.0f;
}

// 2^24 / f of the rows g (lo) and g + 8 (hi) of tile cm, by cm & 1
__device__ __forceinline__ float inv_f_lo(int odd) { return odd ? 1048576.0f : 16777216.0f; }
__device__ __forceinline__ float inv_f_hi(int odd) { return odd ? 262144.0f : 4194304.0f; }

// Write a warp's state as (o[hh][128], m[hh], l[hh]) for hh < G: o of head hh at
// o + hh * os, m and l at m + hh * ms, l + hh * ms.  Reduces l and W over the lanes of
// a column first (the state is not usable afterwards).
template <bool DUAL>
__device__ void state_emit(MmaState& st, int G, float* o, int64_t os, float* m, float* l, int64_t ms) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
#pragma unroll
  for (int s = 4; s < 32; s <<= 1) {
    st.l[0] += __shfl_xor_sync(0xffffffffu, st.l[0], s);
    st.l[1] += __shfl_xor_sync(0xffffffffu, st.l[1], s);
    st.W[0] += __shfl_xor_sync(0xffffffffu, st.W[0], s);
    st.W[1] += __shfl_xor_sync(0xffffffffu, st.W[1], s);
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int hh = 2 * j + e;
    if (hh < G && (!DUAL || j < 2)) {
      float* dst = o + hh * os;
#pragma unroll
      for (int cm = 0; cm < 8; ++cm) {
        const int d0 = 16 * g + 8 * (cm >> 2) + 2 * (cm & 3);
        const float v0 = fmaf(st.O[cm][e], inv_f_lo(cm & 1), st.W[e]);
        const float v1 = fmaf(st.O[cm][2 + e], inv_f_hi(cm & 1), st.W[e]);
        *reinterpret_cast<float2*>(dst + d0) = make_float2(v0, v1);
      }
      if (g == 0) {
        m[hh * ms] = st.m[e];
        l[hh * ms] = st.l[e];
      }
    }
  }
}

// ---- raw tokens (sink + residual) staged in shared memory -------------------------------
// nt <= 8 tokens: key rows at stg, value rows at stg + kRawBytes (source dtype).  Scores
// in fp32 (lane: channels 4 lane .. 4 lane + 3, reduced over the warp), four tokens at
// a time; the probabilities are accumulated into the state's tiles, each lane for its
// own 16 channels 16 g .. 16 g + 15.
template <bool DUAL, int GM, typename Q>
__device__ void raw_item(MmaState& st, const uint8_t* stg, int nt, int dtype, const Q& qv) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const int hc = DUAL ? 2 * (j & 1) : 2 * j;           // heads hc, hc + 1 of this lane
  const float keep = (!DUAL || j < 2) ? 1.0f : 0.0f;   // DUAL mirror lanes accumulate nothing
  const float lkeep = g == 0 ? 1.0f : 0.0f;            // l is summed over the 8 lanes of a column
  const int esz = dtype == KVQ_F32 ? 4 : 2;
  const uint8_t* Kr = stg;
  const uint8_t* Vr = stg + kRawBytes;
#pragma unroll 1
  for (int t = 0; t < nt; t += 4) {
    float sc[4][GM];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float4 k = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t + e < nt) k = load4(Kr + (t + e) * 128 * esz, 4 * lane, dtype);
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        const float4 q = qv.get(hh);
        float part = q.x * k.x;
        part = fmaf(q.y, k.y, part);
        part = fmaf(q.z, k.z, part);
        part = fmaf(q.w, k.w, part);
        sc[e][hh] = part;
      }
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1)
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) sc[e][hh] += __shfl_xor_sync(0xffffffffu, sc[e][hh], s);
    // this lane's two heads
    float s0[4], s1[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float a0 = sc[e][0], a1 = sc[e][1];
#pragma unroll
      for (int hh = 2; hh < GM; hh += 2) {
        if (hc == hh) {
          a0 = sc[e][hh];
          a1 = sc[e][hh + 1];
        }
      }
      s0[e] = t + e < nt ? a0 : -INFINITY;
      s1[e] = t + e < nt ? a1 : -INFINITY;
    }
    const float mn0 = fmaxf(st.m[0], fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s0[2], s0[3])));
    const float mn1 = fmaxf(st.m[1], fmaxf(fmaxf(s1[0], s1[1]), fmaxf(s1[2], s1[3])));
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
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (t + e < nt) {
        const float p0 = ex2(s0[e] - mn0), p1 = ex2(s1[e] - mn1);
        st.l[0] = fmaf(p0, lkeep, st.l[0]);
        st.l[1] = fmaf(p1, lkeep, st.l[1]);
        const float q0 = p0 * keep, q1 = p1 * keep;
        // scaled probabilities of the rows g (lo) and g + 8 (hi), even and odd tiles
        const float a0e = q0 * (1.0f / 16777216.0f), a0o = q0 * (1.0f / 1048576.0f);
        const float b0e = q0 * (1.0f / 4194304.0f), b0o = q0 * (1.0f / 262144.0f);
        const float a1e = q1 * (1.0f / 16777216.0f), a1o = q1 * (1.0f / 1048576.0f);
        const float b1e = q1 * (1.0f / 4194304.0f), b1o = q1 * (1.0f / 262144.0f);
        const uint8_t* vrow = Vr + (t + e) * 128 * esz;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {    // channels 16 g + 4 qd .. + 3
          const float4 v = load4(vrow, 16 * g + 4 * qd, dtype);
          // channels 16g + 4qd + {0,1} -> tile cm = 2 qd (even: rows lo, hi), {2,3} -> cm = 2 qd + 1
          // (cm >> 2 selects the upper 8 channels: qd >= 2)
          const int ce = 2 * qd;   // even tile of this quad
          const int co = ce + 1;
          st.O[ce][0] = fmaf(a0e, v.x, st.O[ce][0]);
          st.O[ce][1] = fmaf(a1e, v.x, st.O[ce][1]);
          st.O[ce][2] = fmaf(b0e, v.y, st.O[ce][2]);
          st.O[ce][3] = fmaf(b1e, v.y, st.O[ce][3]);
          st.O[co][0] = fmaf(a0o, v.z, st.O[co][0]);
          st.O[co][1] = fmaf(a1o, v.z, st.O[co][1]);
          st.O[co][2] = fmaf(b0o, v.w, st.O[co][2]);
          st.O[co][3] = fmaf(b1o, v.w, st.O[co][3]);
        }
      }
    }
  }
}

// The key-product B operand of one group (per lane), its exponent and bias.
// The key-product B operand of a group: k-steps of high (bh) and, without DUAL, low (bl)
// fp16 parts; MIXED adds two k-steps for the 4-bit slots and one bf16 k-step for the raw
// slots (eight 2-bit k-steps, two 4-bit, one raw).
template <bool MIX>
struct KeyOpT {
  uint32_t bh[MIX ? 11 : 8][2], bl[MIX ? 11 : 8][2];
  float mult, bias0, bias1;
};
using KeyOp = KeyOpT<false>;

// The head's pre-scaled queries, channels 4 lane .. 4 lane + 3 of head hh: with DUAL in
// the upper half of the warp's scratch (shared memory), otherwise in registers.
template <bool DUAL, int GM>
struct QVec;
template <int GM>
struct QVec<true, GM> {
  float* s;   // [G][128]
  __device__ __forceinline__ float4 get(int hh) const {
    return *reinterpret_cast<const float4*>(s + hh * 128 + 4 * (threadIdx.x & 31));
  }
  __device__ __forceinline__ void set(int hh, float4 v) {
    *reinterpret_cast<float4*>(s + hh * 128 + 4 * (threadIdx.x & 31)) = v;
  }
};
template <int GM>
struct QVec<false, GM> {
  float v[GM][4];
  __device__ __forceinline__ float4 get(int hh) const { return make_float4(v[hh][0], v[hh][1], v[hh][2], v[hh][3]); }
  __device__ __forceinline__ void set(int hh, float4 x) {
    v[hh][0] = x.x; v[hh][1] = x.y; v[hh][2] = x.z; v[hh][3] = x.w;
  }
};

// Build the key-product B operand of a group from its per-channel scale / zero-point
// (ks, kz in shared memory) and the head's pre-scaled queries.  DUAL: G <= 4, the
// remainder rides in columns 4..7.
//
// Lane l owns channels 4 l + k (k < 4) of every head; channel 4 l + k is row
// 2 ((l & 7) >> 1) + (k >> 1) ... of the fragments of consumer lane 4 hh + (l >> 3): k-step
// kk = 2 ((l & 7) >> 1) + (k >> 1), register k & 1, half l & 1.  The two lanes of a pair
// (l, l ^ 1) fill the two halves of the same four words; one shuffle gives each of them
// two whole words (even lane: k-step kk0 = 2 ((l & 7) >> 1), odd lane: kk0 + 1), stored
// as one 64-bit word pair.
// Scratch word of k-step kk of consumer lane R's fragments: R's four 16-byte quads sit at
// slots 4 R + (q ^ frag_swz(R)) (q = kk / 2), so that both the pair stores of the
// producers and the quad loads of the consumers fall on distinct banks.
__device__ __forceinline__ int frag_swz(int R) { return (R >> 1) & 3; }
__device__ __forceinline__ int frag_word(int R, int kk) {
  return 4 * (4 * R + ((kk >> 1) ^ frag_swz(R))) + 2 * (kk & 1);
}

template <bool DUAL, int GM>
__device__ __forceinline__ void key_operand(const MmaArgs& a, const __half* ks, const __half* kz,
                                            uint32_t* scratch, const QVec<DUAL, GM>& qv, KeyOp& ko) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const int G = a.G;
  const uint2 sv = *reinterpret_cast<const uint2*>(ks + 4 * lane);
  const uint2 zv = *reinterpret_cast<const uint2*>(kz + 4 * lane);
  const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
  const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
  const float2 z01 = __half22float2(*reinterpret_cast<const __half2*>(&zv.x));
  const float2 z23 = __half22float2(*reinterpret_cast<const __half2*>(&zv.y));
  float av[GM][4], dz[GM];
  float amax = 0.0f;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
    if (hh < G) q = qv.get(hh);
    av[hh][0] = q.x * s01.x;
    av[hh][1] = q.y * s01.y;
    av[hh][2] = q.z * s23.x;
    av[hh][3] = q.w * s23.y;
    dz[hh] = fmaf(q.w, z23.y, fmaf(q.z, z23.x, fmaf(q.y, z01.y, q.x * z01.x)));
#pragma unroll
    for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fabsf(av[hh][k]));
  }
  amax = warp_max(amax);
  // one exponent for the group: max |a 2^(24 - e)| < 2^15
  int ex = 0;
  if (amax > 0.0f) ex = (int)((__float_as_uint(amax) >> 23) & 0xff) - 127 + 10;
  ex = max(-100, min(127, ex));
  ko.mult = pow2(ex);
  const float sc = __uint_as_float((uint32_t)max(1, min(254, 127 + 24 - ex)) << 23);
  const float sc16 = sc * 0.0625f;   // odd k: the code sits 4 bits up (factor 16)
  const bool odd = lane & 1;
  const int kk0 = 2 * ((lane & 7) >> 1) + (odd ? 1 : 0);
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    if (hh < G) {
      const float x0 = av[hh][0] * sc, x1 = av[hh][1] * sc16, x2 = av[hh][2] * sc, x3 = av[hh][3] * sc16;
      const __half2 h01 = __floats2half2_rn(x0, x1), h23 = __floats2half2_rn(x2, x3);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      const __half2 l01 = __floats2half2_rn(x0 - f01.x, x1 - f01.y);
      const __half2 l23 = __floats2half2_rn(x2 - f23.x, x3 - f23.y);
      const uint32_t H01 = *reinterpret_cast<const uint32_t*>(&h01), H23 = *reinterpret_cast<const uint32_t*>(&h23);
      const uint32_t L01 = *reinterpret_cast<const uint32_t*>(&l01), L23 = *reinterpret_cast<const uint32_t*>(&l23);
      // even lane keeps k = 0, 1 and sends k = 2, 3; odd lane the reverse
      const uint32_t rh = __shfl_xor_sync(0xffffffffu, odd ? H01 : H23, 1);
      const uint32_t rl = __shfl_xor_sync(0xffffffffu, odd ? L01 : L23, 1);
      const uint32_t mh = odd ? H23 : H01, ml = odd ? L23 : L01;
      // word (kk, reg r) = (even lane's half, odd lane's half) of k = 2 (kk - kk0e) + r
      const uint2 wh = odd ? make_uint2(__byte_perm(rh, mh, 0x5410), __byte_perm(rh, mh, 0x7632))
                           : make_uint2(__byte_perm(mh, rh, 0x5410), __byte_perm(mh, rh, 0x7632));
      const uint2 wl = odd ? make_uint2(__byte_perm(rl, ml, 0x5410), __byte_perm(rl, ml, 0x7632))
                           : make_uint2(__byte_perm(ml, rl, 0x5410), __byte_perm(ml, rl, 0x7632));
      const int dl = 4 * hh + (lane >> 3);   // consumer lane
      *reinterpret_cast<uint2*>(scratch + frag_word(dl, kk0)) = wh;
      if (DUAL) *reinterpret_cast<uint2*>(scratch + frag_word(dl + 16, kk0)) = wl;   // column hh + 4
      else *reinterpret_cast<uint2*>(scratch + 32 * 16 + frag_word(dl, kk0)) = wl;
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
      const uint4 x = src[u ^ frag_swz(lane)];
      ko.bh[2 * u][0] = x.x; ko.bh[2 * u][1] = x.y; ko.bh[2 * u + 1][0] = x.z; ko.bh[2 * u + 1][1] = x.w;
    }
    if (!DUAL) {
      const uint4* srl = reinterpret_cast<const uint4*>(scratch) + 32 * 4 + lane * 4;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 x = srl[u ^ frag_swz(lane)];
        ko.bl[2 * u][0] = x.x; ko.bl[2 * u][1] = x.y; ko.bl[2 * u + 1][0] = x.z; ko.bl[2 * u + 1][1] = x.w;
      }
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) ko.bh[kk][0] = ko.bh[kk][1] = ko.bl[kk][0] = ko.bl[kk][1] = 0u;
  }
  __syncwarp();
}

// Per-head sums dz[hh] over the warp, delivered as the biases of the lane's columns
// (heads 2j, 2j + 1; with DUAL heads 2 (j & 1), 2 (j & 1) + 1).
template <bool DUAL, int GM>
__device__ __forceinline__ void head_sums(const float (&dz)[GM], float* b0, float* b1) {
  const int lane = threadIdx.x & 31, j = lane & 3;
  const int h0 = DUAL ? 2 * (j & 1) : 2 * j, h1 = h0 + 1;
  const bool u4 = lane & 16, u3 = lane & 8, u2 = lane & 4;
  if constexpr (GM == 4) {
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
    *b0 = __shfl_sync(0xffffffffu, v3, 16 * ((h0 >> 1) & 1) + 8 * (h0 & 1));
    *b1 = __shfl_sync(0xffffffffu, v3, 16 * ((h1 >> 1) & 1) + 8 * (h1 & 1));
  } else {
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
    *b0 = __shfl_sync(0xffffffffu, v4, ((h0 >> 2) & 1) * 16 + ((h0 >> 1) & 1) * 8 + (h0 & 1) * 4);
    *b1 = __shfl_sync(0xffffffffu, v4, ((h1 >> 2) & 1) * 16 + ((h1 >> 1) & 1) * 8 + (h1 & 1) * 4);
  }
}

__device__ __forceinline__ void split_half2(float x0, float x1, uint32_t* hi, uint32_t* lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(x0 - f.x, x1 - f.y);
  *hi = *reinterpret_cast<const uint32_t*>(&h);
  *lo = *reinterpret_cast<const uint32_t*>(&l);
}
__device__ __forceinline__ void split_bf162(float x0, float x1, uint32_t* hi, uint32_t* lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 f = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - f.x, x1 - f.y);
  *hi = *reinterpret_cast<const uint32_t*>(&h);
  *lo = *reinterpret_cast<const uint32_t*>(&l);
}

// MIXED keys ([MIX] Figure 3 tiers: 8 raw, 24 4-bit, 96 2-bit slots in salience order).
// The score of token t is sum_s B[s] A[t][s] over slots: A holds the codes as fp16
// subnormals in place (2-bit field f of a word: factor 4^f; 4-bit nibble: 1 or 16) and
// the raw slots as bf16; B[s] = q[order[s]] s_s 2^(24 - e) / factor for coded slots and
// q[order[s]] 2^-e for raw ones; sum_s q[order[s]] z_s is the bias.  Lane (g, j) builds its
// own fragments (head g, or with DUAL the low part of head g - 4 for g >= 4) from the
// slot products that the warp first writes to its scratch in slot order.
//
// k-steps of lane j: 2-bit slots, k-step 4 sg + qq: word w = 4 sg + j of the 2-bit
// plane (none when w >= 6), registers 2 qq and 2 qq + 1 of the word, register r being
// (r < 4 ? x : odd_bytes_down(x)) & (0x00030003 << 2 (r & 3)), whose low / high halves
// hold slots (r < 4 ? 0 : 4) + (r & 3) and that + 8 of the word; 4-bit slots, k-step
// 8 + qq: word j of the 4-bit plane (none for j = 3), registers 2 qq, 2 qq + 1, register r
// being (r < 2 ? x : odd(x)) & (r even ? 0x000F000F : 0x00F000F0) with slots r, r + 4;
// raw slots, k-step 10 (bf16): word j of the raw plane = slots 2 j, 2 j + 1, the upper
// eight k-columns empty.
template <bool DUAL, int GM>
__device__ __forceinline__ void key_operand_mixed(const MmaArgs& a, const uint8_t* stage, uint32_t* scratch,
                                                  const QVec<DUAL, GM>& qv, KeyOpT<true>& ko) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const int G = a.G;
  const uint8_t* ord = stage + kMixOrd;
  const __half* ks = reinterpret_cast<const __half*>(stage + kHalfK + kHalfV + kHalfVM);
  const __half* kz = ks + 128;
  float* av = reinterpret_cast<float*>(scratch);   // [GM][kAv] slot products, slot order
  int ch[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) ch[i] = ord[4 * lane + i] & 127;   // a channel of the head
  float qs[GM][4];
  if constexpr (DUAL) {
#pragma unroll
    for (int hh = 0; hh < GM; ++hh)
#pragma unroll
      for (int i = 0; i < 4; ++i) qs[hh][i] = qv.s[hh * 128 + ch[i]];
  } else {   // the queries live in registers by channel: go through the scratch once
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) *reinterpret_cast<float4*>(av + hh * kAv + 4 * lane) = qv.get(hh);
    __syncwarp();
#pragma unroll
    for (int hh = 0; hh < GM; ++hh)
#pragma unroll
      for (int i = 0; i < 4; ++i) qs[hh][i] = av[hh * kAv + ch[i]];
    __syncwarp();
  }
  float sv[4], zv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int sl = 4 * lane + i;
    sv[i] = sl >= 8 ? __half2float(ks[sl - 8]) : 0.0f;
    zv[i] = sl >= 8 ? __half2float(kz[sl - 8]) : 0.0f;
  }
  float dz[GM];
  float amax = 0.0f;
#pragma unroll
  for (int hh = 0; hh < GM; ++hh) {
    dz[hh] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x = qs[hh][i] * sv[i];
      dz[hh] = fmaf(qs[hh][i], zv[i], dz[hh]);
      amax = fmaxf(amax, fabsf(x));
      if (lane >= 2) qs[hh][i] = x;   // lanes 0, 1 hold the raw slots 0..7: keep q
    }
  }
  amax = warp_max(amax);
  int ex = 0;
  if (amax > 0.0f) ex = (int)((__float_as_uint(amax) >> 23) & 0xff) - 127 + 10;
  ex = max(-100, min(127, ex));
  ko.mult = pow2(ex);
  // coded slots: 2^(24 - ex) (the codes enter as c 2^-24); raw slots: 2^-ex, so that after
  // the accumulator is scaled by 2^ex both give q . k (powers of two: exact)
  const float sc = lane >= 2 ? __uint_as_float((uint32_t)max(1, min(254, 127 + 24 - ex)) << 23)
                             : __uint_as_float((uint32_t)max(1, min(254, 127 - ex)) << 23);
#pragma unroll
  for (int hh = 0; hh < GM; ++hh)
    *reinterpret_cast<float4*>(av + hh * kAv + 4 * lane) =
        make_float4(qs[hh][0] * sc, qs[hh][1] * sc, qs[hh][2] * sc, qs[hh][3] * sc);
  head_sums<DUAL, GM>(dz, &ko.bias0, &ko.bias1);
  __syncwarp();
  const int hd = DUAL ? (g & 3) : g;
  const bool live = hd < G;
  const bool low_lane = DUAL && g >= 4;   // columns 4..7 carry the low parts
  const float* ah = av + (live ? hd : 0) * kAv;
  auto put = [&](int k, float v0, float v1, float v2, float v3) {
    uint32_t h0, l0, h1, l1;
    split_half2(v0, v1, &h0, &l0);
    split_half2(v2, v3, &h1, &l1);
    if (DUAL) {
      ko.bh[k][0] = low_lane ? l0 : h0;
      ko.bh[k][1] = low_lane ? l1 : h1;
    } else {
      ko.bh[k][0] = h0; ko.bh[k][1] = h1;
      ko.bl[k][0] = l0; ko.bl[k][1] = l1;
    }
  };
  // 2-bit slots 32 + 16 w + p
#pragma unroll
  for (int sg = 0; sg < 2; ++sg) {
    const int w = 4 * sg + j;
    const bool ok = live && w < 6;
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 2 * qq + e, f = r & 3;
        const int p = (r < 4 ? 0 : 4) + f;
        const float inv = f == 0 ? 1.0f : f == 1 ? 0.25f : f == 2 ? 0.0625f : 0.015625f;
        v[2 * e] = ok ? ah[32 + 16 * w + p] * inv : 0.0f;
        v[2 * e + 1] = ok ? ah[32 + 16 * w + p + 8] * inv : 0.0f;
      }
      put(4 * sg + qq, v[0], v[1], v[2], v[3]);
    }
  }
  // 4-bit slots 8 + 8 w + p
  {
    const bool ok = live && j < 3;
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 2 * qq + e;
        const float inv = (r & 1) ? 0.0625f : 1.0f;
        v[2 * e] = ok ? ah[8 + 8 * j + r] * inv : 0.0f;
        v[2 * e + 1] = ok ? ah[8 + 8 * j + r + 4] * inv : 0.0f;
      }
      put(8 + qq, v[0], v[1], v[2], v[3]);
    }
  }
  // raw slots 2 j, 2 j + 1 (bf16)
  {
    uint32_t h0, l0;
    split_bf162(live ? ah[2 * j] : 0.0f, live ? ah[2 * j + 1] : 0.0f, &h0, &l0);
    if (DUAL) {
      ko.bh[10][0] = low_lane ? l0 : h0;
      ko.bh[10][1] = 0u;
    } else {
      ko.bh[10][0] = h0; ko.bh[10][1] = 0u;
      ko.bl[10][0] = l0; ko.bl[10][1] = 0u;
    }
  }
  __syncwarp();
}

// 64 tokens (one half of a group) held in a ring stage: key codes [64][16] words,
// value codes [32 pairs][16] words, value scale / zero-point [64] each.
template <bool DUAL, bool MIX>
__device__ __forceinline__ void mma_half(MmaState& st, const uint8_t* stage, const KeyOpT<MIX>& ko,
                                         int tvalid) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const uint32_t* kc = reinterpret_cast<const uint32_t*>(stage);
  const uint32_t* vc = reinterpret_cast<const uint32_t*>(stage + kHalfK);
  const __half* vs = reinterpret_cast<const __half*>(stage + kHalfK + kHalfV);
  const __half* vz = vs + 64;

  // ---- scores of the 64 tokens (4 tiles of 16) ----
  // all four tiles' code words first, then the k-steps tile by tile so that consecutive
  // products go to different accumulators
  float S[4][4];
  if constexpr (MIX) {
    // per tile: the 2-bit words 4 sg + j, the 4-bit word j and the raw word j of rows
    // g and g + 8 (k-step layout in key_operand_mixed)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      S[mt][0] = S[mt][1] = S[mt][2] = S[mt][3] = 0.0f;
      const int r0 = 16 * mt + g, r1 = r0 + 8;
#pragma unroll
      for (int sg = 0; sg < 2; ++sg) {
        const int w = 4 * sg + j;
        uint32_t x0 = 0u, x1 = 0u;
        if (w < 6) {
          x0 = *reinterpret_cast<const uint32_t*>(stage + kMixLo + r0 * 24 + 4 * w);
          x1 = *reinterpret_cast<const uint32_t*>(stage + kMixLo + r1 * 24 + 4 * w);
        }
        const uint32_t y0 = odd_bytes_down(x0), y1 = odd_bytes_down(x1);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const uint32_t s0 = qq < 2 ? x0 : y0, s1 = qq < 2 ? x1 : y1;
          const uint32_t ma = 0x00030003u << (2 * ((2 * qq) & 3)), mb = 0x00030003u << (2 * ((2 * qq + 1) & 3));
          mma16816(S[mt], s0 & ma, s1 & ma, s0 & mb, s1 & mb, ko.bh[4 * sg + qq][0], ko.bh[4 * sg + qq][1]);
          if (!DUAL)
            mma16816(S[mt], s0 & ma, s1 & ma, s0 & mb, s1 & mb, ko.bl[4 * sg + qq][0], ko.bl[4 * sg + qq][1]);
        }
      }
      {
        uint32_t x0 = 0u, x1 = 0u;
        if (j < 3) {
          x0 = *reinterpret_cast<const uint32_t*>(stage + kMixMid + r0 * 12 + 4 * j);
          x1 = *reinterpret_cast<const uint32_t*>(stage + kMixMid + r1 * 12 + 4 * j);
        }
        const uint32_t y0 = odd_bytes_down(x0), y1 = odd_bytes_down(x1);
        mma16816(S[mt], x0 & 0x000F000Fu, x1 & 0x000F000Fu, x0 & 0x00F000F0u, x1 & 0x00F000F0u, ko.bh[8][0], ko.bh[8][1]);
        mma16816(S[mt], y0 & 0x000F000Fu, y1 & 0x000F000Fu, y0 & 0x00F000F0u, y1 & 0x00F000F0u, ko.bh[9][0], ko.bh[9][1]);
        if (!DUAL) {
          mma16816(S[mt], x0 & 0x000F000Fu, x1 & 0x000F000Fu, x0 & 0x00F000F0u, x1 & 0x00F000F0u, ko.bl[8][0], ko.bl[8][1]);
          mma16816(S[mt], y0 & 0x000F000Fu, y1 & 0x000F000Fu, y0 & 0x00F000F0u, y1 & 0x00F000F0u, ko.bl[9][0], ko.bl[9][1]);
        }
      }
      {
        const uint32_t x0 = *reinterpret_cast<const uint32_t*>(stage + kMixRaw + r0 * 16 + 4 * j);
        const uint32_t x1 = *reinterpret_cast<const uint32_t*>(stage + kMixRaw + r1 * 16 + 4 * j);
        mma16816_bf16(S[mt], x0, x1, 0u, 0u, ko.bh[10][0], ko.bh[10][1]);
        if (!DUAL) mma16816_bf16(S[mt], x0, x1, 0u, 0u, ko.bl[10][0], ko.bl[10][1]);
      }
    }
  } else {
  uint4 wlo[4], whi[4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    S[mt][0] = S[mt][1] = S[mt][2] = S[mt][3] = 0.0f;
    wlo[mt] = *reinterpret_cast<const uint4*>(kc + (16 * mt + g) * 16 + 4 * j);
    whi[mt] = *reinterpret_cast<const uint4*>(kc + (16 * mt + g + 8) * 16 + 4 * j);
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const uint32_t x0 = w == 0 ? wlo[mt].x : w == 1 ? wlo[mt].y : w == 2 ? wlo[mt].z : wlo[mt].w;
      const uint32_t x1 = w == 0 ? whi[mt].x : w == 1 ? whi[mt].y : w == 2 ? whi[mt].z : whi[mt].w;
      const uint32_t p0 = odd_bytes_down(x0), p1 = odd_bytes_down(x1);
      // k-step 2w: nibbles 0 (f 1) and 1 (f 16) of each half; k-step 2w + 1: nibbles 2, 3
      mma16816(S[mt], x0 & 0x000F000Fu, x1 & 0x000F000Fu, x0 & 0x00F000F0u, x1 & 0x00F000F0u,
               ko.bh[2 * w][0], ko.bh[2 * w][1]);
      mma16816(S[mt], p0 & 0x000F000Fu, p1 & 0x000F000Fu, p0 & 0x00F000F0u, p1 & 0x00F000F0u,
               ko.bh[2 * w + 1][0], ko.bh[2 * w + 1][1]);
      if (!DUAL) {
        mma16816(S[mt], x0 & 0x000F000Fu, x1 & 0x000F000Fu, x0 & 0x00F000F0u, x1 & 0x00F000F0u,
                 ko.bl[2 * w][0], ko.bl[2 * w][1]);
        mma16816(S[mt], p0 & 0x000F000Fu, p1 & 0x000F000Fu, p0 & 0x00F000F0u, p1 & 0x00F000F0u,
                 ko.bl[2 * w + 1][0], ko.bl[2 * w + 1][1]);
      }
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
    // P = p s_t as an fp16 high part and an fp16 remainder (about 22 bits): two products
    // with the same value codes into the same accumulators
    uint32_t h0, l0, h1, l1;
    split_half2(p00 * sk0, p01 * sk0, &h0, &l0);
    split_half2(p10 * sk1, p11 * sk1, &h1, &l1);
    const uint32_t pb0 = movtrans(h0), pb1 = movtrans(h1);
    const uint32_t pr0 = movtrans(l0), pr1 = movtrans(l1);
    const uint2 va = *reinterpret_cast<const uint2*>(vc + (8 * mt + j) * 16 + 2 * g);
    const uint2 vb = *reinterpret_cast<const uint2*>(vc + (8 * mt + j + 4) * 16 + 2 * g);
    const uint32_t ya = odd_bytes_down(va.x), yb = odd_bytes_down(vb.x);
    const uint32_t za = odd_bytes_down(va.y), zb = odd_bytes_down(vb.y);
    // fields at bits 0, 2, 4, 6 of each half: factors 1, 4, 16, 64
    const uint32_t A[8][4] = {
        {va.x & 0x00030003u, va.x & 0x000C000Cu, vb.x & 0x00030003u, vb.x & 0x000C000Cu},
        {va.x & 0x00300030u, va.x & 0x00C000C0u, vb.x & 0x00300030u, vb.x & 0x00C000C0u},
        {ya & 0x00030003u, ya & 0x000C000Cu, yb & 0x00030003u, yb & 0x000C000Cu},
        {ya & 0x00300030u, ya & 0x00C000C0u, yb & 0x00300030u, yb & 0x00C000C0u},
        {va.y & 0x00030003u, va.y & 0x000C000Cu, vb.y & 0x00030003u, vb.y & 0x000C000Cu},
        {va.y & 0x00300030u, va.y & 0x00C000C0u, vb.y & 0x00300030u, vb.y & 0x00C000C0u},
        {za & 0x00030003u, za & 0x000C000Cu, zb & 0x00030003u, zb & 0x000C000Cu},
        {za & 0x00300030u, za & 0x00C000C0u, zb & 0x00300030u, zb & 0x00C000C0u}};
#pragma unroll
    for (int cm = 0; cm < 8; ++cm) {
      mma16816(st.O[cm], A[cm][0], A[cm][1], A[cm][2], A[cm][3], pb0, pb1);
      mma16816(st.O[cm], A[cm][0], A[cm][1], A[cm][2], A[cm][3], pr0, pr1);
    }
  }
}

// ---- per-warp staging with cp.async ----------------------------------------------------
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copy one half group (64 rows) of head `head`, group `gi` into a stage buffer, with the
// group's key scale / zero-point when `with_key`: every lane moves 16-byte chunks.
template <bool MIX>
__device__ __forceinline__ void load_half(const MmaArgs& a, uint8_t* buf, int64_t head, int gi, int hf,
                                          bool with_key) {
  const int lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)gi * 128 + 64 * hf;
  const uint8_t* vc = a.v_codes + head * a.v_slab_bytes + t0 * 32;
  if constexpr (MIX) {
    // the group's planes: raw [128][8] 16-bit (2048 B), 4-bit [128][3] words (1536 B),
    // 2-bit [128][6] words; this half's rows of each
    const uint8_t* gb = a.k_codes + head * a.k_slab_bytes + (int64_t)gi * a.k_group_bytes;
#pragma unroll
    for (int e = 0; e < 2; ++e) cp_async16(buf + kMixRaw + 16 * (lane + 32 * e), gb + 1024 * hf + 16 * (lane + 32 * e));
    for (int c = lane; c < 48; c += 32) cp_async16(buf + kMixMid + 16 * c, gb + 2048 + 768 * hf + 16 * c);
#pragma unroll
    for (int e = 0; e < 3; ++e)
      cp_async16(buf + kMixLo + 16 * (lane + 32 * e), gb + 3584 + 1536 * hf + 16 * (lane + 32 * e));
  } else {
    const uint8_t* kc = a.k_codes + head * a.k_slab_bytes + t0 * 64;
#pragma unroll
    for (int e = 0; e < kHalfK / 512; ++e) cp_async16(buf + 16 * (lane + 32 * e), kc + 16 * (lane + 32 * e));
  }
#pragma unroll
  for (int e = 0; e < kHalfV / 512; ++e)
    cp_async16(buf + kHalfK + 16 * (lane + 32 * e), vc + 16 * (lane + 32 * e));
  if (lane < 16) {   // value scale (lanes 0..7) and zero-point (lanes 8..15), 64 rows each
    const __half* src = (lane < 8 ? a.v_scale : a.v_zero) + head * a.C + t0 + 8 * (lane & 7);
    cp_async16(buf + kHalfK + kHalfV + 16 * lane, src);
  }
  if (with_key) {
    if constexpr (MIX) {   // slot order into the key region; 120 scales (lanes 0..14), zero-points (16..30)
      const int64_t grp = head * a.ng + gi;
      if (lane < 8) cp_async16(buf + kMixOrd + 16 * lane, a.k_order + grp * 128 + 16 * lane);
      if ((lane & 15) < 15) {
        const __half* src = (lane < 16 ? a.k_scale : a.k_zero) + grp * 120 + 8 * (lane & 15);
        cp_async16(buf + kHalfK + kHalfV + kHalfVM + 16 * lane, src);
      }
    } else {   // the group's key scale (lanes 0..15) and zero-point (16..31)
      const __half* src = (lane < 16 ? a.k_scale : a.k_zero) + (head * a.ng + gi) * 128 + 8 * (lane & 15);
      cp_async16(buf + kHalfK + kHalfV + kHalfVM + 16 * lane, src);
    }
  }
}

// Copy raw item r of head `head` (its key rows, then its value rows at +kRawBytes).
__device__ __forceinline__ void load_raw(const MmaArgs& a, uint8_t* buf, int64_t head, int r) {
  const int lane = threadIdx.x & 31;
  const int lg = a.src_dtype == KVQ_F32 ? 5 : 4;   // log2 of the 16-byte chunks per row
  const int rowb = 16 << lg;                       // bytes per row
  const int nraw = a.n_sink + a.t_res;
  const int t0 = r * a.rt, nt = min(a.rt, nraw - t0);
  const int per = nt << lg;
  for (int c = lane; c < 2 * per; c += 32) {
    const int kv = c >= per, rem = c - (kv ? per : 0);
    const int t = rem >> lg, ch = rem & ((1 << lg) - 1);
    const int tok = t0 + t;
    const bool sink = tok < a.n_sink;
    const void* arr = kv ? (sink ? a.sink_v : a.res_v) : (sink ? a.sink_k : a.res_k);
    const int64_t row = head * (sink ? a.n_sink : a.res_cap) + (sink ? tok : tok - a.n_sink);
    cp_async16(buf + kv * kRawBytes + t * rowb + ch * 16,
               reinterpret_cast<const uint8_t*>(arr) + row * rowb + ch * 16);
  }
}

// ---- final combine of one query-head row over its valid slots -------------------------
// Lane owns channels 4 lane .. 4 lane + 3.  The slots are read eight at a time, all loads
// of a batch issued before any of them is used.
__device__ __forceinline__ void combine_row(const float* m, const float* l, const float* o, int S,
                                            int64_t row, int s_lo, int s_hi, int lane, void* out,
                                            int out_dtype, float* lse) {
  const float* mrow = m + row * S;
  const float* lrow = l + row * S;
  float M = -INFINITY, L = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = s_lo; s0 <= s_hi; s0 += 8) {
    float mv[8], lv[8];
    float4 ov[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int s = s0 + u;
      mv[u] = -INFINITY;
      lv[u] = 0.0f;
      ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s <= s_hi) {
        mv[u] = __ldcg(mrow + s);
        lv[u] = __ldcg(lrow + s);
        ov[u] = __ldcg(reinterpret_cast<const float4*>(o + (row * S + s) * 128) + lane);
      }
    }
    float Mc = M;
#pragma unroll
    for (int u = 0; u < 8; ++u) Mc = fmaxf(Mc, mv[u]);
    if (M != -INFINITY && Mc != M) {   // earlier batches were weighted against M
      const float c = ex2(M - Mc);
      L *= c;
      acc.x *= c; acc.y *= c; acc.z *= c; acc.w *= c;
    }
    M = Mc;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (mv[u] == -INFINITY) continue;
      const float f = ex2(mv[u] - M);
      L = fmaf(f, lv[u], L);
      acc.x = fmaf(f, ov[u].x, acc.x);
      acc.y = fmaf(f, ov[u].y, acc.y);
      acc.z = fmaf(f, ov[u].z, acc.z);
      acc.w = fmaf(f, ov[u].w, acc.w);
    }
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;   // L = 0: a row with no tokens
  const int64_t i = row * 128 + 4 * lane;
  // natural log of the row's softmax denominator (scores were kept as log2 units)
  if (lse && lane == 0) lse[row] = (M + __log2f(L)) * 0.6931471805599453f;
  if (out_dtype == KVQ_F32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + i) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    store_elem(out, i + 0, out_dtype, acc.x * inv);
    store_elem(out, i + 1, out_dtype, acc.y * inv);
    store_elem(out, i + 2, out_dtype, acc.z * inv);
    store_elem(out, i + 3, out_dtype, acc.w * inv);
  }
}

// Four query channels 4 lane .. 4 lane + 3 taken into the Walsh-Hadamard basis of the keys.
__device__ __forceinline__ float4 rotate_q(float4 x, int lane, float c) {
  float v[4] = {x.x, x.y, x.z, x.w};
  wht128_quad_unscaled(v, lane);
  return make_float4(v[0] * c, v[1] * c, v[2] * c, v[3] * c);
}

// ---- the kernel --------------------------------------------------------------------------
template <bool DUAL, bool ROT, bool MIX>
__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(MmaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int GM = DUAL ? 4 : 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kCW + warp;
  const int64_t i0 = item_start(gw, a.I, a.W), i1 = item_start(gw + 1, a.I, a.W);
  const int U = a.U;
  uint8_t* ring = smem + (size_t)warp * (kBuffers * kStageBytes);
  uint32_t* my_scratch = reinterpret_cast<uint32_t*>(smem + (size_t)kCW * kBuffers * kStageBytes) +
                         warp * (kScratchBytes / 4);
  int* last_head = reinterpret_cast<int*>(smem + (size_t)kCW * (kBuffers * kStageBytes + kScratchBytes));
  const int nraw = a.n_sink + a.t_res;

  // load cursor: one work item ahead of the compute cursor (odd raw positions carry none)
  int64_t lhead = i0 / U, li = i0;
  int lr = (int)(i0 - lhead * U);
  int issued = 0;
  auto advance_load = [&]() {
    ++li;
    if (++lr == U) {
      lr = 0;
      ++lhead;
    }
  };
  auto issue_next = [&]() {
    while (li < i1 && lr < a.nrp && (lr & 1)) advance_load();
    if (li < i1) {
      uint8_t* buf = ring + (issued % kBuffers) * kStageBytes;
      if (lr < a.nrp) {
        load_raw(a, buf, lhead, lr >> 1);
      } else {
        const int p = lr - a.nrp;
        load_half<MIX>(a, buf, lhead, p >> 1, p & 1, (p & 1) == 0 || li == i0);
      }
      advance_load();
    }
    cp_async_commit();   // an empty group keeps the group count uniform
    ++issued;
  };
#pragma unroll 1
  for (int e = 0; e < kBuffers - 1; ++e) issue_next();

  MmaState st;
  state_reset(st);
  QVec<DUAL, GM> qv;
  if constexpr (DUAL) qv.s = reinterpret_cast<float*>(my_scratch) + (kScratchBytes / 4 - 512);   // last 2 KiB
  KeyOpT<MIX> ko;
  int64_t head = i0 / U, cur_head = -1;
  int r = (int)(i0 - head * U);
  bool qbad = false, qrot = false;
  int consumed = 0;
#pragma unroll 1
  for (int64_t i = i0; i < i1; ++i) {
    if (head != cur_head) {
      if (cur_head >= 0) {   // the range crosses into the next head: slot 0 of this one
        const int64_t row0 = cur_head * a.G;
        state_emit<DUAL>(st, a.G, a.ws_o + row0 * a.S * 128, (int64_t)a.S * 128, a.ws_m + row0 * a.S,
                         a.ws_l + row0 * a.S, a.S);
        state_reset(st);
      }
      cur_head = head;
      if constexpr (ROT) qrot = r >= a.nrp;
      // this head's queries, pre-scaled, for channels 4 lane .. 4 lane + 3 (as given for
      // raw tokens; in the Walsh-Hadamard basis for the packed keys of a rotating format)
#pragma unroll
      for (int hh = 0; hh < GM; ++hh) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (hh < a.G) x = load4(a.q, (head * a.G + hh) * 128 + 4 * lane, a.q_dtype);
        qbad |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
        if constexpr (ROT) {
          if (qrot) x = rotate_q(x, lane, a.rot_scale);
        }
        qv.set(hh, make_float4(x.x * a.qscale, x.y * a.qscale, x.z * a.qscale, x.w * a.qscale));
      }
    }
    if (r < a.nrp && (r & 1)) {   // second position of a raw item: no work
      if (++r == U) {
        r = 0;
        ++head;
      }
      continue;
    }
    if constexpr (ROT) {   // a head's raw items come first: at most one switch per head
      if (r >= a.nrp && !qrot) {
        qrot = true;
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) {
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (hh < a.G) x = load4(a.q, (head * a.G + hh) * 128 + 4 * lane, a.q_dtype);
          x = rotate_q(x, lane, a.rot_scale);
          qv.set(hh, make_float4(x.x * a.qscale, x.y * a.qscale, x.z * a.qscale, x.w * a.qscale));
        }
      }
    }
    // the next item goes into the buffer consumed last time, then this one is waited
    // for: the warp's own copy of the next item overlaps its math on this one
    issue_next();
    cp_async_wait<kBuffers - 1>();
    __syncwarp();
    const uint8_t* stg = ring + (consumed % kBuffers) * kStageBytes;
    if (r < a.nrp) {
      raw_item<DUAL, GM>(st, stg, min(a.rt, nraw - (r >> 1) * a.rt), a.src_dtype, qv);
    } else {
      const int p = r - a.nrp, gi = p >> 1, hf = p & 1;
      if (hf == 0 || i == i0) {
        const __half* ks = reinterpret_cast<const __half*>(stg + kHalfK + kHalfV + kHalfVM);
        if constexpr (MIX) key_operand_mixed<DUAL, GM>(a, stg, my_scratch, qv, ko);
        else key_operand<DUAL, GM>(a, ks, ks + 128, my_scratch, qv, ko);
      }
      const int tvalid = (int)min((int64_t)64, a.t_quant - (int64_t)gi * 128 - 64 * hf);
      mma_half<DUAL, MIX>(st, stg, ko, tvalid);
    }
    __syncwarp();
    ++consumed;
    if (++r == U) {
      r = 0;
      ++head;
    }
  }
  cp_async_wait<0>();
  __syncwarp();
  if (__any_sync(0xffffffffu, qbad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);

  // ---- merge of the warps' last heads inside the CTA ----
  // Every warp, empty ones included, belongs to the head of item i1 - 1; its record
  // (its own ring, now idle) holds its state of that head (empty: m = -inf, l = 0, o = 0).
  const int lh = i1 > 0 ? (int)((i1 - 1) / U) : -1;
  float* rec = reinterpret_cast<float*>(ring);
  if (lh >= 0) state_emit<DUAL>(st, a.G, rec, 128, rec + 8 * 128, rec + 8 * 128 + 8, 1);
  if (lane == 0) last_head[warp] = lh;
  __syncthreads();
  const int G = a.G;
  int w0 = 0;
#pragma unroll 1
  while (w0 < kCW) {
    const int h = last_head[w0];
    int w1 = w0;
    while (w1 + 1 < kCW && last_head[w1 + 1] == h) ++w1;
    if (h >= 0) {
      const int64_t ca = first_ending_warp(h, U, a.I, a.W) / kCW;
      const int slot = 1 + (int)((int64_t)blockIdx.x - ca);
#pragma unroll 1
      for (int idx = threadIdx.x; idx < G * 128; idx += kThreads) {
        const int hh = idx >> 7, d = idx & 127;
        float M = -INFINITY;
        for (int w = w0; w <= w1; ++w) {
          const float* rw = reinterpret_cast<const float*>(smem + (size_t)w * (kBuffers * kStageBytes));
          M = fmaxf(M, rw[8 * 128 + hh]);
        }
        float o = 0.0f, l = 0.0f;
        for (int w = w0; w <= w1; ++w) {
          const float* rw = reinterpret_cast<const float*>(smem + (size_t)w * (kBuffers * kStageBytes));
          const float mw = rw[8 * 128 + hh];
          if (mw != -INFINITY) {
            const float f = ex2(mw - M);
            o = fmaf(f, rw[hh * 128 + d], o);
            l = fmaf(f, rw[8 * 128 + 8 + hh], l);
          }
        }
        const int64_t sl = ((int64_t)h * G + hh) * a.S + slot;
        a.ws_o[sl * 128 + d] = o;
        if (d == 0) {
          a.ws_m[sl] = M;
          a.ws_l[sl] = l;
        }
      }
    }
    w0 = w1 + 1;
  }
}

// ==== K4/V2 keys with G <= 4: the lean kernel ============================================
// Same partition, math encoding and partial-state contract as decode_mma_kernel, arranged
// so that every lane owns one query head:
//  - Each half group (64 tokens: key and value codes, value scale / zero-point and, for
//    the half that opens a group, the group's key scale / zero-point) arrives in a stage
//    of the warp's two-stage ring by 1-D bulk copies (the TMA engine; this GPU's memory
//    only, no multicast) on one mbarrier per stage.  Lane 0 issues the copies of the
//    next half (predicated, no divergent branch) before the warp waits for the current
//    one; waits are bounded.
//  - The key product's N columns are (head 0 high, head 0 remainder, head 1 high, ...):
//    lane (g, j) ends with the high part and the remainder of head j for tokens g and
//    g + 8 of the tile and adds them in place; the online softmax then runs on two
//    values per lane and tile, with m, l and W scalars per lane.
//  - The value product's B operand carries the probabilities P = p s_t of a tile as an
//    fp16 high part and an fp16 remainder (about 22 bits): column 2h holds head h's high
//    parts and column 2h + 1 its remainders.  Packed per lane as (high, remainder) of
//    token g (and of token g + 8), one 8x8 transpose (movmatrix) each puts exactly the
//    B fragment in place: lane (2h, j') receives the high parts of tokens 2j', 2j' + 1
//    of head h, lane (2h + 1, j') their remainders.
//  - The key-product B operand of a group is built with every (head, channel) product
//    formed once: lane L forms head L / 8, channels 16 (L % 8) .. + 15, and the fragments
//    reach their lanes through the warp's scratch.  Each head has its own exponent.
//  - A warp's range covers at most two heads; each is a run of raw items (staged with
//    cp.async in the same stages, the next one in flight) and a run of halves, walked
//    with 32-bit counters.
constexpr int kQBytes = 4 * 128 * 4;            // pre-scaled queries of up to four heads
constexpr int kBScratch = 32 * 16 * 4;          // key-operand fragments on their way to lanes
constexpr int kKMetaBytes = 2 * 128 * 4;        // the group's key scale / zero-point as fp32
constexpr int kLeanWarpBytes = kBuffers * kStageBytes + kQBytes + kBScratch + kKMetaBytes;
constexpr int kWaitRounds = 1000;               // try_wait rounds (each up to 1 ms) before giving up
static_assert(kRecordFloats * 4 <= kBuffers * kStageBytes, "merge record fits the ring");
static_assert(2 * kRawBytes <= kStageBytes, "raw item fits a stage");
static_assert(64 * 8 <= kBScratch, "value scale / zero-point pairs fit the scratch");

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// On lane 0 only (pred != 0): arrive on `bar` expecting `bytes` of transfers.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes, uint32_t pred) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %2, 0;\n @p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n}" ::"r"(
          smem_u32(bar)),
      "r"(bytes), "r"(pred)
      : "memory");
}
// On lane 0 only: 1-D bulk copy global -> this CTA's shared memory completing `bytes` on
// `bar` (addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint32_t pred) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " @p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n}" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "r"(pred)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `parity`; false when kWaitRounds rounds pass first.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  bool ok = false;
  for (int it = 0; it < kWaitRounds && !ok; ++it) ok = mbar_try_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void mma16816_n(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movtrans_n(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Copies of half p of slab `head` (key codes, value codes, value scale / zero-point
// and, when `with_key`, the key scale / zero-point of its group) into a stage, on lane 0.
__device__ __forceinline__ void issue_half(const MmaArgs& a, uint8_t* buf, uint64_t* bar, int64_t head, int p,
                                           bool with_key) {
  const uint32_t l0 = (threadIdx.x & 31) == 0;
  const int64_t t0 = 64 * (int64_t)p;
  mbar_expect_tx(bar, kHalfK + kHalfV + kHalfVM + (with_key ? kHalfKM : 0), l0);
  bulk_g2s(buf, a.k_codes + head * a.k_slab_bytes + t0 * 64, kHalfK, bar, l0);
  bulk_g2s(buf + kHalfK, a.v_codes + head * a.v_slab_bytes + t0 * 32, kHalfV, bar, l0);
  bulk_g2s(buf + kHalfK + kHalfV, a.v_scale + head * a.C + t0, 128, bar, l0);
  bulk_g2s(buf + kHalfK + kHalfV + 128, a.v_zero + head * a.C + t0, 128, bar, l0);
  if (with_key) {
    const int64_t grp = head * a.ng + (p >> 1);
    bulk_g2s(buf + kHalfK + kHalfV + kHalfVM, a.k_scale + grp * 128, 256, bar, l0);
    bulk_g2s(buf + kHalfK + kHalfV + kHalfVM + 256, a.k_zero + grp * 128, 256, bar, l0);
  }
}

// ---- the fused append: one group of every head, in warp-sized units -------------------
// Unit j of a head (kFusedUnits of them, flags at head * 32 + j): j < 16 takes key channels
// 8 j .. 8 j + 7 of the group's rows (lane l: rows l, l + 32, l + 64, l + 96; the channel
// statistics meet over the warp), j >= 16 value rows 16 (j - 16) .. + 15 (two lanes per row,
// 64 channels each).  Same rules, arithmetic and
// layouts as the append kernels: asym_params for the metadata, pack8 for the codes, the
// pair layout for the 2-bit value rows ([KVQ] "Approach"; [K4V2]).
constexpr int kFusedUnits = 32;
__device__ void fused_key_unit(const MmaArgs& a, int64_t head, int j) {
  const int lane = threadIdx.x & 31;
  const int64_t b = head / a.Hkv, h = head % a.Hkv;
  const int c0 = 8 * j;
  float x[4][8], mn[8], mx[8];
  float fin = 0.0f;   // x * 0 is 0 for finite x and NaN otherwise
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    mn[c] = INFINITY;
    mx[c] = -INFINITY;
  }
  const int64_t base = b * a.app_sb + h * a.app_sh + c0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = lane + 32 * k;
#pragma unroll
    for (int c = 0; c < 8; ++c) x[k][c] = 0.0f;
    if (r < a.app_n) {
      load8(a.app_k, base + r * a.app_st, a.src_dtype, x[k]);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        fin = fmaf(x[k][c], 0.0f, fin);
        mn[c] = fminf(mn[c], x[k][c]);
        mx[c] = fmaxf(mx[c], x[k][c]);
      }
    }
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      mn[c] = fminf(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], o));
      mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], o));
    }
  // lane c < 8 forms channel c's scale / zero-point and stores them; all lanes get all eight
  float m0 = mn[0], m1 = mx[0];
#pragma unroll
  for (int c = 1; c < 8; ++c)
    if (lane == c) {
      m0 = mn[c];
      m1 = mx[c];
    }
  __half s, z;
  const bool good = asym_params(m0, m1, 4, &s, &z);
  if (lane < 8) {
    const int64_t mi = (head * a.ng + a.dep_lo / 128) * 128 + c0 + lane;
    const_cast<__half*>(a.k_scale)[mi] = s;
    const_cast<__half*>(a.k_zero)[mi] = z;
  }
  const float sf = __half2float(s), zf = __half2float(z), rf = __frcp_rn(sf);
  float s8[8], z8[8], r8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    s8[c] = __shfl_sync(0xffffffffu, sf, c);
    z8[c] = __shfl_sync(0xffffffffu, zf, c);
    r8[c] = __shfl_sync(0xffffffffu, rf, c);
  }
  uint8_t* codes = const_cast<uint8_t*>(a.k_codes) + head * a.k_slab_bytes + a.dep_lo * 64 + c0 / 2;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = lane + 32 * k;
    if (r < a.app_n) *reinterpret_cast<uint32_t*>(codes + r * 64) = pack8(x[k], s8, r8, z8, 4).x;
  }
  if (__any_sync(0xffffffffu, !(fin == 0.0f)) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);
  if (__any_sync(0xffffffffu, lane < 8 && !good) && lane == 0) flag(a.status, KVQ_DEV_RANGE);
}

__device__ void fused_value_unit(const MmaArgs& a, int64_t head, int j) {
  const int lane = threadIdx.x & 31;
  const int64_t b = head / a.Hkv, h = head % a.Hkv;
  const int r = 8 * j + (lane >> 2), part = lane & 3, c0 = 32 * part;   // row in the group
  const bool ok = r < a.app_n;
  float x[4][8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int c = 0; c < 8; ++c) x[k][c] = 0.0f;
    if (ok) load8(a.app_v, b * a.app_sb + h * a.app_sh + r * a.app_st + c0 + 8 * k, a.src_dtype, x[k]);
  }
  float mn = INFINITY, mx = -INFINITY, fin = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      fin = fmaf(x[k][c], 0.0f, fin);
      mn = fminf(mn, x[k][c]);
      mx = fmaxf(mx, x[k][c]);
    }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __half sh, zh;
  const bool good = asym_params(mn, mx, 2, &sh, &zh);
  const int64_t t = a.dep_lo + r;
  if (ok && part == 0) {
    const_cast<__half*>(a.v_scale)[head * a.C + t] = sh;
    const_cast<__half*>(a.v_zero)[head * a.C + t] = zh;
  }
  const float sv = __half2float(sh), zv = __half2float(zh), rv = __frcp_rn(sv);
  float s8[8], z8[8], r8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    s8[c] = sv;
    z8[c] = zv;
    r8[c] = rv;
  }
  const bool even = (t & 1) == 0;
  const bool lone = even && r + 1 >= a.app_n;
  uint32_t* dst = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.v_codes) + head * a.v_slab_bytes) +
                  (t / 2) * 16 + part * 4;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t hw = pack8(x[k], s8, r8, z8, 2).x & 0xffffu;
    const uint32_t other = __shfl_xor_sync(0xffffffffu, hw, 4);
    if (ok && even) dst[k] = hw | ((lone ? 0u : other) << 16);
  }
  if (__any_sync(0xffffffffu, ok && !(fin == 0.0f)) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);
  if (__any_sync(0xffffffffu, ok && !good) && lane == 0) flag(a.status, KVQ_DEV_RANGE);
}

// Warp gw's units (gw, gw + W, ...), each announced by its flag once its rows are visible
// to the other SMs' bulk copies.
__device__ void fused_append(const MmaArgs& a, int64_t gw) {
  const int64_t units = a.heads * kFusedUnits;
#pragma unroll 1
  for (int64_t u = gw; u < units; u += a.W) {
    const int64_t head = u / kFusedUnits;
    const int j = (int)(u % kFusedUnits);
    if (j < 16) fused_key_unit(a, head, j);
    else fused_value_unit(a, head, j - 16);
    __threadfence();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
    if ((threadIdx.x & 31) == 0) atomicExch(a.flags + head * 32 + j, a.epoch);
  }
}

// Waits (bounded) until the kFusedUnits units of `head` are done; a wait that runs out sets
// KVQ_DEV_TIMEOUT and goes on.
constexpr int kFlagRounds = 1 << 22;   // polls, each followed by a sleep of about 0.25 us
__device__ __noinline__ void fused_wait(const uint32_t* flags, uint32_t epoch, int32_t* status, int64_t head) {
  const uint32_t* f = flags + head * 32 + (threadIdx.x & 31);
#pragma unroll 1
  for (int it = 0; it < kFlagRounds; ++it) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (__all_sync(0xffffffffu, v == epoch || (threadIdx.x & 31) >= kFusedUnits)) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      return;
    }
    __nanosleep(256);
  }
  if ((threadIdx.x & 31) == 0) flag(status, KVQ_DEV_TIMEOUT);
}

__device__ __forceinline__ void cp_async16_lean(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// Raw item r of raw head `head` (nraw raw tokens: its key rows, then its value rows at
// +kRawBytes) into a stage with cp.async, every lane moving 16-byte chunks; committed as
// one group.
__device__ __forceinline__ void stage_raw(const MmaArgs& a, uint8_t* buf, int64_t head, int r, int nraw) {
  const int lane = threadIdx.x & 31;
  const int lg = a.src_dtype == KVQ_F32 ? 5 : 4;   // log2 of the 16-byte chunks per row
  const int rowb = 16 << lg;
  const int t0 = r * a.rt, nt = min(a.rt, nraw - t0);
  const int per = nt << lg;
  for (int c = lane; c < 2 * per; c += 32) {
    const int kv = c >= per, rem = c - (kv ? per : 0);
    const int t = rem >> lg, ch = rem & ((1 << lg) - 1);
    const int tok = t0 + t;
    const bool sink = tok < a.n_sink;
    const void* arr = kv ? (sink ? a.sink_v : a.res_v) : (sink ? a.sink_k : a.res_k);
    const int64_t row = head * (sink ? a.n_sink : a.res_cap) + (sink ? tok : tok - a.n_sink);
    cp_async16_lean(buf + kv * kRawBytes + t * rowb + ch * 16, reinterpret_cast<const uint8_t*>(arr) + row * rowb + ch * 16);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Online-softmax state of lane (g, j) for head j: O[cm][0] + O[cm][1] and O[cm][2] +
// O[cm][3] are channels d0 = 16 g + 8 (cm >> 2) + 2 (cm & 3) and d0 + 1 (the high-part
// and remainder columns of the value product); m, l, W the running max, sum and sum of
// p z (l and W summed over the lanes g of the column at the end).
struct LeanState {
  float O[8][4];
  float m, l, W;
};

__device__ __forceinline__ void lean_reset(LeanState& st) {
#pragma unroll
  for (int cm = 0; cm < 8; ++cm) st.O[cm][0] = st.O[cm][1] = st.O[cm][2] = st.O[cm][3] = 0.0f;
  st.m = -INFINITY;
  st.l = st.W = 0.0f;
}

__device__ __forceinline__ void lean_rescale(LeanState& st, float mnew) {
  if (__any_sync(0xffffffffu, mnew != st.m)) {
    const float c = ex2(st.m - mnew);
#pragma unroll
    for (int cm = 0; cm < 8; ++cm) {
      st.O[cm][0] *= c;
      st.O[cm][1] *= c;
      st.O[cm][2] *= c;
      st.O[cm][3] *= c;
    }
    st.l *= c;
    st.W *= c;
    st.m = mnew;
  }
}

// Writes the state as (o[hh][128], m[hh], l[hh]) for hh < G (o of head hh at o + hh os,
// m and l at m + hh ms, l + hh ms); the state is not usable afterwards.
__device__ void lean_emit(LeanState& st, int G, float* o, int64_t os, float* m, float* l, int64_t ms) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
#pragma unroll
  for (int s = 4; s < 32; s <<= 1) {
    st.l += __shfl_xor_sync(0xffffffffu, st.l, s);
    st.W += __shfl_xor_sync(0xffffffffu, st.W, s);
  }
  if (j < G) {
    float* dst = o + j * os;
#pragma unroll
    for (int cm = 0; cm < 8; ++cm) {
      const int d0 = 16 * g + 8 * (cm >> 2) + 2 * (cm & 3);
      *reinterpret_cast<float2*>(dst + d0) =
          make_float2(fmaf(st.O[cm][0] + st.O[cm][1], inv_f_lo(cm & 1), st.W),
                      fmaf(st.O[cm][2] + st.O[cm][3], inv_f_hi(cm & 1), st.W));
    }
    if (g == 0) {
      m[j * ms] = st.m;
      l[j * ms] = st.l;
    }
  }
}

// Sixteen consecutive elements (element offset c0, a multiple of 8) of a raw row in
// shared memory, as fp32.
__device__ __forceinline__ void load16(const uint8_t* row, int c0, int dtype, float* v) {
  if (dtype == KVQ_F32) {
    const float4* p = reinterpret_cast<const float4*>(row) + c0 / 4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 x = p[u];
      v[4 * u] = x.x; v[4 * u + 1] = x.y; v[4 * u + 2] = x.z; v[4 * u + 3] = x.w;
    }
    return;
  }
  const uint4* p = reinterpret_cast<const uint4*>(row) + c0 / 8;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const uint4 x = p[u];
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (dtype == KVQ_F16) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        v[8 * u + 2 * k] = f.x;
        v[8 * u + 2 * k + 1] = f.y;
      } else {
        v[8 * u + 2 * k] = __uint_as_float(w[k] << 16);
        v[8 * u + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
      }
    }
  }
}

// Shared-memory rows of 128 channels (queries, key scale / zero-point) keep channel quad
// c / 4 = 4 b + u (16-channel block b, quad u inside it) at float4 slot 8 u + b: the eight
// lanes of a load phase that read quad u of blocks 0..7 then read one contiguous 128 bytes.
__device__ __forceinline__ int qslot(int quad) { return 8 * (quad & 3) + (quad >> 2); }

// Raw tokens (sink + residual, nt <= 8) staged at stg (key rows, value rows at
// +kRawBytes): fp32 scores on CUDA cores, lane (g, j) over channels 16 g .. 16 g + 15 of
// head j, summed over the lanes g; the probabilities go into the state's tiles scaled
// by each row's field factor f / 2^24.
__device__ void lean_raw(LeanState& st, const uint8_t* stg, int nt, int dtype, const float* qs) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  const float lkeep = g == 0 ? 1.0f : 0.0f;   // l is summed over the eight lanes of a column
  const int rowb = dtype == KVQ_F32 ? 512 : 256;
  float q[16];
  {
    const float4* p = reinterpret_cast<const float4*>(qs + j * 128);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 x = p[8 * u + g];
      q[4 * u] = x.x; q[4 * u + 1] = x.y; q[4 * u + 2] = x.z; q[4 * u + 3] = x.w;
    }
  }
  float sc[8];
  float mx = -INFINITY;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    sc[t] = -INFINITY;
    if (t < nt) {
      float k[16];
      load16(stg + t * rowb, 16 * g, dtype, k);
      float part = q[0] * k[0];
#pragma unroll
      for (int c = 1; c < 16; ++c) part = fmaf(q[c], k[c], part);
      part += __shfl_xor_sync(0xffffffffu, part, 4);
      part += __shfl_xor_sync(0xffffffffu, part, 8);
      part += __shfl_xor_sync(0xffffffffu, part, 16);
      sc[t] = part;
      mx = fmaxf(mx, part);
    }
  }
  lean_rescale(st, fmaxf(st.m, mx));
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    if (t < nt) {
      const float p = ex2(sc[t] - st.m);
      st.l = fmaf(p, lkeep, st.l);
      const float pe = p * (1.0f / 16777216.0f), po = p * (1.0f / 1048576.0f);
      const float qe = p * (1.0f / 4194304.0f), qo = p * (1.0f / 262144.0f);
      float v[16];
      load16(stg + kRawBytes + t * rowb, 16 * g, dtype, v);
#pragma unroll
      for (int cm = 0; cm < 8; ++cm) {
        const int i0 = 8 * (cm >> 2) + 2 * (cm & 3);
        st.O[cm][0] = fmaf((cm & 1) ? po : pe, v[i0], st.O[cm][0]);
        st.O[cm][2] = fmaf((cm & 1) ? qo : qe, v[i0 + 1], st.O[cm][2]);
      }
    }
  }
}

// The key-product B operand of a group: b[2 kk + r] is register r of k-step kk for
// column g' = 2 h + part of lane (g', j') (part 0: the fp16 high part, 1: the remainder
// of q~[h][c] s[c] 2^(24 - e_h) / f_c over the channels 32 j' .. 32 j' + 31 in the order
// of the key unpack); mult = 2^e_j and bias = sum_c q~[j][c] z[c] of the lane's head j.
struct LeanKey {
  uint32_t b[16];
  float mult, bias;
};

// ks, kz: the group's key scale / zero-point as fp32 [128] in shared memory, qs the queries
// [4][128]; channel quads at qslot().
__device__ __forceinline__ void lean_key_operand(const float* ks, const float* kz, const float* qs,
                                                 uint32_t* scr, LeanKey& ko) {
  const int lane = threadIdx.x & 31;
  const int hL = lane >> 3, cb = lane & 7;   // head, 16-channel block formed by this lane
  float a[16];
  float amax = 0.0f, dz = 0.0f;
  {
    const float4* q4 = reinterpret_cast<const float4*>(qs + hL * 128);
    const float4* s4 = reinterpret_cast<const float4*>(ks);
    const float4* z4 = reinterpret_cast<const float4*>(kz);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 qv = q4[8 * u + cb], sv = s4[8 * u + cb], zv = z4[8 * u + cb];
      a[4 * u] = qv.x * sv.x;
      a[4 * u + 1] = qv.y * sv.y;
      a[4 * u + 2] = qv.z * sv.z;
      a[4 * u + 3] = qv.w * sv.w;
      dz = fmaf(qv.x, zv.x, dz);
      dz = fmaf(qv.y, zv.y, dz);
      dz = fmaf(qv.z, zv.z, dz);
      dz = fmaf(qv.w, zv.w, dz);
#pragma unroll
      for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fabsf(a[4 * u + k]));
    }
  }
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
    dz += __shfl_xor_sync(0xffffffffu, dz, s);
  }
  // the head's exponent: max |a 2^(24 - e)| < 2^15
  int ex = 0;
  if (amax > 0.0f) ex = (int)((__float_as_uint(amax) >> 23) & 0xff) - 127 + 10;
  ex = max(-100, min(127, ex));
  const float mult = pow2(ex);
  const float sc = __uint_as_float((uint32_t)max(1, min(254, 127 + 24 - ex)) << 23);
  const float sc16 = sc * 0.0625f;   // channels at the odd nibble of a byte (factor 16)
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {   // channel pairs (p, p + 4) of word 2 cb + u
      // odd p: the A element is a whole byte, c_p-1 + 16 c_p, weighted a_p sc / 16; even p:
      // the A element c_p alone, weighted a_p sc - a_p+1 sc / 16, so that each channel
      // still enters with its own weight
      float y0, y1;
      if (p & 1) {
        y0 = a[8 * u + p] * sc16;
        y1 = a[8 * u + p + 4] * sc16;
      } else {
        y0 = fmaf(-a[8 * u + p + 1], sc16, a[8 * u + p] * sc);
        y1 = fmaf(-a[8 * u + p + 5], sc16, a[8 * u + p + 4] * sc);
      }
      split_half2(y0, y1, &hw[p], &lw[p]);
    }
    // register quad w of reader lane R sits at uint4 slot 32 w + (R ^ 4 (w / 2)): a read
    // phase of eight lanes is one contiguous 128 bytes, and the two stores of a lane pair
    // (w, w + 2) land in different bank groups
    const int W = 2 * cb + u, jd = W >> 2, w = W & 3, sw = 4 * (w >> 1);
    *reinterpret_cast<uint4*>(scr + (32 * w + ((4 * (2 * hL) + jd) ^ sw)) * 4) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(scr + (32 * w + ((4 * (2 * hL + 1) + jd) ^ sw)) * 4) =
        make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint4 x = *reinterpret_cast<const uint4*>(scr + (32 * u + (lane ^ (4 * (u >> 1)))) * 4);
    ko.b[4 * u] = x.x; ko.b[4 * u + 1] = x.y; ko.b[4 * u + 2] = x.z; ko.b[4 * u + 3] = x.w;
  }
  ko.mult = __shfl_sync(0xffffffffu, mult, 8 * (lane & 3));
  ko.bias = __shfl_sync(0xffffffffu, dz, 8 * (lane & 3));
  __syncwarp();
}

// The scores of the half's 64 tokens (4 tiles of 16) from its key codes [64][16] words in
// shared memory: lane (g, j) takes words 4j .. 4j + 3 of rows 16 mt + g and 16 mt + g + 8.
__device__ __forceinline__ void lean_scores(float (&S)[4][4], const uint4* kc4, const LeanKey& ko) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
  uint4 kw[8];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    S[mt][0] = S[mt][1] = S[mt][2] = S[mt][3] = 0.0f;
    kw[2 * mt] = kc4[(16 * mt + g) * 4 + j];
    kw[2 * mt + 1] = kc4[(16 * mt + g + 8) * 4 + j];
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const uint4 lo = kw[2 * mt], hi = kw[2 * mt + 1];
      const uint32_t x0 = w == 0 ? lo.x : w == 1 ? lo.y : w == 2 ? lo.z : lo.w;
      const uint32_t x1 = w == 0 ? hi.x : w == 1 ? hi.y : w == 2 ? hi.z : hi.w;
      const uint32_t p0 = odd_bytes_down(x0), p1 = odd_bytes_down(x1);
      // low nibble alone, then the whole byte (low + 16 high; the byte of p as it stands)
      mma16816_n(S[mt], x0 & 0x000F000Fu, x1 & 0x000F000Fu, x0 & 0x00FF00FFu, x1 & 0x00FF00FFu, ko.b[4 * w],
                 ko.b[4 * w + 1]);
      mma16816_n(S[mt], p0 & 0x000F000Fu, p1 & 0x000F000Fu, p0, p1, ko.b[4 * w + 2], ko.b[4 * w + 3]);
    }
  }
}

// Online softmax of the half on head j (tokens g and g + 8 of every tile): l and W
// updated, the probability operands of the half's value product returned in pb (tile mt:
// pb[mt][0] = the (high, remainder) columns of tokens 2j', 2j' + 1 and pb[mt][1] of tokens
// 2j' + 8, 2j' + 9, as the B fragment of m16n8k16).  sz: the half's value scale /
// zero-point as fp32 pairs in shared memory.  The value product of any earlier half must
// already be in st.O (a new maximum rescales it).
__device__ __forceinline__ void lean_softmax(LeanState& st, const float (&S)[4][4], const LeanKey& ko,
                                             int tvalid, const float2* sz, uint32_t (&pb)[4][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2;
  float x[4][2];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    x[mt][0] = S[mt][0] + S[mt][1];
    x[mt][1] = S[mt][2] + S[mt][3];
  }
  if (tvalid < 64) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      if (16 * mt + g >= tvalid) x[mt][0] = -INFINITY;
      if (16 * mt + g + 8 >= tvalid) x[mt][1] = -INFINITY;
    }
  }
  float lm = fmaxf(fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1])),
                   fmaxf(fmaxf(x[2][0], x[2][1]), fmaxf(x[3][0], x[3][1])));
  lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 4));
  lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 8));
  lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 16));
  lean_rescale(st, fmaxf(st.m, fmaf(lm, ko.mult, ko.bias)));
  const float bm = ko.bias - st.m;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const float p0 = ex2(fmaf(x[mt][0], ko.mult, bm)), p1 = ex2(fmaf(x[mt][1], ko.mult, bm));
    const float2 a0 = sz[16 * mt + g], a1 = sz[16 * mt + g + 8];
    st.l += p0 + p1;
    st.W = fmaf(p0, a0.y, fmaf(p1, a1.y, st.W));
    uint32_t ph, pl;   // high parts and remainders of (P of token g, P of token g + 8)
    split_half2(p0 * a0.x, p1 * a1.x, &ph, &pl);
    pb[mt][0] = movtrans_n(__byte_perm(ph, pl, 0x5410));   // (high, remainder) of token g
    pb[mt][1] = movtrans_n(__byte_perm(ph, pl, 0x7632));   // of token g + 8
  }
}

// The value words of a half in this lane's fragment registers: vw[2 mt] = pair g of pair
// row 8 mt + j, vw[2 mt + 1] = pair g of pair row 8 mt + j + 4 (vc2: [32 pair rows][8]).
__device__ __forceinline__ void lean_value_words(uint2 (&vw)[8], const uint2* vc2) {
  const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    vw[2 * mt] = vc2[(8 * mt + j) * 8 + g];
    vw[2 * mt + 1] = vc2[(8 * mt + j + 4) * 8 + g];
  }
}

// The value product of a half: st.O += V^T P from its value words and probability operands.
__device__ __forceinline__ void lean_pv(LeanState& st, const uint2 (&vw)[8], const uint32_t (&pb)[4][2]) {
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const uint2 va = vw[2 * mt], vb = vw[2 * mt + 1];
    const uint32_t b0 = pb[mt][0], b1 = pb[mt][1];
    const uint32_t ya = odd_bytes_down(va.x), yb = odd_bytes_down(vb.x);
    const uint32_t za = odd_bytes_down(va.y), zb = odd_bytes_down(vb.y);
    // fields at bits 0, 2, 4, 6 of each half: factors 1, 4, 16, 64
    mma16816_n(st.O[0], va.x & 0x00030003u, va.x & 0x000C000Cu, vb.x & 0x00030003u, vb.x & 0x000C000Cu, b0, b1);
    mma16816_n(st.O[1], va.x & 0x00300030u, va.x & 0x00C000C0u, vb.x & 0x00300030u, vb.x & 0x00C000C0u, b0, b1);
    mma16816_n(st.O[2], ya & 0x00030003u, ya & 0x000C000Cu, yb & 0x00030003u, yb & 0x000C000Cu, b0, b1);
    mma16816_n(st.O[3], ya & 0x00300030u, ya & 0x00C000C0u, yb & 0x00300030u, yb & 0x00C000C0u, b0, b1);
    mma16816_n(st.O[4], va.y & 0x00030003u, va.y & 0x000C000Cu, vb.y & 0x00030003u, vb.y & 0x000C000Cu, b0, b1);
    mma16816_n(st.O[5], va.y & 0x00300030u, va.y & 0x00C000C0u, vb.y & 0x00300030u, vb.y & 0x00C000C0u, b0, b1);
    mma16816_n(st.O[6], za & 0x00030003u, za & 0x000C000Cu, zb & 0x00030003u, zb & 0x000C000Cu, b0, b1);
    mma16816_n(st.O[7], za & 0x00300030u, za & 0x00C000C0u, zb & 0x00300030u, zb & 0x00C000C0u, b0, b1);
  }
}

// The value scale / zero-point pairs of tokens 2 lane, 2 lane + 1 as fp32 into szbuf
// (tokens past tvalid get (0, 0)).
__device__ __forceinline__ void lean_sz(uint32_t s2, uint32_t z2, int tvalid, float* szbuf) {
  const int lane = threadIdx.x & 31;
  float2 s = __half22float2(*reinterpret_cast<const __half2*>(&s2));
  float2 z = __half22float2(*reinterpret_cast<const __half2*>(&z2));
  if (2 * lane >= tvalid) s.x = z.x = 0.0f;
  if (2 * lane + 1 >= tvalid) s.y = z.y = 0.0f;
  reinterpret_cast<float4*>(szbuf)[lane] = make_float4(s.x, z.x, s.y, z.y);
}

// The head's queries, pre-scaled, channels 4 lane .. 4 lane + 3 of heads 0..3 (rows
// qhead * G + hh of q; as given for raw tokens, in the Walsh-Hadamard basis for the
// packed keys of a rotating format) into qs [4][128].
template <bool ROT>
__device__ __forceinline__ void lean_load_queries(const MmaArgs& a, int64_t qhead, bool rotated, float* qs,
                                                  bool& qbad) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (hh < a.G) x = load4(a.q, (qhead * a.G + hh) * 128 + 4 * lane, a.q_dtype);
    qbad |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
    if constexpr (ROT) {
      if (rotated) x = rotate_q(x, lane, a.rot_scale);
    }
    reinterpret_cast<float4*>(qs + hh * 128)[qslot(lane)] =
        make_float4(x.x * a.qscale, x.y * a.qscale, x.z * a.qscale, x.w * a.qscale);
  }
  __syncwarp();
}

// The warp's shared-memory areas and ring counters.
struct LeanWarp {
  uint8_t* ring;      // kBuffers stages
  float* qs;          // [4][128] queries, channel quads at qslot()
  uint32_t* scr;      // key-operand fragments / value scale and zero-point pairs
  float* kmeta;       // the group's key scale / zero-point as fp32, [2][128]
  uint64_t* bars;     // one mbarrier per stage
  int nbulk, ncons;   // halves issued to / consumed from the ring
  bool dep_done;      // the preceding kernel is known to be complete
};

// One warp's run over one KV head: raw items [ra, rb) (nraw raw tokens in all, rows of
// raw head `rawhead`), then packed halves [ha, hb) of the head's tq packed tokens.
// Queries are rows qhead * G + hh of q.  slab_of(p, &slab, &ph) names the slab holding
// half p and the half's index in it (the contiguous cache: the head's slab and p; a
// paged pool: the block's slab and p & 1).  Returns false when a wait ran out.
template <bool ROT, typename SlabOf, bool FUSE = false>
__device__ __forceinline__ bool lean_run(const MmaArgs& a, LeanState& st, LeanWarp& w, int64_t qhead,
                                         int64_t rawhead, int nraw, int64_t tq, int ra, int rb, int ha, int hb,
                                         const SlabOf& slab_of, bool& qbad) {
  const int lane = threadIdx.x & 31;
  if (ra < rb) {   // staged with cp.async in the ring, the next item in flight
    lean_load_queries<ROT>(a, qhead, false, w.qs, qbad);
    stage_raw(a, w.ring, rawhead, ra, nraw);
#pragma unroll 1
    for (int r = ra; r < rb; ++r) {
      if (r + 1 < rb) stage_raw(a, w.ring + ((r + 1 - ra) & 1) * kStageBytes, rawhead, r + 1, nraw);
      else asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 1;" ::: "memory");
      __syncwarp();
      lean_raw(st, w.ring + ((r - ra) & 1) * kStageBytes, min(a.rt, nraw - r * a.rt), a.src_dtype, w.qs);
      __syncwarp();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // the ring's next writers are bulk copies (async proxy) after these generic writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
  }
  if (ha >= hb) return true;
  lean_load_queries<ROT>(a, qhead, ROT, w.qs, qbad);
  // two halves in flight; a half's stage is released once its value words are in
  // registers, and its value product runs during the next half's key product
  if constexpr (FUSE) w.dep_done = false;   // fused append: its flags are per head
  auto issue = [&](int q) {
    if ((FUSE || a.defer) && !w.dep_done) {   // the group of half q (codes and metadata) meets the append
      const int64_t g0 = 128 * (int64_t)(q >> 1);
      if (g0 < a.dep_hi && g0 + 128 > a.dep_lo) {
        // fused: the head's units are done (the contiguous cache: slab = head = qhead)
        if constexpr (FUSE) fused_wait(a.flags, a.epoch, a.status, qhead);
        else griddep_wait();
        w.dep_done = true;
      }
    }
    int64_t slab;
    int ph;
    slab_of(q, &slab, &ph);
    issue_half(a, w.ring + (w.nbulk & 1) * kStageBytes, &w.bars[w.nbulk & 1], slab, ph, q == ha || (q & 1) == 0);
    ++w.nbulk;
  };
#pragma unroll 1
  for (int q = ha; q < min(hb, ha + kBuffers); ++q) issue(q);
  LeanKey ko;
  // the pending value product (zero operands before the first half: it adds nothing, and
  // the two products stay in one block for the scheduler)
  uint2 vw[8];
  uint32_t pb[4][2];
#pragma unroll
  for (int u = 0; u < 8; ++u) vw[u] = make_uint2(0u, 0u);
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) pb[mt][0] = pb[mt][1] = 0u;
#pragma unroll 1
  for (int p = ha; p < hb; ++p) {
    const int sb2 = w.ncons & 1;
    if (!mbar_wait(&w.bars[sb2], (uint32_t)(w.ncons >> 1) & 1u)) return false;
    const uint8_t* stg = w.ring + sb2 * kStageBytes;
    if ((p & 1) == 0 || p == ha) {   // the group's key operand
      // lane L takes the channel quad stored at slot L (qslot of quad 4 (L & 7) + L / 8): the
      // stores below are then one contiguous 512 bytes
      const int quad = 4 * (lane & 7) + (lane >> 3);
      const uint2 sv = reinterpret_cast<const uint2*>(stg + kHalfK + kHalfV + kHalfVM)[quad];
      const uint2 zv = reinterpret_cast<const uint2*>(stg + kHalfK + kHalfV + kHalfVM + 256)[quad];
      const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
      const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
      const float2 z01 = __half22float2(*reinterpret_cast<const __half2*>(&zv.x));
      const float2 z23 = __half22float2(*reinterpret_cast<const __half2*>(&zv.y));
      reinterpret_cast<float4*>(w.kmeta)[lane] = make_float4(s01.x, s01.y, s23.x, s23.y);
      reinterpret_cast<float4*>(w.kmeta + 128)[lane] = make_float4(z01.x, z01.y, z23.x, z23.y);
      __syncwarp();
      lean_key_operand(w.kmeta, w.kmeta + 128, w.qs, w.scr, ko);
    }
    const int tvalid = (int)min((int64_t)64, tq - 64 * (int64_t)p);
    const uint32_t* vsz = reinterpret_cast<const uint32_t*>(stg + kHalfK + kHalfV);
    lean_sz(vsz[lane], vsz[32 + lane], tvalid, reinterpret_cast<float*>(w.scr));
    float S[4][4];
    lean_scores(S, reinterpret_cast<const uint4*>(stg), ko);
    lean_pv(st, vw, pb);   // the previous half's value product
    __syncwarp();          // the scale / zero-point pairs
    lean_softmax(st, S, ko, tvalid, reinterpret_cast<const float2*>(w.scr), pb);
    lean_value_words(vw, reinterpret_cast<const uint2*>(stg + kHalfK));
    __syncwarp();          // stage and scratch reads done before they are written again
    ++w.ncons;
    if (p + kBuffers < hb) issue(p + kBuffers);   // the freed stage takes the half after the next
  }
  lean_pv(st, vw, pb);
  return true;
}

// Waits for the copies still in flight (after a wait ran out) so that the ring can be
// reused, then flags the timeout.
__device__ __forceinline__ void lean_drain(const MmaArgs& a, LeanWarp& w) {
  for (int c = w.ncons; c < w.nbulk; ++c) mbar_wait(&w.bars[c & 1], (uint32_t)(c >> 1) & 1u);
  if ((threadIdx.x & 31) == 0) flag(a.status, KVQ_DEV_TIMEOUT);
}

// The warp areas of warp `warp` in a CTA of nw warps (stages, queries, scratch, key
// metadata per warp, then the mbarriers of every warp).
__device__ __forceinline__ LeanWarp lean_warp(uint8_t* smem, int warp, int nw) {
  LeanWarp w;
  w.ring = smem + (size_t)warp * kLeanWarpBytes;
  w.qs = reinterpret_cast<float*>(w.ring + kBuffers * kStageBytes);
  w.scr = reinterpret_cast<uint32_t*>(w.ring + kBuffers * kStageBytes + kQBytes);
  w.kmeta = reinterpret_cast<float*>(w.ring + kBuffers * kStageBytes + kQBytes + kBScratch);
  w.bars = reinterpret_cast<uint64_t*>(smem + (size_t)nw * kLeanWarpBytes) + kBuffers * warp;
  w.nbulk = w.ncons = 0;
  w.dep_done = false;
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int b = 0; b < kBuffers; ++b) mbar_init(&w.bars[b], 1);
    mbar_fence_init();
  }
  __syncwarp();
  return w;
}

// Merges the records of warps [w0, w1] of the CTA (each warp's ring: o[G][128], m[G],
// l[G] of one head) and writes the merged state of query rows h G + hh into slot `slot`.
__device__ __forceinline__ void lean_merge(const MmaArgs& a, uint8_t* smem, int w0, int w1, int64_t h, int slot,
                                           int nthreads) {
  const int G = a.G;
#pragma unroll 1
  for (int idx = threadIdx.x; idx < G * 128; idx += nthreads) {
    const int hh = idx >> 7, d = idx & 127;
    float M = -INFINITY;
    for (int w = w0; w <= w1; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + (size_t)w * kLeanWarpBytes);
      M = fmaxf(M, rw[8 * 128 + hh]);
    }
    float o = 0.0f, l = 0.0f;
    for (int w = w0; w <= w1; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + (size_t)w * kLeanWarpBytes);
      const float mw = rw[8 * 128 + hh];
      if (mw != -INFINITY) {
        const float f = ex2(mw - M);
        o = fmaf(f, rw[hh * 128 + d], o);
        l = fmaf(f, rw[8 * 128 + 8 + hh], l);
      }
    }
    const int64_t sl = (h * G + hh) * a.S + slot;
    a.ws_o[sl * 128 + d] = o;
    if (d == 0) {
      a.ws_m[sl] = M;
      a.ws_l[sl] = l;
    }
  }
}

template <bool ROT, bool FUSE>
__global__ void __launch_bounds__(kThreads, 1) decode_k4v2_kernel(MmaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  // launched with launch_pdl: without a deferred wait the cache and q are complete from
  // here on; with one (an append just before), see MmaArgs::defer
  if (!a.defer) griddep_wait();
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kCW + warp;
  const int64_t i0 = item_start(gw, a.I, a.W), i1 = item_start(gw + 1, a.I, a.W);
  const int U = a.U;
  if constexpr (FUSE) fused_append(a, gw);
  LeanWarp w = lean_warp(smem, warp, kCW);
  int* last_head = reinterpret_cast<int*>(smem + (size_t)kCW * kLeanWarpBytes + kCW * kBuffers * 8);
  const int nraw = a.n_sink + a.t_res;
  const int G = a.G;
  const int nrp = a.nrp;

  LeanState st;
  lean_reset(st);
  bool qbad = false, timed_out = false;
  // The warp's range of positions covers at most two heads (a range never exceeds U).
  const int64_t hA = i0 / U;
  const int64_t endA = min(i1, (hA + 1) * (int64_t)U);
#pragma unroll 1
  for (int segi = 0; segi < 2 && !timed_out; ++segi) {
    const int64_t head = hA + segi;
    const int64_t sb = segi == 0 ? i0 : (hA + 1) * (int64_t)U;
    const int64_t se = segi == 0 ? endA : i1;
    if (se <= sb) continue;
    const int pb = (int)(sb - head * U), pe = (int)(se - head * U);   // positions in the head's row
    if (segi == 1) {   // the range crosses into the next head: slot 0 of the first one
      const int64_t row0 = hA * G;
      lean_emit(st, G, a.ws_o + row0 * a.S * 128, (int64_t)a.S * 128, a.ws_m + row0 * a.S,
                a.ws_l + row0 * a.S, a.S);
      lean_reset(st);
    }
    // raw items with work: r with 2 r in [pb, pe) and 2 r < nrp; packed halves [ha, hb)
    const int ra = (pb + 1) >> 1, rb = (min(pe, nrp) + 1) >> 1;
    const int ha = max(pb, nrp) - nrp, hb = max(pe, nrp) - nrp;
    auto slab_of = [&](int p, int64_t* slab, int* ph) {
      *slab = head;
      *ph = p;
    };
    timed_out = !lean_run<ROT, decltype(slab_of), FUSE>(a, st, w, head, head, nraw, a.t_quant, ra, rb, ha, hb,
                                                        slab_of, qbad);
  }
  if (timed_out) lean_drain(a, w);
  __syncwarp();
  if (__any_sync(0xffffffffu, qbad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);
  // this grid completes only after the one before it, so that the kernels after it on
  // the stream find the append done as well
  if (a.defer) griddep_wait();

  // ---- merge of the warps' last heads inside the CTA (as decode_mma_kernel) ----
  const int lh = i1 > 0 ? (int)((i1 - 1) / U) : -1;
  float* rec = reinterpret_cast<float*>(w.ring);
  if (lh >= 0) lean_emit(st, G, rec, 128, rec + 8 * 128, rec + 8 * 128 + 8, 1);
  if (lane == 0) last_head[warp] = lh;
  __syncthreads();
  int w0 = 0;
#pragma unroll 1
  while (w0 < kCW) {
    const int h = last_head[w0];
    int w1 = w0;
    while (w1 + 1 < kCW && last_head[w1 + 1] == h) ++w1;
    if (h >= 0) {
      const int64_t ca = first_ending_warp(h, U, a.I, a.W) / kCW;
      lean_merge(a, smem, w0, w1, h, 1 + (int)((int64_t)blockIdx.x - ca), kThreads);
    }
    w0 = w1 + 1;
  }
}

// ==== paged cache with per-sequence lengths ==============================================
// Grid (chunk, sequence x KV head).  Each KV head of a sequence is a row of positions as
// above (two per raw item, one per packed half), with the sequence's own lengths; CTA
// (c, head) takes positions [c kPagedChunk, (c + 1) kPagedChunk) of that row, its kPagedWarps
// warps a contiguous quarter each, and writes one partial state per query row into slot c
// (m = -inf for an empty chunk).  Half p of a sequence lives in block block_table[s][p / 2],
// at half p % 2 of that block's slab; a warp reads the block ids of its groups once, and
// every id is checked against the pool before any copy uses it.
constexpr int kPagedWarps = 4;
constexpr int kPagedThreads = kPagedWarps * 32;
constexpr int kPagedChunk = 64;   // positions per CTA
static_assert(kPagedChunk % kPagedWarps == 0, "chunk splits over the warps");
static_assert(kPagedChunk / kPagedWarps / 2 + 1 <= 32, "a warp's block ids fit its lanes");

struct PagedArgs {
  MmaArgs a;                 // pool arrays as slabs of one group (C = g, ng = 1); raw arrays per sequence
  const int32_t* table;      // [num_seqs][max_blocks]
  const int32_t* t_quant;    // [num_seqs]
  const int32_t* t_res;      // [num_seqs]
  int max_blocks, num_blocks;
  int64_t max_t_quant;
  int max_t_res;
};

// Positions of a head row: two per raw item of rt tokens, then one per packed half.
__device__ __forceinline__ int row_positions(int nraw, int rt, int64_t tq, int* nrp) {
  *nrp = 2 * ((nraw + rt - 1) / rt);
  if (tq <= 0) return *nrp;
  const int64_t ngv = (tq + 127) / 128, rem = tq - (ngv - 1) * 128;
  return *nrp + (int)(2 * (ngv - 1) + (rem > 64 ? 2 : 1));
}

template <bool ROT>
__global__ void __launch_bounds__(kPagedThreads, 1) decode_paged_kernel(PagedArgs pa) {
  extern __shared__ __align__(128) uint8_t smem[];
  griddep_wait();   // launched with launch_pdl: the cache, tables and q are complete
  griddep_launch_dependents();
  const MmaArgs& a = pa.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int64_t head = blockIdx.y;   // sequence s, KV head kvh
  const int s = (int)(head / a.Hkv), kvh = (int)(head % a.Hkv);
  LeanWarp w = lean_warp(smem, warp, kPagedWarps);

  // the sequence's lengths, clamped to the bounds the launch was sized for
  int64_t tq = pa.t_quant[s];
  int tr = pa.t_res[s];
  bool oob = false;
  const int64_t tq_cap = min(pa.max_t_quant, (int64_t)pa.max_blocks * 128);
  if (tq < 0 || tq > tq_cap) { oob = true; tq = tq < 0 ? 0 : tq_cap; }
  if (tr < 0 || tr > pa.max_t_res) { oob = true; tr = tr < 0 ? 0 : pa.max_t_res; }
  const int nraw = a.n_sink + tr;
  int nrp;
  const int U = row_positions(nraw, a.rt, tq, &nrp);
  const int per = kPagedChunk / kPagedWarps;
  const int p0 = min(U, c * kPagedChunk + warp * per), p1 = min(U, c * kPagedChunk + (warp + 1) * per);

  LeanState st;
  lean_reset(st);
  bool qbad = false;
  if (p0 < p1) {
    const int ra = (p0 + 1) >> 1, rb = (min(p1, nrp) + 1) >> 1;
    const int ha = max(p0, nrp) - nrp, hb = max(p1, nrp) - nrp;
    // the block ids of the warp's groups, lane i holding group (ha / 2) + i
    const int g0 = ha >> 1;
    int blk = 0;
    if (ha < hb && g0 + lane <= (hb - 1) >> 1) {
      const int gi = g0 + lane;
      blk = pa.table[(int64_t)s * pa.max_blocks + gi];
      if (blk < 0 || blk >= pa.num_blocks) { oob = true; blk = 0; }
    }
    auto slab_of = [&](int p, int64_t* slab, int* ph) {
      const int b = __shfl_sync(0xffffffffu, blk, (p >> 1) - g0);
      *slab = (int64_t)b * a.Hkv + kvh;
      *ph = p & 1;
    };
    if (!lean_run<ROT>(a, st, w, head, head, nraw, tq, ra, rb, ha, hb, slab_of, qbad)) lean_drain(a, w);
  }
  __syncwarp();
  if (__any_sync(0xffffffffu, qbad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);
  if (__any_sync(0xffffffffu, oob) && lane == 0) flag(a.status, KVQ_DEV_BOUNDS);
  // every warp's state (empty ones: m = -inf) into its record, then one slot per CTA
  float* rec = reinterpret_cast<float*>(w.ring);
  lean_emit(st, a.G, rec, 128, rec + 8 * 128, rec + 8 * 128 + 8, 1);
  __syncthreads();
  lean_merge(a, smem, 0, kPagedWarps - 1, head, c, kPagedThreads);
}

// The merge of a row's slots for the paged path (slots with m = -inf are empty; a row
// with no tokens at all gets zeros).
struct CombArgsPaged {
  int S;
  int64_t rows;
  const float* m;
  const float* l;
  const float* o;
  void* out;
  int out_dtype;
};
__global__ void __launch_bounds__(128) combine_paged_kernel(CombArgsPaged a) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  combine_row(a.m, a.l, a.o, a.S, row, 0, a.S - 1, lane, a.out, a.out_dtype, nullptr);
}

size_t lean_smem() {
  return (size_t)kCW * kLeanWarpBytes + (size_t)kCW * kBuffers * 8 + kCW * sizeof(int);
}

// ---- combine for this path: the valid slots of a head follow from the partition ---------
struct CombArgsMma {
  int G, S;
  int64_t rows, U, I, W;
  const float* m;
  const float* l;
  const float* o;
  void* out;
  int out_dtype;
  float* lse;   // nullable
};

// One warp per query-head row.
__global__ void __launch_bounds__(128) combine_mma_kernel(CombArgsMma a) {
  griddep_wait();   // launched with launch_pdl: the split kernel's states are complete
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  int s_lo, s_hi;
  head_slots(row / a.G, a.U, a.I, a.W, kCW, &s_lo, &s_hi);
  combine_row(a.m, a.l, a.o, a.S, row, s_lo, s_hi, lane, a.out, a.out_dtype, a.lse);
}

// per-warp rings of item stages, per-warp scratch, then the warps' last heads
static_assert(kStageBytes % 128 == 0, "stage alignment");
size_t mma_smem() {
  return (size_t)kCW * kBuffers * kStageBytes + (size_t)kCW * kScratchBytes + kCW * sizeof(int);
}

// Positions of a head: two per raw item of rt tokens, then one per packed half.
struct Items {
  int rt, nrp, nh, U;
};
Items head_items(const Layout& L, int64_t t_quant, int t_res) {
  Items it;
  it.rt = kRawBytes / (128 * (L.src_dtype == KVQ_F32 ? 4 : 2));
  const int nraw = L.n_sink + t_res;
  it.nrp = 2 * ((nraw + it.rt - 1) / it.rt);
  const int64_t ngv = (t_quant + 127) / 128;
  const int64_t rem = t_quant - (ngv - 1) * 128;
  it.nh = (int)(2 * (ngv - 1) + (rem > 64 ? 2 : 1));
  it.U = it.nrp + it.nh;
  return it;
}

}  // namespace

bool mma_path_ok(const Layout& L, int Hq) {
  const Side& K = L.side[0];
  const Side& V = L.side[1];
  const int G = Hq / L.Hkv;
  const bool k4 = K.scheme == KVQ_ASYM && K.bits == 4 && K.axis == KVQ_AXIS_CHANNEL;
  // MIXED keys with the [MIX] Figure 3 tiers (8 raw bf16, 24 4-bit, 96 2-bit slots)
  const bool mix = K.scheme == KVQ_MIXED && L.mixed_hi == 8 && L.mixed_mid == 24 &&
                   L.src_dtype == KVQ_BF16;
  return L.D == 128 && L.g == 128 && (k4 || mix) && V.scheme == KVQ_ASYM && V.bits == 2 &&
         V.axis == KVQ_AXIS_TOKEN && L.rope == 0 && G >= 1 && G <= 8;
}

bool fused_append_ok(const Layout& L, int Hq, const DecodePlan& p, int64_t t0, int64_t n) {
  const Side& K = L.side[0];
  const Side& V = L.side[1];
  return p.fast && mma_path_ok(L, Hq) && Hq / L.Hkv <= 4 && K.scheme == KVQ_ASYM && K.bits == 4 &&
         K.axis == KVQ_AXIS_CHANNEL && !L.k_rotate && V.scheme == KVQ_ASYM && V.bits == 2 &&
         (L.src_dtype == KVQ_F16 || L.src_dtype == KVQ_BF16) && n >= 1 && n <= 128 && t0 % 128 == 0 &&
         t0 + n <= L.C;
}

// Partition of the fast path (t_quant >= 1): CTAs, slots per query head.  At least one
// warp per head, so that no warp range is longer than a head's row of items.
void plan_mma(const Layout& L, int64_t t_quant, int t_res, int max_ctas, DecodePlan& p) {
  const int64_t heads = (int64_t)L.B * L.Hkv;
  const Items it = head_items(L, t_quant, t_res);
  const int64_t I = heads * it.U;
  int64_t cap = device_sm_count();
  if (max_ctas > 0) cap = std::min<int64_t>(cap, max_ctas);
  int64_t grid = std::min<int64_t>(cap, (I + kCW - 1) / kCW);
  grid = std::max<int64_t>(grid, (heads + kCW - 1) / kCW);
  grid = std::max<int64_t>(grid, 1);
  const int64_t W = grid * kCW;
  int64_t span = 1;
  for (int64_t h = 0; h < heads; ++h) {
    const int64_t ca = first_ending_warp(h, it.U, I, W) / kCW, cb = last_ending_warp(h, it.U, I, W) / kCW;
    span = std::max(span, cb - ca + 1);
  }
  p.S = (int)(1 + span);
  p.grid_ctas = (int)grid;
  p.raw_slot = -1;
  p.raw_pieces = it.nrp;
  p.n_packed_splits = it.nh;
  p.split_groups = it.rt;
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
  a.k_order = L.k_order;
  a.k_group_bytes = L.mixed_group_bytes;
  a.q = q;
  a.q_dtype = q_dtype;
  a.qscale = scale * kLog2e;
  a.k_rotate = L.k_rotate;
  a.rot_scale = L.rot_scale;
  a.nrp = p.raw_pieces;
  a.rt = p.split_groups;
  a.U = p.raw_pieces + p.n_packed_splits;
  a.I = (int64_t)L.B * L.Hkv * a.U;
  a.W = (int64_t)p.grid_ctas * kCW;
  a.S = p.S;
  a.ws_m = ws_m;
  a.ws_l = ws_l;
  a.ws_o = ws_o;
  a.status = d_status;
  a.defer = p.defer;
  a.dep_lo = p.dep_lo;
  a.dep_hi = p.dep_hi;
  a.fuse = p.fuse;
  a.app_n = p.app_n;
  a.app_k = p.app_k;
  a.app_v = p.app_v;
  a.app_sb = p.app_sb;
  a.app_sh = p.app_sh;
  a.app_st = p.app_st;
  a.flags = p.flags;
  a.epoch = p.epoch;
  a.heads = (int64_t)L.B * L.Hkv;
  const bool mix = L.side[0].scheme == KVQ_MIXED;
  if (!mix && a.G <= 4) {
    const size_t smem = lean_smem();
    // the fused append takes no rotated keys (fused_append_ok)
    auto kern = a.fuse ? decode_k4v2_kernel<false, true>
              : (a.k_rotate ? decode_k4v2_kernel<true, false> : decode_k4v2_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(p.grid_ctas), dim3(kThreads), smem, s, a);
  }
  const size_t smem = mma_smem();
  auto kern = mix ? (a.G <= 4 ? decode_mma_kernel<true, false, true> : decode_mma_kernel<false, false, true>)
            : (a.k_rotate ? decode_mma_kernel<false, true, false> : decode_mma_kernel<false, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<p.grid_ctas, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

bool paged_path_ok(const Layout& L, int Hq) {
  const Side& K = L.side[0];
  const Side& V = L.side[1];
  const int G = Hq / L.Hkv;
  return L.D == 128 && L.g == 128 && K.scheme == KVQ_ASYM && K.bits == 4 && K.axis == KVQ_AXIS_CHANNEL &&
         V.scheme == KVQ_ASYM && V.bits == 2 && V.axis == KVQ_AXIS_TOKEN && L.rope == 0 && G >= 1 && G <= 4;
}

int paged_slots(const Layout& L, int64_t max_t_quant, int max_t_res) {
  const int rt = kRawBytes / (128 * (L.src_dtype == KVQ_F32 ? 4 : 2));
  const int nraw = L.n_sink + max_t_res;
  int64_t U = 2 * ((nraw + rt - 1) / rt);
  if (max_t_quant > 0) {
    const int64_t ngv = (max_t_quant + 127) / 128, rem = max_t_quant - (ngv - 1) * 128;
    U += 2 * (ngv - 1) + (rem > 64 ? 2 : 1);
  }
  return (int)std::max<int64_t>(1, (U + kPagedChunk - 1) / kPagedChunk);
}

cudaError_t launch_decode_paged(const Layout& L, const PagedDecode& pd, int S, const void* q, int q_dtype, int Hq,
                                float scale, float* ws_m, float* ws_l, float* ws_o, void* out, int out_dtype,
                                int32_t* d_status, cudaStream_t s) {
  PagedArgs pa;
  MmaArgs& a = pa.a;
  std::memset(&pa, 0, sizeof(pa));
  a.k_codes = reinterpret_cast<const uint8_t*>(L.side[0].codes);
  a.v_codes = reinterpret_cast<const uint8_t*>(L.side[1].codes);
  a.k_scale = reinterpret_cast<const __half*>(L.side[0].scale);
  a.k_zero = reinterpret_cast<const __half*>(L.side[0].zero);
  a.v_scale = reinterpret_cast<const __half*>(L.side[1].scale);
  a.v_zero = reinterpret_cast<const __half*>(L.side[1].zero);
  a.k_slab_bytes = L.side[0].code_slab_bytes;   // one group per slab
  a.v_slab_bytes = L.side[1].code_slab_bytes;
  a.C = L.C;
  a.ng = L.ng;
  a.Hkv = L.Hkv;
  a.Hq = Hq;
  a.G = Hq / L.Hkv;
  a.n_sink = L.n_sink;
  a.res_cap = L.res_cap;
  a.src_dtype = L.src_dtype;
  a.sink_k = pd.sink[0];
  a.sink_v = pd.sink[1];
  a.res_k = pd.res[0];
  a.res_v = pd.res[1];
  a.q = q;
  a.q_dtype = q_dtype;
  a.qscale = scale * kLog2e;
  a.k_rotate = L.k_rotate;
  a.rot_scale = L.rot_scale;
  a.rt = kRawBytes / (128 * (L.src_dtype == KVQ_F32 ? 4 : 2));
  a.S = S;
  a.ws_m = ws_m;
  a.ws_l = ws_l;
  a.ws_o = ws_o;
  a.status = d_status;
  pa.table = pd.table;
  pa.t_quant = pd.t_quant;
  pa.t_res = pd.t_res;
  pa.max_blocks = pd.max_blocks;
  pa.num_blocks = L.B;
  pa.max_t_quant = pd.max_t_quant;
  pa.max_t_res = pd.max_t_res;
  const size_t smem = (size_t)kPagedWarps * kLeanWarpBytes + (size_t)kPagedWarps * kBuffers * 8;
  auto kern = L.k_rotate ? decode_paged_kernel<true> : decode_paged_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((unsigned)S, (unsigned)((int64_t)pd.num_seqs * L.Hkv)), dim3(kPagedThreads), smem, s,
                 pa);
  if (e != cudaSuccess) return e;
  CombArgsPaged c;
  c.S = S;
  c.rows = (int64_t)pd.num_seqs * Hq;
  c.m = ws_m;
  c.l = ws_l;
  c.o = ws_o;
  c.out = out;
  c.out_dtype = out_dtype;
  return launch_pdl(combine_paged_kernel, dim3((unsigned)((c.rows + 3) / 4)), dim3(128), 0, s, c);
}

cudaError_t launch_combine_mma(const Layout& L, const DecodePlan& p, int Hq, const float* ws_m,
                               const float* ws_l, const float* ws_o, void* out, int out_dtype,
                               float* lse, cudaStream_t s) {
  CombArgsMma c;
  c.G = Hq / L.Hkv;
  c.S = p.S;
  c.rows = (int64_t)L.B * Hq;
  c.U = p.raw_pieces + p.n_packed_splits;
  c.I = (int64_t)L.B * L.Hkv * c.U;
  c.W = (int64_t)p.grid_ctas * kCW;
  c.m = ws_m;
  c.l = ws_l;
  c.o = ws_o;
  c.out = out;
  c.out_dtype = out_dtype;
  c.lse = lse;
  return launch_pdl(combine_mma_kernel, dim3((unsigned)((c.rows + 3) / 4)), dim3(128), 0, s, c);
}

}  // namespace kvq
