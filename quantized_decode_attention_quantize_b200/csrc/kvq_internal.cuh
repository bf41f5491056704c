// Internal declarations shared by the kernels and the host layer of libkvq.
// Not part of the public ABI (include/kvq.h is).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

// ---------------------------------------------------------------------------
// Layout: everything a kernel needs to address the cache, derived on the host
// from kvq_format + kvq_cache and passed by value.
// ---------------------------------------------------------------------------
struct Side {
  int scheme, bits, axis, nout;
  int64_t code_slab_bytes;   // bytes of codes per (b, kv-head) slab
  int64_t meta_slab_elems;   // scale / zero elements per slab
  int code_row_bytes;        // packed bytes per token row (MIXED: per row of all planes)
  void* codes;
  void* scale;
  void* zero;
  const __half* lut;
  const float* lutf;         // KQV: fp32 centroids
};

struct Layout {
  int D, g, src_dtype, B, Hkv;
  int64_t C;                 // capacity (tokens), multiple of g
  int ng;                    // C / g
  int n_sink, res_cap, rope;
  float rope_base;
  int k_rotate;              // keys stored in the Walsh-Hadamard basis
  float rot_scale;           // fl32(1 / sqrt(D))
  int mixed_hi, mixed_mid, mixed_lo, mixed_group_bytes;
  Side side[2];
  uint8_t* k_order;
  int32_t* k_out_rowptr;
  uint8_t* k_out_col;
  __half* k_out_val;
  uint8_t* v_out_col;
  __half* v_out_val;
  void* sink[2];
  void* res[2];
  int raw_bytes;             // element size of src_dtype
  const float* sketch;       // KQV: the D x D sketch matrix
};

// Host helpers (api.cpp)
kvq_status make_layout(const kvq_format* f, const kvq_cache* c, Layout* L);

// Launchers (each .cu file), return cudaError_t of the launch.
cudaError_t launch_quantize(const Layout& L, int which, const void* src, int64_t sb,
                            int64_t sh, int64_t st, int64_t t0, int64_t n,
                            int32_t* d_status, cudaStream_t s);
bool asym_fast_ok(const Layout& L, int which);
cudaError_t launch_quantize_asym(const Layout& L, int which, const void* src, int64_t sb,
                                 int64_t sh, int64_t st, int64_t t0, int64_t n,
                                 int32_t* d_status, cudaStream_t s);
// blocks (nullable): a paged pool, sequence b's group going to block blocks[b] (L: the
// pool as one group per slab, L.B = the number of sequences, num_blocks the pool's blocks)
cudaError_t launch_quantize_asym_kv(const Layout& L, const void* ksrc, const void* vsrc, int64_t sb,
                                    int64_t sh, int64_t st, int64_t t0, int64_t n, int32_t* d_status,
                                    cudaStream_t s, const int32_t* blocks = nullptr, int num_blocks = 0);
cudaError_t launch_dequantize(const Layout& L, int which, int64_t t0, int64_t n, void* out,
                              int out_dtype, int32_t* d_status, cudaStream_t s);
// KQV (quantize_kqv.cu)
cudaError_t launch_quantize_kqv(const Layout& L, int which, const void* src, int64_t sb, int64_t sh,
                                int64_t st, int64_t t0, int64_t n, int32_t* d_status, cudaStream_t s);
cudaError_t launch_dequantize_kqv(const Layout& L, int which, int64_t t0, int64_t n, void* out, int out_dtype,
                                  cudaStream_t s);
cudaError_t launch_salience(const Layout& L, const void* q, int64_t qsb, int64_t qsh,
                            int64_t qst, const void* k, int64_t ksb, int64_t ksh, int64_t kst,
                            int B, int Hq, int Hkv, int R, double* sal, uint8_t* order,
                            int64_t osb, int64_t osh, int32_t* d_status, cudaStream_t s);

struct DecodePlan {
  int S;                // partial slots per query head
  int split_groups;     // generic path: packed groups per split; fast path: tokens per raw item
  int n_packed_splits;  // generic path: splits over the packed region; fast path: packed halves per head
  int raw_slot;         // generic path: slot of the raw (sink + residual) tokens, -1 if none
  int raw_pieces;       // fast path: raw positions per head (two per raw item)
  int fast;             // 1 when the tensor-core K4/V2 kernel runs the packed region
  int grid_ctas;        // CTAs of the split kernel
  // set by the append-and-decode entry point: the split kernel follows the append of
  // packed rows [dep_lo, dep_hi) directly and may read the other rows before it completes
  int defer = 0;
  int64_t dep_lo = 0, dep_hi = 0;
  // set by the append-and-decode entry point when the split kernel does the append itself
  // (fused_append_ok): one group at dep_lo of app_n rows from these sources, flags in the
  // workspace, a fresh epoch per call
  int fuse = 0;
  int app_n = 0;
  const void* app_k = nullptr;
  const void* app_v = nullptr;
  int64_t app_sb = 0, app_sh = 0, app_st = 0;
  uint32_t* flags = nullptr;
  uint32_t epoch = 0;
};
DecodePlan plan_decode(const Layout& L, int Hq, int64_t t_quant, int t_res, int num_splits);
size_t workspace_bytes(const Layout& L, int Hq, const DecodePlan& p);
bool fast_path_ok(const Layout& L, int Hq);
// The split kernel can take the append of n rows at t0 itself (one group; K4 per channel,
// V2 per token, not rotated, 16-bit sources, the G <= 4 tensor-core kernel).
bool fused_append_ok(const Layout& L, int Hq, const DecodePlan& p, int64_t t0, int64_t n);
cudaError_t launch_decode_partial(const Layout& L, const DecodePlan& p, const void* q,
                                  int q_dtype, int Hq, int64_t t_quant, int t_res, float scale,
                                  void* ws, int32_t* d_status, cudaStream_t s);
cudaError_t launch_combine(const Layout& L, int Hq, const DecodePlan& p, const void* ws, void* out,
                           int out_dtype, float* lse, cudaStream_t s);
// out = sum_r w_r out_r / sum_r w_r with w_r = exp(lse_r - max_r lse_r) over n parts
// (outs [n][rows][D] fp32, lses [n][rows] fp32).
cudaError_t launch_merge_states(int n, int64_t rows, int D, const float* outs, const float* lses,
                                void* out, int out_dtype, float* lse_out, cudaStream_t s);
int device_sm_count();

// Paged cache (the 4-bit / 2-bit tensor-core format, G <= 4): the pool layout L has one
// group per slab (C = g, B = num_blocks).
struct PagedDecode {
  const int32_t* table;
  const int32_t* t_quant;
  const int32_t* t_res;
  int num_seqs, max_blocks;
  int64_t max_t_quant;
  int max_t_res;
  const void* sink[2];
  const void* res[2];
};
bool paged_path_ok(const Layout& L, int Hq);
int paged_slots(const Layout& L, int64_t max_t_quant, int max_t_res);
cudaError_t launch_decode_paged(const Layout& L, const PagedDecode& pd, int S, const void* q, int q_dtype, int Hq,
                                float scale, float* ws_m, float* ws_l, float* ws_o, void* out, int out_dtype,
                                int32_t* d_status, cudaStream_t s);

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float load_elem(const void* p, int64_t i, int dtype) {
  if (dtype == KVQ_F32) return reinterpret_cast<const float*>(p)[i];
  if (dtype == KVQ_F16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ void store_elem(void* p, int64_t i, int dtype, float v) {
  if (dtype == KVQ_F32) reinterpret_cast<float*>(p)[i] = v;
  else if (dtype == KVQ_F16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

__device__ __forceinline__ void flag(int32_t* st, int bits) {
  if (st) atomicOr(st, bits);
}

// Asymmetric b-bit metadata: z = fp16 toward -inf of mn, s = fp16 toward +inf of
// fl32(fl32(mx - z) / (2^b - 1)), s = 1 when that is zero.
__device__ __forceinline__ bool asym_params(float mn, float mx, int bits, __half* s_out,
                                            __half* z_out) {
  __half z = __float2half_rd(mn);
  float zf = __half2float(z);
  float d = __fsub_rn(mx, zf);
  float t = __fdiv_rn(d, (float)((1 << bits) - 1));
  __half s = __float2half_ru(t);
  float sf = __half2float(s);
  if (sf == 0.0f) s = __float2half_rn(1.0f);
  *s_out = s;
  *z_out = z;
  return isfinite(zf) && isfinite(__half2float(s));
}

__device__ __forceinline__ int asym_code(float x, float s, float z, int maxc) {
  float q = __fdiv_rn(__fsub_rn(x, z), s);
  float r = rintf(q);
  r = fminf(fmaxf(r, 0.0f), (float)maxc);
  return (int)r;
}

// The same code without a division in the common case, given rs = fl32(1 / s): for the
// in-range quotients of a group (|q| <= 2^8) q1 = fl32(fl32(x - z) * rs) is within
// 2^-22 |q| + 2^-24 |q| < 2^-13 of the exact quotient, so q1 and fl32(fl32(x - z) / s)
// round to the same integer unless q1 lies within 2^-12 of a half-integer; there the
// quotient is taken exactly.  Out-of-range quotients clip to the same end either way.
__device__ __forceinline__ int asym_code_r(float x, float s, float rs, float z, int maxc) {
  const float u = __fsub_rn(x, z);
  float q = __fmul_rn(u, rs);
  if (fabsf(q - floorf(q) - 0.5f) < 0x1p-12f) q = __fdiv_rn(u, s);
  float r = rintf(q);
  r = fminf(fmaxf(r, 0.0f), (float)maxc);
  return (int)r;
}

// nuq3 metadata: z = fp16 nearest of fl32(fl32(mx + mn) * 0.5),
// s = fp16 toward +inf of max(fl32(mx - z), fl32(z - mn)), s = 1 when zero.
__device__ __forceinline__ bool nuq_params(float mn, float mx, __half* s_out, __half* z_out) {
  float h = __fmul_rn(__fadd_rn(mx, mn), 0.5f);
  __half z = __float2half_rn(h);
  float zf = __half2float(z);
  float a = __fsub_rn(mx, zf);
  float b = __fsub_rn(zf, mn);
  __half s = __float2half_ru(fmaxf(a, b));
  if (__half2float(s) == 0.0f) s = __float2half_rn(1.0f);
  *s_out = s;
  *z_out = z;
  return isfinite(zf) && isfinite(__half2float(s));
}

// Nearest of the eight centroids via the seven fp32 midpoints (an exact midpoint
// goes to the lower centroid).
__device__ __forceinline__ int nuq_code(float x, float s, float z, const float* mids) {
  float y = __fdiv_rn(__fsub_rn(x, z), s);
  int c = 0;
#pragma unroll
  for (int j = 0; j < 7; ++j) c += (y > mids[j]) ? 1 : 0;
  return c;
}

// Programmatic dependent launch.  A kernel launched with launch_pdl may begin while the
// kernel before it on the stream is still running; it must call griddep_wait() before it
// reads or writes any memory that earlier work on the stream produces or still reads
// (griddep_wait returns once that grid has completed and its writes are visible).
// griddep_launch_dependents() lets the next such kernel be scheduled early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---- append-time code packing (the append kernels and the split kernel's fused append) ----
// 8 consecutive elements (16 bytes for 16-bit sources, two 16-byte loads for fp32)
__device__ __forceinline__ void load8(const void* base, int64_t i, int dtype, float* out) {
  if (dtype == KVQ_F32) {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i + 4);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (dtype == KVQ_F16) {
        out[2 * j] = half_bits_to_float((uint16_t)(w[j] & 0xffffu));
        out[2 * j + 1] = half_bits_to_float((uint16_t)(w[j] >> 16));
      } else {
        out[2 * j] = __uint_as_float(w[j] << 16);
        out[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    }
  }
}

// 8 codes of `bits` bits packed LSB-first (bits = 2: 16 bits, 4: 32 bits; 8: two words).
// Each code is rint_even(fl32(fl32(x - z) / s)) clipped to [0, 2^bits - 1], found as
// asym_code_r does: from q = fl32(fl32(x - z) * rs), rs = fl32(1 / s), which is within
// 2^-13 of the exact quotient for in-range codes, so that q and the IEEE quotient round to
// the same integer unless q lies within 2^-12 of a half-integer.  Such elements (rare) take
// the quotient instead, behind one branch per eight codes.
__device__ __forceinline__ uint2 pack8(const float* x, const float* s, const float* rs, const float* z,
                                       int bits) {
  const float maxc = (float)((1 << bits) - 1);
  float q[8];
  bool near = false;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    q[j] = __fmul_rn(__fsub_rn(x[j], z[j]), rs[j]);
    near |= fabsf(q[j] - rintf(q[j])) > 0.5f - 0x1p-12f;
  }
  if (near) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (fabsf(q[j] - rintf(q[j])) > 0.5f - 0x1p-12f) q[j] = __fdiv_rn(__fsub_rn(x[j], z[j]), s[j]);
  }
  uint32_t c[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) c[j] = (uint32_t)fminf(fmaxf(rintf(q[j]), 0.0f), maxc);
  uint32_t lo = 0, hi = 0;
  if (bits == 8) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      lo |= c[j] << (8 * j);
      hi |= c[4 + j] << (8 * j);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) lo |= c[j] << (bits * j);
  }
  return make_uint2(lo, hi);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace kvq
