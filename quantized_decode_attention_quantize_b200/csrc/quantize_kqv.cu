// KQV quantization and reconstruction ([TQ] "Quantization Schemes": rotated keys by
// n-bit scalar MSE codes of their direction, rotated values by (n-1)-bit codes plus a
// one-bit QJL sketch of the residual; "Theoretical Framework" for the codebook).
//
// One warp per token row of D = 128 channels, lane l owning channels 4 l .. 4 l + 3.
// The stored format fixes every decision in fp32 with one IEEE rounding per operation:
//   y  = fp32 Walsh-Hadamard butterfly (strides 1, 2 inside the lane, 4 .. 64 across
//        lanes) and one product with fl32(1 / sqrt(D));
//   T  = pairwise-tree sum over the channel index: levels 1 and 2 inside the lane, levels
//        3 .. 7 by xor-shuffles over lanes 1, 2, 4, 8, 16 (addition is commutative, so
//        both lanes of a pair hold the same bits);
//   n  = sqrt(T(y^2)), u = y / n, code = #{j : u > fl32(fl32(C_j + C_{j+1}) * 0.5)};
//   values: r = y - fl32(n C[code]), rn = sqrt(T(r^2)), sign bit i = (T(S_i . r) >= 0)
//        with the sketch matrix S staged in shared memory.
#include <cmath>

#include "decode_common.cuh"
#include "wht.cuh"

namespace kvq {
namespace {

constexpr int kQW = 8;                 // warps per CTA
constexpr int kD = 128;
constexpr float kSketchScale = 0.009791516697777345f;   // sqrt(pi / 2) / 128

struct KqvArgs {
  Layout L;
  int which;
  const void* src;
  int64_t sb, sh, st, t0, n;
  void* out;          // dequantize: [B][Hkv][n][D] out_dtype
  int out_dtype;
  int32_t* status;
};

__device__ __forceinline__ float tree128(float a0, float a1, float a2, float a3) {
  float s = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
  return s;
}

// Four consecutive source elements (fp32, fp16 or bf16), exactly widened to fp32.
__device__ __forceinline__ void load4(const void* p, int64_t i, int dtype, float (&x)[4]) {
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

// Packs the lane's 4-channel field of `bpc` bits per channel into the row layout
// (channel c at word c / (32 / bpc), bit bpc * (c % (32 / bpc))) and lets the first lane
// of each word store it at words[lane / (8 / bpc)].  bpc in {1, 2, 4}.
__device__ __forceinline__ void store_plane(uint32_t* words, uint32_t field, int bpc, int lane) {
  const int lpw = 8 / bpc;   // lanes per word
  uint32_t v = field << (4 * bpc * (lane % lpw));
  for (int o = 1; o < lpw; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
  if (lane % lpw == 0) words[lane / lpw] = v;
}

// Stores the codes of the lane's channels (b bits each; b = 3 as the two planes).
__device__ __forceinline__ void store_codes(uint32_t* row, const int (&code)[4], int b, int lane) {
  if (b == 3) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      lo |= (uint32_t)(code[j] & 3) << (2 * j);
      hi |= (uint32_t)(code[j] >> 2) << j;
    }
    store_plane(row, lo, 2, lane);
    store_plane(row + kD / 16, hi, 1, lane);
  } else {
    uint32_t f = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) f |= (uint32_t)code[j] << (b * j);
    store_plane(row, f, b, lane);
  }
}

// Codes of the lane's channels from a packed row.
__device__ __forceinline__ void load_codes(const uint32_t* row, int b, int lane, int (&code)[4]) {
  if (b == 3) {
    const uint32_t lo = row[lane / 4] >> (8 * (lane % 4));
    const uint32_t hi = row[kD / 16 + lane / 8] >> (4 * (lane % 8));
#pragma unroll
    for (int j = 0; j < 4; ++j) code[j] = (int)(((lo >> (2 * j)) & 3u) | (((hi >> j) & 1u) << 2));
  } else {
    const int lpw = 8 / b;
    const uint32_t f = row[lane / lpw] >> (4 * b * (lane % lpw));
#pragma unroll
    for (int j = 0; j < 4; ++j) code[j] = (int)((f >> (b * j)) & ((1u << b) - 1));
  }
}

__global__ void __launch_bounds__(kQW * 32) kqv_quantize_kernel(KqvArgs a) {
  extern __shared__ __align__(16) float sk[];   // values: S [128][128]
  const Layout& L = a.L;
  const Side& S = L.side[a.which];
  const bool val = a.which == KVQ_VALUES;
  const int b = val ? S.bits - 1 : S.bits;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (val) {
    const float4* g = reinterpret_cast<const float4*>(L.sketch);
    for (int i = threadIdx.x; i < kD * kD / 4; i += blockDim.x) reinterpret_cast<float4*>(sk)[i] = g[i];
    __syncthreads();
  }
  // midpoints of the fp32 codebook (at most 15)
  const float* C = reinterpret_cast<const float*>(S.lutf);
  const int K = 1 << b;
  float mids[15];
#pragma unroll
  for (int j = 0; j < 15; ++j) {
    mids[j] = INFINITY;
    if (j + 1 < K) mids[j] = __fmul_rn(__fadd_rn(C[j], C[j + 1]), 0.5f);
  }
  const float clane = C[lane & (K - 1)];       // lane i holds C[i mod K]
  const int words = val ? S.bits * kD / 32 : b * kD / 32;
  int bad = 0;
  const int64_t rows = (int64_t)L.B * L.Hkv * a.n;
  for (int64_t r = (int64_t)blockIdx.x * kQW + warp; r < rows; r += (int64_t)gridDim.x * kQW) {
    const int64_t head = r / a.n, t = r % a.n;
    const int64_t bb = head / L.Hkv, h = head % L.Hkv;
    float y[4];
    load4(a.src, bb * a.sb + h * a.sh + t * a.st + 4 * lane, L.src_dtype, y);
#pragma unroll
    for (int j = 0; j < 4; ++j) bad |= !isfinite(y[j]);
    wht128_quad_unscaled(y, lane);
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = __fmul_rn(y[j], L.rot_scale);
    const float nrm = __fsqrt_rn(tree128(__fmul_rn(y[0], y[0]), __fmul_rn(y[1], y[1]),
                                         __fmul_rn(y[2], y[2]), __fmul_rn(y[3], y[3])));
    int code[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float u = nrm > 0.0f ? __fdiv_rn(y[j], nrm) : 0.0f;
      int c = 0;
#pragma unroll
      for (int m = 0; m < 15; ++m) c += u > mids[m];
      code[j] = c;
    }
    const int64_t pos = a.t0 + t;
    uint32_t* row = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(S.codes) + head * S.code_slab_bytes) +
                    pos * words;
    store_codes(row, code, b, lane);
    if (lane == 0) reinterpret_cast<float*>(S.scale)[head * L.C + pos] = nrm;
    if (val) {
      float rr[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float cj = __shfl_sync(0xffffffffu, clane, code[j]);
        rr[j] = __fsub_rn(y[j], __fmul_rn(nrm, cj));
      }
      const float rn = __fsqrt_rn(tree128(__fmul_rn(rr[0], rr[0]), __fmul_rn(rr[1], rr[1]),
                                          __fmul_rn(rr[2], rr[2]), __fmul_rn(rr[3], rr[3])));
      if (lane == 0) reinterpret_cast<float*>(S.zero)[head * L.C + pos] = rn;
      uint32_t* sw = row + b * kD / 32;
      for (int w = 0; w < kD / 32; ++w) {
        uint32_t word = 0;
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
          const float4 s4 = reinterpret_cast<const float4*>(sk + (w * 32 + k) * kD)[lane];
          const float ti = tree128(__fmul_rn(s4.x, rr[0]), __fmul_rn(s4.y, rr[1]), __fmul_rn(s4.z, rr[2]),
                                   __fmul_rn(s4.w, rr[3]));
          word |= (uint32_t)(ti >= 0.0f) << k;
        }
        if (lane == 0) sw[w] = word;
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) flag(a.status, KVQ_DEV_NONFINITE);
}

// Reconstruction: k^ = H (n C[code]); v^ = H (n C[code] + fl32(kappa rn) sum_i s_i S_i),
// the sum over i in index order, kappa = sqrt(pi / 2) / D.
__global__ void __launch_bounds__(kQW * 32) kqv_dequant_kernel(KqvArgs a) {
  const Layout& L = a.L;
  const Side& S = L.side[a.which];
  const bool val = a.which == KVQ_VALUES;
  const int b = val ? S.bits - 1 : S.bits;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* C = reinterpret_cast<const float*>(S.lutf);
  const float clane = C[lane & ((1 << b) - 1)];
  const int words = val ? S.bits * kD / 32 : b * kD / 32;
  const int64_t rows = (int64_t)L.B * L.Hkv * a.n;
  for (int64_t r = (int64_t)blockIdx.x * kQW + warp; r < rows; r += (int64_t)gridDim.x * kQW) {
    const int64_t head = r / a.n, t = r % a.n, pos = a.t0 + t;
    const uint32_t* row = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(S.codes) +
                                                            head * S.code_slab_bytes) + pos * words;
    int code[4];
    load_codes(row, b, lane, code);
    const float nrm = reinterpret_cast<const float*>(S.scale)[head * L.C + pos];
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = __fmul_rn(nrm, __shfl_sync(0xffffffffu, clane, code[j]));
    if (val) {
      const float rs = __fmul_rn(kSketchScale, reinterpret_cast<const float*>(S.zero)[head * L.C + pos]);
      const uint32_t* sw = row + b * kD / 32;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int i = 0; i < kD; ++i) {
        const float4 s4 = reinterpret_cast<const float4*>(L.sketch + (int64_t)i * kD)[lane];
        const bool plus = (sw[i >> 5] >> (i & 31)) & 1u;
        acc[0] = plus ? __fadd_rn(acc[0], s4.x) : __fsub_rn(acc[0], s4.x);
        acc[1] = plus ? __fadd_rn(acc[1], s4.y) : __fsub_rn(acc[1], s4.y);
        acc[2] = plus ? __fadd_rn(acc[2], s4.z) : __fsub_rn(acc[2], s4.z);
        acc[3] = plus ? __fadd_rn(acc[3], s4.w) : __fsub_rn(acc[3], s4.w);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) y[j] = __fadd_rn(y[j], __fmul_rn(rs, acc[j]));
    }
    wht128_quad_unscaled(y, lane);
    const int64_t o = (head * a.n + t) * kD + 4 * lane;
#pragma unroll
    for (int j = 0; j < 4; ++j) store_elem(a.out, o + j, a.out_dtype, __fmul_rn(y[j], L.rot_scale));
  }
}

int kqv_grid(const Layout& L, int64_t n) {
  const int64_t rows = (int64_t)L.B * L.Hkv * n;
  const int64_t want = (rows + kQW - 1) / kQW, cap = (int64_t)device_sm_count() * 4;
  return (int)(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_quantize_kqv(const Layout& L, int which, const void* src, int64_t sb, int64_t sh,
                                int64_t st, int64_t t0, int64_t n, int32_t* d_status, cudaStream_t s) {
  KqvArgs a;
  a.L = L;
  a.which = which;
  a.src = src;
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.t0 = t0;
  a.n = n;
  a.out = nullptr;
  a.out_dtype = 0;
  a.status = d_status;
  const size_t smem = which == KVQ_VALUES ? (size_t)kD * kD * sizeof(float) : 0;
  cudaError_t e = cudaFuncSetAttribute(kqv_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(kD * kD * sizeof(float)));
  if (e != cudaSuccess) return e;
  kqv_quantize_kernel<<<kqv_grid(L, n), kQW * 32, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_kqv(const Layout& L, int which, int64_t t0, int64_t n, void* out, int out_dtype,
                                  cudaStream_t s) {
  KqvArgs a;
  a.L = L;
  a.which = which;
  a.src = nullptr;
  a.sb = a.sh = a.st = 0;
  a.t0 = t0;
  a.n = n;
  a.out = out;
  a.out_dtype = out_dtype;
  a.status = nullptr;
  kqv_dequant_kernel<<<kqv_grid(L, n), kQW * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
