// Key-only rotation ([K4V2] "Rotation Integration"; [TQ] KQV scheme): the orthonormal
// Sylvester-ordered Walsh-Hadamard transform y = H_D x / sqrt(D) of a D-vector held by
// one warp.  The stored format fixes its fp32 evaluation: the butterfly over strides
// h = 1, 2, ..., D/2, where pair (i, i + h) becomes (a + b, a - b) with each sum
// rounded, then one rounded product with c = fl32(1 / sqrt(D)).  Each output of a stage
// is one IEEE sum of two values of the previous stage, so any distribution of the
// elements over lanes gives the same bits; the explicit _rn intrinsics keep the
// compiler from contracting the final product into a later operation.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Lane holds x[j] = element lane + 32 j, j < NJ (D = 32 NJ).  Strides below 32 pair
// lanes (partner lane ^ h), the others pair registers (j, j + h / 32); both run in
// increasing order.  Ends with the product by c (c = 1 skips nothing: x * 1 is exact).
template <int NJ>
__device__ __forceinline__ void wht_strided(float* x, int lane, float c) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const bool upper = lane & h;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, x[j], h);
      x[j] = upper ? __fsub_rn(o, x[j]) : __fadd_rn(x[j], o);
    }
  }
#pragma unroll
  for (int hj = 1; hj < NJ; hj <<= 1) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      if (!(j & hj)) {
        const float a = x[j], b = x[j + hj];
        x[j] = __fadd_rn(a, b);
        x[j + hj] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) x[j] = __fmul_rn(x[j], c);
}

template <int NJ>
__device__ __forceinline__ void wht_tile_rows_t(float* tile, int rows, float c) {
  constexpr int D = 32 * NJ;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = warp; r < rows; r += nw) {
    float x[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) x[j] = tile[r * D + lane + 32 * j];
    wht_strided<NJ>(x, lane, c);
#pragma unroll
    for (int j = 0; j < NJ; ++j) tile[r * D + lane + 32 * j] = x[j];
  }
}

// Rotates rows [0, rows) of a [rows][D] fp32 shared-memory tile in place, one warp per
// row (warps w, w + nw, ...).  The caller synchronises before and after.
__device__ __forceinline__ void wht_tile_rows(float* tile, int rows, int D, float c) {
  switch (D) {
    case 32: wht_tile_rows_t<1>(tile, rows, c); break;
    case 64: wht_tile_rows_t<2>(tile, rows, c); break;
    case 128: wht_tile_rows_t<4>(tile, rows, c); break;
    default: wht_tile_rows_t<8>(tile, rows, c); break;
  }
}

// D = 128 with lane holding the four consecutive elements 4 lane .. 4 lane + 3: strides
// 1 and 2 within the lane, 4 .. 64 across lanes (partner lane ^ (h / 4)).  Without the
// final product (the caller folds c into its own scale).
__device__ __forceinline__ void wht128_quad_unscaled(float (&x)[4], int lane) {
  float a = x[0], b = x[1];
  x[0] = __fadd_rn(a, b);
  x[1] = __fsub_rn(a, b);
  a = x[2]; b = x[3];
  x[2] = __fadd_rn(a, b);
  x[3] = __fsub_rn(a, b);
  a = x[0]; b = x[2];
  x[0] = __fadd_rn(a, b);
  x[2] = __fsub_rn(a, b);
  a = x[1]; b = x[3];
  x[1] = __fadd_rn(a, b);
  x[3] = __fsub_rn(a, b);
#pragma unroll
  for (int hl = 1; hl < 32; hl <<= 1) {
    const bool upper = lane & hl;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, x[j], hl);
      x[j] = upper ? __fsub_rn(o, x[j]) : __fadd_rn(x[j], o);
    }
  }
}

}  // namespace kvq
