// Element-wise reconstruction of packed cache entries (dense part, before the sparse
// outlier overrides).  Used by the dequantize kernel and by the generic decode path.
//
//   SYM8  x^ = fl32(code * s)                      [AXES] "What rows and columns mean"
//   ASYM  x^ = fl32(code * s + z)   (exact product, one rounding)
//   NUQ   x^ = fl32(C[code] * s + z) (exact product, one rounding)  [KVQ] "Approach"
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// sin and cos of the RoPE angle pos * theta (radians, up to ~1e5 at long context): the
// angle is first reduced modulo 2 pi in double (one fused multiply-add with the double
// nearest to 2 pi; error ~1e-11 rad at 131k tokens), so that the library sincos works on
// |r| <= pi.
__device__ __forceinline__ void angle_sincos(double pos, double theta, float* s, float* c) {
  const double two_pi = 6.283185307179586;
  const double x = pos * theta;
  const double r = fma(-rint(x * (1.0 / two_pi)), two_pi, x);
  double sd, cd;
  sincos(r, &sd, &cd);
  *s = (float)sd;
  *c = (float)cd;
}

__device__ __forceinline__ float meta_f16(const void* p, int64_t i) {
  return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

// Dense reconstruction of packed row t (0 <= t < C), channel c of slab sl.
// Not valid for MIXED (see mixed_slot_value).
__device__ __forceinline__ float deq_dense(const Layout& L, int which, int64_t sl, int64_t t,
                                           int c) {
  const Side& S = L.side[which];
  const int D = L.D;
  const int64_t gi = t / L.g;
  switch (S.scheme) {
    case KVQ_NONE: {
      const uint8_t* base = reinterpret_cast<const uint8_t*>(S.codes) + sl * S.code_slab_bytes;
      return load_elem(base, t * D + c, L.src_dtype);
    }
    case KVQ_SYM8: {
      const int8_t* codes = reinterpret_cast<const int8_t*>(S.codes) + sl * S.code_slab_bytes;
      const float* sc = reinterpret_cast<const float*>(S.scale);
      float s;
      if (S.axis == KVQ_AXIS_TENSOR) s = sc[sl * L.ng + gi];
      else if (S.axis == KVQ_AXIS_TOKEN) s = sc[sl * L.C + t];
      else s = sc[(sl * L.ng + gi) * D + c];
      return __fmul_rn((float)codes[t * D + c], s);
    }
    case KVQ_ASYM: {
      const uint8_t* base = reinterpret_cast<const uint8_t*>(S.codes) + sl * S.code_slab_bytes;
      const int b = S.bits;
      uint32_t code;
      if (b == 8) {
        code = base[t * D + c];
      } else if (which == KVQ_KEYS) {
        const int per = 32 / b, W = D / per;
        const uint32_t w = reinterpret_cast<const uint32_t*>(base)[t * W + c / per];
        code = (w >> (b * (c % per))) & ((1u << b) - 1);
      } else {
        const int per = 16 / b, WP = D / per;
        const uint32_t w = reinterpret_cast<const uint32_t*>(base)[(t >> 1) * WP + c / per];
        code = (w >> (16 * (int)(t & 1) + b * (c % per))) & ((1u << b) - 1);
      }
      const int64_t mi = which == KVQ_KEYS ? (sl * L.ng + gi) * D + c : sl * L.C + t;
      return __fmaf_rn((float)code, meta_f16(S.scale, mi), meta_f16(S.zero, mi));
    }
    case KVQ_NUQ: {
      const uint32_t* base = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const uint8_t*>(S.codes) + sl * S.code_slab_bytes);
      const int W = 3 * D / 32;
      const uint32_t lo = (base[t * W + c / 16] >> (2 * (c % 16))) & 3u;
      const uint32_t hi = (base[t * W + D / 16 + c / 32] >> (c % 32)) & 1u;
      const float cv = __half2float(S.lut[lo | (hi << 2)]);
      const int64_t mi = which == KVQ_KEYS ? (sl * L.ng + gi) * D + c : sl * L.C + t;
      return __fmaf_rn(cv, meta_f16(S.scale, mi), meta_f16(S.zero, mi));
    }
  }
  return 0.0f;
}

// MIXED keys: reconstruction of storage slot j of packed row t.
__device__ __forceinline__ float mixed_slot_value(const Layout& L, int64_t sl, int64_t t, int j) {
  const int D = L.D, g = L.g, hi = L.mixed_hi, mid = L.mixed_mid, lo = L.mixed_lo;
  const int64_t gi = t / g;
  const int r = (int)(t % g);
  const uint8_t* gbase = reinterpret_cast<const uint8_t*>(L.side[0].codes) +
                         (sl * L.ng + gi) * (int64_t)L.mixed_group_bytes;
  if (j < hi) {
    const uint16_t bits = reinterpret_cast<const uint16_t*>(gbase)[r * hi + j];
    return L.src_dtype == KVQ_F16 ? half_bits_to_float(bits) : __uint_as_float((uint32_t)bits << 16);
  }
  uint32_t code;
  if (j < hi + mid) {
    const int e = j - hi;
    const uint32_t w = reinterpret_cast<const uint32_t*>(gbase + g * hi * 2)[r * (mid / 8) + e / 8];
    code = (w >> (4 * (e % 8))) & 15u;
  } else {
    const int e = j - hi - mid;
    const uint32_t w =
        reinterpret_cast<const uint32_t*>(gbase + g * hi * 2 + g * mid / 2)[r * (lo / 16) + e / 16];
    code = (w >> (2 * (e % 16))) & 3u;
  }
  const int64_t mi = (sl * L.ng + gi) * (D - hi) + (j - hi);
  return __fmaf_rn((float)code, meta_f16(L.side[0].scale, mi), meta_f16(L.side[0].zero, mi));
}

}  // namespace kvq
