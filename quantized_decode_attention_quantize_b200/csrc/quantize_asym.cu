// Append-time quantization for the asymmetric b-bit formats (b = 2, 4, 8): keys per
// channel over a token group, values per token ([KVQ] "Approach"; [K4V2]).  Same rules
// as the general quantize kernel, tiled for parallelism: a key group is split into
// blocks of 32 channels (the statistics of a channel never leave its block), values
// into blocks of 32 tokens.  Loads are 16-byte vectors, stores are packed words.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 256;
constexpr int kCB = 32;     // channels per key block
constexpr int kTB = 32;     // tokens per value block

struct AArgs {
  Layout L;
  const void* src;
  int64_t sb, sh, st, t0, n;
  int32_t* status;
};

// 8 consecutive elements (16 bytes for 16-bit sources, two 16-byte loads for fp32)
__device__ __forceinline__ void load8(const void* base, int64_t i, int dtype, float* out, int* bad) {
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
#pragma unroll
  for (int j = 0; j < 8; ++j) *bad |= !isfinite(out[j]);
}

__global__ void __launch_bounds__(kThreads) asym_keys_kernel(AArgs a) {
  __shared__ float tile[256 * kCB];
  __shared__ float pmin[8][kCB], pmax[8][kCB];
  __shared__ float sf[kCB], zf[kCB];
  __shared__ int flags;
  const Layout& L = a.L;
  const Side& S = L.side[KVQ_KEYS];
  const int D = L.D, g = L.g, bits = S.bits, maxc = (1 << bits) - 1;
  const int64_t ts = a.t0 + (int64_t)blockIdx.x * g;
  const int ln = (int)min((int64_t)g, a.t0 + a.n - ts);
  const int gi = (int)(ts / g);
  const int cb = blockIdx.y * kCB;
  const int head = blockIdx.z;
  const int b = head / L.Hkv, h = head % L.Hkv;
  if (threadIdx.x == 0) flags = 0;
  int bad = 0;
  // stage [ln][32] channels: 4 vectors of 8 per row
  for (int v = threadIdx.x; v < ln * (kCB / 8); v += kThreads) {
    const int r = v / (kCB / 8), c8 = (v % (kCB / 8)) * 8;
    const int64_t off = (int64_t)b * a.sb + (int64_t)h * a.sh + (ts - a.t0 + r) * a.st + cb + c8;
    load8(a.src, off, L.src_dtype, tile + r * kCB + c8, &bad);
  }
  __syncthreads();
  if (bad) atomicOr(&flags, 1);
  // per-channel min / max: 8 row slices per channel
  {
    const int c = threadIdx.x % kCB, slice = threadIdx.x / kCB;
    float mn = INFINITY, mx = -INFINITY;
    for (int r = slice; r < ln; r += 8) {
      const float x = tile[r * kCB + c];
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    pmin[slice][c] = mn;
    pmax[slice][c] = mx;
  }
  __syncthreads();
  if (threadIdx.x < kCB) {
    const int c = threadIdx.x;
    float mn = pmin[0][c], mx = pmax[0][c];
#pragma unroll
    for (int k = 1; k < 8; ++k) {
      mn = fminf(mn, pmin[k][c]);
      mx = fmaxf(mx, pmax[k][c]);
    }
    __half s, z;
    if (!asym_params(mn, mx, bits, &s, &z)) atomicOr(&flags, 2);
    const int64_t mi = ((int64_t)head * L.ng + gi) * D + cb + c;
    reinterpret_cast<__half*>(S.scale)[mi] = s;
    reinterpret_cast<__half*>(S.zero)[mi] = z;
    sf[c] = __half2float(s);
    zf[c] = __half2float(z);
  }
  __syncthreads();
  uint8_t* codes = reinterpret_cast<uint8_t*>(S.codes) + (int64_t)head * S.code_slab_bytes;
  if (bits == 8) {
    for (int v = threadIdx.x; v < ln * (kCB / 4); v += kThreads) {
      const int r = v / (kCB / 4), c4 = (v % (kCB / 4)) * 4;
      uint32_t w = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) w |= (uint32_t)asym_code(tile[r * kCB + c4 + j], sf[c4 + j], zf[c4 + j], maxc) << (8 * j);
      *reinterpret_cast<uint32_t*>(codes + (ts + r) * D + cb + c4) = w;
    }
  } else {
    const int per = 32 / bits, wpb = kCB / per, W = D / per;   // words per row-block, per row
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes) + ts * W + cb / per;
    for (int v = threadIdx.x; v < ln * wpb; v += kThreads) {
      const int r = v / wpb, w = v % wpb;
      uint32_t word = 0;
      for (int j = 0; j < per; ++j) {
        const int c = w * per + j;
        word |= (uint32_t)asym_code(tile[r * kCB + c], sf[c], zf[c], maxc) << (bits * j);
      }
      dst[r * W + w] = word;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && flags)
    flag(a.status, ((flags & 1) ? KVQ_DEV_NONFINITE : 0) | ((flags & 2) ? KVQ_DEV_RANGE : 0));
}

__global__ void __launch_bounds__(kThreads) asym_values_kernel(AArgs a) {
  extern __shared__ __align__(16) uint8_t vsm[];   // [kTB][D] codes
  __shared__ int flags;
  const Layout& L = a.L;
  const Side& S = L.side[KVQ_VALUES];
  const int D = L.D, bits = S.bits, maxc = (1 << bits) - 1;
  const int64_t tb = a.t0 + (int64_t)blockIdx.x * kTB;
  const int nt = (int)min((int64_t)kTB, a.t0 + a.n - tb);
  const int head = blockIdx.y;
  const int b = head / L.Hkv, h = head % L.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) flags = 0;
  __syncthreads();
  int bad = 0, rbad = 0;
  // one warp per token row: lane owns D / 32 consecutive channels (multiple of 8 when
  // D >= 256, else handled by the 8-wide loads of 32 / (D / 8) lanes)
  for (int r = warp; r < nt; r += kThreads / 32) {
    const int64_t off = (int64_t)b * a.sb + (int64_t)h * a.sh + (tb - a.t0 + r) * a.st;
    float x[8];
    const int nvec = D / 8;                  // 8-wide vectors per row (4..32)
    float mn = INFINITY, mx = -INFINITY;
    if (lane < nvec) {
      load8(a.src, off + 8 * lane, L.src_dtype, x, &bad);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        mn = fminf(mn, x[j]);
        mx = fmaxf(mx, x[j]);
      }
    }
    mn = warp_min(mn);
    mx = warp_max(mx);
    __half s, z;
    const bool ok = asym_params(mn, mx, bits, &s, &z);
    if (lane == 0) {
      rbad |= !ok;
      reinterpret_cast<__half*>(S.scale)[(int64_t)head * L.C + tb + r] = s;
      reinterpret_cast<__half*>(S.zero)[(int64_t)head * L.C + tb + r] = z;
    }
    if (lane < nvec) {
      const float sfv = __half2float(s), zfv = __half2float(z);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) lo |= (uint32_t)asym_code(x[j], sfv, zfv, maxc) << (8 * j);
#pragma unroll
      for (int j = 0; j < 4; ++j) hi |= (uint32_t)asym_code(x[4 + j], sfv, zfv, maxc) << (8 * j);
      *reinterpret_cast<uint2*>(vsm + r * D + 8 * lane) = make_uint2(lo, hi);
    }
  }
  if (bad) atomicOr(&flags, 1);
  if (rbad) atomicOr(&flags, 2);
  __syncthreads();
  uint8_t* codes = reinterpret_cast<uint8_t*>(S.codes) + (int64_t)head * S.code_slab_bytes;
  if (bits == 8) {
    for (int v = threadIdx.x; v < nt * D / 16; v += kThreads)
      reinterpret_cast<uint4*>(codes + tb * D)[v] = reinterpret_cast<const uint4*>(vsm)[v];
  } else {
    // pair layout: word w of pair u holds (16 / b) channels of token 2u (low half) and 2u + 1
    const int per = 16 / bits, WP = D / per, P = (nt + 1) / 2;
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes) + (tb / 2) * WP;
    for (int v = threadIdx.x; v < P * WP; v += kThreads) {
      const int u = v / WP, w = v % WP;
      uint32_t lo = 0, hi = 0;
      for (int j = 0; j < per; ++j) lo |= (uint32_t)vsm[(2 * u) * D + w * per + j] << (bits * j);
      if (2 * u + 1 < nt)
        for (int j = 0; j < per; ++j) hi |= (uint32_t)vsm[(2 * u + 1) * D + w * per + j] << (bits * j);
      dst[v] = lo | (hi << 16);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && flags)
    flag(a.status, ((flags & 1) ? KVQ_DEV_NONFINITE : 0) | ((flags & 2) ? KVQ_DEV_RANGE : 0));
}

}  // namespace

bool asym_fast_ok(const Layout& L, int which) {
  const Side& S = L.side[which];
  if (S.scheme != KVQ_ASYM) return false;
  if (which == KVQ_KEYS) return S.axis == KVQ_AXIS_CHANNEL && L.g <= 256 && L.D % kCB == 0;
  return S.axis == KVQ_AXIS_TOKEN && L.D >= 32 && L.D <= 256;
}

cudaError_t launch_quantize_asym(const Layout& L, int which, const void* src, int64_t sb, int64_t sh,
                                 int64_t st, int64_t t0, int64_t n, int32_t* d_status, cudaStream_t s) {
  AArgs a;
  a.L = L;
  a.src = src;
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.t0 = t0;
  a.n = n;
  a.status = d_status;
  if (which == KVQ_KEYS) {
    dim3 grid((unsigned)((n + L.g - 1) / L.g), L.D / kCB, L.B * L.Hkv);
    asym_keys_kernel<<<grid, kThreads, 0, s>>>(a);
  } else {
    dim3 grid((unsigned)((n + kTB - 1) / kTB), L.B * L.Hkv);
    asym_values_kernel<<<grid, kThreads, (size_t)kTB * L.D, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace kvq
