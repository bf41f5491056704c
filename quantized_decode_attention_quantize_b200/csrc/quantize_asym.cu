// Append-time quantization for the asymmetric b-bit formats (b = 2, 4, 8): keys per
// channel over a token group, values per token ([KVQ] "Approach"; [K4V2]).  Same rules
// as the general quantize kernel, laid out for latency: every thread issues all of its
// 16-byte loads first, keeps its values in registers, reduces with warp shuffles and
// packs its own codes into words, so an append of one group costs about one DRAM round
// trip.  Keys: a CTA takes 32 channels of one group (the statistics of a channel never
// leave it); values: a CTA takes 32 tokens.
#include "kvq_internal.cuh"
#include "wht.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 256;
constexpr int kCB = 32;     // channels per key block (64 when g <= 128 and D % 64 == 0)
constexpr int kMaxKeyRows = 4;   // rows per thread: g <= 256 over 64 row slices

struct AArgs {
  Layout L;
  const void* src;
  int64_t sb, sh, st, t0, n;
  int32_t* status;
  // paged destination: sequence b's group goes to pool block blocks[b] (slab blocks[b] *
  // Hkv + h of a layout with one group per slab); null for a contiguous cache
  const int32_t* blocks;
  int num_blocks;
};

// The destination slab of source head `head` = (b, h): the head itself, or in a paged
// pool the slab of its block (false, with KVQ_DEV_BOUNDS raised once, when the block id
// is out of range).
__device__ __forceinline__ bool dest_slab(const AArgs& a, int head, int b, int h, int64_t* slab) {
  if (a.blocks == nullptr) {
    *slab = head;
    return true;
  }
  const int blk = a.blocks[b];
  if (blk < 0 || blk >= a.num_blocks) {
    if (threadIdx.x == 0) flag(a.status, KVQ_DEV_BOUNDS);
    return false;
  }
  *slab = (int64_t)blk * a.L.Hkv + h;
  return true;
}

// Keys over a block of CB channels (32 or 64).  Thread t of the CTA: vector v = t mod VPC
// (channels cb + 8 v .. + 7, VPC = CB / 8) of rows rs, rs + NS, ... with rs = t / VPC over
// NS = 256 / VPC row slices (CB = 64: g <= 4 NS = 128; CB = 32: g <= 256).  The min / max
// of a channel meet first over the lanes of a warp with equal v, then over the 8 warps.
template <int CB>
__device__ __forceinline__ void asym_keys_block(const AArgs& a, int bx, int by, int bz) {
  constexpr int VPC = CB / 8, NS = kThreads / VPC;
  __shared__ float pmin[8][CB], pmax[8][CB];
  __shared__ float sf[CB], zf[CB], rf[CB];
  __shared__ int flags;
  const Layout& L = a.L;
  const Side& S = L.side[KVQ_KEYS];
  const int D = L.D, g = L.g, bits = S.bits;
  const int64_t ts = a.t0 + (int64_t)bx * g;
  const int ln = (int)min((int64_t)g, a.t0 + a.n - ts);
  const int gi = (int)(ts / g);
  const int cb = by * CB;
  const int head = bz;
  const int b = head / L.Hkv, h = head % L.Hkv;
  int64_t slab;
  if (!dest_slab(a, head, b, h, &slab)) return;   // uniform over the CTA
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int v = threadIdx.x % VPC, rs = threadIdx.x / VPC;
  if (threadIdx.x == 0) flags = 0;
  float x[kMaxKeyRows][8];
  const int64_t base = (int64_t)b * a.sb + (int64_t)h * a.sh + (ts - a.t0) * a.st + cb + 8 * v;
#pragma unroll
  for (int k = 0; k < kMaxKeyRows; ++k) {
    const int r = rs + NS * k;
#pragma unroll
    for (int c = 0; c < 8; ++c) x[k][c] = 0.0f;
    if (r < ln) load8(a.src, base + r * a.st, L.src_dtype, x[k]);
  }
  int bad = 0;
  float mn[8], mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    mn[c] = INFINITY;
    mx[c] = -INFINITY;
  }
  float fin = 0.0f;   // x * 0 is 0 for finite x and NaN otherwise
#pragma unroll
  for (int k = 0; k < kMaxKeyRows; ++k) {
    if (rs + NS * k < ln) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        fin = fmaf(x[k][c], 0.0f, fin);
        mn[c] = fminf(mn[c], x[k][c]);
        mx[c] = fmaxf(mx[c], x[k][c]);
      }
    }
  }
  bad = !(fin == 0.0f);
  // over the row slices of the warp (lanes with equal v)
#pragma unroll
  for (int o = VPC; o < 32; o <<= 1)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      mn[c] = fminf(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], o));
      mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], o));
    }
  __syncthreads();   // flags initialised
  if (lane < VPC) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      pmin[warp][8 * v + c] = mn[c];
      pmax[warp][8 * v + c] = mx[c];
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&flags, 1);
  __syncthreads();
  if (threadIdx.x < CB) {
    const int c = threadIdx.x;
    float m0 = pmin[0][c], m1 = pmax[0][c];
#pragma unroll
    for (int k = 1; k < 8; ++k) {
      m0 = fminf(m0, pmin[k][c]);
      m1 = fmaxf(m1, pmax[k][c]);
    }
    __half s, z;
    if (!asym_params(m0, m1, bits, &s, &z)) atomicOr(&flags, 2);
    const int64_t mi = (slab * L.ng + gi) * D + cb + c;
    reinterpret_cast<__half*>(S.scale)[mi] = s;
    reinterpret_cast<__half*>(S.zero)[mi] = z;
    sf[c] = __half2float(s);
    zf[c] = __half2float(z);
    rf[c] = __frcp_rn(sf[c]);
  }
  __syncthreads();
  float s8[8], z8[8], r8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    s8[c] = sf[8 * v + c];
    z8[c] = zf[8 * v + c];
    r8[c] = rf[8 * v + c];
  }
  uint8_t* codes = reinterpret_cast<uint8_t*>(S.codes) + slab * S.code_slab_bytes;
  const int rowb = D * bits / 8;   // bytes per code row
#pragma unroll
  for (int k = 0; k < kMaxKeyRows; ++k) {
    const int r = rs + NS * k;
    if (NS * k >= g) break;   // uniform: no slice has a row k
    const bool ok = r < ln;
    const uint2 w = pack8(x[k], s8, r8, z8, bits);
    uint8_t* row = codes + (ts + r) * rowb;
    if (bits == 8) {
      if (ok) *reinterpret_cast<uint2*>(row + cb + 8 * v) = w;
    } else if (bits == 4) {
      if (ok) *reinterpret_cast<uint32_t*>(row + (cb + 8 * v) / 2) = w.x;
    } else {   // 2-bit: 16 channels per word, this lane's 8 are its low (v even) or high half
      const uint32_t other = __shfl_xor_sync(0xffffffffu, w.x, 1);
      if (ok && (v & 1) == 0) *reinterpret_cast<uint32_t*>(row + (cb + 8 * v) / 4) = w.x | (other << 16);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && flags)
    flag(a.status, ((flags & 1) ? KVQ_DEV_NONFINITE : 0) | ((flags & 2) ? KVQ_DEV_RANGE : 0));
}

// Values.  LPT = D / 32 lanes per token, each holding 32 consecutive channels; a warp takes
// 32 / LPT consecutive tokens and the CTA's 8 warps value_tokens(D) = 256 / LPT tokens.
// A token's min / max meet over its LPT lanes; its scale / zero-point, computed by every
// lane of the token alike, is stored by the first.  In the pair layout (b < 8) the partner
// token of a pair sits in lane ^ LPT.
__host__ __device__ __forceinline__ int value_tokens(int D) { return 256 * 32 / D; }

__device__ __forceinline__ void asym_values_block(const AArgs& a, int bx, int by) {
  __shared__ int vflags;
  int& flags = vflags;
  const Layout& L = a.L;
  const Side& S = L.side[KVQ_VALUES];
  const int D = L.D, bits = S.bits;
  const int LPT = D / 32, TPC = value_tokens(D);
  const int64_t tb = a.t0 + (int64_t)bx * TPC;
  const int nt = (int)min((int64_t)TPC, a.t0 + a.n - tb);
  const int head = by;
  const int b = head / L.Hkv, h = head % L.Hkv;
  int64_t slab;
  if (!dest_slab(a, head, b, h, &slab)) return;   // uniform over the CTA
  const int lane = threadIdx.x & 31;
  const int t = threadIdx.x / LPT;   // token within the block
  const int part = threadIdx.x % LPT, c0 = 32 * part;
  const bool ok = t < nt;
  if (threadIdx.x == 0) flags = 0;
  float x[4][8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int c = 0; c < 8; ++c) x[k][c] = 0.0f;
    if (ok) load8(a.src, (int64_t)b * a.sb + (int64_t)h * a.sh + (tb - a.t0 + t) * a.st + c0 + 8 * k,
                  L.src_dtype, x[k]);
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
  for (int o = 1; o < LPT; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __syncthreads();   // flags initialised
  __half sh, zh;
  const bool good = asym_params(mn, mx, bits, &sh, &zh);
  if (ok && part == 0) {
    reinterpret_cast<__half*>(S.scale)[slab * L.C + tb + t] = sh;
    reinterpret_cast<__half*>(S.zero)[slab * L.C + tb + t] = zh;
  }
  const float sv = __half2float(sh), zv = __half2float(zh), rv = __frcp_rn(sv);
  float s8[8], z8[8], r8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    s8[j] = sv;
    z8[j] = zv;
    r8[j] = rv;
  }
  uint2 w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = pack8(x[k], s8, r8, z8, bits);
  uint8_t* codes = reinterpret_cast<uint8_t*>(S.codes) + slab * S.code_slab_bytes;
  if (bits == 8) {
    if (ok) {
#pragma unroll
      for (int k = 0; k < 4; ++k) *reinterpret_cast<uint2*>(codes + (tb + t) * D + c0 + 8 * k) = w[k];
    }
  } else {
    // pair layout: word j of pair u holds 16 / bits channels of token 2u (low half) and of
    // token 2u + 1 (high half); the lane's 32 channels are 2 bits half words
    uint32_t hw[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (bits == 2) {
        hw[k] = w[k].x & 0xffffu;
      } else {
        hw[2 * k] = w[k].x & 0xffffu;
        hw[2 * k + 1] = w[k].x >> 16;
      }
    }
    const int nh = 2 * bits;   // half words of the lane
    const bool even = (tb + t) % 2 == 0;
    const bool lone = even && t + 1 >= nt;   // no partner: its half stays zero
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes) + ((tb + t) / 2) * (D * bits / 16) + part * nh;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < nh) {
        const uint32_t other = __shfl_xor_sync(0xffffffffu, hw[k], LPT);
        if (ok && even) dst[k] = hw[k] | ((lone ? 0u : other) << 16);
      }
    }
  }
  if (__any_sync(0xffffffffu, ok && (!(fin == 0.0f))) && lane == 0) atomicOr(&flags, 1);
  if (__any_sync(0xffffffffu, ok && !good) && lane == 0) atomicOr(&flags, 2);
  __syncthreads();
  if (threadIdx.x == 0 && flags)
    flag(a.status, ((flags & 1) ? KVQ_DEV_NONFINITE : 0) | ((flags & 2) ? KVQ_DEV_RANGE : 0));
}

// Keys of a rotating format (D = 128, g <= 128): a CTA takes one whole group, since the
// Walsh-Hadamard transform mixes all channels of a row.  Warp w holds rows w, w + 8, ...
// (16 at most); lane l holds channels 4 l .. 4 l + 3 of each, loaded as one 8-byte (16-bit
// source) or 16-byte (fp32) vector.  Rows are transformed in registers (strides 1, 2 in
// the lane, 4 .. 64 across lanes, then the product with fl32(1/sqrt(D))), the per-channel
// min / max go through shared memory across the 8 warps, and the codes of four channels
// are packed by the lane and merged with its neighbours' by shuffles into row words.
constexpr int kRotRows = 16;
__device__ __forceinline__ void asym_keys_rot_block(const AArgs& a, int bx, int head) {
  __shared__ float pmin[8][128], pmax[8][128];
  __shared__ float sf[128], zf[128];
  __shared__ int flags;
  const Layout& L = a.L;
  const Side& S = L.side[KVQ_KEYS];
  const int g = L.g, bits = S.bits;
  const int64_t ts = a.t0 + (int64_t)bx * g;
  const int ln = (int)min((int64_t)g, a.t0 + a.n - ts);
  const int gi = (int)(ts / g);
  const int b = head / L.Hkv, h = head % L.Hkv;
  int64_t slab;
  if (!dest_slab(a, head, b, h, &slab)) return;   // uniform over the CTA
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) flags = 0;
  float x[kRotRows][4];
  const int64_t base = (int64_t)b * a.sb + (int64_t)h * a.sh + (ts - a.t0) * a.st + 4 * lane;
#pragma unroll
  for (int k = 0; k < kRotRows; ++k) {
    const int r = warp + 8 * k;
    if (r < ln) {
      const int64_t i = base + r * a.st;
      if (L.src_dtype == KVQ_F32) {
        const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.src) + i);
        x[k][0] = v.x; x[k][1] = v.y; x[k][2] = v.z; x[k][3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a.src) + i);
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (L.src_dtype == KVQ_F16) {
            x[k][2 * j] = half_bits_to_float((uint16_t)(w[j] & 0xffffu));
            x[k][2 * j + 1] = half_bits_to_float((uint16_t)(w[j] >> 16));
          } else {
            x[k][2 * j] = __uint_as_float(w[j] << 16);
            x[k][2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
          }
        }
      }
    } else {
      x[k][0] = x[k][1] = x[k][2] = x[k][3] = 0.0f;
    }
  }
  int bad = 0;
  float mn[4], mx[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    mn[j] = INFINITY;
    mx[j] = -INFINITY;
  }
#pragma unroll
  for (int k = 0; k < kRotRows; ++k) {
    if (warp + 8 * k < ln) {   // warp-uniform: the shuffles of the transform see all lanes
#pragma unroll
      for (int j = 0; j < 4; ++j) bad |= !isfinite(x[k][j]);
      wht128_quad_unscaled(x[k], lane);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[k][j] = __fmul_rn(x[k][j], L.rot_scale);
        mn[j] = fminf(mn[j], x[k][j]);
        mx[j] = fmaxf(mx[j], x[k][j]);
      }
    }
  }
  __syncthreads();   // flags initialised
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    pmin[warp][4 * lane + j] = mn[j];
    pmax[warp][4 * lane + j] = mx[j];
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&flags, 1);
  __syncthreads();
  if (threadIdx.x < 128) {
    const int c = threadIdx.x;
    float m0 = pmin[0][c], m1 = pmax[0][c];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      m0 = fminf(m0, pmin[w][c]);
      m1 = fmaxf(m1, pmax[w][c]);
    }
    __half sh, zh;
    if (!asym_params(m0, m1, bits, &sh, &zh)) atomicOr(&flags, 2);
    const int64_t mi = (slab * L.ng + gi) * 128 + c;
    reinterpret_cast<__half*>(S.scale)[mi] = sh;
    reinterpret_cast<__half*>(S.zero)[mi] = zh;
    sf[c] = __half2float(sh);
    zf[c] = __half2float(zh);
  }
  __syncthreads();
  float s4[4], z4[4], r4[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    s4[j] = sf[4 * lane + j];
    z4[j] = zf[4 * lane + j];
    r4[j] = __frcp_rn(s4[j]);
  }
  const int maxc = (1 << bits) - 1;
  uint8_t* codes = reinterpret_cast<uint8_t*>(S.codes) + slab * S.code_slab_bytes;
  const int rowb = 128 * bits / 8;
#pragma unroll
  for (int k = 0; k < kRotRows; ++k) {
    const int r = warp + 8 * k;
    if (r < ln) {   // warp-uniform
      uint32_t v = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) v |= (uint32_t)asym_code_r(x[k][j], s4[j], r4[j], z4[j], maxc) << (bits * j);
      uint8_t* row = codes + (ts + r) * rowb;
      if (bits == 8) {
        *reinterpret_cast<uint32_t*>(row + 4 * lane) = v;
      } else if (bits == 4) {   // word lane / 2: this lane's 16 bits at 16 (lane & 1)
        v <<= 16 * (lane & 1);
        v |= __shfl_xor_sync(0xffffffffu, v, 1);
        if ((lane & 1) == 0) reinterpret_cast<uint32_t*>(row)[lane >> 1] = v;
      } else {                  // 2-bit: word lane / 4, this lane's 8 bits at 8 (lane & 3)
        v <<= 8 * (lane & 3);
        v |= __shfl_xor_sync(0xffffffffu, v, 1);
        v |= __shfl_xor_sync(0xffffffffu, v, 2);
        if ((lane & 3) == 0) reinterpret_cast<uint32_t*>(row)[lane >> 2] = v;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && flags)
    flag(a.status, ((flags & 1) ? KVQ_DEV_NONFINITE : 0) | ((flags & 2) ? KVQ_DEV_RANGE : 0));
}

__global__ void __launch_bounds__(kThreads) asym_keys_rot_kernel(AArgs a) {
  asym_keys_rot_block(a, blockIdx.x, blockIdx.y);
}

// A rotating format's append in one launch: blocks [0, nk) take one key group each
// (group, head), the rest are value blocks.
__global__ void __launch_bounds__(kThreads) asym_kv_rot_kernel(AArgs ak, AArgs av, int kgx, int nk,
                                                               int vgx) {
  const int b = blockIdx.x;
  if (b < nk) {
    asym_keys_rot_block(ak, b % kgx, b / kgx);
  } else {
    const int v = b - nk;
    asym_values_block(av, v % vgx, v / vgx);
  }
}

template <int CB>
// Four CTAs per SM, as asym_kv_kernel.
__global__ void __launch_bounds__(kThreads, 4) asym_keys_kernel(AArgs a) {
  asym_keys_block<CB>(a, blockIdx.x, blockIdx.y, blockIdx.z);
}

__global__ void __launch_bounds__(kThreads, 4) asym_values_kernel(AArgs a) {
  asym_values_block(a, blockIdx.x, blockIdx.y);
}

// Keys and values of one append in one launch: blocks [0, nk) are key blocks
// (group, channel block, head), the rest value blocks (token block, head).
// Four CTAs per SM (64 registers): a full-cache quantize streams at about 1.7 TB/s against
// 1.15 TB/s with two CTAs per SM (92 registers).
template <int CB>
__global__ void __launch_bounds__(kThreads, 4) asym_kv_kernel(AArgs ak, AArgs av, int kgx, int kgy, int nk,
                                                           int vgx) {
  griddep_wait();   // launched with launch_pdl: earlier work on the stream is complete
  griddep_launch_dependents();
  const int b = blockIdx.x;
  if (b < nk) {
    asym_keys_block<CB>(ak, b % kgx, (b / kgx) % kgy, b / (kgx * kgy));
  } else {
    const int v = b - nk;
    asym_values_block(av, v % vgx, v / vgx);
  }
}

// Channels per key block: 64 halves the blocks and the shuffle levels of the min / max
// when its 32 row slices cover the group.
int key_cb(const Layout& L) { return (L.g <= 128 && L.D % 64 == 0) ? 64 : kCB; }

}  // namespace

bool asym_fast_ok(const Layout& L, int which) {
  const Side& S = L.side[which];
  if (S.scheme != KVQ_ASYM) return false;
  if (which == KVQ_KEYS) {
    if (S.axis != KVQ_AXIS_CHANNEL) return false;
    if (L.k_rotate) return L.D == 128 && L.g <= 8 * kRotRows;   // whole rows per CTA
    return L.g <= 64 * kMaxKeyRows && L.D % kCB == 0;
  }
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
  a.blocks = nullptr;
  a.num_blocks = 0;
  if (which == KVQ_KEYS && L.k_rotate) {
    dim3 grid((unsigned)((n + L.g - 1) / L.g), L.B * L.Hkv);
    asym_keys_rot_kernel<<<grid, kThreads, 0, s>>>(a);
  } else if (which == KVQ_KEYS) {
    const int cb = key_cb(L);
    dim3 grid((unsigned)((n + L.g - 1) / L.g), L.D / cb, L.B * L.Hkv);
    if (cb == 64) asym_keys_kernel<64><<<grid, kThreads, 0, s>>>(a);
    else asym_keys_kernel<kCB><<<grid, kThreads, 0, s>>>(a);
  } else {
    const int tpc = value_tokens(L.D);
    dim3 grid((unsigned)((n + tpc - 1) / tpc), L.B * L.Hkv);
    asym_values_kernel<<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace kvq

namespace kvq {

cudaError_t launch_quantize_asym_kv(const Layout& L, const void* ksrc, const void* vsrc, int64_t sb,
                                    int64_t sh, int64_t st, int64_t t0, int64_t n, int32_t* d_status,
                                    cudaStream_t s, const int32_t* blocks, int num_blocks) {
  AArgs ak, av;
  ak.blocks = av.blocks = blocks;
  ak.num_blocks = av.num_blocks = num_blocks;
  ak.L = av.L = L;
  ak.src = ksrc;
  av.src = vsrc;
  ak.sb = av.sb = sb;
  ak.sh = av.sh = sh;
  ak.st = av.st = st;
  ak.t0 = av.t0 = t0;
  ak.n = av.n = n;
  ak.status = av.status = d_status;
  const int cb = key_cb(L);
  const int kgx = (int)((n + L.g - 1) / L.g), kgy = L.k_rotate ? 1 : L.D / cb, heads = L.B * L.Hkv;
  const int vgx = (int)((n + value_tokens(L.D) - 1) / value_tokens(L.D));
  const int64_t nk = (int64_t)kgx * kgy * heads, nv = (int64_t)vgx * heads;
  if (nk + nv > 0x7fffffff) return cudaErrorInvalidConfiguration;
  if (L.k_rotate)
    asym_kv_rot_kernel<<<(unsigned)(nk + nv), kThreads, 0, s>>>(ak, av, kgx, (int)nk, vgx);
  else
    return launch_pdl(cb == 64 ? asym_kv_kernel<64> : asym_kv_kernel<kCB>, dim3((unsigned)(nk + nv)),
                      dim3(kThreads), 0, s, ak, av, kgx, kgy,
                      (int)nk, vgx);
  return cudaGetLastError();
}

}  // namespace kvq
