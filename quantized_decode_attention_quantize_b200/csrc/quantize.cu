// Append-time quantization of K / V token groups into the packed cache.
//
// One CTA per (token group, kv head, batch).  The group's n <= g rows of D source
// values are staged in shared memory as fp32 (128-bit coalesced loads; key rows of a
// rotating format are then Walsh-Hadamard transformed in place), the group
// statistics are reduced (per-channel min/max or absmax by column threads, per-token
// by warp shuffles), metadata are rounded as the format states, and codes are
// encoded and packed into 32-bit words that are stored coalesced.
//
// Rules: [AXES] "What rows and columns mean" (symmetric INT8 and its three
// groupings); [KVQ] "Approach" (keys per channel before RoPE, values per token, nuq3
// with per-vector dense-and-sparse outliers); [MIX] Figure 3 (salience tiers);
// [K4V2] (more bits for keys than values).
#include "kvq_internal.cuh"
#include "wht.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 256;

struct QArgs {
  Layout L;
  int which;
  const void* src;
  int64_t sb, sh, st, t0, n;
  int32_t* status;
};

struct QSmem {
  float* tile;      // [g][D]
  float* sf;        // [256] per channel / slot / row scale (fp32 value)
  float* zf;        // [256]
  float* mids;      // [8]
  uint8_t* codes;   // [g][D]
  uint32_t* omask;  // [g][D/32]
  int* rowptr;      // [g + 1]
  int* flag;        // [1]
};

__device__ __forceinline__ int64_t slab_of(const Layout& L) {
  return (int64_t)blockIdx.z * L.Hkv + blockIdx.y;
}

// ---- staging --------------------------------------------------------------------
__device__ void load_tile(const QArgs& a, int ln, int64_t src_row0, float* tile, int* bad) {
  const Layout& L = a.L;
  const int D = L.D;
  const int esz = L.raw_bytes;
  const int per = 16 / esz;                      // elements per 16-byte vector
  const int vecs = ln * D / per;
  const char* base = reinterpret_cast<const char*>(a.src);
  int local_bad = 0;
  for (int i = threadIdx.x; i < vecs; i += blockDim.x) {
    const int e = i * per;
    const int r = e / D, c = e % D;
    const int64_t off = (int64_t)blockIdx.z * a.sb + (int64_t)blockIdx.y * a.sh +
                        (src_row0 + r) * a.st + c;
    const uint4 v = *reinterpret_cast<const uint4*>(base + off * esz);
    float* dst = tile + r * D + c;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if (L.src_dtype == KVQ_F32) {
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = __uint_as_float(w[j]);
    } else if (L.src_dtype == KVQ_F16) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        dst[2 * j] = half_bits_to_float((uint16_t)(w[j] & 0xffffu));
        dst[2 * j + 1] = half_bits_to_float((uint16_t)(w[j] >> 16));
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        dst[2 * j] = __uint_as_float(w[j] << 16);
        dst[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    }
    for (int j = 0; j < per; ++j) local_bad |= !isfinite(dst[j]);
  }
  if (local_bad) atomicOr(bad, 1);
}

__device__ __forceinline__ void store_raw(void* base, int64_t idx, int dtype, float v) {
  // exact: v is a value of the source dtype
  store_elem(base, idx, dtype, v);
}

// ---- symmetric INT8 ---------------------------------------------------------------
__device__ __forceinline__ float sym8_scale(float m) {
  return m == 0.0f ? 1.0f : __fdiv_rn(m, 127.0f);
}
__device__ __forceinline__ int8_t sym8_code(float x, float s) {
  float r = rintf(__fdiv_rn(x, s));
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return (int8_t)(int)r;
}

__device__ void do_sym8(const QArgs& a, const QSmem& sm, int ln, int64_t ts, int gi) {
  const Layout& L = a.L;
  const Side& S = L.side[a.which];
  const int D = L.D;
  const int64_t sl = slab_of(L);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  float* scale = reinterpret_cast<float*>(S.scale);
  if (S.axis == KVQ_AXIS_TENSOR) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < ln * D; i += blockDim.x) m = fmaxf(m, fabsf(sm.tile[i]));
    m = warp_max(m);
    if (lane == 0) sm.sf[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      float mm = 0.0f;
      for (int w = 0; w < nw; ++w) mm = fmaxf(mm, sm.sf[w]);
      const float s = sym8_scale(mm);
      sm.zf[0] = s;
      scale[sl * L.ng + gi] = s;
    }
    __syncthreads();
    const float s = sm.zf[0];
    for (int i = threadIdx.x; i < ln * D; i += blockDim.x) sm.codes[i] = (uint8_t)sym8_code(sm.tile[i], s);
  } else if (S.axis == KVQ_AXIS_TOKEN) {
    for (int r = warp; r < ln; r += nw) {
      float m = 0.0f;
      for (int c = lane; c < D; c += 32) m = fmaxf(m, fabsf(sm.tile[r * D + c]));
      m = warp_max(m);
      const float s = sym8_scale(m);
      if (lane == 0) scale[sl * L.C + ts + r] = s;
      for (int c = lane; c < D; c += 32) sm.codes[r * D + c] = (uint8_t)sym8_code(sm.tile[r * D + c], s);
    }
  } else {
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      float m = 0.0f;
      for (int r = 0; r < ln; ++r) m = fmaxf(m, fabsf(sm.tile[r * D + c]));
      const float s = sym8_scale(m);
      sm.sf[c] = s;
      scale[(sl * L.ng + gi) * D + c] = s;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < ln * D; i += blockDim.x) sm.codes[i] = (uint8_t)sym8_code(sm.tile[i], sm.sf[i % D]);
  }
  __syncthreads();
  // int8 rows [ts, ts + ln), 16 bytes per store
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(S.codes) + sl * S.code_slab_bytes + ts * D);
  const uint4* srcv = reinterpret_cast<const uint4*>(sm.codes);
  for (int i = threadIdx.x; i < ln * D / 16; i += blockDim.x) dst[i] = srcv[i];
}

// ---- asymmetric b-bit ---------------------------------------------------------------
__device__ void do_asym(const QArgs& a, const QSmem& sm, int ln, int64_t ts, int gi) {
  const Layout& L = a.L;
  const Side& S = L.side[a.which];
  const int D = L.D, bits = S.bits, maxc = (1 << bits) - 1;
  const int64_t sl = slab_of(L);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __half* hs = reinterpret_cast<__half*>(S.scale);
  __half* hz = reinterpret_cast<__half*>(S.zero);
  int range_bad = 0;
  if (a.which == KVQ_KEYS) {  // per channel over the group
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      float mn = sm.tile[c], mx = mn;
      for (int r = 1; r < ln; ++r) {
        const float x = sm.tile[r * D + c];
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
      __half s, z;
      range_bad |= !asym_params(mn, mx, bits, &s, &z);
      hs[(sl * L.ng + gi) * D + c] = s;
      hz[(sl * L.ng + gi) * D + c] = z;
      sm.sf[c] = __half2float(s);
      sm.zf[c] = __half2float(z);
    }
  } else {  // per token row over the D channels
    for (int r = warp; r < ln; r += nw) {
      float mn = INFINITY, mx = -INFINITY;
      for (int c = lane; c < D; c += 32) {
        const float x = sm.tile[r * D + c];
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
      mn = warp_min(mn);
      mx = warp_max(mx);
      __half s, z;
      const bool ok = asym_params(mn, mx, bits, &s, &z);
      if (lane == 0) {
        range_bad |= !ok;
        hs[sl * L.C + ts + r] = s;
        hz[sl * L.C + ts + r] = z;
        sm.sf[r] = __half2float(s);
        sm.zf[r] = __half2float(z);
      }
    }
  }
  if (range_bad) atomicOr(sm.flag, 2);
  __syncthreads();
  const bool per_channel = a.which == KVQ_KEYS;
  auto code_at = [&](int r, int c) -> uint32_t {
    const int m = per_channel ? c : r;
    return (uint32_t)asym_code(sm.tile[r * D + c], sm.sf[m], sm.zf[m], maxc);
  };
  uint8_t* cbase = reinterpret_cast<uint8_t*>(S.codes) + sl * S.code_slab_bytes;
  if (bits == 8) {
    for (int i = threadIdx.x; i < ln * D / 4; i += blockDim.x) {
      const int e = i * 4, r = e / D, c = e % D;
      uint32_t w = 0;
      for (int j = 0; j < 4; ++j) w |= code_at(r, c + j) << (8 * j);
      reinterpret_cast<uint32_t*>(cbase + (ts + r) * D + c)[0] = w;
    }
  } else if (a.which == KVQ_KEYS) {  // row layout
    const int per = 32 / bits, W = D / per;
    uint32_t* dst = reinterpret_cast<uint32_t*>(cbase) + ts * W;
    for (int i = threadIdx.x; i < ln * W; i += blockDim.x) {
      const int r = i / W, w = i % W;
      uint32_t word = 0;
      for (int j = 0; j < per; ++j) word |= code_at(r, w * per + j) << (bits * j);
      dst[i] = word;
    }
  } else {  // pair layout
    const int per = 16 / bits, WP = D / per, P = (ln + 1) / 2;
    uint32_t* dst = reinterpret_cast<uint32_t*>(cbase) + (ts / 2) * WP;
    for (int i = threadIdx.x; i < P * WP; i += blockDim.x) {
      const int u = i / WP, w = i % WP;
      uint32_t lo = 0, hi = 0;
      for (int j = 0; j < per; ++j) lo |= code_at(2 * u, w * per + j) << (bits * j);
      if (2 * u + 1 < ln)
        for (int j = 0; j < per; ++j) hi |= code_at(2 * u + 1, w * per + j) << (bits * j);
      dst[i] = lo | (hi << 16);
    }
  }
}

// ---- nuq3 with per-vector outliers ------------------------------------------------------
__device__ void pack_3bit_rows(const QArgs& a, const QSmem& sm, int ln, int64_t ts) {
  const Layout& L = a.L;
  const Side& S = L.side[a.which];
  const int D = L.D, W = 3 * D / 32, W2 = D / 16;
  const int64_t sl = slab_of(L);
  uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(S.codes) + sl * S.code_slab_bytes) + ts * W;
  for (int i = threadIdx.x; i < ln * W; i += blockDim.x) {
    const int r = i / W, w = i % W;
    uint32_t word = 0;
    if (w < W2) {
      for (int j = 0; j < 16; ++j) word |= (uint32_t)(sm.codes[r * D + w * 16 + j] & 3) << (2 * j);
    } else {
      const int w1 = w - W2;
      for (int j = 0; j < 32; ++j) word |= (uint32_t)(sm.codes[r * D + w1 * 32 + j] >> 2) << j;
    }
    dst[i] = word;
  }
}

__device__ void do_nuq(const QArgs& a, const QSmem& sm, int ln, int64_t ts, int gi) {
  const Layout& L = a.L;
  const Side& S = L.side[a.which];
  const int D = L.D, k = S.nout, g = L.g;
  const int64_t sl = slab_of(L);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __half* hs = reinterpret_cast<__half*>(S.scale);
  __half* hz = reinterpret_cast<__half*>(S.zero);
  if (threadIdx.x < 7) {
    const float c0 = __half2float(S.lut[threadIdx.x]), c1 = __half2float(S.lut[threadIdx.x + 1]);
    sm.mids[threadIdx.x] = __fmul_rn(__fadd_rn(c0, c1), 0.5f);
  }
  const int mw = D / 32;
  for (int i = threadIdx.x; i < ln * mw; i += blockDim.x) sm.omask[i] = 0u;
  __syncthreads();
  int range_bad = 0;
  if (a.which == KVQ_KEYS) {
    // Two threads per channel (adjacent lanes): the even one scans rows [0, h), the odd one
    // rows [h, ln), h = ceil(ln / 2).  Each keeps its own top-k |x| (ties to the lower row:
    // a later row displaces an entry only with a strictly larger magnitude); the global
    // top-k is the top-k of the 2k candidates, rows of the even thread first on ties.
    const int half = threadIdx.x & 1, h2 = (ln + 1) / 2;
    const int r_lo = half ? h2 : 0, r_hi = half ? ln : h2;
    for (int c = threadIdx.x >> 1; c < D; c += blockDim.x >> 1) {
      float ba[8];
      int bi[8];
      int cnt = 0;
      for (int r = r_lo; r < r_hi; ++r) {
        const float v = fabsf(sm.tile[r * D + c]);
        int pos = cnt;
        while (pos > 0 && v > ba[pos - 1]) --pos;
        if (pos < k) {
          const int last = cnt < k ? cnt : k - 1;
          for (int j = last; j > pos; --j) {
            ba[j] = ba[j - 1];
            bi[j] = bi[j - 1];
          }
          ba[pos] = v;
          bi[pos] = r;
          if (cnt < k) ++cnt;
        }
      }
      // merge with the partner's list: candidates of the even thread first
      const int pcnt = __shfl_xor_sync(0xffffffffu, cnt, 1);
      float ca[16];
      int ci[16];
      int n_c = 0;
      for (int j = 0; j < 8; ++j) {
        const float pv = __shfl_xor_sync(0xffffffffu, j < cnt ? ba[j] : 0.0f, 1);
        const int pi = __shfl_xor_sync(0xffffffffu, j < cnt ? bi[j] : 0, 1);
        if (half == 0 && j < cnt) { ca[n_c] = ba[j]; ci[n_c] = bi[j]; ++n_c; }
        if (half == 1 && j < pcnt) { ca[n_c] = pv; ci[n_c] = pi; ++n_c; }
      }
      for (int j = 0; j < 8; ++j) {
        const float pv = __shfl_xor_sync(0xffffffffu, j < cnt ? ba[j] : 0.0f, 1);
        const int pi = __shfl_xor_sync(0xffffffffu, j < cnt ? bi[j] : 0, 1);
        if (half == 0 && j < pcnt) { ca[n_c] = pv; ci[n_c] = pi; ++n_c; }
        if (half == 1 && j < cnt) { ca[n_c] = ba[j]; ci[n_c] = bi[j]; ++n_c; }
      }
      // top-k of the candidates in order (candidates of lower rows come first, so a
      // strict comparison keeps the lower row on ties)
      cnt = 0;
      for (int x = 0; x < n_c; ++x) {
        const float v = ca[x];
        int pos = cnt;
        while (pos > 0 && v > ba[pos - 1]) --pos;
        if (pos < k) {
          const int last = cnt < k ? cnt : k - 1;
          for (int j = last; j > pos; --j) {
            ba[j] = ba[j - 1];
            bi[j] = bi[j - 1];
          }
          ba[pos] = v;
          bi[pos] = ci[x];
          if (cnt < k) ++cnt;
        }
      }
      float mn = INFINITY, mx = -INFINITY;
      for (int r = r_lo; r < r_hi; ++r) {
        bool out = false;
        for (int j = 0; j < cnt; ++j) out |= (bi[j] == r);
        if (!out) {
          const float x = sm.tile[r * D + c];
          mn = fminf(mn, x);
          mx = fmaxf(mx, x);
        }
      }
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      if (!(mn <= mx)) mn = mx = 0.0f;
      __half s, z;
      const bool ok = nuq_params(mn, mx, &s, &z);
      if (half == 0) {
        for (int j = 0; j < cnt; ++j) atomicOr(&sm.omask[bi[j] * mw + c / 32], 1u << (c % 32));
        range_bad |= !ok;
        hs[(sl * L.ng + gi) * D + c] = s;
        hz[(sl * L.ng + gi) * D + c] = z;
      }
      const float sf = __half2float(s), zf = __half2float(z);
      for (int r = r_lo; r < r_hi; ++r) {
        const float x = fminf(fmaxf(sm.tile[r * D + c], mn), mx);
        sm.codes[r * D + c] = (uint8_t)nuq_code(x, sf, zf, sm.mids);
      }
    }
    __syncthreads();
    if (k > 0) {
      // CSR by token row: per-row counts, a block-wide exclusive scan, then each row's
      // entries in channel order
      int* cnt_scan = sm.rowptr;   // [g + 1]
      {
        const int r = threadIdx.x;   // g <= blockDim.x
        int cr = 0;
        if (r < ln)
          for (int w = 0; w < mw; ++w) cr += __popc(sm.omask[r * mw + w]);
        // inclusive scan within the warp, then across warps
        int incl = cr;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        __shared__ int wsum[kThreads / 32];
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; ++w) base += wsum[w];
        if (r < g) cnt_scan[r + 1] = base + incl;
        if (r == 0) cnt_scan[0] = 0;
      }
      __syncthreads();
      int32_t* rp = L.k_out_rowptr + (sl * L.ng + gi) * (g + 1);
      for (int r = threadIdx.x; r <= g; r += blockDim.x) rp[r] = sm.rowptr[r];
      uint8_t* col = L.k_out_col + (sl * L.ng + gi) * (int64_t)D * k;
      __half* val = L.k_out_val + (sl * L.ng + gi) * (int64_t)D * k;
      int vbad = 0;
      for (int r = threadIdx.x; r < ln; r += blockDim.x) {
        int e = sm.rowptr[r];
        for (int w = 0; w < mw; ++w) {
          uint32_t bitsw = sm.omask[r * mw + w];
          while (bitsw) {
            const int b = __ffs(bitsw) - 1;
            bitsw &= bitsw - 1;
            const int c = w * 32 + b;
            const __half hv = __float2half_rn(sm.tile[r * D + c]);
            vbad |= !isfinite(__half2float(hv));
            col[e] = (uint8_t)c;
            val[e] = hv;
            ++e;
          }
        }
      }
      for (int e = sm.rowptr[g] + threadIdx.x; e < D * k; e += blockDim.x) {
        col[e] = 0;
        val[e] = __ushort_as_half((unsigned short)0);
      }
      if (vbad) atomicOr(sm.flag, 2);
    }
  } else {
    // Value rows: each half warp takes one row (lanes 16 h .. 16 h + 15, channels
    // (lane & 15) + 16 j), so a warp works on two rows with one instruction stream and
    // every reduction is four shuffle levels.
    const int hl = lane & 15, hw = lane >> 4;
    const int nj = D / 16;
    const int rows_per_pass = 2 * nw;
    const int passes = (ln + rows_per_pass - 1) / rows_per_pass;
    for (int pass = 0; pass < passes; ++pass) {
      const int r = pass * rows_per_pass + 2 * warp + hw;
      const bool live = r < ln;
      const float* row = sm.tile + (live ? r : 0) * D;
      uint32_t chosen = 0;           // bit j: channel hl + 16 j chosen
      int sel[8];
      for (int e = 0; e < k; ++e) {
        float ba = -1.0f;
        int bc = 1 << 30;
        for (int j = 0; j < nj; ++j) {
          const int c = hl + 16 * j;
          if (!(chosen & (1u << j))) {
            const float v = fabsf(row[c]);
            if (v > ba) { ba = v; bc = c; }
          }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          const float oa = __shfl_xor_sync(0xffffffffu, ba, o);
          const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
          if (oa > ba || (oa == ba && oc < bc)) { ba = oa; bc = oc; }
        }
        sel[e] = bc;
        if ((bc & 15) == hl) chosen |= 1u << (bc >> 4);
      }
      // ascending channel order
      for (int i = 1; i < k; ++i) {
        const int v = sel[i];
        int j = i;
        while (j > 0 && sel[j - 1] > v) { sel[j] = sel[j - 1]; --j; }
        sel[j] = v;
      }
      float mn = INFINITY, mx = -INFINITY;
      for (int j = 0; j < nj; ++j) {
        if (!(chosen & (1u << j))) {
          const float x = row[hl + 16 * j];
          mn = fminf(mn, x);
          mx = fmaxf(mx, x);
        }
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (!(mn <= mx)) mn = mx = 0.0f;
      __half s, z;
      const bool ok = nuq_params(mn, mx, &s, &z);
      const float sf = __half2float(s), zf = __half2float(z);
      if (live) {
        for (int j = 0; j < nj; ++j) {
          const int c = hl + 16 * j;
          const float x = fminf(fmaxf(row[c], mn), mx);
          sm.codes[r * D + c] = (uint8_t)nuq_code(x, sf, zf, sm.mids);
        }
        if (hl == 0) {
          range_bad |= !ok;
          hs[sl * L.C + ts + r] = s;
          hz[sl * L.C + ts + r] = z;
        }
        if (hl < k) {
          int c = sel[0];
          for (int e = 1; e < k; ++e) if (hl == e) c = sel[e];
          const __half hv = __float2half_rn(row[c]);
          range_bad |= !isfinite(__half2float(hv));
          L.v_out_col[(sl * L.C + ts + r) * k + hl] = (uint8_t)c;
          L.v_out_val[(sl * L.C + ts + r) * k + hl] = hv;
        }
      }
    }
  }
  if (range_bad) atomicOr(sm.flag, 2);
  __syncthreads();
  pack_3bit_rows(a, sm, ln, ts);
}

// ---- MixKVQ tiers ------------------------------------------------------------------------
__device__ void do_mixed(const QArgs& a, const QSmem& sm, int ln, int64_t ts, int gi) {
  const Layout& L = a.L;
  const Side& S = L.side[KVQ_KEYS];
  const int D = L.D, g = L.g, hi = L.mixed_hi, mid = L.mixed_mid, lo = L.mixed_lo;
  const int64_t sl = slab_of(L);
  uint8_t* ord = sm.codes;  // [D] slot -> channel
  for (int j = threadIdx.x; j < D; j += blockDim.x) ord[j] = L.k_order[(sl * L.ng + gi) * D + j];
  __syncthreads();
  // permute every staged row into slot order once (a warp per row: gather, then write
  // back), so that the statistics and the codes below read slots contiguously
  {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int per = D / 32;   // slots per lane
    for (int r = warp; r < ln; r += nw) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (e < per) v[e] = sm.tile[r * D + ord[per * lane + e]];
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (e < per) sm.tile[r * D + per * lane + e] = v[e];
    }
  }
  __syncthreads();
  uint8_t* gbase = reinterpret_cast<uint8_t*>(S.codes) + (sl * L.ng + gi) * (int64_t)L.mixed_group_bytes;
  // raw plane [g][hi]
  uint16_t* raw = reinterpret_cast<uint16_t*>(gbase);
  for (int i = threadIdx.x; i < ln * hi; i += blockDim.x) {
    const int r = i / hi, j = i % hi;
    const float v = sm.tile[r * D + j];
    raw[r * hi + j] = L.src_dtype == KVQ_F16 ? __half_as_ushort(__float2half_rn(v))
                                             : (uint16_t)(__float_as_uint(v) >> 16);
  }
  __half* hs = reinterpret_cast<__half*>(S.scale) + (sl * L.ng + gi) * (D - hi);
  __half* hz = reinterpret_cast<__half*>(S.zero) + (sl * L.ng + gi) * (D - hi);
  int range_bad = 0;
  for (int j = hi + threadIdx.x; j < D; j += blockDim.x) {
    const int bits = j < hi + mid ? 4 : 2;
    float mn = sm.tile[j], mx = mn;
#pragma unroll 8
    for (int r = 1; r < ln; ++r) {
      const float x = sm.tile[r * D + j];
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    __half s, z;
    range_bad |= !asym_params(mn, mx, bits, &s, &z);
    hs[j - hi] = s;
    hz[j - hi] = z;
    sm.sf[j] = __half2float(s);
    sm.zf[j] = __half2float(z);
  }
  if (range_bad) atomicOr(sm.flag, 2);
  __syncthreads();
  uint32_t* midp = reinterpret_cast<uint32_t*>(gbase + g * hi * 2);
  uint32_t* lop = reinterpret_cast<uint32_t*>(gbase + g * hi * 2 + g * mid / 2);
  const int Wm = mid / 8, Wl = lo / 16;
  if (D == 128) {
    // a warp per row, lane l on slots 4 l .. 4 l + 3 (one float4 of the slot-ordered row;
    // tier boundaries are multiples of 8 slots, so a lane sits in one tier): 4-bit words
    // join the halves of lanes l, l ^ 1, 2-bit words the bytes of four lanes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int s0 = 4 * lane;
    const bool is_mid = s0 >= hi && s0 < hi + mid, is_lo = s0 >= hi + mid;
    float sf4[4], zf4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sf4[e] = s0 >= hi ? sm.sf[s0 + e] : 0.0f;
      zf4[e] = s0 >= hi ? sm.zf[s0 + e] : 0.0f;
    }
    for (int r = warp; r < ln; r += nw) {
      const float4 x4 = *reinterpret_cast<const float4*>(sm.tile + r * D + s0);
      const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
      uint32_t v4 = 0, v2 = 0;
      if (s0 >= hi) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = asym_code(xs[e], sf4[e], zf4[e], is_mid ? 15 : 3);
          v4 |= (uint32_t)c << (4 * e);
          v2 |= (uint32_t)c << (2 * e);
        }
      }
      v4 <<= 16 * (lane & 1);
      v4 |= __shfl_xor_sync(0xffffffffu, v4, 1);
      v2 <<= 8 * (lane & 3);
      v2 |= __shfl_xor_sync(0xffffffffu, v2, 1);
      v2 |= __shfl_xor_sync(0xffffffffu, v2, 2);
      if (is_mid && (lane & 1) == 0) midp[r * Wm + (s0 - hi) / 8] = v4;
      if (is_lo && (lane & 3) == 0) lop[r * Wl + (s0 - hi - mid) / 16] = v2;
    }
    return;
  }
  for (int i = threadIdx.x; i < ln * (Wm + Wl); i += blockDim.x) {
    const int r = i / (Wm + Wl), w = i % (Wm + Wl);
    const float* row = sm.tile + r * D;
    uint32_t word = 0;
    if (w < Wm) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = hi + w * 8 + e;
        word |= (uint32_t)asym_code(row[j], sm.sf[j], sm.zf[j], 15) << (4 * e);
      }
      midp[r * Wm + w] = word;
    } else {
      const int w2 = w - Wm;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int j = hi + mid + w2 * 16 + e;
        word |= (uint32_t)asym_code(row[j], sm.sf[j], sm.zf[j], 3) << (2 * e);
      }
      lop[r * Wl + w2] = word;
    }
  }
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(QArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const Layout& L = a.L;
  const int D = L.D, g = L.g;
  QSmem sm;
  sm.tile = reinterpret_cast<float*>(smem);
  sm.sf = sm.tile + g * D;
  sm.zf = sm.sf + 256;
  sm.mids = sm.zf + 256;
  sm.codes = reinterpret_cast<uint8_t*>(sm.mids + 8);
  sm.omask = reinterpret_cast<uint32_t*>(sm.codes + g * D);
  sm.rowptr = reinterpret_cast<int*>(sm.omask + g * (D / 32));
  sm.flag = sm.rowptr + (g + 1) + 3;
  if (threadIdx.x == 0) *sm.flag = 0;
  __syncthreads();

  const int64_t ts = a.t0 + (int64_t)blockIdx.x * g;
  const int ln = (int)min((int64_t)g, a.t0 + a.n - ts);
  const int gi = (int)(ts / g);
  load_tile(a, ln, ts - a.t0, sm.tile, sm.flag);
  __syncthreads();
  if (a.which == KVQ_KEYS && L.k_rotate) {   // statistics and codes in the rotated basis
    wht_tile_rows(sm.tile, ln, D, L.rot_scale);
    __syncthreads();
  }
  const Side& S = L.side[a.which];
  switch (S.scheme) {
    case KVQ_NONE: {
      uint8_t* dst = reinterpret_cast<uint8_t*>(S.codes) + slab_of(L) * S.code_slab_bytes +
                     ts * (int64_t)D * L.raw_bytes;
      for (int i = threadIdx.x; i < ln * D; i += blockDim.x) store_raw(dst, i, L.src_dtype, sm.tile[i]);
      break;
    }
    case KVQ_SYM8: do_sym8(a, sm, ln, ts, gi); break;
    case KVQ_ASYM: do_asym(a, sm, ln, ts, gi); break;
    case KVQ_NUQ: do_nuq(a, sm, ln, ts, gi); break;
    case KVQ_MIXED: do_mixed(a, sm, ln, ts, gi); break;
  }
  __syncthreads();
  if (threadIdx.x == 0 && *sm.flag) {
    int bitsv = 0;
    if (*sm.flag & 1) bitsv |= KVQ_DEV_NONFINITE;
    if (*sm.flag & 2) bitsv |= KVQ_DEV_RANGE;
    flag(a.status, bitsv);
  }
}

size_t quantize_smem(const Layout& L) {
  const size_t g = L.g, D = L.D;
  return g * D * 4 + 2 * 256 * 4 + 8 * 4 + g * D + g * (D / 32) * 4 + (g + 1 + 4) * 4 + 16;
}

}  // namespace

cudaError_t launch_quantize(const Layout& L, int which, const void* src, int64_t sb, int64_t sh,
                            int64_t st, int64_t t0, int64_t n, int32_t* d_status,
                            cudaStream_t s) {
  if (asym_fast_ok(L, which)) return launch_quantize_asym(L, which, src, sb, sh, st, t0, n, d_status, s);
  if (L.side[which].scheme == KVQ_KQV) return launch_quantize_kqv(L, which, src, sb, sh, st, t0, n, d_status, s);
  QArgs a;
  a.L = L;
  a.which = which;
  a.src = src;
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.t0 = t0;
  a.n = n;
  a.status = d_status;
  const size_t smem = quantize_smem(L);
  cudaError_t e = cudaFuncSetAttribute(quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int groups = (int)((n + L.g - 1) / L.g);
  dim3 grid(groups, L.Hkv, L.B);
  quantize_kernel<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
