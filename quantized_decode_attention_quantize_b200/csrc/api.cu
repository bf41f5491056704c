// Host layer of the C ABI: argument validation, array sizes, layout derivation and
// kernel dispatch.  No allocation, no synchronisation, no global state.
#include <cmath>
#include <cstring>
#include <vector>

#include "kvq_internal.cuh"

#include <atomic>
#include <chrono>

using namespace kvq;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int dtype_bytes(int dt) { return dt == KVQ_F32 ? 4 : 2; }

bool valid_dtype(int dt) { return dt == KVQ_F32 || dt == KVQ_F16 || dt == KVQ_BF16; }

// Per-side check: returns KVQ_OK / KVQ_ERR_INVALID / KVQ_ERR_UNSUPPORTED.
kvq_status check_side(const kvq_format* f, int which) {
  const int scheme = which == KVQ_KEYS ? f->k_scheme : f->v_scheme;
  const int bits = which == KVQ_KEYS ? f->k_bits : f->v_bits;
  const int axis = which == KVQ_KEYS ? f->k_axis : f->v_axis;
  const int nout = which == KVQ_KEYS ? f->k_outliers : f->v_outliers;
  const int want_axis = which == KVQ_KEYS ? KVQ_AXIS_CHANNEL : KVQ_AXIS_TOKEN;
  switch (scheme) {
    case KVQ_NONE:
      return nout == 0 ? KVQ_OK : KVQ_ERR_INVALID;
    case KVQ_SYM8:
      if (bits != 8 || nout != 0) return KVQ_ERR_INVALID;
      if (axis < KVQ_AXIS_TENSOR || axis > KVQ_AXIS_CHANNEL) return KVQ_ERR_INVALID;
      return KVQ_OK;
    case KVQ_ASYM:
      if (bits != 2 && bits != 4 && bits != 8) return KVQ_ERR_INVALID;
      if (nout != 0) return KVQ_ERR_INVALID;
      if (axis < KVQ_AXIS_TENSOR || axis > KVQ_AXIS_CHANNEL) return KVQ_ERR_INVALID;
      return axis == want_axis ? KVQ_OK : KVQ_ERR_UNSUPPORTED;
    case KVQ_NUQ:
      if (bits != 3 || nout < 0 || nout > 8) return KVQ_ERR_INVALID;
      if (axis < KVQ_AXIS_TENSOR || axis > KVQ_AXIS_CHANNEL) return KVQ_ERR_INVALID;
      if (which == KVQ_KEYS && nout > f->group_tokens) return KVQ_ERR_INVALID;
      return axis == want_axis ? KVQ_OK : KVQ_ERR_UNSUPPORTED;
    case KVQ_MIXED: {
      if (which != KVQ_KEYS) return KVQ_ERR_UNSUPPORTED;
      if (f->src_dtype == KVQ_F32) return KVQ_ERR_UNSUPPORTED;
      const int lo = f->head_dim - f->mixed_hi - f->mixed_mid;
      if (f->mixed_hi < 0 || f->mixed_mid < 0 || lo < 0) return KVQ_ERR_INVALID;
      if (f->mixed_hi % 8 || f->mixed_mid % 8 || lo % 16) return KVQ_ERR_INVALID;
      return KVQ_OK;
    }
    case KVQ_KQV:
      // keys b in {2, 3, 4} bits; values a budget of b in {2, 3, 4} (b - 1 code bits + sketch)
      if (bits < 2 || bits > 4 || nout != 0) return KVQ_ERR_INVALID;
      if (axis < KVQ_AXIS_TENSOR || axis > KVQ_AXIS_CHANNEL) return KVQ_ERR_INVALID;
      return axis == KVQ_AXIS_TOKEN ? KVQ_OK : KVQ_ERR_UNSUPPORTED;
    default:
      return KVQ_ERR_INVALID;
  }
}

int64_t code_row_bytes(const kvq_format* f, int which) {
  const int scheme = which == KVQ_KEYS ? f->k_scheme : f->v_scheme;
  const int bits = which == KVQ_KEYS ? f->k_bits : f->v_bits;
  const int D = f->head_dim;
  switch (scheme) {
    case KVQ_NONE: return (int64_t)D * dtype_bytes(f->src_dtype);
    case KVQ_SYM8: return D;
    case KVQ_ASYM: return (int64_t)D * bits / 8;
    case KVQ_NUQ: return 3 * (int64_t)D / 8;
    case KVQ_KQV: return (int64_t)D * bits / 8;   // values: b - 1 code bits and the sketch bit
    case KVQ_MIXED: {
      const int lo = D - f->mixed_hi - f->mixed_mid;
      return 2 * f->mixed_hi + f->mixed_mid / 2 + lo / 4;
    }
  }
  return 0;
}

// (scale elements, zero elements) per slab
void meta_elems(const kvq_format* f, int which, int64_t C, int64_t* ns, int64_t* nz) {
  const int scheme = which == KVQ_KEYS ? f->k_scheme : f->v_scheme;
  const int axis = which == KVQ_KEYS ? f->k_axis : f->v_axis;
  const int64_t ng = C / f->group_tokens, D = f->head_dim;
  *ns = *nz = 0;
  if (scheme == KVQ_SYM8) {
    *ns = axis == KVQ_AXIS_TENSOR ? ng : axis == KVQ_AXIS_TOKEN ? C : ng * D;
  } else if (scheme == KVQ_ASYM || scheme == KVQ_NUQ) {
    *ns = *nz = axis == KVQ_AXIS_CHANNEL ? ng * D : C;
  } else if (scheme == KVQ_MIXED) {
    *ns = *nz = ng * (D - f->mixed_hi);
  } else if (scheme == KVQ_KQV) {
    *ns = C;                                  // row norms
    *nz = which == KVQ_VALUES ? C : 0;        // residual norms
  }
}

int meta_elem_bytes(const kvq_format* f, int which) {
  const int scheme = which == KVQ_KEYS ? f->k_scheme : f->v_scheme;
  return scheme == KVQ_SYM8 || scheme == KVQ_KQV ? 4 : 2;
}

// LUT bytes: NUQ fp16 [8]; KQV fp32 [2^code bits]
int64_t lut_bytes(const kvq_format* f, int which) {
  const int scheme = which == KVQ_KEYS ? f->k_scheme : f->v_scheme;
  const int bits = which == KVQ_KEYS ? f->k_bits : f->v_bits - 1;
  if (scheme == KVQ_NUQ) return 16;
  if (scheme == KVQ_KQV) return 4 * ((int64_t)1 << bits);
  return 0;
}

}  // namespace

extern "C" {

int32_t kvq_version(void) { return (KVQ_VERSION_MAJOR << 16) | KVQ_VERSION_MINOR; }

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported format or shape";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

kvq_status kvq_format_check(const kvq_format* f) {
  if (!f) return KVQ_ERR_INVALID;
  const int D = f->head_dim, g = f->group_tokens;
  if (D != 32 && D != 64 && D != 128 && D != 256) return KVQ_ERR_INVALID;
  if (g < 16 || g > 256 || g % 16 || (int64_t)g * D > 32768) return KVQ_ERR_INVALID;
  if (!valid_dtype(f->src_dtype)) return KVQ_ERR_INVALID;
  if (f->n_sink < 0 || f->n_sink > 4096 || f->residual_cap < 0 || f->residual_cap > (1 << 20))
    return KVQ_ERR_INVALID;
  if (f->rope != 0 && f->rope != 1) return KVQ_ERR_INVALID;
  if (f->rope && !(f->rope_base > 1.0f)) return KVQ_ERR_INVALID;
  if (f->rope && D < 64) return KVQ_ERR_UNSUPPORTED;
  if (f->k_rotate != 0 && f->k_rotate != 1) return KVQ_ERR_INVALID;
  if (f->k_rotate && (f->rope || (f->k_scheme != KVQ_SYM8 && f->k_scheme != KVQ_ASYM &&
                                  f->k_scheme != KVQ_NUQ)))
    return KVQ_ERR_UNSUPPORTED;
  // KQV codes keys and values together, D = 128, its own rotation, no RoPE
  if ((f->k_scheme == KVQ_KQV) != (f->v_scheme == KVQ_KQV)) return KVQ_ERR_UNSUPPORTED;
  if (f->k_scheme == KVQ_KQV && (D != 128 || f->rope || f->k_rotate)) return KVQ_ERR_UNSUPPORTED;
  kvq_status a = check_side(f, KVQ_KEYS);
  if (a == KVQ_ERR_INVALID) return a;
  kvq_status b = check_side(f, KVQ_VALUES);
  if (b == KVQ_ERR_INVALID) return b;
  if (a != KVQ_OK) return a;
  return b;
}

kvq_status kvq_kqv_codebook(int32_t bits, int32_t d, float* centroids) {
  if (bits < 1 || bits > 4 || d < 3 || d > 4096 || !centroids) return KVQ_ERR_INVALID;
  // midpoint quadrature on [-R, R], R = min(1, 14 / sqrt(d)): the density beyond 14
  // standard deviations (1 / sqrt(d)) carries no mass at double precision
  const int N = 400000, K = 1 << bits;
  const double R = std::fmin(1.0, 14.0 / std::sqrt((double)d));
  const double logc = std::lgamma(d / 2.0) - std::lgamma(0.5) - std::lgamma((d - 1) / 2.0);
  std::vector<double> x(N), w(N);
  double tot = 0.0;
  for (int i = 0; i < N; ++i) {
    x[i] = ((i + 0.5) / N) * 2.0 * R - R;
    w[i] = std::fabs(x[i]) < 1.0 ? std::exp(logc + (d - 3) / 2.0 * std::log1p(-x[i] * x[i])) : 0.0;
    tot += w[i];
  }
  for (int i = 0; i < N; ++i) w[i] /= tot;
  // start at the quantiles (k + 1/2) / K of the grid's distribution, linearly interpolated
  double c[16], t[15];
  {
    double cdf = 0.0, prev_cdf = 0.0;
    int k = 0, i = 0;
    while (k < K) {
      const double target = (k + 0.5) / K;
      while (i < N && cdf < target) {
        prev_cdf = cdf;
        cdf += w[i++];
      }
      if (i == 0) {
        c[k] = x[0];
      } else if (cdf <= prev_cdf) {
        c[k] = x[i - 1];
      } else {
        const double f = (target - prev_cdf) / (cdf - prev_cdf);
        c[k] = i >= 2 ? x[i - 2] + f * (x[i - 1] - x[i - 2]) : x[i - 1];
      }
      ++k;
    }
  }
  for (int it = 0; it < 300; ++it) {
    for (int j = 0; j + 1 < K; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
    double mass[16] = {0}, mom[16] = {0};
    int cell = 0;
    for (int i = 0; i < N; ++i) {
      while (cell < K - 1 && t[cell] < x[i]) ++cell;   // cell = #{ j : t_j < x }
      mass[cell] += w[i];
      mom[cell] += w[i] * x[i];
    }
    double nc[16];
    for (int j = 0; j < K; ++j) nc[j] = mass[j] > 0.0 ? mom[j] / mass[j] : c[j];
    for (int j = 0; j < K; ++j) c[j] = 0.5 * (nc[j] - nc[K - 1 - j]);   // symmetric density
  }
  for (int j = 0; j < K; ++j) centroids[j] = (float)c[j];
  return KVQ_OK;
}

size_t kvq_cache_array_bytes(const kvq_format* f, int32_t B, int32_t H, int64_t C, int32_t id) {
  if (kvq_format_check(f) != KVQ_OK || B <= 0 || H <= 0 || C < 0 || C % f->group_tokens)
    return 0;
  const int64_t slabs = (int64_t)B * H, D = f->head_dim, g = f->group_tokens, ng = C / g;
  const int64_t raw = dtype_bytes(f->src_dtype);
  int64_t ns, nz;
  const bool kout = f->k_scheme == KVQ_NUQ && f->k_outliers > 0;
  const bool vout = f->v_scheme == KVQ_NUQ && f->v_outliers > 0;
  switch (id) {
    case KVQ_ARR_K_CODES: return slabs * C * code_row_bytes(f, KVQ_KEYS);
    case KVQ_ARR_V_CODES: return slabs * C * code_row_bytes(f, KVQ_VALUES);
    case KVQ_ARR_K_SCALE: meta_elems(f, KVQ_KEYS, C, &ns, &nz); return slabs * ns * meta_elem_bytes(f, KVQ_KEYS);
    case KVQ_ARR_K_ZERO: meta_elems(f, KVQ_KEYS, C, &ns, &nz); return slabs * nz * meta_elem_bytes(f, KVQ_KEYS);
    case KVQ_ARR_V_SCALE: meta_elems(f, KVQ_VALUES, C, &ns, &nz); return slabs * ns * meta_elem_bytes(f, KVQ_VALUES);
    case KVQ_ARR_V_ZERO: meta_elems(f, KVQ_VALUES, C, &ns, &nz); return slabs * nz * meta_elem_bytes(f, KVQ_VALUES);
    case KVQ_ARR_K_ORDER: return f->k_scheme == KVQ_MIXED ? slabs * ng * D : 0;
    case KVQ_ARR_K_OUT_ROWPTR: return kout ? slabs * ng * (g + 1) * 4 : 0;
    case KVQ_ARR_K_OUT_COL: return kout ? slabs * ng * D * f->k_outliers : 0;
    case KVQ_ARR_K_OUT_VAL: return kout ? slabs * ng * D * f->k_outliers * 2 : 0;
    case KVQ_ARR_V_OUT_COL: return vout ? slabs * C * f->v_outliers : 0;
    case KVQ_ARR_V_OUT_VAL: return vout ? slabs * C * f->v_outliers * 2 : 0;
    case KVQ_ARR_K_LUT: return lut_bytes(f, KVQ_KEYS);
    case KVQ_ARR_V_LUT: return lut_bytes(f, KVQ_VALUES);
    case KVQ_ARR_V_SKETCH: return f->v_scheme == KVQ_KQV ? D * D * 4 : 0;
    case KVQ_ARR_SINK_K:
    case KVQ_ARR_SINK_V: return slabs * f->n_sink * D * raw;
    case KVQ_ARR_RES_K:
    case KVQ_ARR_RES_V: return slabs * f->residual_cap * D * raw;
  }
  return 0;
}

}  // extern "C"

namespace kvq {

kvq_status make_layout(const kvq_format* f, const kvq_cache* c, Layout* L) {
  kvq_status st = kvq_format_check(f);
  if (st != KVQ_OK) return st;
  if (!c || c->batch <= 0 || c->kv_heads <= 0 || c->capacity < 0 ||
      c->capacity % f->group_tokens)
    return KVQ_ERR_INVALID;
  std::memset(L, 0, sizeof(*L));
  L->D = f->head_dim;
  L->g = f->group_tokens;
  L->src_dtype = f->src_dtype;
  L->raw_bytes = dtype_bytes(f->src_dtype);
  L->B = c->batch;
  L->Hkv = c->kv_heads;
  L->C = c->capacity;
  L->ng = (int)(c->capacity / f->group_tokens);
  L->n_sink = f->n_sink;
  L->res_cap = f->residual_cap;
  L->rope = f->rope;
  L->rope_base = f->rope_base;
  L->k_rotate = f->k_rotate;
  L->rot_scale = (float)(1.0 / std::sqrt((double)f->head_dim));
  L->mixed_hi = f->mixed_hi;
  L->mixed_mid = f->mixed_mid;
  L->mixed_lo = f->head_dim - f->mixed_hi - f->mixed_mid;
  L->mixed_group_bytes = (int)(f->group_tokens * code_row_bytes(f, KVQ_KEYS));
  for (int w = 0; w < 2; ++w) {
    Side& s = L->side[w];
    s.scheme = w == 0 ? f->k_scheme : f->v_scheme;
    s.bits = w == 0 ? f->k_bits : f->v_bits;
    s.axis = w == 0 ? f->k_axis : f->v_axis;
    s.nout = s.scheme == KVQ_NUQ ? (w == 0 ? f->k_outliers : f->v_outliers) : 0;
    s.code_row_bytes = (int)code_row_bytes(f, w);
    s.code_slab_bytes = s.code_row_bytes * c->capacity;
    int64_t ns, nz;
    meta_elems(f, w, c->capacity, &ns, &nz);
    s.meta_slab_elems = ns;
    s.codes = w == 0 ? c->k_codes : c->v_codes;
    s.scale = w == 0 ? c->k_scale : c->v_scale;
    s.zero = w == 0 ? c->k_zero : c->v_zero;
    s.lut = reinterpret_cast<const __half*>(w == 0 ? c->k_lut : c->v_lut);
    if (!s.codes || !aligned16(s.codes)) return KVQ_ERR_INVALID;
    if (ns && (!s.scale || !aligned16(s.scale))) return KVQ_ERR_INVALID;
    if (nz && (!s.zero || !aligned16(s.zero))) return KVQ_ERR_INVALID;
    if (s.scheme == KVQ_NUQ && (!s.lut || !aligned16(s.lut))) return KVQ_ERR_INVALID;
    s.lutf = reinterpret_cast<const float*>(w == 0 ? c->k_lut : c->v_lut);
    if (s.scheme == KVQ_KQV && (!s.lutf || !aligned16(s.lutf))) return KVQ_ERR_INVALID;
  }
  L->sketch = reinterpret_cast<const float*>(c->v_sketch);
  if (f->v_scheme == KVQ_KQV && (!L->sketch || !aligned16(L->sketch))) return KVQ_ERR_INVALID;
  L->k_order = reinterpret_cast<uint8_t*>(c->k_order);
  if (f->k_scheme == KVQ_MIXED && (!L->k_order || !aligned16(L->k_order))) return KVQ_ERR_INVALID;
  if (f->k_scheme == KVQ_NUQ && f->k_outliers > 0) {
    L->k_out_rowptr = reinterpret_cast<int32_t*>(c->k_out_rowptr);
    L->k_out_col = reinterpret_cast<uint8_t*>(c->k_out_col);
    L->k_out_val = reinterpret_cast<__half*>(c->k_out_val);
    if (!L->k_out_rowptr || !L->k_out_col || !L->k_out_val || !aligned16(L->k_out_rowptr) ||
        !aligned16(L->k_out_col) || !aligned16(L->k_out_val))
      return KVQ_ERR_INVALID;
  }
  if (f->v_scheme == KVQ_NUQ && f->v_outliers > 0) {
    L->v_out_col = reinterpret_cast<uint8_t*>(c->v_out_col);
    L->v_out_val = reinterpret_cast<__half*>(c->v_out_val);
    if (!L->v_out_col || !L->v_out_val || !aligned16(L->v_out_col) || !aligned16(L->v_out_val))
      return KVQ_ERR_INVALID;
  }
  L->sink[0] = c->sink_k;
  L->sink[1] = c->sink_v;
  L->res[0] = c->res_k;
  L->res[1] = c->res_v;
  return KVQ_OK;
}

int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

}  // namespace kvq

extern "C" {

static kvq_status quantize_common(int which, const kvq_format* f, const kvq_cache* c,
                                  const void* src, int64_t sb, int64_t sh, int64_t st,
                                  int64_t t0, int64_t n, int32_t* d_status, void* stream) {
  Layout L;
  kvq_status s = make_layout(f, c, &L);
  if (s != KVQ_OK) return s;
  if (n < 0 || t0 < 0 || t0 % L.g || t0 + n > L.C) return KVQ_ERR_INVALID;
  if (n == 0) return KVQ_OK;
  if (!src || !aligned16(src)) return KVQ_ERR_INVALID;
  const int64_t eb = dtype_bytes(L.src_dtype);
  if (st < L.D || sb < 0 || sh < 0) return KVQ_ERR_INVALID;
  if ((st * eb) % 16 || (sh * eb) % 16 || (sb * eb) % 16) return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  cudaError_t e = launch_quantize(L, which, src, sb, sh, st, t0, n, d_status,
                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_quantize_keys(const kvq_format* f, const kvq_cache* c, const void* src,
                             int64_t sb, int64_t sh, int64_t st, int64_t t0, int64_t n,
                             int32_t* d_status, void* stream) {
  return quantize_common(KVQ_KEYS, f, c, src, sb, sh, st, t0, n, d_status, stream);
}

kvq_status kvq_quantize_values(const kvq_format* f, const kvq_cache* c, const void* src,
                               int64_t sb, int64_t sh, int64_t st, int64_t t0, int64_t n,
                               int32_t* d_status, void* stream) {
  return quantize_common(KVQ_VALUES, f, c, src, sb, sh, st, t0, n, d_status, stream);
}

kvq_status kvq_quantize_kv(const kvq_format* f, const kvq_cache* c, const void* k_src,
                           const void* v_src, int64_t sb, int64_t sh, int64_t st, int64_t t0,
                           int64_t n, int32_t* d_status, void* stream) {
  Layout L;
  kvq_status s = make_layout(f, c, &L);
  if (s != KVQ_OK) return s;
  if (n < 0 || t0 < 0 || t0 % L.g || t0 + n > L.C) return KVQ_ERR_INVALID;
  if (n == 0) return KVQ_OK;
  if (!k_src || !v_src || !aligned16(k_src) || !aligned16(v_src)) return KVQ_ERR_INVALID;
  const int64_t eb = dtype_bytes(L.src_dtype);
  if (st < L.D || sb < 0 || sh < 0) return KVQ_ERR_INVALID;
  if ((st * eb) % 16 || (sh * eb) % 16 || (sb * eb) % 16) return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  if (asym_fast_ok(L, KVQ_KEYS) && asym_fast_ok(L, KVQ_VALUES)) {
    cudaError_t e = launch_quantize_asym_kv(L, k_src, v_src, sb, sh, st, t0, n, d_status,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
  }
  s = quantize_common(KVQ_KEYS, f, c, k_src, sb, sh, st, t0, n, d_status, stream);
  if (s != KVQ_OK) return s;
  return quantize_common(KVQ_VALUES, f, c, v_src, sb, sh, st, t0, n, d_status, stream);
}

kvq_status kvq_dequantize(const kvq_format* f, const kvq_cache* c, int32_t which, int64_t t0,
                          int64_t n, void* out, int32_t out_dtype, int32_t* d_status,
                          void* stream) {
  Layout L;
  kvq_status s = make_layout(f, c, &L);
  if (s != KVQ_OK) return s;
  if (which != KVQ_KEYS && which != KVQ_VALUES) return KVQ_ERR_INVALID;
  if (n < 0 || t0 < 0 || t0 + n > L.C) return KVQ_ERR_INVALID;
  if (!valid_dtype(out_dtype)) return KVQ_ERR_INVALID;
  if (n == 0) return KVQ_OK;
  if (!out || !aligned16(out)) return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  cudaError_t e = launch_dequantize(L, which, t0, n, out, out_dtype, d_status,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_key_salience(const kvq_format* f, const void* q, int64_t qsb, int64_t qsh,
                            int64_t qst, const void* k, int64_t ksb, int64_t ksh, int64_t kst,
                            int32_t B, int32_t Hq, int32_t Hkv, int32_t R, double* sal,
                            uint8_t* order, int64_t osb, int64_t osh, int32_t* d_status,
                            void* stream) {
  kvq_status s = kvq_format_check(f);
  if (s != KVQ_OK) return s;
  if (!q || !k || !order || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || R <= 0)
    return KVQ_ERR_INVALID;
  const int D = f->head_dim;
  if (qst < D || kst < D || qsb < 0 || qsh < 0 || ksb < 0 || ksh < 0 || osb < 0 || osh < 0)
    return KVQ_ERR_INVALID;
  if (sal && (reinterpret_cast<uintptr_t>(sal) & 7)) return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  Layout L;
  std::memset(&L, 0, sizeof(L));
  L.D = D;
  L.src_dtype = f->src_dtype;
  cudaError_t e = launch_salience(L, q, qsb, qsh, qst, k, ksb, ksh, kst, B, Hq, Hkv, R, sal,
                                  order, osb, osh, d_status,
                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

static kvq_status decode_args(const kvq_format* f, int32_t B, int32_t Hq, int32_t Hkv,
                              int64_t t_quant, int32_t t_res, int32_t num_splits) {
  kvq_status s = kvq_format_check(f);
  if (s != KVQ_OK) return s;
  if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv) return KVQ_ERR_INVALID;
  if ((int64_t)(Hq / Hkv) * f->head_dim > 2048 || Hq / Hkv > 16) return KVQ_ERR_UNSUPPORTED;
  if (f->k_scheme == KVQ_KQV && Hq / Hkv > 8) return KVQ_ERR_UNSUPPORTED;
  if (t_quant < 0 || t_res < 0 || t_res > f->residual_cap || num_splits < 0)
    return KVQ_ERR_INVALID;
  if (f->n_sink + t_quant + t_res <= 0) return KVQ_ERR_INVALID;
  return KVQ_OK;
}

static void plan_layout(const kvq_format* f, int32_t B, int32_t Hkv, Layout* L) {
  std::memset(L, 0, sizeof(*L));
  L->D = f->head_dim;
  L->g = f->group_tokens;
  L->B = B;
  L->Hkv = Hkv;
  L->n_sink = f->n_sink;
  L->side[0].scheme = f->k_scheme;
  L->side[0].bits = f->k_bits;
  L->side[0].axis = f->k_axis;
  L->side[0].nout = f->k_scheme == KVQ_NUQ ? f->k_outliers : 0;
  L->side[1].scheme = f->v_scheme;
  L->side[1].bits = f->v_bits;
  L->side[1].axis = f->v_axis;
  L->side[1].nout = f->v_scheme == KVQ_NUQ ? f->v_outliers : 0;
  L->rope = f->rope;
  L->src_dtype = f->src_dtype;
  // every format field the decode planner reads (the tiers select the MIXED kernel)
  L->mixed_hi = f->mixed_hi;
  L->mixed_mid = f->mixed_mid;
  L->mixed_lo = f->head_dim - f->mixed_hi - f->mixed_mid;
  L->k_rotate = f->k_rotate;
}

size_t kvq_decode_workspace_bytes(const kvq_format* f, int32_t B, int32_t Hq, int32_t Hkv,
                                  int64_t t_quant, int32_t t_res, int32_t num_splits) {
  if (decode_args(f, B, Hq, Hkv, t_quant, t_res, num_splits) != KVQ_OK) return 0;
  Layout L;
  plan_layout(f, B, Hkv, &L);
  DecodePlan p = plan_decode(L, Hq, t_quant, t_res, num_splits);
  return workspace_bytes(L, Hq, p);
}

int32_t kvq_decode_partial_slots(const kvq_format* f, int32_t B, int32_t Hq, int32_t Hkv,
                                 int64_t t_quant, int32_t t_res, int32_t num_splits) {
  if (decode_args(f, B, Hq, Hkv, t_quant, t_res, num_splits) != KVQ_OK) return 0;
  Layout L;
  plan_layout(f, B, Hkv, &L);
  return plan_decode(L, Hq, t_quant, t_res, num_splits).S;
}

// Validation and plan of a decode call; nothing is launched.
static kvq_status decode_prepare(const kvq_format* f, const kvq_cache* c, const void* q,
                                 int32_t q_dtype, int32_t Hq, int64_t t_quant, int32_t t_res,
                                 float scale, void* ws, size_t ws_bytes, int32_t num_splits,
                                 int32_t* d_status, Layout* L, DecodePlan* p) {
  kvq_status s = make_layout(f, c, L);
  if (s != KVQ_OK) return s;
  s = decode_args(f, L->B, Hq, L->Hkv, t_quant, t_res, num_splits);
  if (s != KVQ_OK) return s;
  if (t_quant > L->C) return KVQ_ERR_INVALID;
  if (!q || !aligned16(q) || !valid_dtype(q_dtype) || !(scale > 0.0f)) return KVQ_ERR_INVALID;
  if (L->n_sink && (!L->sink[0] || !L->sink[1] || !aligned16(L->sink[0]) || !aligned16(L->sink[1])))
    return KVQ_ERR_INVALID;
  if (t_res && (!L->res[0] || !L->res[1] || !aligned16(L->res[0]) || !aligned16(L->res[1])))
    return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  *p = plan_decode(*L, Hq, t_quant, t_res, num_splits);
  if (!ws || !aligned16(ws)) return KVQ_ERR_INVALID;
  if (ws_bytes < workspace_bytes(*L, Hq, *p)) return KVQ_ERR_WORKSPACE;
  return KVQ_OK;
}

static kvq_status partial_common(const kvq_format* f, const kvq_cache* c, const void* q,
                                 int32_t q_dtype, int32_t Hq, int64_t t_quant, int32_t t_res,
                                 float scale, void* ws, size_t ws_bytes, int32_t num_splits,
                                 int32_t* d_status, void* stream, Layout* L, DecodePlan* p) {
  kvq_status s = decode_prepare(f, c, q, q_dtype, Hq, t_quant, t_res, scale, ws, ws_bytes, num_splits,
                                d_status, L, p);
  if (s != KVQ_OK) return s;
  cudaError_t e = launch_decode_partial(*L, *p, q, q_dtype, Hq, t_quant, t_res, scale, ws, d_status,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_decode_partial(const kvq_format* f, const kvq_cache* c, const void* q,
                              int32_t q_dtype, int32_t Hq, int64_t t_quant, int32_t t_res,
                              float scale, void* ws, size_t ws_bytes, int32_t num_splits,
                              int32_t* d_status, void* stream) {
  Layout L;
  DecodePlan p;
  return partial_common(f, c, q, q_dtype, Hq, t_quant, t_res, scale, ws, ws_bytes, num_splits,
                        d_status, stream, &L, &p);
}

kvq_status kvq_decode_combine(const kvq_format* f, int32_t B, int32_t Hq, int32_t Hkv,
                              int64_t t_quant, int32_t t_res, int32_t num_splits, const void* ws,
                              size_t ws_bytes, void* out, int32_t out_dtype, void* stream) {
  kvq_status s = decode_args(f, B, Hq, Hkv, t_quant, t_res, num_splits);
  if (s != KVQ_OK) return s;
  if (!out || !aligned16(out) || !valid_dtype(out_dtype) || !ws || !aligned16(ws))
    return KVQ_ERR_INVALID;
  Layout L;
  plan_layout(f, B, Hkv, &L);
  DecodePlan p = plan_decode(L, Hq, t_quant, t_res, num_splits);
  if (ws_bytes < workspace_bytes(L, Hq, p)) return KVQ_ERR_WORKSPACE;
  cudaError_t e = launch_combine(L, Hq, p, ws, out, out_dtype, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_decode_combine_lse(const kvq_format* f, int32_t B, int32_t Hq, int32_t Hkv,
                                  int64_t t_quant, int32_t t_res, int32_t num_splits, const void* ws,
                                  size_t ws_bytes, float* out, float* lse, void* stream) {
  kvq_status s = decode_args(f, B, Hq, Hkv, t_quant, t_res, num_splits);
  if (s != KVQ_OK) return s;
  if (!out || !aligned16(out) || !lse || !aligned16(lse) || !ws || !aligned16(ws)) return KVQ_ERR_INVALID;
  Layout L;
  plan_layout(f, B, Hkv, &L);
  DecodePlan p = plan_decode(L, Hq, t_quant, t_res, num_splits);
  if (ws_bytes < workspace_bytes(L, Hq, p)) return KVQ_ERR_WORKSPACE;
  cudaError_t e = launch_combine(L, Hq, p, ws, out, KVQ_F32, lse, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_merge_states(int32_t n_parts, int64_t rows, int32_t head_dim, const float* outs,
                            const float* lses, void* out, int32_t out_dtype, float* lse_out,
                            void* stream) {
  if (n_parts < 1 || n_parts > 4096 || rows < 1 || rows > ((int64_t)1 << 31)) return KVQ_ERR_INVALID;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128 && head_dim != 256) return KVQ_ERR_INVALID;
  if (!outs || !aligned16(outs) || !lses || !aligned16(lses) || !out || !aligned16(out) ||
      !valid_dtype(out_dtype) || (lse_out && !aligned16(lse_out)))
    return KVQ_ERR_INVALID;
  cudaError_t e = launch_merge_states(n_parts, rows, head_dim, outs, lses, out, out_dtype, lse_out,
                                      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// A value per call of the fused append that the flags of an earlier call (or a fresh
// workspace) do not hold: a per-process counter from a clock-seeded start, never 0.
static uint32_t next_epoch() {
  static std::atomic<uint32_t> counter{(uint32_t)std::chrono::steady_clock::now().time_since_epoch().count() |
                                       1u};
  uint32_t e;
  do {
    e = counter.fetch_add(1, std::memory_order_relaxed);
  } while (e == 0);
  return e;
}

kvq_status kvq_append_decode_attention(const kvq_format* f, const kvq_cache* c, const void* k_src,
                                       const void* v_src, int64_t sb, int64_t sh, int64_t st, int64_t t0,
                                       int64_t n, const void* q, int32_t q_dtype, int32_t Hq, int64_t t_quant,
                                       int32_t t_res, float scale, void* out, int32_t out_dtype, void* ws,
                                       size_t ws_bytes, int32_t num_splits, int32_t* d_status, void* stream) {
  // every argument of both halves is checked before anything is launched
  if (!out || !aligned16(out) || !valid_dtype(out_dtype)) return KVQ_ERR_INVALID;
  Layout L;
  DecodePlan p;
  kvq_status s = decode_prepare(f, c, q, q_dtype, Hq, t_quant, t_res, scale, ws, ws_bytes, num_splits, d_status,
                                &L, &p);
  if (s != KVQ_OK) return s;
  if (n < 0 || t0 < 0 || t0 % L.g || t0 + n > L.C) return KVQ_ERR_INVALID;
  if (n > 0) {
    if (!k_src || !v_src || !aligned16(k_src) || !aligned16(v_src)) return KVQ_ERR_INVALID;
    const int64_t eb = dtype_bytes(L.src_dtype);
    if (st < L.D || sb < 0 || sh < 0) return KVQ_ERR_INVALID;
    if ((st * eb) % 16 || (sh * eb) % 16 || (sb * eb) % 16) return KVQ_ERR_INVALID;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (n > 0) {
    if (fused_append_ok(L, Hq, p, t0, n)) {
      // the split kernel quantizes the group itself before its decode (no append launch)
      p.fuse = 1;
      p.dep_lo = t0;
      p.dep_hi = t0 + n;
      p.app_n = (int)n;
      p.app_k = k_src;
      p.app_v = v_src;
      p.app_sb = sb;
      p.app_sh = sh;
      p.app_st = st;
      p.epoch = next_epoch();
    } else if (asym_fast_ok(L, KVQ_KEYS) && asym_fast_ok(L, KVQ_VALUES)) {
      // one append kernel directly before the split kernel: the split kernel reads the
      // rows the append does not touch without waiting for it
      if (launch_quantize_asym_kv(L, k_src, v_src, sb, sh, st, t0, n, d_status, cs) != cudaSuccess)
        return KVQ_ERR_CUDA;
      p.defer = 1;
      p.dep_lo = t0;
      p.dep_hi = t0 + n;
    } else {
      if (launch_quantize(L, KVQ_KEYS, k_src, sb, sh, st, t0, n, d_status, cs) != cudaSuccess ||
          launch_quantize(L, KVQ_VALUES, v_src, sb, sh, st, t0, n, d_status, cs) != cudaSuccess)
        return KVQ_ERR_CUDA;
    }
  }
  if (launch_decode_partial(L, p, q, q_dtype, Hq, t_quant, t_res, scale, ws, d_status, cs) != cudaSuccess)
    return KVQ_ERR_CUDA;
  cudaError_t e = launch_combine(L, Hq, p, ws, out, out_dtype, nullptr, cs);
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_decode_attention(const kvq_format* f, const kvq_cache* c, const void* q,
                                int32_t q_dtype, int32_t Hq, int64_t t_quant, int32_t t_res,
                                float scale, void* out, int32_t out_dtype, void* ws,
                                size_t ws_bytes, int32_t num_splits, int32_t* d_status,
                                void* stream) {
  if (!out || !aligned16(out) || !valid_dtype(out_dtype)) return KVQ_ERR_INVALID;
  Layout L;
  DecodePlan p;
  kvq_status s = partial_common(f, c, q, q_dtype, Hq, t_quant, t_res, scale, ws, ws_bytes,
                                num_splits, d_status, stream, &L, &p);
  if (s != KVQ_OK) return s;
  cudaError_t e = launch_combine(L, Hq, p, ws, out, out_dtype, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}


static kvq_status paged_layout(const kvq_format* f, const kvq_paged_cache* pc, Layout* L) {
  if (!pc) return KVQ_ERR_INVALID;
  kvq_status st = make_layout(f, &pc->pool, L);
  if (st != KVQ_OK) return st;
  if (pc->pool.capacity != f->group_tokens) return KVQ_ERR_INVALID;
  if (pc->num_seqs < 1 || pc->max_blocks < 1 || !pc->block_table ||
      (reinterpret_cast<uintptr_t>(pc->block_table) & 3))
    return KVQ_ERR_INVALID;
  return KVQ_OK;
}

kvq_status kvq_quantize_kv_paged(const kvq_format* f, const kvq_paged_cache* pc, const void* k_src,
                                 const void* v_src, int64_t sb, int64_t sh, int64_t st, const int32_t* blocks,
                                 int64_t n, int32_t* d_status, void* stream) {
  Layout L;
  kvq_status s = paged_layout(f, pc, &L);
  if (s != KVQ_OK) return s;
  if (!(asym_fast_ok(L, KVQ_KEYS) && asym_fast_ok(L, KVQ_VALUES))) return KVQ_ERR_UNSUPPORTED;
  if (n < 1 || n > L.g) return KVQ_ERR_INVALID;
  if (!blocks || (reinterpret_cast<uintptr_t>(blocks) & 3)) return KVQ_ERR_INVALID;
  if (!k_src || !v_src || !aligned16(k_src) || !aligned16(v_src)) return KVQ_ERR_INVALID;
  const int64_t eb = dtype_bytes(L.src_dtype);
  if (st < L.D || sb < 0 || sh < 0) return KVQ_ERR_INVALID;
  if ((st * eb) % 16 || (sh * eb) % 16 || (sb * eb) % 16) return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  const int num_blocks = L.B;
  Layout Ls = L;
  Ls.B = pc->num_seqs;   // the grid covers the sequences; destinations go through `blocks`
  cudaError_t e = launch_quantize_asym_kv(Ls, k_src, v_src, sb, sh, st, 0, n, d_status,
                                          reinterpret_cast<cudaStream_t>(stream), blocks, num_blocks);
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

static size_t paged_ws_bytes(const Layout& L, int num_seqs, int Hq, int S) {
  const size_t rows = (size_t)num_seqs * Hq * S;
  const size_t a16 = (rows * 4 + 15) & ~(size_t)15;
  return 2 * a16 + ((rows * L.D * 4 + 15) & ~(size_t)15);
}

static kvq_status paged_args(const kvq_format* f, int32_t num_seqs, int32_t Hq, int32_t Hkv, int64_t max_tq,
                             int32_t max_tr, Layout* L) {
  kvq_status s = kvq_format_check(f);
  if (s != KVQ_OK) return s;
  if (num_seqs < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv) return KVQ_ERR_INVALID;
  if (max_tq < 0 || max_tr < 0 || max_tr > f->residual_cap || f->n_sink + max_tq + max_tr < 1)
    return KVQ_ERR_INVALID;
  plan_layout(f, 1, Hkv, L);
  L->src_dtype = f->src_dtype;
  if (!paged_path_ok(*L, Hq)) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

size_t kvq_decode_paged_workspace_bytes(const kvq_format* f, int32_t num_seqs, int32_t Hq, int32_t Hkv,
                                        int64_t max_tq, int32_t max_tr) {
  Layout L;
  if (paged_args(f, num_seqs, Hq, Hkv, max_tq, max_tr, &L) != KVQ_OK) return 0;
  return paged_ws_bytes(L, num_seqs, Hq, paged_slots(L, max_tq, max_tr));
}

kvq_status kvq_decode_attention_paged(const kvq_format* f, const kvq_paged_cache* pc, const int32_t* t_quant,
                                      const int32_t* t_res, int64_t max_tq, int32_t max_tr, const void* q,
                                      int32_t q_dtype, int32_t Hq, float scale, void* out, int32_t out_dtype,
                                      void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  Layout L;
  kvq_status s = paged_layout(f, pc, &L);
  if (s != KVQ_OK) return s;
  Layout Lp;
  s = paged_args(f, pc->num_seqs, Hq, L.Hkv, max_tq, max_tr, &Lp);
  if (s != KVQ_OK) return s;
  if (max_tq > (int64_t)pc->max_blocks * L.g) return KVQ_ERR_INVALID;
  if (!t_quant || !t_res || (reinterpret_cast<uintptr_t>(t_quant) & 3) || (reinterpret_cast<uintptr_t>(t_res) & 3))
    return KVQ_ERR_INVALID;
  if (!q || !aligned16(q) || !valid_dtype(q_dtype) || !(scale > 0.0f)) return KVQ_ERR_INVALID;
  if (!out || !aligned16(out) || !valid_dtype(out_dtype)) return KVQ_ERR_INVALID;
  if (L.n_sink && (!pc->sink_k || !pc->sink_v || !aligned16(pc->sink_k) || !aligned16(pc->sink_v)))
    return KVQ_ERR_INVALID;
  if (max_tr && (!pc->res_k || !pc->res_v || !aligned16(pc->res_k) || !aligned16(pc->res_v)))
    return KVQ_ERR_INVALID;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)) return KVQ_ERR_INVALID;
  const int S = paged_slots(L, max_tq, max_tr);
  if ((int64_t)S > 65535 || (int64_t)pc->num_seqs * L.Hkv > 65535) return KVQ_ERR_UNSUPPORTED;
  if (!ws || !aligned16(ws)) return KVQ_ERR_INVALID;
  if (ws_bytes < paged_ws_bytes(L, pc->num_seqs, Hq, S)) return KVQ_ERR_WORKSPACE;
  const size_t rows = (size_t)pc->num_seqs * Hq * S;
  const size_t a16 = (rows * 4 + 15) & ~(size_t)15;
  float* ws_m = reinterpret_cast<float*>(ws);
  float* ws_l = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + a16);
  float* ws_o = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + 2 * a16);
  PagedDecode pd;
  pd.table = pc->block_table;
  pd.t_quant = t_quant;
  pd.t_res = t_res;
  pd.num_seqs = pc->num_seqs;
  pd.max_blocks = pc->max_blocks;
  pd.max_t_quant = max_tq;
  pd.max_t_res = max_tr;
  pd.sink[0] = pc->sink_k;
  pd.sink[1] = pc->sink_v;
  pd.res[0] = pc->res_k;
  pd.res[1] = pc->res_v;
  cudaError_t e = launch_decode_paged(L, pd, S, q, q_dtype, Hq, scale, ws_m, ws_l, ws_o, out, out_dtype, d_status,
                                      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // extern "C"
