/*
 * kvq.h -- C ABI of the packed low-bit KV cache and of decode attention over it.
 *
 * One shared library (libkvq.so) built for sm_100a.  Every entry point is a plain
 * C function taking plain pointers and sizes; there are no C++ or framework types
 * in any signature.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Ownership.  The caller owns every buffer.  The library allocates no memory,
 *    keeps no global state, never synchronises the stream and never frees anything.
 *    Array sizes come from kvq_cache_array_bytes() / kvq_decode_workspace_bytes().
 *  - Pointers.  Arguments documented as "device" must point to device memory of the
 *    current CUDA device and be 16-byte aligned.  "host" pointers are read during
 *    the call only.
 *  - Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued on it and the call returns without waiting.
 *  - Host errors.  Arguments are validated before anything is launched: a bad
 *    argument returns KVQ_ERR_INVALID, a valid but unimplemented combination returns
 *    KVQ_ERR_UNSUPPORTED, and nothing is enqueued in either case.  A failed launch
 *    returns KVQ_ERR_CUDA.
 *  - Device errors.  `d_status` (device int32, may be NULL) receives bits OR-ed in by
 *    the kernels: KVQ_DEV_NONFINITE when an input element is NaN or Inf (the inputs
 *    are rejected, as the INT8 page prescribes: the affected outputs are
 *    unspecified), KVQ_DEV_RANGE when a scale, zero-point or outlier value does not
 *    fit fp16, KVQ_DEV_TIMEOUT when a bounded in-kernel wait expired.  The caller
 *    zeroes the word and reads it back when it wants to know.
 *  - Layouts.  B = batch, Hkv = KV heads, Hq = query heads, G = Hq / Hkv, D = head
 *    dimension.  Query head h reads KV head h / G (contiguous GQA grouping).
 *    Every cache array is [B][Hkv][slab] with the per-(b, kv-head) slab laid out as
 *    described at each array below; slabs are contiguous and in (b, kv-head) order.
 *
 * Sources (web pages; section named after the title):
 *  [AXES]   "KV quantization axes: why Key and Value need separate reasoning",
 *           sections "What rows and columns mean", "Separate the two error paths",
 *           "Scales occupy bytes too".
 *  [KVQ]    "KVQuant: Towards 10 Million Context Length LLM Inference with KV Cache
 *           Quantization", sections "Approach", "Key results", "Measured effects".
 *  [MIX]    "MixKVQ: Query-Aware Mixed-Precision KV Cache Quantization for
 *           Long-Context Reasoning", Figures 3 and 4.
 *  [K4V2]   "Quantize What Counts: More for Keys, Less for Values", Technical
 *           Summary ("Key Contributions", "Results", "Rotation Integration").
 *  [TQ]     "Statistical Inference and Quality Measures of KV Cache Quantisations
 *           Inspired by TurboQuant", Technical Summary (the KQV scheme's
 *           Walsh-Hadamard transform, "Fat-Tail Robustness").
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_VERSION_MAJOR 0
#define KVQ_VERSION_MINOR 2

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID = 1,      /* bad argument: null, misaligned, out of range, shape mismatch */
  KVQ_ERR_UNSUPPORTED = 2,  /* well-formed request this library does not implement */
  KVQ_ERR_CUDA = 3,         /* a CUDA call or a kernel launch failed */
  KVQ_ERR_WORKSPACE = 4     /* workspace smaller than kvq_decode_workspace_bytes() */
} kvq_status;

/* Bits OR-ed into the caller's device status word.  KVQ_DEV_TIMEOUT: a bounded wait
 * inside a kernel ran out (the kernel stopped early; its outputs are unspecified).
 * KVQ_DEV_BOUNDS: a device-side length or block id was out of range (paged entry
 * points); the work it named was skipped and the affected outputs are unspecified. */
enum { KVQ_DEV_NONFINITE = 1, KVQ_DEV_RANGE = 2, KVQ_DEV_TIMEOUT = 4, KVQ_DEV_BOUNDS = 8 };

/* Element types of sources, raw tokens, queries and outputs. */
enum { KVQ_F32 = 0, KVQ_F16 = 1, KVQ_BF16 = 2 };

/* Quantization schemes.
 *  KVQ_NONE  : the "codes" array holds the raw source values (src_dtype).
 *  KVQ_SYM8  : symmetric INT8 of [AXES] "What rows and columns mean":
 *                m = max|x| over the group; s = fl32(m / 127), s = 1 when m == 0;
 *                code = clip(rint_even(fl32(x / s)), -127, 127); x^ = fl32(code * s).
 *              Scales are fp32.  Axis TENSOR: one scale per token group of
 *              `group_tokens` tokens over all channels; TOKEN: one scale per token
 *              row; CHANNEL: one scale per channel per token group.
 *  KVQ_ASYM  : asymmetric b-bit (b = 2, 4, 8) with fp16 scale and zero-point, the
 *              min/max form of the low-bit quantizers the KVQuant page compares
 *              against (KIVI):  z = fp16_down(min), s = fp16_up(fl32(fl32(max - z)
 *              / (2^b - 1))), s = 1 when that is 0;
 *              code = clip(rint_even(fl32(fl32(x - z) / s)), 0, 2^b - 1);
 *              x^ = fl32(code * s + z)  (code * s is exact in fp32).
 *              Keys: axis CHANNEL (per channel over a token group, [KVQ] "Approach");
 *              values: axis TOKEN (per token over the D channels).
 *  KVQ_NUQ   : 3-bit non-uniform codebook ("nuq3", [KVQ] "Approach") with per-vector
 *              dense-and-sparse outliers.  For a vector (a key channel over its token
 *              group, or a value token row) the n_outliers largest |x| (ties: lower
 *              index) are kept as fp16 in a sparse side list and excluded from the
 *              statistics; mn/mx over the rest; z = fp16_near(fl32(fl32(mx + mn) * 0.5)),
 *              s = fp16_up(max(fl32(mx - z), fl32(z - mn))), s = 1 when 0;
 *              y = fl32(fl32(x' - z) / s) with x' = x clipped to [mn, mx];
 *              code = #{ j in 0..6 : y > fl32(fl32(C[j] + C[j+1]) * 0.5) } for the
 *              eight ascending fp16 centroids C (the LUT); x^ = fl32(C[code] * s + z),
 *              replaced by the stored fp16 value at outlier positions.
 *  KVQ_MIXED : keys only, salience-selected tiers of [MIX] Figure 3: per token group
 *              an order[] (slot -> channel, by descending salience, see
 *              kvq_key_salience); slots [0, mixed_hi) keep the raw 16-bit source,
 *              slots [mixed_hi, mixed_hi + mixed_mid) use KVQ_ASYM 4-bit and the rest
 *              KVQ_ASYM 2-bit, both per channel over the group.
 *  KVQ_KQV   : the KQV scheme of [TQ] ("Quantization Schemes"), keys and values
 *              together (both sides KVQ_KQV, axis TOKEN, D = 128, no outliers, rope or
 *              k_rotate).  Each token row x is rotated, y = the fp32 Walsh-Hadamard
 *              transform described at k_rotate, and coded by its direction: with the
 *              pairwise-tree fp32 sum T over the channels (level 1 adds elements 2i and
 *              2i + 1, every later level the results 2i and 2i + 1 of the one before),
 *              n = fl32(sqrt(T(fl32(y_c * y_c)))), u_c = fl32(y_c / n) (0 when n = 0),
 *              code_c = #{ j : u_c > fl32(fl32(C[j] + C[j+1]) * 0.5) } for the 2^b
 *              ascending fp32 centroids C of the LUT (b = k_bits for keys, v_bits - 1
 *              for values: v_bits is the value budget including the sketch bit).  Values
 *              add a one-bit sketch of the residual: yh_c = fl32(n * C[code_c]),
 *              r_c = fl32(y_c - yh_c), rn = fl32(sqrt(T(fl32(r_c * r_c)))), and for each
 *              row i of the D x D fp32 matrix S (cache->v_sketch) sign bit
 *              s_i = (T_c(fl32(S[i][c] * r_c)) >= 0).  Reconstruction (real-valued):
 *              k^ = H (n C[code]),  v^ = H (n C[code] + sqrt(pi/2) / D * rn * S^T s),
 *              s_i = +1 for a set bit and -1 otherwise, H the orthonormal transform.
 */
enum { KVQ_NONE = 0, KVQ_SYM8 = 1, KVQ_ASYM = 2, KVQ_NUQ = 3, KVQ_MIXED = 4, KVQ_KQV = 5 };

/* Grouping axes ([AXES]: tensor / token / channel scales). */
enum { KVQ_AXIS_TENSOR = 0, KVQ_AXIS_TOKEN = 1, KVQ_AXIS_CHANNEL = 2 };

/* Which half of the cache. */
enum { KVQ_KEYS = 0, KVQ_VALUES = 1 };

typedef struct kvq_format {
  int32_t head_dim;      /* D: 32, 64, 128 or 256                                          */
  int32_t group_tokens;  /* g: tokens per group (channel / tensor axes and the unit of
                            appends); a multiple of 16 in [16, 256], g * D <= 32768        */
  int32_t src_dtype;     /* KVQ_F32 / KVQ_F16 / KVQ_BF16: quantize inputs and raw tokens   */
  int32_t k_scheme, k_bits, k_axis, k_outliers;
  int32_t v_scheme, v_bits, v_axis, v_outliers;
  int32_t mixed_hi;      /* KVQ_MIXED: raw 16-bit key channels per group (multiple of 8)   */
  int32_t mixed_mid;     /* KVQ_MIXED: 4-bit key channels per group (multiple of 8); the
                            remaining D - hi - mid (a multiple of 16) are 2-bit            */
  int32_t n_sink;        /* tokens [0, n_sink) are kept raw (attention sink, [KVQ])       */
  int32_t residual_cap;  /* capacity of the raw window of recent tokens ([MIX] Figure 4)  */
  int32_t rope;          /* 1: keys are stored pre-RoPE and decode rotates every key at
                            its absolute position ([KVQ] "Approach")                      */
  float rope_base;       /* RoPE base (10000); rotate-half pairs (i, i + D/2),
                            theta_i = base^(-2i/D)                                       */
  int32_t k_rotate;      /* 1: key-only rotation ([K4V2] "Rotation Integration", [TQ]):
                            every key row x is replaced, before its statistics, by
                            y = H_D x / sqrt(D), the orthonormal Sylvester-ordered
                            Walsh-Hadamard transform, evaluated in fp32 as the butterfly
                            over strides 1, 2, ..., D/2 (pair (i, i+h) -> (a+b, a-b),
                            each rounded) and one product with fl32(1/sqrt(D)).  Codes,
                            metadata and outliers then live in the rotated basis;
                            kvq_dequantize maps keys back with the same transform (its
                            own inverse) and decode rotates the query instead, since
                            q'.y = q.x.  Raw sink and residual keys stay unrotated.
                            Keys of scheme SYM8, ASYM or NUQ, without rope.            */
} kvq_format;

/* Cache arrays.  Per (b, kv-head) slab, with capacity C tokens (a multiple of g),
 * ngroups = C / g, packed token index i = absolute position - n_sink:
 *
 *  k_codes / v_codes
 *    NONE   [C][D] src_dtype.
 *    SYM8   [C][D] int8.
 *    ASYM8  [C][D] uint8.
 *    ASYM4 / ASYM2, keys: [C][D*b/32] uint32, "row" layout: channel c sits in word
 *           c / (32/b) at bit b * (c % (32/b)) (LSB first).
 *    ASYM4 / ASYM2, values: [C/2][D*b/16] uint32, "pair" layout: tokens 2u and 2u+1
 *           share words; word w holds channels (16/b)*w .. (16/b)*(w+1)-1 of token 2u
 *           in its low 16 bits and of token 2u+1 in its high 16 bits, channel c at bit
 *           b * (c % (16/b)) of its half.  A missing odd token leaves its half zero.
 *    NUQ (3-bit), keys and values: [C][3*D/32] uint32 per token row: D/16 words of
 *           the low two code bits in the row layout, then D/32 words of the high bit
 *           (channel c at bit c % 32 of word c / 32).
 *    KQV, keys: [C][b*D/32] uint32 per token row, b = k_bits in {2, 3, 4}: the row
 *           layout for b = 2 and 4, the NUQ layout (two planes) for b = 3.
 *    KQV, values: [C][(b + 1)*D/32] uint32 per token row, b = v_bits - 1 in {1, 2, 3}:
 *           the codes as for keys (b = 1: row layout), then D/32 words of sketch bits
 *           (bit i at bit i % 32 of word i / 32).
 *    MIXED (keys): [ngroups][g * (2*hi + mid/2 + lo/4)] bytes per group: the raw
 *           plane [g][hi] src_dtype, then the 4-bit plane [g][mid/8] uint32 and the
 *           2-bit plane [g][lo/16] uint32, both in the row layout over slots.
 *  k_scale / k_zero
 *    SYM8   fp32 scale only: TENSOR [ngroups], TOKEN [C], CHANNEL [ngroups][D].
 *    ASYM, NUQ (channel axis)  fp16 [ngroups][D].
 *    MIXED  fp16 [ngroups][D - hi], indexed by slot - hi.
 *    KQV    k_scale: fp32 [C], the row norms n; no k_zero.
 *  v_scale / v_zero
 *    SYM8   fp32 as for keys.   ASYM, NUQ (token axis): fp16 [C].
 *    KQV    v_scale: fp32 [C], the row norms n; v_zero: fp32 [C], the residual norms rn.
 *  k_order             MIXED: uint8 [ngroups][D], slot -> channel.
 *  k_out_rowptr        NUQ keys with outliers: int32 [ngroups][g + 1]; CSR row
 *                      pointers by token row of the group, relative to the group's
 *                      first entry at (group * D * k_outliers).
 *  k_out_col, k_out_val  uint8 channel / fp16 value [ngroups][D * k_outliers],
 *                      sorted by (token row, channel) within the group.
 *  v_out_col, v_out_val  NUQ values with outliers: uint8 / fp16 [C][v_outliers]; a
 *                      CSR whose row pointer is implicit (k entries per token row),
 *                      sorted by channel within the row.
 *  k_lut / v_lut       NUQ: fp16 [8] ascending centroids in [-1, 1].
 *                      KQV: fp32 [2^b] ascending centroids (see kvq_kqv_codebook).
 *  v_sketch            KQV: fp32 [D][D], the sketch matrix S (row i = direction i);
 *                      one matrix for the whole cache, read by quantize, dequantize
 *                      and decode (the method's random draw, made by the caller).
 *  sink_k / sink_v     [n_sink][D] src_dtype (raw, pre-RoPE keys).
 *  res_k / res_v       [residual_cap][D] src_dtype (raw, pre-RoPE keys).
 * Unused arrays may be NULL.
 */
typedef struct kvq_cache {
  int32_t batch, kv_heads;
  int64_t capacity;
  void *k_codes, *k_scale, *k_zero, *k_order;
  void *k_out_rowptr, *k_out_col, *k_out_val;
  void *v_codes, *v_scale, *v_zero;
  void *v_out_col, *v_out_val;
  const void *k_lut, *v_lut;
  void *sink_k, *sink_v, *res_k, *res_v;
  const void* v_sketch;
} kvq_cache;

/* Array identifiers for kvq_cache_array_bytes (same order as kvq_cache). */
enum {
  KVQ_ARR_K_CODES = 0, KVQ_ARR_K_SCALE, KVQ_ARR_K_ZERO, KVQ_ARR_K_ORDER,
  KVQ_ARR_K_OUT_ROWPTR, KVQ_ARR_K_OUT_COL, KVQ_ARR_K_OUT_VAL,
  KVQ_ARR_V_CODES, KVQ_ARR_V_SCALE, KVQ_ARR_V_ZERO,
  KVQ_ARR_V_OUT_COL, KVQ_ARR_V_OUT_VAL,
  KVQ_ARR_K_LUT, KVQ_ARR_V_LUT,
  KVQ_ARR_SINK_K, KVQ_ARR_SINK_V, KVQ_ARR_RES_K, KVQ_ARR_RES_V,
  KVQ_ARR_V_SKETCH,
  KVQ_ARR_COUNT
};

/* Library version as (major << 16) | minor. */
int32_t kvq_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* kvq_status_string(kvq_status status);

/* Checks a format: KVQ_OK, KVQ_ERR_INVALID or KVQ_ERR_UNSUPPORTED.  Host only. */
kvq_status kvq_format_check(const kvq_format* fmt);

/* Bytes of one cache array for `batch` x `kv_heads` slabs of `capacity` tokens
 * (a multiple of group_tokens); 0 for an array the format does not use, and 0 for an
 * invalid format.  Host only.  With SYM8 K-channel / V-token, capacity = g = N this
 * reproduces the byte accounting 2ND + 4D + 4N of [AXES] "Scales occupy bytes too". */
size_t kvq_cache_array_bytes(const kvq_format* fmt, int32_t batch, int32_t kv_heads,
                             int64_t capacity, int32_t array_id);

/* Quantize n new key (or value) tokens into packed rows [t0, t0 + n) of the cache
 * ([AXES], [KVQ] "Approach", [K4V2]).  `src` is device memory holding
 * src[b][h][t][c] at element offset b*stride_b + h*stride_h + t*stride_t + c, in
 * fmt->src_dtype (stride_t >= D; every stride * element size a multiple of 16 bytes).
 * t0 must be a multiple of group_tokens (appends are whole groups; a partial last
 * group is allowed and a later call at the same t0 rewrites it), t0 + n <= capacity.
 * Keys of a MIXED format read the group's order from cache->k_order.  Writes codes,
 * scales, zero-points and outlier lists of the touched groups only. */
kvq_status kvq_quantize_keys(const kvq_format* fmt, const kvq_cache* cache,
                             const void* src, int64_t stride_b, int64_t stride_h,
                             int64_t stride_t, int64_t t0, int64_t n,
                             int32_t* d_status, void* stream);
kvq_status kvq_quantize_values(const kvq_format* fmt, const kvq_cache* cache,
                               const void* src, int64_t stride_b, int64_t stride_h,
                               int64_t stride_t, int64_t t0, int64_t n,
                               int32_t* d_status, void* stream);

/* Keys and values of one append: the same as kvq_quantize_keys(k_src) followed by
 * kvq_quantize_values(v_src) on the same stream, both sources with the same strides,
 * and bit for bit the same cache contents.  When both sides use the asymmetric
 * per-channel / per-token kernels (the K4/V2 decode format among them) it is one
 * launch instead of two. */
kvq_status kvq_quantize_kv(const kvq_format* fmt, const kvq_cache* cache, const void* k_src,
                           const void* v_src, int64_t stride_b, int64_t stride_h,
                           int64_t stride_t, int64_t t0, int64_t n, int32_t* d_status,
                           void* stream);

/* The Lloyd-Max centroids of KVQ_KQV ([TQ] "Theoretical Framework": a coordinate of a
 * uniformly random unit vector in head_dim dimensions has the density
 * (1 - x^2)^((d - 3) / 2) / B(1/2, (d - 1) / 2) on [-1, 1]): the 2^bits ascending
 * centroids minimising the mean squared error under that density (thresholds at the
 * midpoints, centroids at the conditional means, iterated to a fixed point by
 * quadrature in double and kept symmetric), rounded to fp32.  bits in 1..4, head_dim
 * in 3..4096.  `centroids` is host memory of 2^bits floats.  Host only; about a tenth
 * of a second. */
kvq_status kvq_kqv_codebook(int32_t bits, int32_t head_dim, float* centroids);

/* Reconstruct packed rows [t0, t0 + n) of keys or values (which = KVQ_KEYS/VALUES)
 * into `out` (device, [B][Hkv][n][D] contiguous, out_dtype).  fp32 output is the exact
 * x^ of the scheme; fp16 / bf16 output is that fp32 value rounded to nearest-even.
 * Outlier positions return their stored fp16 value; MIXED raw channels return the
 * stored source value.  No RoPE is applied.  KQV rows are the real-valued k^ / v^ of
 * the scheme evaluated in fp32 (products with the centroids, the sketch sum S^T s in
 * channel order, the Walsh-Hadamard butterfly), so they match it to fp32 rounding,
 * not bit for bit. */
kvq_status kvq_dequantize(const kvq_format* fmt, const kvq_cache* cache, int32_t which,
                          int64_t t0, int64_t n, void* out, int32_t out_dtype,
                          int32_t* d_status, void* stream);

/* MixKVQ key-channel salience over one window of R tokens ([MIX] Figures 3 and 4):
 *   I_d = (sum over the G query heads of the KV group, then over the R rows, of
 *          |Q[d]|, accumulated in fp64 in that order) / (G * R)
 *   S_d = max_r K[r][d] - min_r K[r][d]            (fp64)
 *   A_d = I_d * S_d                                  (fp64)
 * order_out receives the D channels sorted by descending A_d (ties: lower channel
 * first) at order_out[b*order_stride_b + h*order_stride_h + slot]; salience_out
 * (device fp64 [B][Hkv][D], may be NULL) receives A_d.  q: [b][hq][r][c] at
 * b*q_stride_b + hq*q_stride_h + r*q_stride_t + c; k likewise with kv heads; both in
 * fmt->src_dtype. */
kvq_status kvq_key_salience(const kvq_format* fmt, const void* q, int64_t q_stride_b,
                            int64_t q_stride_h, int64_t q_stride_t, const void* k,
                            int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_t,
                            int32_t batch, int32_t q_heads, int32_t kv_heads, int32_t R,
                            double* salience_out, uint8_t* order_out,
                            int64_t order_stride_b, int64_t order_stride_h,
                            int32_t* d_status, void* stream);

/* Workspace bytes for kvq_decode_attention with these sizes; num_splits = 0 selects
 * the split count the attention call would choose (depends on the current device's
 * SM count). */
size_t kvq_decode_workspace_bytes(const kvq_format* fmt, int32_t batch, int32_t q_heads,
                                  int32_t kv_heads, int64_t t_quant, int32_t t_residual,
                                  int32_t num_splits);

/* Decode attention over the cache ([AXES] "Separate the two error paths"):
 *   out[b][h] = sum_t softmax_t(softmax_scale * q[b][h] . k^_t) v^_t
 * over all T = n_sink + t_quant + t_residual tokens: the raw sink tokens, packed rows
 * [0, t_quant) and raw residual rows [0, t_residual), with k^ rotated at its absolute
 * position when fmt->rope.  q: device [B][Hq][D] in q_dtype (already rotated when
 * rope); out: device [B][Hq][D] in out_dtype.  Split-KV: num_splits (0 = automatic)
 * partial softmax states are written to `workspace` and merged by a second kernel. */
kvq_status kvq_decode_attention(const kvq_format* fmt, const kvq_cache* cache,
                                const void* q, int32_t q_dtype, int32_t q_heads,
                                int64_t t_quant, int32_t t_residual, float softmax_scale,
                                void* out, int32_t out_dtype, void* workspace,
                                size_t workspace_bytes, int32_t num_splits,
                                int32_t* d_status, void* stream);

/* One decode step with its append ([MIX] Figure 4: the full recent window is quantized
 * into the packed cache and the step then attends over all tokens; [KVQ] "Approach"):
 * the same as kvq_quantize_kv(fmt, cache, k_src, v_src, stride_b, stride_h, stride_t, t0,
 * n) followed by kvq_decode_attention(fmt, cache, q, ...) on the same stream, with the
 * same results bit for bit.  Every argument of both is checked before anything is
 * launched; n = 0 appends nothing.  For one group (t0 a multiple of 128, n <= 128) of a
 * K4-per-channel / V2-per-token cache with unrotated keys and 16-bit sources decoded by
 * the G <= 4 tensor-core split kernel, that kernel quantizes the group itself before its
 * decode (warp-sized units, each announced by a flag in the workspace; a warp waits for
 * its head's flags before it copies that group).  Otherwise, when the format's append is
 * one kernel and the tensor-core split kernel decodes it, the split kernel starts while
 * the append still runs and waits for it only where it reaches the appended rows. */
kvq_status kvq_append_decode_attention(const kvq_format* fmt, const kvq_cache* cache,
                                       const void* k_src, const void* v_src, int64_t stride_b,
                                       int64_t stride_h, int64_t stride_t, int64_t t0, int64_t n,
                                       const void* q, int32_t q_dtype, int32_t q_heads,
                                       int64_t t_quant, int32_t t_residual, float softmax_scale,
                                       void* out, int32_t out_dtype, void* workspace,
                                       size_t workspace_bytes, int32_t num_splits,
                                       int32_t* d_status, void* stream);

/* The two halves of kvq_decode_attention, for callers that time, overlap or
 * distribute them (for instance a sequence split over several GPUs that gathers the
 * partial states before merging them).  kvq_decode_partial runs the split kernel and
 * leaves the partial softmax states in `workspace`; kvq_decode_combine merges them
 * into `out`.  Both must be called with the same format, sizes and num_splits as the
 * workspace was sized for.  Workspace layout (fp32, each part padded to 16 bytes):
 *   m[B][Hq][S], l[B][Hq][S], o[B][Hq][S][D]   with S = kvq_decode_partial_slots();
 * slot s holds, for one query head, the running max m (log2 domain, i.e. of
 * scale * log2(e) * q . k), l = sum 2^(score - m) and o = sum 2^(score - m) v over
 * its share of the tokens (m = -inf, l = 0 for an empty share). */
int32_t kvq_decode_partial_slots(const kvq_format* fmt, int32_t batch, int32_t q_heads,
                                 int32_t kv_heads, int64_t t_quant, int32_t t_residual,
                                 int32_t num_splits);
kvq_status kvq_decode_partial(const kvq_format* fmt, const kvq_cache* cache, const void* q,
                              int32_t q_dtype, int32_t q_heads, int64_t t_quant,
                              int32_t t_residual, float softmax_scale, void* workspace,
                              size_t workspace_bytes, int32_t num_splits, int32_t* d_status,
                              void* stream);
kvq_status kvq_decode_combine(const kvq_format* fmt, int32_t batch, int32_t q_heads,
                              int32_t kv_heads, int64_t t_quant, int32_t t_residual,
                              int32_t num_splits, const void* workspace, size_t workspace_bytes,
                              void* out, int32_t out_dtype, void* stream);

/* Sequence split ([KVQ] "Approach": contexts spread over several GPUs).  Each part of a
 * context (a disjoint set of tokens: its own cache with its own sink / packed / residual
 * tokens, typically one per GPU) runs kvq_decode_partial as usual and then this combine,
 * which writes out[B][Hq][D] fp32 and lse[B][Hq] fp32, the natural log of the part's
 * softmax denominator: lse = log sum_t exp(softmax_scale * q . k_t).  Arguments and
 * errors otherwise as kvq_decode_combine (out and lse device, 16-byte aligned). */
kvq_status kvq_decode_combine_lse(const kvq_format* fmt, int32_t batch, int32_t q_heads,
                                  int32_t kv_heads, int64_t t_quant, int32_t t_residual,
                                  int32_t num_splits, const void* workspace,
                                  size_t workspace_bytes, float* out, float* lse, void* stream);

/* Merge of n_parts such results, gathered into outs[n_parts][rows][head_dim] and
 * lses[n_parts][rows] (device fp32, 16-byte aligned; rows = B * Hq): for every row,
 * out = sum_r w_r outs[r] / sum_r w_r with w_r = exp(lses[r] - max_r lses[r]); a part
 * with lse = -inf (no tokens) has weight 0, and a row whose every part has lse = -inf
 * gets out = 0 and lse_out = -inf.  out is written in out_dtype; lse_out
 * (nullable) receives the merged log-denominator.  The gather itself (one all-gather
 * of (head_dim + 1) * 4 bytes per query row and part) belongs to the caller's
 * collective library.  KVQ_ERR_INVALID for n_parts outside [1, 4096], rows outside
 * [1, 2^31], an unsupported head_dim, or bad pointers. */
kvq_status kvq_merge_states(int32_t n_parts, int64_t rows, int32_t head_dim, const float* outs,
                            const float* lses, void* out, int32_t out_dtype, float* lse_out,
                            void* stream);

/* ---- Paged cache with per-sequence lengths ---------------------------------------
 * A serving cache grows by whole token groups flushed from each sequence's raw window
 * ([MIX] Figure 4) and holds sequences of different lengths side by side ([MIX]
 * Figure 5 measures memory and throughput of such batches).  The pages give no
 * layout; this one is the plainest:
 *  - The packed arrays are a pool of num_blocks blocks, each holding one token group of
 *    every KV head, laid out exactly as a kvq_cache with batch = num_blocks, kv_heads
 *    and capacity = group_tokens (size each pool array with kvq_cache_array_bytes on
 *    those numbers; the group's key metadata sits at group 0 of its block).
 *  - Sequence s owns blocks block_table[s][0 .. ceil(t_quant[s] / group_tokens)), in
 *    token order; a block may belong to one sequence at a time.
 *  - The raw sink and residual arrays are per sequence, [num_seqs][kv_heads][...] as in
 *    kvq_cache.
 * Every group is quantized on its own, so a sequence's packed bytes are the same as in
 * a contiguous cache.  Formats: the 4-bit per-channel key / 2-bit per-token value
 * format with D = 128, group_tokens = 128, no RoPE and no MIXED keys (key rotation
 * allowed); decode needs q_heads / kv_heads <= 4.  Other combinations return
 * KVQ_ERR_UNSUPPORTED. */
typedef struct kvq_paged_cache {
  kvq_cache pool;             /* batch = num_blocks, capacity = group_tokens; its sink /
                                 residual pointers are not used                         */
  int32_t num_seqs;
  int32_t max_blocks;         /* columns of block_table                                 */
  const int32_t* block_table; /* device [num_seqs][max_blocks], physical block ids      */
  void *sink_k, *sink_v;      /* device [num_seqs][kv_heads][n_sink][D] src_dtype        */
  void *res_k, *res_v;        /* device [num_seqs][kv_heads][residual_cap][D] src_dtype  */
} kvq_paged_cache;

/* Quantize the first n (1 <= n <= group_tokens) tokens of one new token group of every
 * sequence into pool block blocks[s] (device int32 [num_seqs]): keys and values, in one
 * launch.  k_src / v_src: [s][h][t][c] at s*stride_b + h*stride_h + t*stride_t + c
 * (rules as kvq_quantize_kv).  A block id outside [0, num_blocks) sets KVQ_DEV_BOUNDS and
 * that sequence is skipped.  The 4-bit / 2-bit asymmetric format above only. */
kvq_status kvq_quantize_kv_paged(const kvq_format* fmt, const kvq_paged_cache* cache,
                                 const void* k_src, const void* v_src, int64_t stride_b,
                                 int64_t stride_h, int64_t stride_t, const int32_t* blocks,
                                 int64_t n, int32_t* d_status, void* stream);

/* Workspace bytes for kvq_decode_attention_paged with these bounds on the lengths. */
size_t kvq_decode_paged_workspace_bytes(const kvq_format* fmt, int32_t num_seqs, int32_t q_heads,
                                        int32_t kv_heads, int64_t max_t_quant, int32_t max_t_res);

/* Decode attention over a paged cache, every sequence over its own tokens: its n_sink
 * sink tokens, packed tokens [0, t_quant[s]) and residual rows [0, t_res[s]).
 * t_quant, t_res: device int32 [num_seqs]; max_t_quant / max_t_res are host bounds on
 * them (max_t_quant <= max_blocks * group_tokens, max_t_res <= residual_cap) that size
 * the launch and the workspace; a device length beyond its bound is clamped and sets
 * KVQ_DEV_BOUNDS, and so does a block id outside [0, num_blocks) (its group is then read
 * from block 0).  A sequence with no tokens at all gets out = 0.  q, out: device
 * [num_seqs][q_heads][D].  Otherwise as kvq_decode_attention.  One kernel computes the
 * partial states of chunks of each sequence's tokens, a second merges them. */
kvq_status kvq_decode_attention_paged(const kvq_format* fmt, const kvq_paged_cache* cache,
                                      const int32_t* t_quant, const int32_t* t_res,
                                      int64_t max_t_quant, int32_t max_t_res, const void* q,
                                      int32_t q_dtype, int32_t q_heads, float softmax_scale,
                                      void* out, int32_t out_dtype, void* workspace,
                                      size_t workspace_bytes, int32_t* d_status, void* stream);

/* Decode attention without a caller workspace, for callers that cannot allocate
 * device memory at all -- for example a serving process whose allocator reserved
 * every byte at start-up, or a plugin host that forbids allocation once running --
 * and so can neither call cudaMalloc nor pass `workspace`.  The pages describe no
 * such interface; it has no counterpart there.
 *
 * Same arguments, kernels and results as kvq_decode_attention, minus the workspace:
 * the partial softmax states go to a fixed array of KVQ_NOALLOC_SCRATCH_BYTES inside
 * the library (every GPU that loads the library holds it until the process exits).
 * Nothing is allocated and nothing is freed.  Returns KVQ_ERR_WORKSPACE when the
 * call would need more than KVQ_NOALLOC_SCRATCH_BYTES (see
 * kvq_decode_workspace_bytes).  The first call on a device looks up the array's
 * device address (with that device current) and keeps it, with the context it belongs
 * to, for later calls; make that first call outside any stream capture.  A later call
 * in another context of the device (after cudaDeviceReset, say) looks the address up
 * again, and that call too should come outside any stream capture.  All calls on a
 * device share the one array and it keeps the last call's contents: calls that overlap
 * on the GPU (on different streams, or from different host threads) race with one
 * another. */
#define KVQ_NOALLOC_SCRATCH_BYTES (16u << 20)
kvq_status kvq_decode_attention_noalloc(const kvq_format* fmt, const kvq_cache* cache,
                                        const void* q, int32_t q_dtype, int32_t q_heads,
                                        int64_t t_quant, int32_t t_residual, float softmax_scale,
                                        void* out, int32_t out_dtype, int32_t num_splits,
                                        int32_t* d_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H_ */
