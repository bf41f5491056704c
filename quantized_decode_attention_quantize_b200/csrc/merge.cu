// Merge of decode results computed over disjoint token ranges (a sequence split: each
// range, e.g. on its own GPU, runs the split kernel and the combine with its log-sum-exp;
// the results are gathered and merged here).  For query row i over parts r:
//
//   out_i = sum_r exp(lse_ri - M_i) out_ri / sum_r exp(lse_ri - M_i),   M_i = max_r lse_ri
//   lse_i = M_i + log sum_r exp(lse_ri - M_i)
//
// the same log-sum-exp merge the combine applies to the partial states of one range
// ([KVQ] "Approach": long contexts split over devices; the softmax normaliser is the
// only quantity the parts must agree on).
#include "kvq_internal.cuh"

namespace kvq {
namespace {

struct MergeArgs {
  int n, D;
  int64_t rows;
  const float* outs;   // [n][rows][D]
  const float* lses;   // [n][rows]
  void* out;
  int out_dtype;
  float* lse_out;      // nullable
};

// One warp per row; lane holds D / 32 channels (c = lane + 32 j).
__global__ void __launch_bounds__(128) merge_states_kernel(MergeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  float M = -INFINITY;
  for (int r = 0; r < a.n; ++r) M = fmaxf(M, a.lses[(int64_t)r * a.rows + row]);
  float W = 0.0f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int nj = a.D / 32;
  for (int r = 0; r < a.n; ++r) {
    const float lr = a.lses[(int64_t)r * a.rows + row];
    if (lr == -INFINITY) continue;   // a part with no tokens
    const float w = __expf(lr - M);
    W += w;
    const float* o = a.outs + ((int64_t)r * a.rows + row) * a.D;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < nj) acc[j] = fmaf(w, o[lane + 32 * j], acc[j]);
  }
  // a row that no part has tokens for (every lse = -inf): zeros and lse = -inf
  const float inv = W > 0.0f ? 1.0f / W : 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < nj) store_elem(a.out, row * a.D + lane + 32 * j, a.out_dtype, acc[j] * inv);
  if (a.lse_out && lane == 0) a.lse_out[row] = W > 0.0f ? M + logf(W) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge_states(int n, int64_t rows, int D, const float* outs, const float* lses,
                                void* out, int out_dtype, float* lse_out, cudaStream_t s) {
  MergeArgs a;
  a.n = n;
  a.D = D;
  a.rows = rows;
  a.outs = outs;
  a.lses = lses;
  a.out = out;
  a.out_dtype = out_dtype;
  a.lse_out = lse_out;
  merge_states_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
