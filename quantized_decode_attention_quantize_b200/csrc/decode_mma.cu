// Tensor-core split-KV decode over packed K4 / V2 (placeholder until the kernel lands).
#include "kvq_internal.cuh"

namespace kvq {

bool mma_path_ok(const Layout& L, int Hq) {
  (void)L;
  (void)Hq;
  return false;
}

int mma_ctas_per_sm() { return 1; }

cudaError_t launch_decode_mma(const Layout&, const DecodePlan&, const void*, int, int, int64_t, int,
                              float, float*, float*, float*, int32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kvq
