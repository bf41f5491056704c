// kvq_decode_attention_noalloc: decode attention for callers that cannot allocate
// device memory.
//
// Some callers can neither call cudaMalloc nor hand the library a workspace: a
// serving process whose allocator reserved all device memory at start-up and owns
// every later allocation, or a plugin host that forbids allocation once it is
// running.  This entry point takes the split kernel's scratch (the partial softmax
// states) from a fixed array compiled into the library instead of a caller
// workspace.  Everything else -- inputs, outputs, kernels -- is the same as
// kvq_decode_attention.
#include <atomic>
#include <mutex>

#include "kvq_internal.cuh"

// The scratch: KVQ_NOALLOC_SCRATCH_BYTES per device, held by every GPU that loads the
// library until the process exits.  In host code this name is only a stand-in for the
// device array, never a device address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char kvq_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

namespace {

// The driver's cuCtxGetCurrent, reached through the runtime (no link against libcuda).
typedef int (*CtxGetCurrentFn)(void**);

CtxGetCurrentFn ctx_get_current() {
  static std::atomic<CtxGetCurrentFn> fn{nullptr};
  CtxGetCurrentFn f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && p != nullptr) {
      f = reinterpret_cast<CtxGetCurrentFn>(p);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

constexpr int kMaxDevices = 64;
// Per device: the context the address was looked up in, and the address.
std::mutex g_lock;
void* g_scratch_ctx[kMaxDevices];
void* g_scratch_addr[kMaxDevices];

// Device address of the scratch on the current device.  It is looked up (with that
// device current) the first time and again whenever the current context is not the one
// it was looked up in: after cudaDeviceReset, for instance, the library's device code is
// loaded anew in a new context, and an address kept from the old one is no longer mapped.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return cudaErrorInitializationError;
  void* ctx = nullptr;
  if (get(&ctx) != 0) return cudaErrorInitializationError;
  std::lock_guard<std::mutex> hold(g_lock);
  if (ctx == nullptr || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, kvq_noalloc_scratch);   // makes the device's context current
    if (e != cudaSuccess) return e;
    if (get(&ctx) != 0 || ctx == nullptr) return cudaErrorInitializationError;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_format* fmt, const kvq_cache* cache,
                                                   const void* q, int32_t q_dtype, int32_t q_heads,
                                                   int64_t t_quant, int32_t t_residual,
                                                   float softmax_scale, void* out, int32_t out_dtype,
                                                   int32_t num_splits, int32_t* d_status,
                                                   void* stream) {
  if (!fmt || !cache) return KVQ_ERR_INVALID;
  const size_t need = kvq_decode_workspace_bytes(fmt, cache->batch, q_heads, cache->kv_heads,
                                                 t_quant, t_residual, num_splits);
  if (need == 0) return kvq_format_check(fmt) != KVQ_OK ? kvq_format_check(fmt) : KVQ_ERR_INVALID;
  if (need > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return KVQ_ERR_CUDA;
  // Nothing in the scratch needs to start at zero: every partial state the combine
  // reads is written by the split kernel of the same call.
  return kvq_decode_attention(fmt, cache, q, q_dtype, q_heads, t_quant, t_residual, softmax_scale,
                              out, out_dtype, scratch, (size_t)KVQ_NOALLOC_SCRATCH_BYTES, num_splits,
                              d_status, stream);
}
