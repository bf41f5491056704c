// Reconstruction of packed rows into fp32 / fp16 / bf16.
//
// One CTA per (32-token chunk, kv head, batch): the dense values are written into a
// shared-memory tile (MIXED keys scatter slot -> channel through the group's order),
// the chunk's sparse outliers overwrite their positions, keys of a rotating format are
// transformed back to the original basis, and the tile is stored
// coalesced in the output dtype (fp32 exact, 16-bit by round-to-nearest-even).
#include "decode_common.cuh"
#include "wht.cuh"

namespace kvq {
namespace {

constexpr int kTok = 32;
constexpr int kThreads = 256;

struct DqArgs {
  Layout L;
  int which;
  int64_t t0, n;
  void* out;
  int out_dtype;
};

__global__ void __launch_bounds__(kThreads) dequant_kernel(DqArgs a) {
  extern __shared__ __align__(16) float tile[];  // [kTok][D]
  const Layout& L = a.L;
  const int D = L.D;
  const int64_t sl = (int64_t)blockIdx.z * L.Hkv + blockIdx.y;
  const int64_t tb = a.t0 + (int64_t)blockIdx.x * kTok;
  const int nt = (int)min((int64_t)kTok, a.t0 + a.n - tb);
  const Side& S = L.side[a.which];
  if (S.scheme == KVQ_MIXED) {
    for (int i = threadIdx.x; i < nt * D; i += blockDim.x) {
      const int r = i / D, j = i % D;
      const int64_t t = tb + r;
      const int c = L.k_order[(sl * L.ng + t / L.g) * D + j];
      tile[r * D + c] = mixed_slot_value(L, sl, t, j);
    }
  } else {
    for (int i = threadIdx.x; i < nt * D; i += blockDim.x) {
      const int r = i / D, c = i % D;
      tile[i] = deq_dense(L, a.which, sl, tb + r, c);
    }
  }
  __syncthreads();
  if (S.nout > 0) {
    for (int r = threadIdx.x; r < nt; r += blockDim.x) {
      const int64_t t = tb + r;
      if (a.which == KVQ_KEYS) {
        const int64_t gi = t / L.g;
        const int rr = (int)(t % L.g);
        const int32_t* rp = L.k_out_rowptr + (sl * L.ng + gi) * (L.g + 1);
        const int64_t e0 = (sl * L.ng + gi) * (int64_t)D * S.nout;
        for (int e = rp[rr]; e < rp[rr + 1]; ++e)
          tile[r * D + L.k_out_col[e0 + e]] = __half2float(L.k_out_val[e0 + e]);
      } else {
        for (int e = 0; e < S.nout; ++e) {
          const int64_t idx = (sl * L.C + t) * S.nout + e;
          tile[r * D + L.v_out_col[idx]] = __half2float(L.v_out_val[idx]);
        }
      }
    }
    __syncthreads();
  }
  if (a.which == KVQ_KEYS && L.k_rotate) {   // back from the rotated basis (own inverse)
    wht_tile_rows(tile, nt, D, L.rot_scale);
    __syncthreads();
  }
  const int64_t obase = (sl * a.n + (tb - a.t0)) * D;
  for (int i = threadIdx.x; i < nt * D; i += blockDim.x) store_elem(a.out, obase + i, a.out_dtype, tile[i]);
}

}  // namespace

cudaError_t launch_dequantize(const Layout& L, int which, int64_t t0, int64_t n, void* out,
                              int out_dtype, int32_t* d_status, cudaStream_t s) {
  (void)d_status;
  if (L.side[which].scheme == KVQ_KQV) return launch_dequantize_kqv(L, which, t0, n, out, out_dtype, s);
  DqArgs a;
  a.L = L;
  a.which = which;
  a.t0 = t0;
  a.n = n;
  a.out = out;
  a.out_dtype = out_dtype;
  const size_t smem = (size_t)kTok * L.D * sizeof(float);
  dim3 grid((unsigned)((n + kTok - 1) / kTok), L.Hkv, L.B);
  dequant_kernel<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
