// MixKVQ key-channel salience ([MIX] Figure 3: A = I * S; Figure 4: recomputed over
// each window of R buffered tokens).
//
// One CTA per (kv head, batch), one thread per channel d.  The window rows are staged
// through shared memory in chunks of 64 rows, double-buffered with asynchronous 16-byte
// copies (element copies where the strides do not allow them) by all threads.  I_d sums |Q[d]| over the G query heads of the group and
// the R window rows in fp64, head-major then row, and divides by G * R; S_d is the fp64 range of K[:, d]; A_d = I_d * S_d.  The rank of a
// channel is the number of channels with a larger A (or an equal A and a lower
// index), so order[rank] = d sorts by descending salience with ties to the lower
// channel.  Every fp64 step is a single IEEE operation, so the result is the same
// bit pattern the plain sequential definition gives.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

struct SalArgs {
  int D, dtype, B, Hq, Hkv, R;
  const void* q;
  int64_t qsb, qsh, qst;
  const void* k;
  int64_t ksb, ksh, kst;
  double* sal;
  uint8_t* order;
  int64_t osb, osh;
  int32_t* status;
  int q_vec, k_vec;   // 16-byte staging loads allowed (aligned base and strides)
};

constexpr int kRC = 64;   // window rows per staged chunk

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// Rows [r0, r0 + nr) of a [R][D] window (element offsets base + r * rstride + c) into
// buf[r - r0][c], by all D threads of the CTA: asynchronous 16-byte copies when the
// base and strides allow (completed by the caller's wait), element copies otherwise.
__device__ __forceinline__ void stage_rows(uint8_t* buf, const void* src, int64_t base, int64_t rstride,
                                           int r0, int nr, int D, int esz, bool vec) {
  const uint8_t* s8 = reinterpret_cast<const uint8_t*>(src);
  if (vec) {
    const int vpr = D * esz / 16;
    for (int v = threadIdx.x; v < nr * vpr; v += blockDim.x) {
      const int row = v / vpr, cv = v - row * vpr;
      cp_async16(buf + (size_t)row * D * esz + cv * 16, s8 + (base + (int64_t)(r0 + row) * rstride) * esz + cv * 16);
    }
  } else {
    for (int i = threadIdx.x; i < nr * D; i += blockDim.x) {
      const int row = i / D, c = i - row * D;
      const uint8_t* from = s8 + (base + (int64_t)(r0 + row) * rstride + c) * esz;
      uint8_t* to = buf + (size_t)i * esz;
      for (int e = 0; e < esz; ++e) to[e] = from[e];
    }
  }
}

// The window as one sequence of chunks: query rows of head 0, 1, ..., G - 1 (R rows each,
// kRC at a time), then the key rows.  Two staging buffers: chunk c + 1 is in flight while
// chunk c is summed, so the fp64 chain of each channel overlaps the loads.
// One staged element as fp32 (exact), for source dtype DT.
template <int DT>
__device__ __forceinline__ float staged(const uint8_t* buf, int i) {
  if constexpr (DT == KVQ_F32) return reinterpret_cast<const float*>(buf)[i];
  const uint16_t h = reinterpret_cast<const uint16_t*>(buf)[i];
  if constexpr (DT == KVQ_F16) return half_bits_to_float(h);
  return __uint_as_float((uint32_t)h << 16);
}

template <int DT>
__global__ void __launch_bounds__(256) salience_kernel(SalArgs a) {
  extern __shared__ __align__(16) uint8_t sbuf[];   // [2][kRC][D] source elements
  __shared__ double A[256];
  __shared__ int bad;
  const int d = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = a.Hq / a.Hkv;
  const int D = a.D;
  constexpr int esz = DT == KVQ_F32 ? 4 : 2;
  const size_t bufb = (size_t)kRC * D * esz;
  const int cpw = (a.R + kRC - 1) / kRC;            // chunks per window
  const int nq = G * cpw, n = nq + cpw;
  const int64_t kb = (int64_t)b * a.ksb + (int64_t)h * a.ksh;
  auto issue = [&](int c) {
    if (c < n) {
      uint8_t* buf = sbuf + (c & 1) * bufb;
      const int w = c < nq ? c % cpw : c - nq;
      const int r0 = w * kRC, nr = min(kRC, a.R - r0);
      if (c < nq) {
        const int64_t qb = (int64_t)b * a.qsb + (int64_t)(h * G + c / cpw) * a.qsh;
        stage_rows(buf, a.q, qb, a.qst, r0, nr, D, esz, a.q_vec);
      } else {
        stage_rows(buf, a.k, kb, a.kst, r0, nr, D, esz, a.k_vec);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (d == 0) bad = 0;
  double acc = 0.0;
  float mn = INFINITY, mx = -INFINITY;
  int nonfinite = 0;
  issue(0);
  for (int c = 0; c < n; ++c) {
    issue(c + 1);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();   // chunk c staged by every thread
    const uint8_t* buf = sbuf + (c & 1) * bufb;
    const int w = c < nq ? c % cpw : c - nq;
    const int nr = min(kRC, a.R - w * kRC);
    if (c < nq) {      // head-major, then row: the order of the plain definition
      // (a NaN or an infinity among the |Q| carries through to acc, checked at the end)
#pragma unroll 16
      for (int r = 0; r < nr; ++r) acc = __dadd_rn(acc, (double)fabsf(staged<DT>(buf, r * D + d)));
    } else {
#pragma unroll 16
      for (int r = 0; r < nr; ++r) {
        const float x = staged<DT>(buf, r * D + d);
        nonfinite |= !(fabsf(x) <= 3.402823466e38f);   // NaN and +-inf
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
    }
    __syncthreads();   // before chunk c + 2 overwrites this buffer
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  nonfinite |= !isfinite(acc);
  const double intensity = __ddiv_rn(acc, (double)G * (double)a.R);
  const double range = __dsub_rn((double)mx, (double)mn);
  const double sal = __dmul_rn(intensity, range);
  A[d] = sal;
  if (nonfinite) atomicOr(&bad, 1);
  __syncthreads();
  int rank = 0;
#pragma unroll 16
  for (int e = 0; e < a.D; ++e) {
    const double v = A[e];
    rank += (v > sal || (v == sal && e < d)) ? 1 : 0;
  }
  a.order[(int64_t)b * a.osb + (int64_t)h * a.osh + rank] = (uint8_t)d;
  if (a.sal) a.sal[((int64_t)b * a.Hkv + h) * a.D + d] = sal;
  if (d == 0 && bad) flag(a.status, KVQ_DEV_NONFINITE);
}

}  // namespace

cudaError_t launch_salience(const Layout& L, const void* q, int64_t qsb, int64_t qsh, int64_t qst,
                            const void* k, int64_t ksb, int64_t ksh, int64_t kst, int B, int Hq,
                            int Hkv, int R, double* sal, uint8_t* order, int64_t osb, int64_t osh,
                            int32_t* d_status, cudaStream_t s) {
  SalArgs a;
  a.D = L.D;
  a.dtype = L.src_dtype;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.R = R;
  a.q = q;
  a.qsb = qsb;
  a.qsh = qsh;
  a.qst = qst;
  a.k = k;
  a.ksb = ksb;
  a.ksh = ksh;
  a.kst = kst;
  a.sal = sal;
  a.order = order;
  a.osb = osb;
  a.osh = osh;
  a.status = d_status;
  const int esz = L.src_dtype == KVQ_F32 ? 4 : 2;
  auto vec_ok = [&](const void* p, int64_t s1, int64_t s2, int64_t s3) {
    return (reinterpret_cast<uintptr_t>(p) % 16 == 0) && (s1 * esz) % 16 == 0 && (s2 * esz) % 16 == 0 &&
           (s3 * esz) % 16 == 0 && (L.D * esz) % 16 == 0;
  };
  a.q_vec = vec_ok(q, qsb, qsh, qst);
  a.k_vec = vec_ok(k, ksb, ksh, kst);
  const size_t smem = 2 * (size_t)kRC * L.D * esz;
  auto kern = L.src_dtype == KVQ_F32 ? salience_kernel<KVQ_F32>
             : L.src_dtype == KVQ_F16 ? salience_kernel<KVQ_F16> : salience_kernel<KVQ_BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(Hkv, B);
  kern<<<grid, L.D, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
