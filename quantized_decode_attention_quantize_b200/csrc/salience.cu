// MixKVQ key-channel salience ([MIX] Figure 3: A = I * S; Figure 4: recomputed over
// each window of R buffered tokens).
//
// One CTA per (kv head, batch), one thread per channel d.  I_d sums |Q[d]| over the
// G query heads of the group and the R window rows in fp64, head-major then row, and
// divides by G * R; S_d is the fp64 range of K[:, d]; A_d = I_d * S_d.  The rank of a
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
};

__global__ void __launch_bounds__(256) salience_kernel(SalArgs a) {
  __shared__ double A[256];
  __shared__ int bad;
  const int d = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = a.Hq / a.Hkv;
  if (d == 0) bad = 0;
  __syncthreads();
  double acc = 0.0;
  int nonfinite = 0;
  for (int hh = 0; hh < G; ++hh) {
    const int64_t qb = (int64_t)b * a.qsb + (int64_t)(h * G + hh) * a.qsh + d;
#pragma unroll 8
    for (int r = 0; r < a.R; ++r) {
      const float x = load_elem(a.q, qb + (int64_t)r * a.qst, a.dtype);
      nonfinite |= !isfinite(x);
      acc = __dadd_rn(acc, fabs((double)x));
    }
  }
  const double intensity = __ddiv_rn(acc, (double)G * (double)a.R);
  const int64_t kb = (int64_t)b * a.ksb + (int64_t)h * a.ksh + d;
  float mn = INFINITY, mx = -INFINITY;
  for (int r = 0; r < a.R; ++r) {
    const float x = load_elem(a.k, kb + (int64_t)r * a.kst, a.dtype);
    nonfinite |= !isfinite(x);
    mn = fminf(mn, x);
    mx = fmaxf(mx, x);
  }
  const double range = __dsub_rn((double)mx, (double)mn);
  const double sal = __dmul_rn(intensity, range);
  A[d] = sal;
  if (nonfinite) atomicOr(&bad, 1);
  __syncthreads();
  int rank = 0;
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
  dim3 grid(Hkv, B);
  salience_kernel<<<grid, L.D, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
