// Rotary position embedding at logical positions.
//
// SpecOPD review (jaehun.me) §3.2(a): RoPE uses each token's logical
// position, not the packing order; paper summary (rustineverything.app)
// §2.1: a branch token's position is the anchor position plus its offset.
// The pages fix no convention; this library uses the half-split pairing
// (d, d + D/2) with angle pos * base^(-2k/D).
//
// Precision: the angle pos * theta_k can reach ~3e4 rad, where an fp32
// product alone would lose ~2e-3 rad.  The angle is therefore formed and
// reduced to [-pi, pi] in double precision (theta_k is computed on the host
// in double), and only the reduced angle goes through fp32 sincosf.
//
// Memory-bound elementwise kernel: one thread per (row, head, pair k).
#include "common.cuh"
#include "kernels.h"

namespace specopd {

struct RopeTheta {
  double theta[128];  // D/2 <= 128
};

template <typename T>
__global__ void rope_kernel(const T* __restrict__ x, T* __restrict__ y,
                            const int32_t* __restrict__ pos, int n, int H, int D,
                            const RopeTheta th) {
  const int half = D >> 1;
  const long long total = (long long)n * H * half;
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(g % half);
    const long long th_idx = g / half;  // t*H + h
    const int t = (int)(th_idx / H);
    const double ang = (double)pos[t] * th.theta[k];
    const double red = ang - two_pi * rint(ang * inv_two_pi);
    float sn, cs;
    sincosf((float)red, &sn, &cs);
    const long long base = th_idx * D;
    const float x1 = Elt<T>::to_f(x[base + k]);
    const float x2 = Elt<T>::to_f(x[base + k + half]);
    y[base + k] = Elt<T>::from_f(x1 * cs - x2 * sn);
    y[base + k + half] = Elt<T>::from_f(x2 * cs + x1 * sn);
  }
}

cudaError_t launch_rope(specopd_dtype dt, const void* x, void* y, const int32_t* pos, int n, int H,
                        int D, const double* theta_host, cudaStream_t st) {
  RopeTheta th;
  for (int k = 0; k < D / 2; ++k) th.theta[k] = theta_host[k];
  const long long total = (long long)n * H * (D / 2);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (dt == SPECOPD_F32)
    rope_kernel<float><<<(int)blocks, threads, 0, st>>>((const float*)x, (float*)y, pos, n, H, D, th);
  else
    rope_kernel<__nv_bfloat16><<<(int)blocks, threads, 0, st>>>(
        (const __nv_bfloat16*)x, (__nv_bfloat16*)y, pos, n, H, D, th);
  return cudaGetLastError();
}

}  // namespace specopd
