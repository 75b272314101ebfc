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
// Memory-bound elementwise kernel: one thread per (row, pair k, group of
// eight heads), so each angle is evaluated once per eight heads.
#include "common.cuh"
#include "kernels.h"

namespace specopd {

struct RopeTheta {
  double theta[128];  // D/2 <= 128
};

// Up to two tensors rotated at the same positions (branch q and k).
struct RopeJob {
  const void* x;
  void* y;
  int H;  // heads; 0 = no job
};

constexpr int kRopeHeadGroup = 8;  // heads per thread: loads batched ahead of the stores

// One thread per (row t, pair k, group of 8 heads of one tensor): the angle
// is reduced and its sine/cosine evaluated once per group, and the 16 loads
// of the group are issued before any store (the tensor may be rotated in
// place, so loads and stores of one head cannot be reordered by the compiler).
// Position of row t: pos[t], or, with pos == NULL, its index within its
// trunk sequence (t - cu[s] for cu[s] <= t < cu[s+1]; cu has S + 1 entries).
__device__ __forceinline__ int row_position(const int32_t* __restrict__ pos,
                                            const int32_t* __restrict__ cu, int S, long long t) {
  if (pos) return pos[t];
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return (int)(t - cu[lo]);
}

template <typename T>
__global__ void rope_kernel(const RopeJob j0, const RopeJob j1, const int32_t* __restrict__ pos,
                            const int32_t* __restrict__ cu, int S, int n, int D,
                            const RopeTheta th) {
  const int half = D >> 1;
  const int g0 = (j0.H + kRopeHeadGroup - 1) / kRopeHeadGroup;
  const int g1 = (j1.H + kRopeHeadGroup - 1) / kRopeHeadGroup;
  const int ng = g0 + g1;
  const long long total = (long long)n * ng * half;
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(g % half);
    const long long rest = g / half;
    const int grp = (int)(rest % ng);
    const long long t = rest / ng;
    const bool first = grp < g0;
    const RopeJob& J = first ? j0 : j1;
    const int hb = (first ? grp : grp - g0) * kRopeHeadGroup;
    const int nh = min(kRopeHeadGroup, J.H - hb);
    const double ang = (double)row_position(pos, cu, S, t) * th.theta[k];
    const double red = ang - two_pi * rint(ang * inv_two_pi);
    float sn, cs;
    sincosf((float)red, &sn, &cs);
    const T* x = reinterpret_cast<const T*>(J.x) + (t * J.H + hb) * D + k;
    T* y = reinterpret_cast<T*>(J.y) + (t * J.H + hb) * D + k;
    float x1[kRopeHeadGroup], x2[kRopeHeadGroup];
#pragma unroll
    for (int i = 0; i < kRopeHeadGroup; ++i) {
      if (i < nh) {
        x1[i] = Elt<T>::to_f(x[(long long)i * D]);
        x2[i] = Elt<T>::to_f(x[(long long)i * D + half]);
      }
    }
#pragma unroll
    for (int i = 0; i < kRopeHeadGroup; ++i) {
      if (i < nh) {
        y[(long long)i * D] = Elt<T>::from_f(x1[i] * cs - x2[i] * sn);
        y[(long long)i * D + half] = Elt<T>::from_f(x2[i] * cs + x1[i] * sn);
      }
    }
  }
}

namespace {
cudaError_t rope_launch(specopd_dtype dt, const void* x0, void* y0, int H0, const void* x1,
                        void* y1, int H1, const int32_t* pos, const int32_t* cu, int S, int n,
                        int D, const double* theta_host, cudaStream_t st) {
  RopeTheta th;
  for (int k = 0; k < D / 2; ++k) th.theta[k] = theta_host[k];
  const RopeJob j0{x0, y0, H0};
  const RopeJob j1{x1, y1, x1 ? H1 : 0};
  const long long groups = (H0 + kRopeHeadGroup - 1) / kRopeHeadGroup +
                           (j1.H + kRopeHeadGroup - 1) / kRopeHeadGroup;
  const long long total = (long long)n * groups * (D / 2);
  if (total == 0) return cudaSuccess;
  const int threads = 128;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (dt == SPECOPD_F32)
    rope_kernel<float><<<(int)blocks, threads, 0, st>>>(j0, j1, pos, cu, S, n, D, th);
  else
    rope_kernel<__nv_bfloat16><<<(int)blocks, threads, 0, st>>>(j0, j1, pos, cu, S, n, D, th);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_rope2(specopd_dtype dt, const void* x0, void* y0, int H0, const void* x1,
                         void* y1, int H1, const int32_t* pos, int n, int D,
                         const double* theta_host, cudaStream_t st) {
  return rope_launch(dt, x0, y0, H0, x1, y1, H1, pos, nullptr, 0, n, D, theta_host, st);
}

cudaError_t launch_rope_trunk(specopd_dtype dt, const void* x, void* y, const int32_t* cu_trunk,
                              int S, int n, int H, int D, const double* theta_host,
                              cudaStream_t st) {
  return rope_launch(dt, x, y, H, nullptr, nullptr, 0, nullptr, cu_trunk, S, n, D, theta_host, st);
}

cudaError_t launch_rope(specopd_dtype dt, const void* x, void* y, const int32_t* pos, int n, int H,
                        int D, const double* theta_host, cudaStream_t st) {
  return launch_rope2(dt, x, y, H, nullptr, nullptr, 0, pos, n, D, theta_host, st);
}

}  // namespace specopd
