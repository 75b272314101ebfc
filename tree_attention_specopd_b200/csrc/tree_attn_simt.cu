// Tree-masked GQA attention of branch rows, fp32 SIMT variant.
//
// SpecOPD review (jaehun.me) §3.2(a): the trunk K/V is cached once and each
// branch query reads only itself and its ancestors: for branch row
// r = (s, b, i) the visible keys are trunk positions 0..a_b of sequence s
// and branch nodes (s, b, 1..i).  Siblings and later trunk tokens are never
// touched, so no mask is materialised.
//
// This variant serves fp32 workloads (tiny problems where tensor cores do
// not apply).  One CTA per (branch row, kv head); one warp per query head
// of the GQA group; keys are visited in order with an online softmax, each
// lane owning D/32 output dims.  q and branch k arrive already rotated.
#include "common.cuh"
#include "kernels.h"

namespace specopd {

template <int DPL>  // dims per lane = D / 32
__global__ void __launch_bounds__(1024) attn_simt_kernel(
    const AttnProblem p, const float* __restrict__ q_rot, const float* __restrict__ k_rot,
    const float* __restrict__ v_br, const float* __restrict__ k_tr,
    const float* __restrict__ v_tr, const int32_t* __restrict__ cu_trunk,
    const int32_t* __restrict__ anchors, float* __restrict__ out, float* __restrict__ lse) {
  const int r = blockIdx.x;
  const int hk = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= p.G) return;
  const int h = hk * p.G + warp;
  const int D = p.D;
  const int Wm1 = p.W - 1;
  const int bid = r / Wm1;
  const int i = r % Wm1 + 1;
  const int s = bid / p.B;
  const int a = anchors[bid];
  const int t0 = cu_trunk[s];
  const int Ts = cu_trunk[s + 1] - t0;
  float* o = out + ((long long)r * p.Hq + h) * D;
  if (a < 0 || a >= Ts) {
    if (lane == 0) set_status(SPECOPD_DEV_ANCHOR_RANGE);
    for (int d = lane; d < D; d += 32) o[d] = __int_as_float(0x7fc00000);
    if (lse && lane == 0) lse[(long long)r * p.Hq + h] = __int_as_float(0x7fc00000);
    return;
  }
  float q[DPL];
  const float* qp = q_rot + ((long long)r * p.Hq + h) * D + lane * DPL;
#pragma unroll
  for (int d = 0; d < DPL; ++d) q[d] = qp[d] * p.scale;
  float acc[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) acc[d] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int first = bid * Wm1;  // branch node (s,b,1) as a branch row index
  const int nkeys = a + 1 + i;
  for (int kk = 0; kk < nkeys; ++kk) {
    const float* kp;
    const float* vp;
    if (kk <= a) {
      const long long row = (long long)(t0 + kk) * p.Hkv + hk;
      kp = k_tr + row * D;
      vp = v_tr + row * D;
    } else {
      const long long row = (long long)(first + (kk - a - 1)) * p.Hkv + hk;
      kp = k_rot + row * D;
      vp = v_br + row * D;
    }
    float sdot = 0.f;
#pragma unroll
    for (int d = 0; d < DPL; ++d) sdot = fmaf(q[d], kp[lane * DPL + d], sdot);
    sdot = warp_sum(sdot);
    const float mn = fmaxf(m, sdot);
    const float corr = expf(m - mn);  // m = -inf on the first key -> 0
    const float pk = expf(sdot - mn);
    l = l * corr + pk;
#pragma unroll
    for (int d = 0; d < DPL; ++d) acc[d] = fmaf(pk, vp[lane * DPL + d], acc[d] * corr);
    m = mn;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int d = 0; d < DPL; ++d) o[lane * DPL + d] = acc[d] * inv;
  if (lse && lane == 0) lse[(long long)r * p.Hq + h] = m + logf(l);
}

cudaError_t launch_attn_simt_f32(const AttnProblem& p, const float* q_rot, const float* k_rot,
                                 const float* v_br, const float* k_tr, const float* v_tr,
                                 const int32_t* cu_trunk, const int32_t* anchors, float* out,
                                 float* lse, cudaStream_t st) {
  if (p.R == 0) return cudaSuccess;
  dim3 grid(p.R, p.Hkv);
  dim3 block(32 * p.G);
  if (p.D == 64)
    attn_simt_kernel<2><<<grid, block, 0, st>>>(p, q_rot, k_rot, v_br, k_tr, v_tr, cu_trunk,
                                                anchors, out, lse);
  else if (p.D == 128)
    attn_simt_kernel<4><<<grid, block, 0, st>>>(p, q_rot, k_rot, v_br, k_tr, v_tr, cu_trunk,
                                                anchors, out, lse);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace specopd
