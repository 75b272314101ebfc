// Tree-masked GQA attention of branch rows, fp32 SIMT variant.
//
// SpecOPD review (jaehun.me) §3.2(a): the trunk K/V is cached once and each
// branch query reads only itself and its ancestors: for branch row
// r = (s, b, i) the visible keys are trunk positions 0..a_b of sequence s
// and branch nodes (s, b, 1..i).  Siblings and later trunk tokens are never
// touched, so no mask is materialised.
//
// This variant serves fp32 workloads (tiny problems where tensor cores do
// not apply).  One CTA per (branch row, kv head); one warp per query head of
// the GQA group.  Keys go in blocks of 32: lane l scores key kb + l with a
// full dot product (q, pre-scaled, from shared memory), one warp reduction
// gives the block's max, the running (max, sum, O) is rescaled once per
// block, and P.V runs with the lanes over the output dims (the block's p
// from shared memory).  q and branch k arrive already rotated.
#include "common.cuh"
#include "kernels.h"

namespace specopd {

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int D>
__global__ void __launch_bounds__(1024) attn_simt_kernel(
    const AttnProblem p, const float* __restrict__ q_rot, const float* __restrict__ k_rot,
    const float* __restrict__ v_br, const float* __restrict__ k_tr,
    const float* __restrict__ v_tr, const int32_t* __restrict__ cu_trunk,
    const int32_t* __restrict__ anchors, float* __restrict__ out, float* __restrict__ lse,
    int prefill) {
  constexpr int DPL = D / 32;  // output dims per lane
  extern __shared__ __align__(16) float simt_smem[];
  const int r = blockIdx.x;
  const int hk = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= p.G) return;
  float* sq = simt_smem + warp * (D + 32);  // this head's scaled q
  float* sp = sq + D;                       // p of the current key block
  const int h = hk * p.G + warp;
  // Branch row r = (s, b, i): trunk keys 0..a of sequence s, then branch
  // nodes 1..i.  Trunk prefill (row r = a trunk row): the keys of its own
  // sequence up to itself, i.e. a = its position, no branch keys.
  const int Wm1 = p.W - 1;
  int bid = 0, i = 0, s = 0, a = 0;
  if (prefill) {
    int lo = 0, hi = p.S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cu_trunk[mid] <= r) lo = mid; else hi = mid - 1;
    }
    s = lo;
    a = r - cu_trunk[s];
  } else {
    bid = r / Wm1;
    i = r % Wm1 + 1;
    s = bid / p.B;
    a = anchors[bid];
  }
  const int t0 = cu_trunk[s];
  const int Ts = cu_trunk[s + 1] - t0;
  float* o = out + ((long long)r * p.Hq + h) * D;
  if (a < 0 || a >= Ts) {
    if (lane == 0) set_status(SPECOPD_DEV_ANCHOR_RANGE);
    for (int d = lane; d < D; d += 32) o[d] = __int_as_float(0x7fc00000);
    if (lse && lane == 0) lse[(long long)r * p.Hq + h] = __int_as_float(0x7fc00000);
    return;
  }
  const float* qp = q_rot + ((long long)r * p.Hq + h) * D;
  for (int d = lane; d < D; d += 32) sq[d] = qp[d] * p.scale;
  __syncwarp();
  const int first = bid * Wm1;  // branch node (s,b,1) as a branch row index
  const int nkeys = a + 1 + i;
  auto key_row = [&](int kk) -> long long {
    return kk <= a ? (long long)(t0 + kk) * p.Hkv + hk : (long long)(first + (kk - a - 1)) * p.Hkv + hk;
  };
  float acc[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) acc[d] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int kb = 0; kb < nkeys; kb += 32) {
    const int kk = kb + lane;
    float sc = -INFINITY;
    if (kk < nkeys) {
      const float* kp = (kk <= a ? k_tr : k_rot) + key_row(kk) * D;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int d = 0; d < D; d += 8) {
        const float4 k0 = *reinterpret_cast<const float4*>(kp + d);
        const float4 k1 = *reinterpret_cast<const float4*>(kp + d + 4);
        const float4 q0 = *reinterpret_cast<const float4*>(sq + d);
        const float4 q1 = *reinterpret_cast<const float4*>(sq + d + 4);
        s0 = fmaf(q0.x, k0.x, fmaf(q0.y, k0.y, fmaf(q0.z, k0.z, fmaf(q0.w, k0.w, s0))));
        s1 = fmaf(q1.x, k1.x, fmaf(q1.y, k1.y, fmaf(q1.z, k1.z, fmaf(q1.w, k1.w, s1))));
      }
      sc = s0 + s1;
    }
    const float mn = fmaxf(m, warp_max_f(sc));
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);  // first block: O and l are zero
    const float pk = (kk < nkeys) ? expf(sc - mn) : 0.f;
    l = l * corr + warp_sum(pk);
#pragma unroll
    for (int d = 0; d < DPL; ++d) acc[d] *= corr;
    sp[lane] = pk;
    __syncwarp();
    const int nb = min(32, nkeys - kb);
#pragma unroll 8
    for (int k = 0; k < nb; ++k) {
      const int key = kb + k;
      const float* vp = (key <= a ? v_tr : v_br) + key_row(key) * D + lane * DPL;
      const float pkk = sp[k];
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc[d] = fmaf(pkk, vp[d], acc[d]);
    }
    __syncwarp();  // sp is rewritten by the next block
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
                                 float* lse, cudaStream_t st, bool prefill) {
  const int nq = prefill ? p.T_tot : p.R;
  if (nq == 0) return cudaSuccess;
  if (p.G < 1 || p.G > 32) return cudaErrorInvalidValue;
  dim3 grid(nq, p.Hkv);
  dim3 block(32 * p.G);
  const size_t smem = (size_t)p.G * (p.D + 32) * sizeof(float);
  if (p.D == 64)
    attn_simt_kernel<64><<<grid, block, smem, st>>>(p, q_rot, k_rot, v_br, k_tr, v_tr, cu_trunk,
                                                    anchors, out, lse, prefill ? 1 : 0);
  else if (p.D == 128)
    attn_simt_kernel<128><<<grid, block, smem, st>>>(p, q_rot, k_rot, v_br, k_tr, v_tr, cu_trunk,
                                                     anchors, out, lse, prefill ? 1 : 0);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace specopd
