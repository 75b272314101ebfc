// Proposal-tree construction on the device.
//
// SpecOPD review (jaehun.me) §3.1 and §3.2(a), paper summary
// (rustineverything.app) §2.1-§2.2: a branch's first token has the anchor
// token as parent, later tokens the previous sampled token; its semantic
// position is anchor + offset; the anchor row scores token 1 and branch row
// i scores token i+1, so B branches add B(W-1) rows after the trunk.
//
// One thread per output element: trunk nodes, branch nodes, supervised
// positions.  Integer work only; a few microseconds at the largest
// workloads, so it is a plain grid-stride kernel.
#include "common.cuh"
#include "kernels.h"

namespace specopd {

__global__ void tree_build_kernel(const CuTrunk cu, const int32_t* __restrict__ anchors, int B,
                                  int W, int32_t* __restrict__ parent,
                                  int32_t* __restrict__ sem_pos, int32_t* __restrict__ score_row) {
  const int S = cu.S;
  const int T_tot = cu.T_tot;
  const long long R = (long long)S * B * (W - 1);
  const long long N = (long long)S * B * W;
  const long long total = T_tot + R + N;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    if (g < T_tot) {
      // trunk node: find its sequence (cu is sorted; binary search)
      int lo = 0, hi = S - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu.cu[mid] <= g) lo = mid; else hi = mid - 1;
      }
      const int j = (int)g - cu.cu[lo];
      if (parent) parent[g] = j > 0 ? (int32_t)g - 1 : -1;
      if (sem_pos) sem_pos[g] = j;
    } else if (g < T_tot + R) {
      const long long r = g - T_tot;
      const int bid = (int)(r / (W - 1));
      const int i = (int)(r % (W - 1)) + 1;
      const int s = bid / B;
      const int a = anchors[bid];
      const int Ts = cu.cu[s + 1] - cu.cu[s];
      if (a < 0 || a >= Ts) {
        set_status(SPECOPD_DEV_ANCHOR_RANGE);
        if (parent) parent[g] = -1;
        if (sem_pos) sem_pos[g] = -1;
        continue;
      }
      if (parent) parent[g] = (i == 1) ? cu.cu[s] + a : (int32_t)g - 1;
      if (sem_pos) sem_pos[g] = a + i;
    } else {
      if (!score_row) continue;
      const long long p = g - T_tot - R;
      const int bid = (int)(p / W);
      const int i = (int)(p % W) + 1;
      const int s = bid / B;
      const int a = anchors[bid];
      const int Ts = cu.cu[s + 1] - cu.cu[s];
      if (a < 0 || a >= Ts) {
        set_status(SPECOPD_DEV_ANCHOR_RANGE);
        score_row[p] = -1;
        continue;
      }
      score_row[p] = (i == 1) ? cu.cu[s] + a : (int32_t)(T_tot + (long long)bid * (W - 1) + (i - 2));
    }
  }
}

cudaError_t launch_tree_build(const CuTrunk& cu, const int32_t* anchors, int B, int W,
                              int32_t* parent, int32_t* sem_pos, int32_t* score_row,
                              cudaStream_t st) {
  const long long total = cu.T_tot + (long long)cu.S * B * (W - 1) + (long long)cu.S * B * W;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  tree_build_kernel<<<(int)blocks, threads, 0, st>>>(cu, anchors, B, W, parent, sem_pos, score_row);
  return cudaGetLastError();
}

}  // namespace specopd
