// E2E-TV acceptance-length loss and its gradient w.r.t. the draft logits.
//
// Sources: SpecOPD review (jaehun.me) §1.1 (the single-draft acceptance
// probability is the overlap sum_v min(p_v, q_v) = 1 - TV) and §3.3 (loss
// from prefix products of the overlaps within a branch; target mass outside
// the drafter's support is kept; the gradient holds the sampled tokens and
// the target fixed, no score-function term); paper summary
// (rustineverything.app) §2.3 (loss = 1 - mean over the B*W proposed tokens
// of the prefix product).
//
// Per position n (branch b, offset i):
//   p = softmax(z_t[target_row[n]]), q = softmax(z_d[n])       (fp32)
//   a_n = sum_v min(p_v, q_v),   s_n = sum_{v: q_v < p_v} q_v
//   P_{b,i} = prod_{j<=i} a_{b,j};  loss = 1 - sum P / norm
//   g_n = -(1/norm) P_{b,i-1} S_{b,i},  S_{b,W} = 1, S_{b,j} = 1 + a_{b,j+1} S_{b,j+1}
//   dz_d[n,u] = g_n q_u ([q_u < p_u] - s_n)
// (d a / d z_u = sum_v [q_v<p_v] q_v (delta_vu - q_u) = q_u ([q_u<p_u] - s).)
//
// B200 design (HBM-bound: the algorithmic traffic is one read of both logit
// rows and one write of the gradient):
//  * One persistent launch of thread-block clusters of CL CTAs; each CTA
//    owns a 1/CL slice of the vocabulary.  Work is a queue of tasks claimed
//    with one atomic each, two tasks ahead so the atomic's latency hides
//    behind the current task:
//      A(n): the two logit rows of position n arrive by 1-D bulk copy (TMA)
//            into shared memory; online max / sum-exp, a DSMEM reduction of
//            the statistics over the cluster, the overlap a_n and s_n from
//            shared memory, a second DSMEM reduction; publish (lse, s, a)
//            and count the branch (release, fire-and-forget).
//      G(n): wait (bounded) until all W positions of branch b are counted,
//            load the branch's W overlaps in one parallel read, form g_n,
//            and write dz from the rows, which were copied in (from L2:
//            the A-task read them a few tasks earlier) during the previous
//            task.  G(b, 1) also writes the branch's prefix products and
//            adds the branch to the loss.
//      S(b): (no gradient requested) the prefix products and loss part of
//            G(b, 1) alone.
//    Each CTA double-buffers its shared memory: the next task's bulk copies
//    stream in while the current task computes.  G/S tasks of branch b are
//    queued `lag` branches after its A-tasks, and only ever wait for
//    A-tasks, which never wait and were claimed earlier: the lowest
//    unfinished task is always running, so the queue cannot deadlock
//    whatever the residency of the grid.
//  * The loss is reduced by the last branch to finish, in a fixed order:
//    deterministic.
//  * All math in the log2 domain: x2 = z*log2(e) - lse2 via one FMA, one
//    ex2 per element per pass.  The same FMA sequence decides [q < p] in the
//    A- and the G-task, so s_n and the gradient's mask always agree.
#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace specopd {

constexpr int kTVThreads = 256;
constexpr int kTVWarps = kTVThreads / 32;
constexpr int kTVCtasPerSm = 2;            // independent CTAs per SM hide each other's waits
constexpr int kTVBuffers = 1;              // row-slice buffers per CTA
constexpr int kTVChunks = 4;               // bulk copies per row slice (pipelined)
constexpr int kTVSmemBudget = 104 * 1024;  // bytes of row slices per CTA
constexpr int kTVMaxW = 1024;              // positions per branch held in shared memory
constexpr float kLog2e = 1.4426950408889634f;

enum TaskKind { kTaskA = 0, kTaskG = 1, kTaskS = 2 };

struct TVArgs {
  int nbranch, W, V, N, rows_target, compute_grad;
  int CL, Lc, lag, aligned, total_tasks;
  float inv_norm;
  double norm;
  const void* zt;
  const int32_t* trow;
  const void* zd;
  float* a_out;
  float* prefix;
  float* loss;
  double* numer;
  void* grad;
  float4* rec;       // [N]  (lse2_t, lse2_d, s, unused)
  double* bsum;      // [nbranch]
  unsigned* cnt;     // [nbranch] positions of the branch published
  unsigned* ctl;     // [0] claim, [1] branches done, [2] abort
};

// Task id -> (kind, index).  index = position for A and G, branch for S.
// Queue: slot k holds the W A-tasks of branch k, then the second-kind tasks
// (W G-tasks, or one S-task) of branch k - lag.
__device__ __forceinline__ void decode_task(const TVArgs& A, int t, int& kind, int& idx) {
  const int W = A.W;
  const int per = A.compute_grad ? W : 1;
  const int k0 = min(A.lag, A.nbranch);
  if (t < k0 * W) { kind = kTaskA; idx = t; return; }
  const int t1 = t - k0 * W;
  const int n_mid = max(0, A.nbranch - A.lag);
  const int blk = W + per;
  int b2, j2;
  if (t1 < n_mid * blk) {
    const int k = A.lag + t1 / blk;
    const int w = t1 % blk;
    if (w < W) { kind = kTaskA; idx = k * W + w; return; }
    b2 = k - A.lag;
    j2 = w - W;
  } else {
    const int t2 = t1 - n_mid * blk;
    b2 = n_mid + t2 / per;
    j2 = t2 % per;
  }
  if (A.compute_grad) { kind = kTaskG; idx = b2 * W + j2; }
  else { kind = kTaskS; idx = b2; }
}

template <typename Tin> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;  // elements per 16 bytes
  static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
  }
  // max of the 8 values, with packed bf16x2 comparisons
  static __device__ __forceinline__ float vmax(const uint4& u) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(&u.z);
    const __nv_bfloat162 d = *reinterpret_cast<const __nv_bfloat162*>(&u.w);
    const __nv_bfloat162 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
    return fmaxf(__low2float(m), __high2float(m));
  }
};
template <> struct Vec<float> {
  static constexpr int kN = 4;
  static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  static __device__ __forceinline__ float vmax(const uint4& u) {
    return fmaxf(fmaxf(__uint_as_float(u.x), __uint_as_float(u.y)),
                 fmaxf(__uint_as_float(u.z), __uint_as_float(u.w)));
  }
};

__device__ __forceinline__ void warp_lse2(float& m, float& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse2_combine(m, s, m2, s2);
  }
}

// Cluster barrier without a release by every thread: a release arrive would
// make each thread drain its outstanding global stores (the gradient rows)
// at every barrier.  All threads execute the same aligned instructions (the
// barrier is never reached divergently); the one thread that wrote shared
// memory another CTA reads after the barrier issues a cluster-scope fence
// first (publish_for_cluster), and the wait is an acquire.
__device__ __forceinline__ void publish_for_cluster() {
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
}
__device__ __forceinline__ void cluster_barrier_relaxed() {
  __syncwarp();  // the .aligned form needs a converged warp
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

struct TVShared {
  int task[4];       // claimed task ids, ring indexed by iteration
  int flag;
  float g;           // gradient coefficient of the current G-task
  uint64_t bar[kTVBuffers][kTVChunks];  // bulk-copy completion, per buffer and chunk
  float4 red_lse[kTVWarps];    // per-warp (m_t, s_t, m_d, s_d)
  float2 red_as[kTVWarps];     // per-warp (a, s)
  float4 cl_lse;     // this CTA's statistics, read by the cluster
  float2 cl_as;      // this CTA's (a, s), read by the cluster
  float4 all_lse;    // cluster-combined statistics
  double dred[kTVWarps];
  float sa[kTVMaxW];  // overlaps of one branch
};

template <typename Tin, typename Tg>
__global__ void __launch_bounds__(kTVThreads, kTVCtasPerSm) e2e_tv_kernel(const TVArgs A) {
  extern __shared__ __align__(128) unsigned char tv_smem_raw[];
  TVShared& sh = *reinterpret_cast<TVShared*>(tv_smem_raw);
  Tin* buf0 = reinterpret_cast<Tin*>(tv_smem_raw + ((sizeof(TVShared) + 127) / 128) * 128);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int VN = Vec<Tin>::kN;

  if (tid == 0) {
    for (int bb = 0; bb < kTVBuffers; ++bb)
      for (int c = 0; c < kTVChunks; ++c) mbar_init(&sh.bar[bb][c], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int V = A.V;
  const int W = A.W;
  const int v0 = rank * A.Lc;
  const int len = max(0, min(V, v0 + A.Lc) - v0);
  const int chunk_elems = ((A.Lc / kTVChunks) + 15) / 16 * 16;
  const Tin* zt = reinterpret_cast<const Tin*>(A.zt);
  const Tin* zd = reinterpret_cast<const Tin*>(A.zd);

  auto row_ptrs = [&](int pos, const Tin*& rt, const Tin*& rd) {
    int row = A.trow ? A.trow[pos] : pos;
    if (row < 0 || row >= A.rows_target) row = 0;
    rt = zt + (long long)row * V + v0;
    rd = zd + (long long)pos * V + v0;
  };
  auto buf_t = [&](int bb) { return buf0 + (size_t)bb * 2 * A.Lc; };
  auto buf_d = [&](int bb) { return buf0 + (size_t)bb * 2 * A.Lc + A.Lc; };

  const uint64_t pol_keep = l2_policy_evict_last();
  const uint64_t pol_drop = l2_policy_evict_first();
  // Start the bulk copies of task t's rows into buffer bb (aligned path; A and
  // G tasks only -- S tasks touch no rows).
  auto issue_loads = [&](int t, int bb) {
    if (t >= A.total_tasks || !A.aligned || tid != 0) return;
    int kind, pos;
    decode_task(A, t, kind, pos);
    if (kind == kTaskS) return;
    const Tin *rt, *rd;
    row_ptrs(pos, rt, rd);
    Tin* st = buf_t(bb);
    Tin* sd = buf_d(bb);
    fence_proxy_async_smem();
    for (int c = 0; c < kTVChunks; ++c) {
      const int e0 = c * chunk_elems;
      const int e1 = min(len, e0 + chunk_elems);
      const unsigned bytes = e1 > e0 ? (unsigned)((e1 - e0) * sizeof(Tin)) : 0u;
      mbar_arrive_expect_tx(&sh.bar[bb][c], 2u * bytes);
      if (bytes) {
        // A-task rows are read again by the branch's G-tasks shortly after:
        // keep them in L2 (evict_last); a G-task is their last use.
        const uint64_t pol = kind == kTaskA ? pol_keep : pol_drop;
        bulk_g2s_hint(st + e0, rt + e0, bytes, &sh.bar[bb][c], pol);
        bulk_g2s_hint(sd + e0, rd + e0, bytes, &sh.bar[bb][c], pol);
      }
    }
  };
  // Every A and G task uses its buffer once: buffer bb's k-th use waits for
  // its barriers' phase k.
  unsigned uses[kTVBuffers] = {};

  auto claim = [&]() -> int {
    const int t = (int)atomicAdd(&A.ctl[0], 1u);
    if (__ldcg(&A.ctl[2]) != 0u) return A.total_tasks;  // a wait ran out: stop
    return t > A.total_tasks ? A.total_tasks : t;
  };
  auto broadcast = [&](int slot, int t) {
    for (int r = 0; r < A.CL; ++r) *cluster.map_shared_rank(&sh.task[slot], r) = t;
  };

  // Loss of the last branch to finish: 1 - sum_b bsum[b] / norm, fixed order.
  auto finish_loss = [&]() {
    double acc = 0.0;
    for (int i = tid; i < A.nbranch; i += kTVThreads) acc += __ldcg(&A.bsum[i]);
    acc = warp_sum_d(acc);
    if (lane == 0) sh.dred[warp] = acc;
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
      for (int w = 0; w < kTVWarps; ++w) tot += sh.dred[w];
      A.loss[0] = (float)(1.0 - tot / A.norm);
      if (A.numer) A.numer[0] = tot;
    }
  };

  // Wait until branch b's W positions are published, then stage its overlaps
  // in sh.sa (all threads of the CTA take part).  Returns false on timeout.
  auto stage_branch = [&](int b) -> bool {
    if (tid == 0) {
      const bool ok = wait_flag_geq(&A.cnt[b], (unsigned)W);
      if (!ok) atomicExch(&A.ctl[2], 1u);
      sh.flag = ok ? 1 : 0;
    }
    __syncthreads();
    const bool ok = sh.flag != 0;
    if (ok)
      for (int i = tid; i < W; i += kTVThreads) sh.sa[i] = __ldcg(&A.a_out[b * W + i]);
    __syncthreads();
    return ok;
  };
  // Prefix products of branch b from sh.sa; writes prefix[] and bsum[b] and
  // counts the branch; the last branch reduces the loss.  Rank 0 only.
  auto scan_branch = [&](int b) {
    if (tid == 0) {
      float P = 1.f;
      double sumP = 0.0;
      for (int i = 0; i < W; ++i) {
        P *= sh.sa[i];
        A.prefix[b * W + i] = P;
        sumP += (double)P;
      }
      A.bsum[b] = sumP;
      __threadfence();
      const unsigned done = atomicAdd(&A.ctl[1], 1u);
      sh.flag = (done == (unsigned)A.nbranch - 1u) ? 1 : 0;
      if (sh.flag) __threadfence();
    }
    __syncthreads();
    if (sh.flag) finish_loss();
  };

  if (rank == 0 && tid == 0) {
    const int t0 = claim();
    const int t1 = claim();
    broadcast(0, t0);
    broadcast(1, t1);
    publish_for_cluster();
  }
  cluster_barrier_relaxed();
  if (kTVBuffers == 2) issue_loads(sh.task[0], 0);

  for (int k = 0;; ++k) {
    const int t = sh.task[k & 3];
    if (t >= A.total_tasks) break;

    // The barrier publishes task k+1 (broadcast at the end of task k-1 by
    // rank 0's thread 0) and ends every thread's use of the buffer that the
    // copies issued next land in (task k-1's).  With two buffers the copies
    // of task k+1 stream in while task k computes; with one, the other CTA
    // on the SM covers the copy of task k.
    cluster_barrier_relaxed();
    issue_loads(sh.task[(k + kTVBuffers - 1) & 3], (k + kTVBuffers - 1) % kTVBuffers);
    // Claim task k+2 (warp 1, so thread 0's copies are not delayed); the id
    // is only needed when it is broadcast at the end of this task.
    int t_ahead = A.total_tasks;
    if (rank == 0 && tid == 32) t_ahead = claim();

    const int bb = k % kTVBuffers;
    Tin* st = buf_t(bb);
    Tin* sd = buf_d(bb);
    int kind, idx;
    decode_task(A, t, kind, idx);
    unsigned parity = 0;
    if (kind != kTaskS) {
      parity = uses[bb] & 1u;
      if (A.aligned) {
        ++uses[bb];
      } else {
        const Tin *rt, *rd;
        row_ptrs(idx, rt, rd);
        for (int e = tid; e < len; e += kTVThreads) {
          st[e] = rt[e];
          sd[e] = rd[e];
        }
        __syncthreads();
      }
    }

    if (kind == kTaskA) {
      // ---------------------------------------------------------- A-task
      const int pos = idx, b = pos / W;
      bool task_row_ok = true;
      if (rank == 0 && tid == 0 && A.trow) {
        const int trow = A.trow[pos];  // read early; used when publishing
        task_row_ok = (trow >= 0 && trow < A.rows_target);
      }
      // pass 0: row maxima of this slice (packed compares), chunk by chunk as
      // the copies land; pass 1: sum of 2^(x - max) from shared memory.
      float mt = -INFINITY, md = -INFINITY;
      for (int c = 0; c < kTVChunks; ++c) {
        const int e0 = c * chunk_elems;
        const int e1 = min(len, e0 + chunk_elems);
        if (A.aligned && !mbar_wait(&sh.bar[bb][c], parity) && tid == 0) atomicExch(&A.ctl[2], 1u);
        if (e1 <= e0) continue;
        const int nv = (e1 - e0) / VN;
        for (int vi = tid; vi < nv; vi += kTVThreads) {
          mt = fmaxf(mt, Vec<Tin>::vmax(*reinterpret_cast<const uint4*>(st + e0 + vi * VN)));
          md = fmaxf(md, Vec<Tin>::vmax(*reinterpret_cast<const uint4*>(sd + e0 + vi * VN)));
        }
        for (int e = e0 + nv * VN + tid; e < e1; e += kTVThreads) {  // ragged tail
          mt = fmaxf(mt, Elt<Tin>::to_f(st[e]));
          md = fmaxf(md, Elt<Tin>::to_f(sd[e]));
        }
      }
      mt *= kLog2e;
      md *= kLog2e;
      // Same element-to-thread mapping as pass 0, so each thread's maximum
      // covers exactly the elements it sums.
      float ssum_t = 0.f, ssum_d = 0.f;
      if (mt != -INFINITY || md != -INFINITY) {
        for (int c = 0; c < kTVChunks; ++c) {
          const int e0 = c * chunk_elems;
          const int e1 = min(len, e0 + chunk_elems);
          if (e1 <= e0) continue;
          const int nv = (e1 - e0) / VN;
          for (int vi = tid; vi < nv; vi += kTVThreads) {
            const uint4 ut = *reinterpret_cast<const uint4*>(st + e0 + vi * VN);
            const uint4 ud = *reinterpret_cast<const uint4*>(sd + e0 + vi * VN);
            float ft[VN], fd[VN];
            Vec<Tin>::unpack(ut, ft);
            Vec<Tin>::unpack(ud, fd);
            // independent partial sums: no serial FADD chain across the vector
            float at[VN], ad[VN];
#pragma unroll
            for (int q = 0; q < VN; ++q) {
              at[q] = exp2f(__fmaf_rn(ft[q], kLog2e, -mt));
              ad[q] = exp2f(__fmaf_rn(fd[q], kLog2e, -md));
            }
#pragma unroll
            for (int w = VN / 2; w > 0; w >>= 1)
#pragma unroll
              for (int q = 0; q < w; ++q) {
                at[q] += at[q + w];
                ad[q] += ad[q + w];
              }
            ssum_t += at[0];
            ssum_d += ad[0];
          }
          for (int e = e0 + nv * VN + tid; e < e1; e += kTVThreads) {
            ssum_t += exp2f(__fmaf_rn(Elt<Tin>::to_f(st[e]), kLog2e, -mt));
            ssum_d += exp2f(__fmaf_rn(Elt<Tin>::to_f(sd[e]), kLog2e, -md));
          }
        }
      }
      // A -inf maximum means this thread saw no finite entry of that row: no
      // mass (the NaNs formed above are dropped; the combine skips -inf).
      if (mt == -INFINITY) ssum_t = 0.f;
      if (md == -INFINITY) ssum_d = 0.f;
      warp_lse2(mt, ssum_t);
      warp_lse2(md, ssum_d);
      if (lane == 0) sh.red_lse[warp] = make_float4(mt, ssum_t, md, ssum_d);
      __syncthreads();
      if (warp == 0) {
        float4 v = lane < kTVWarps ? sh.red_lse[lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        warp_lse2(v.x, v.y);
        warp_lse2(v.z, v.w);
        if (lane == 0) {
          sh.cl_lse = v;
          publish_for_cluster();
        }
      }
      cluster_barrier_relaxed();
      if (warp == 0) {
        // lane r reads rank r's statistics: one DSMEM round trip
        float4 v = lane < A.CL ? *cluster.map_shared_rank(&sh.cl_lse, lane)
                               : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        warp_lse2(v.x, v.y);
        warp_lse2(v.z, v.w);
        if (lane == 0) sh.all_lse = v;
      }
      __syncthreads();
      const float4 L = sh.all_lse;
      const float lse2_t = L.x + log2f(L.y);
      const float lse2_d = L.z + log2f(L.w);
      float pa = 0.f, ps = 0.f;
      {
        const int nv = len / VN;
        for (int vi = tid; vi < nv; vi += kTVThreads) {
          const uint4 ut = *reinterpret_cast<const uint4*>(st + vi * VN);
          const uint4 ud = *reinterpret_cast<const uint4*>(sd + vi * VN);
          float ft[VN], fd[VN];
          Vec<Tin>::unpack(ut, ft);
          Vec<Tin>::unpack(ud, fd);
          float ea[VN], es[VN];
#pragma unroll
          for (int q = 0; q < VN; ++q) {
            const float lt = __fmaf_rn(ft[q], kLog2e, -lse2_t);
            const float ld = __fmaf_rn(fd[q], kLog2e, -lse2_d);
            ea[q] = exp2f(fminf(lt, ld));
            es[q] = (ld < lt) ? ea[q] : 0.f;
          }
#pragma unroll
          for (int w = VN / 2; w > 0; w >>= 1)
#pragma unroll
            for (int q = 0; q < w; ++q) {
              ea[q] += ea[q + w];
              es[q] += es[q + w];
            }
          pa += ea[0];
          ps += es[0];
        }
        for (int e = nv * VN + tid; e < len; e += kTVThreads) {
          const float lt = __fmaf_rn(Elt<Tin>::to_f(st[e]), kLog2e, -lse2_t);
          const float ld = __fmaf_rn(Elt<Tin>::to_f(sd[e]), kLog2e, -lse2_d);
          const float ex = exp2f(fminf(lt, ld));
          pa += ex;
          ps += (ld < lt) ? ex : 0.f;
        }
      }
      pa = warp_sum(pa);
      ps = warp_sum(ps);
      if (lane == 0) sh.red_as[warp] = make_float2(pa, ps);
      __syncthreads();
      if (warp == 0) {
        float2 v = lane < kTVWarps ? sh.red_as[lane] : make_float2(0.f, 0.f);
        v.x = warp_sum(v.x);
        v.y = warp_sum(v.y);
        if (lane == 0) {
          sh.cl_as = v;
          publish_for_cluster();
        }
      }
      cluster_barrier_relaxed();
      if (rank == 0 && warp == 0) {
        float2 v = lane < A.CL ? *cluster.map_shared_rank(&sh.cl_as, lane) : make_float2(0.f, 0.f);
        v.x = warp_sum(v.x);
        v.y = warp_sum(v.y);
        if (lane == 0) {
          const bool row_ok = task_row_ok;
          const bool finite = (L.x != -INFINITY) && (L.z != -INFINITY);
          if (!row_ok) set_status(SPECOPD_DEV_ROW_RANGE);
          if (!finite) set_status(SPECOPD_DEV_ALL_NEG_INF);
          if (!row_ok || !finite) v = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
          A.rec[pos] = make_float4(lse2_t, lse2_d, v.y, 0.f);
          A.a_out[pos] = v.x;
          // release: the two stores above are visible before the count
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&A.cnt[b]) : "memory");
        }
      }
    } else if (kind == kTaskG) {
      // ---------------------------------------------------------- G-task
      const int pos = idx, b = pos / W, i = pos % W;
      if (A.aligned) {
        for (int c = 0; c < kTVChunks; ++c)
          if (!mbar_wait(&sh.bar[bb][c], parity) && tid == 0) atomicExch(&A.ctl[2], 1u);
      }
      const bool ok = stage_branch(b);
      if (ok && tid == 0) {
        // g = -(1/norm) P_{i-1} S_i  (no division by any overlap)
        float P = 1.f;
        for (int j = 0; j < i; ++j) P *= sh.sa[j];
        float S = 1.f;
        for (int j = W - 1; j > i; --j) S = fmaf(sh.sa[j], S, 1.f);
        sh.g = -A.inv_norm * P * S;
      }
      __syncthreads();
      // G(b, 1) publishes the branch's prefix products before its gradient
      // stores, so its fence does not wait for them.
      if (ok && i == 0 && rank == 0) scan_branch(b);
      if (ok && len > 0) {
        const float4 r = __ldcg(&A.rec[pos]);
        const float lse2_t = r.x, lse2_d = r.y, s_val = r.z, g = sh.g;
        Tg* gout = reinterpret_cast<Tg*>(A.grad) + (long long)pos * V + v0;
        if (A.aligned) {
          const int nv = len / VN;
          for (int vi = tid; vi < nv; vi += kTVThreads) {
            const uint4 ut = *reinterpret_cast<const uint4*>(st + vi * VN);
            const uint4 ud = *reinterpret_cast<const uint4*>(sd + vi * VN);
            float ft[VN], fd[VN], o[VN];
            Vec<Tin>::unpack(ut, ft);
            Vec<Tin>::unpack(ud, fd);
#pragma unroll
            for (int q = 0; q < VN; ++q) {
              const float lt = __fmaf_rn(ft[q], kLog2e, -lse2_t);
              const float ld = __fmaf_rn(fd[q], kLog2e, -lse2_d);
              const float qv = exp2f(ld);
              o[q] = g * qv * (((ld < lt) ? 1.f : 0.f) - s_val);
            }
            if constexpr (sizeof(Tg) == 4) {
#pragma unroll
              for (int q = 0; q < VN; q += 4)
                __stcs(reinterpret_cast<float4*>(gout + vi * VN + q),
                       make_float4(o[q], o[q + 1], o[q + 2], o[q + 3]));
            } else {
#pragma unroll
              for (int q = 0; q < VN; q += 8) {
                uint4 u;
                u.x = pack_bf16x2(o[q], o[q + 1]);
                u.y = pack_bf16x2(o[q + 2], o[q + 3]);
                u.z = pack_bf16x2(o[q + 4], o[q + 5]);
                u.w = pack_bf16x2(o[q + 6], o[q + 7]);
                __stcs(reinterpret_cast<uint4*>(gout + vi * VN + q), u);
              }
            }
          }
        } else {
          for (int e = tid; e < len; e += kTVThreads) {
            const float lt = __fmaf_rn(Elt<Tin>::to_f(st[e]), kLog2e, -lse2_t);
            const float ld = __fmaf_rn(Elt<Tin>::to_f(sd[e]), kLog2e, -lse2_d);
            const float qv = exp2f(ld);
            gout[e] = Elt<Tg>::from_f(g * qv * (((ld < lt) ? 1.f : 0.f) - s_val));
          }
        }
      }
    } else {
      // ---------------------------------------------------------- S-task
      if (rank == 0 && stage_branch(idx)) scan_branch(idx);
    }
    if (rank == 0 && tid == 32) {
      broadcast((k + 2) & 3, t_ahead);
      publish_for_cluster();
    }
  }
  // Rank 0 may still be reading a peer's shared memory (DSMEM) from the last
  // task; no CTA of the cluster may exit before every peer is done with it.
  cluster_barrier_relaxed();
}

// ------------------------------------------------------------------ host
namespace {

struct TVLayout {
  size_t rec, bsum, cnt, ctl, total, zero_begin, zero_bytes;
};

TVLayout tv_layout(const TVProblem& p) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  TVLayout L;
  size_t off = 0;
  L.rec = off;   off = up(off + sizeof(float4) * (size_t)p.N);
  L.bsum = off;  off = up(off + sizeof(double) * (size_t)p.nbranch);
  L.cnt = off;   off += sizeof(unsigned) * (size_t)p.nbranch;
  L.ctl = off;   off = up(off + 4 * sizeof(unsigned));
  L.zero_begin = L.cnt;
  L.zero_bytes = off - L.cnt;
  L.total = off;
  return L;
}

int elt_size(specopd_dtype d) { return d == SPECOPD_BF16 ? 2 : 4; }

template <typename Tin, typename Tg>
void* tv_kernel_ptr() {
  return reinterpret_cast<void*>(&e2e_tv_kernel<Tin, Tg>);
}

void* pick_kernel(specopd_dtype in, specopd_dtype g) {
  if (in == SPECOPD_BF16)
    return g == SPECOPD_BF16 ? tv_kernel_ptr<__nv_bfloat16, __nv_bfloat16>()
                             : tv_kernel_ptr<__nv_bfloat16, float>();
  return g == SPECOPD_BF16 ? tv_kernel_ptr<float, __nv_bfloat16>() : tv_kernel_ptr<float, float>();
}

std::mutex g_occ_mu;
std::map<std::tuple<int, void*, int, int>, int> g_occ_cache;  // (dev, fn, CL, smem) -> clusters

}  // namespace

size_t tv_workspace(const TVProblem& p) { return tv_layout(p).total; }

cudaError_t launch_e2e_tv(const TVProblem& p, const void* z_target, const int32_t* target_row,
                          const void* z_draft, float* a, float* prefix, float* loss, double* numer,
                          void* grad, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const TVLayout L = tv_layout(p);
  if (ws_bytes < L.total) return cudaErrorInvalidValue;
  if (p.W > kTVMaxW) return cudaErrorInvalidConfiguration;
  const int es = elt_size(p.logit_dtype);
  const int gs = elt_size(p.grad_dtype);
  // Cluster size: smallest CL whose per-CTA slices of two tasks fit the budget.
  int CL = (int)((2ll * kTVBuffers * p.V * es + kTVSmemBudget - 1) / kTVSmemBudget);
  if (CL < 1) CL = 1;
  int Lc = (p.V + CL - 1) / CL;
  Lc = (Lc + 15) / 16 * 16;
  CL = (p.V + Lc - 1) / Lc;
  if (CL > 16) return cudaErrorInvalidConfiguration;
  const size_t smem = ((sizeof(TVShared) + 127) / 128) * 128 + 2ull * kTVBuffers * Lc * es;

  TVArgs A;
  A.nbranch = p.nbranch; A.W = p.W; A.V = p.V; A.N = p.N; A.rows_target = p.rows_target;
  A.compute_grad = p.compute_grad && grad != nullptr;
  A.CL = CL; A.Lc = Lc;
  const bool ptr_ok = ((uintptr_t)z_target % 16 == 0) && ((uintptr_t)z_draft % 16 == 0) &&
                      (!A.compute_grad || (uintptr_t)grad % 16 == 0);
  A.aligned = ptr_ok && ((size_t)p.V * es % 16 == 0) && (!A.compute_grad || (size_t)p.V * gs % 16 == 0);
  A.norm = p.norm_count;
  A.inv_norm = (float)(1.0 / p.norm_count);
  A.zt = z_target; A.trow = target_row; A.zd = z_draft;
  A.a_out = a; A.prefix = prefix; A.loss = loss; A.numer = numer; A.grad = grad;
  char* w = reinterpret_cast<char*>(ws);
  A.rec = reinterpret_cast<float4*>(w + L.rec);
  A.bsum = reinterpret_cast<double*>(w + L.bsum);
  A.cnt = reinterpret_cast<unsigned*>(w + L.cnt);
  A.ctl = reinterpret_cast<unsigned*>(w + L.ctl);

  void* fn = pick_kernel(p.logit_dtype, p.grad_dtype);
  cudaError_t e = cudaMemsetAsync(w + L.zero_begin, 0, L.zero_bytes, stream);
  if (e != cudaSuccess) return e;

  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kTVThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  int nclusters = 0;
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    auto key = std::make_tuple(dev, fn, CL, (int)smem);
    auto it = g_occ_cache.find(key);
    // The attribute is per function: set it on every launch (another problem
    // size may have lowered it since).
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (CL > 8) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    if (it != g_occ_cache.end()) {
      nclusters = it->second;
    } else {
      int nsm = 148;
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
      cfg.gridDim = dim3(CL * std::max(1, nsm / CL));
      e = cudaOccupancyMaxActiveClusters(&nclusters, fn, &cfg);
      if (e != cudaSuccess) return e;
      if (nclusters < 1) return cudaErrorInvalidConfiguration;
      g_occ_cache[key] = nclusters;
    }
  }
  A.total_tasks = p.N + (A.compute_grad ? p.N : p.nbranch);
  if (nclusters > A.total_tasks) nclusters = A.total_tasks;
  // G-tasks of a branch start ~2 rounds of the whole grid after its A-tasks,
  // so they rarely wait, while its rows are still resident in L2.
  A.lag = (2 * nclusters + p.W - 1) / p.W + 1;
  cfg.gridDim = dim3(CL * nclusters);
  void* args[] = {&A};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace specopd
