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
//  * One persistent launch of thread-block clusters.  Work is a queue of
//    tasks claimed with one atomic per task:
//      A(n): bulk-copy (TMA 1-D) the two logit rows of position n into the
//            cluster's shared memory, each CTA holding a 1/CL slice; online
//            max / sum-exp, a DSMEM reduction of the statistics, then the
//            overlap a_n and s_n from shared memory (no second HBM read),
//            another DSMEM reduction.  The A-task that completes a branch
//            (atomic count) runs the branch's prefix scan and gradient
//            coefficients; the one that completes the last branch reduces
//            the loss in a fixed order (deterministic).
//      G(n): wait (bounded) until branch b is scanned, stream the two rows
//            again -- by queue construction they were read a few tasks ago
//            and are still resident in the 126 MB L2 -- and write dz.
//    G-tasks of branch b are queued `lag` branches after its A-tasks, and a
//    G-task only ever waits for A-tasks claimed before it, which never wait:
//    the queue cannot deadlock whatever the residency of the grid.
//  * All math in the log2 domain: x2 = z*log2(e) - lse2 via one FMA, one
//    ex2 per element per pass.  The same FMA sequence decides [q < p] in the
//    A- and the G-task, so s_n and the gradient's mask always agree.
#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace specopd {

constexpr int kTVThreads = 512;
constexpr int kTVWarps = kTVThreads / 32;
constexpr int kTVChunks = 4;            // bulk copies per row slice (pipelined)
constexpr int kTVSmemBudget = 210 * 1024;  // bytes of row slices per CTA (2 tasks)
constexpr float kLog2e = 1.4426950408889634f;

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
  float4* rec;       // [N]  (lse2_t, lse2_d, s, g)
  double* bsum;      // [nbranch]
  unsigned* cnt;     // [nbranch]
  unsigned* ready;   // [nbranch]
  unsigned* ctl;     // [0] claim, [1] branches done, [2] abort
};

// Task id -> (is_A, position).  See the queue description above.
__device__ __forceinline__ void decode_task(const TVArgs& A, int t, bool& isA, int& pos) {
  const int W = A.W;
  if (!A.compute_grad) { isA = true; pos = t; return; }
  const int k0 = min(A.lag, A.nbranch);
  if (t < k0 * W) { isA = true; pos = t; return; }
  const int t1 = t - k0 * W;
  const int n_mid = max(0, A.nbranch - A.lag);
  if (t1 < n_mid * 2 * W) {
    const int k = A.lag + t1 / (2 * W);
    const int w = t1 % (2 * W);
    if (w < W) { isA = true; pos = k * W + w; }
    else { isA = false; pos = (k - A.lag) * W + (w - W); }
    return;
  }
  isA = false;
  pos = n_mid * W + (t1 - n_mid * 2 * W);
}

template <typename Tin> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;  // elements per 16 bytes
  static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
  }
};
template <> struct Vec<float> {
  static constexpr int kN = 4;
  static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};

// Online (max, sum 2^(x - max)) over a group of values already in log2 units.
template <int K>
__device__ __forceinline__ void online_update(float& m, float& s, const float* x2) {
  float mx = x2[0];
#pragma unroll
  for (int k = 1; k < K; ++k) mx = fmaxf(mx, x2[k]);
  const float mn = fmaxf(m, mx);
  if (mn == -INFINITY) return;
  float acc = (m == -INFINITY) ? 0.f : s * exp2f(m - mn);
#pragma unroll
  for (int k = 0; k < K; ++k) acc += exp2f(x2[k] - mn);
  m = mn;
  s = acc;
}

// Block-wide combine of per-thread (m, s) pairs; result valid in all threads.
__device__ __forceinline__ void block_lse2(float& m, float& s, float2* red /*[kTVWarps]*/) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse2_combine(m, s, m2, s2);
  }
  const int warp = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[warp] = make_float2(m, s);
  __syncthreads();
  m = -INFINITY; s = 0.f;
  for (int w = 0; w < kTVWarps; ++w) lse2_combine(m, s, red[w].x, red[w].y);
}

__device__ __forceinline__ float block_sum(float v, float* red /*[kTVWarps]*/) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < kTVWarps; ++w) t += red[w];
  return t;
}

struct TVShared {
  int task[2];      // claimed task ids, by iteration parity
  int flag;
  int pad;
  uint64_t bar[2][kTVChunks];  // bulk-copy completion, per buffer and chunk
  float4 cl_red1;   // this CTA's (m_t, s_t, m_d, s_d) for the cluster reduction
  float2 cl_red2;   // this CTA's (a, s) partial
  float2 wred[kTVWarps];
  float fred[kTVWarps];
  float fred2[kTVWarps];
  double dred[kTVWarps];
};

// Row addresses of task t for this CTA's slice.
struct TaskRows {
  bool isA, row_ok;
  int pos, b;
};

__device__ __forceinline__ TaskRows task_rows(const TVArgs& A, int t) {
  TaskRows tr;
  decode_task(A, t, tr.isA, tr.pos);
  tr.b = tr.pos / A.W;
  const int row = A.trow ? A.trow[tr.pos] : tr.pos;
  tr.row_ok = (row >= 0 && row < A.rows_target);
  return tr;
}

template <typename Tin, typename Tg>
__global__ void __launch_bounds__(kTVThreads, 1) e2e_tv_kernel(const TVArgs A) {
  extern __shared__ __align__(128) unsigned char tv_smem_raw[];
  TVShared& sh = *reinterpret_cast<TVShared*>(tv_smem_raw);
  Tin* buf0 = reinterpret_cast<Tin*>(tv_smem_raw + ((sizeof(TVShared) + 127) / 128) * 128);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  constexpr int VN = Vec<Tin>::kN;

  if (tid == 0) {
    for (int bb = 0; bb < 2; ++bb)
      for (int c = 0; c < kTVChunks; ++c) mbar_init(&sh.bar[bb][c], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int V = A.V;
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
  // Buffer bb holds the slices (st, sd) of one task: [Lc] target, [Lc] draft.
  auto buf_t = [&](int bb) { return buf0 + (size_t)bb * 2 * A.Lc; };
  auto buf_d = [&](int bb) { return buf0 + (size_t)bb * 2 * A.Lc + A.Lc; };

  // Issue the asynchronous bulk copies of task t into buffer bb (aligned path).
  auto issue_loads = [&](int t, int bb) {
    if (t >= A.total_tasks || !A.aligned || tid != 0) return;
    bool isA;
    int pos;
    decode_task(A, t, isA, pos);
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
        bulk_g2s(st + e0, rt + e0, bytes, &sh.bar[bb][c]);
        bulk_g2s(sd + e0, rd + e0, bytes, &sh.bar[bb][c]);
      }
    }
  };

  auto claim = [&](int slot) {
    if (rank == 0 && tid == 0) {
      int t = A.total_tasks;
      if (*((volatile unsigned*)&A.ctl[2]) == 0u) t = (int)atomicAdd(&A.ctl[0], 1u);
      if (t > A.total_tasks) t = A.total_tasks;
      for (int r = 0; r < A.CL; ++r) *cluster.map_shared_rank(&sh.task[slot], r) = t;
    }
  };

  claim(0);
  cluster.sync();
  issue_loads(sh.task[0], 0);

  for (int k = 0;; ++k) {
    const int t = sh.task[k & 1];
    if (t >= A.total_tasks) break;
    // Claim the next task now and start its copies into the other buffer, so
    // they stream while this task computes.  The cluster barrier also ends
    // every thread's use of that buffer (task k-1).
    claim((k + 1) & 1);
    cluster.sync();
    issue_loads(sh.task[(k + 1) & 1], (k + 1) & 1);

    const int bb = k & 1;
    const unsigned parity = (unsigned)(k >> 1) & 1u;
    Tin* st = buf_t(bb);
    Tin* sd = buf_d(bb);
    const TaskRows tr = task_rows(A, t);
    const int pos = tr.pos, b = tr.b;
    if (!A.aligned) {
      const Tin *rt, *rd;
      row_ptrs(pos, rt, rd);
      for (int e = tid; e < len; e += kTVThreads) {
        st[e] = rt[e];
        sd[e] = rd[e];
      }
      __syncthreads();
    }

    if (tr.isA) {
      // ---------------------------------------------------------- A-task
      // pass 1: online max / sum-exp of both rows (log2 units), chunk by chunk
      float mt = -INFINITY, ssum_t = 0.f, md = -INFINITY, ssum_d = 0.f;
      for (int c = 0; c < kTVChunks; ++c) {
        const int e0 = c * chunk_elems;
        const int e1 = min(len, e0 + chunk_elems);
        if (A.aligned && !mbar_wait(&sh.bar[bb][c], parity) && tid == 0) atomicExch(&A.ctl[2], 1u);
        if (e1 <= e0) continue;
        const int nv = (e1 - e0) / VN;
        for (int vi = tid; vi < nv; vi += kTVThreads) {
          const uint4 ut = *reinterpret_cast<const uint4*>(st + e0 + vi * VN);
          const uint4 ud = *reinterpret_cast<const uint4*>(sd + e0 + vi * VN);
          float ft[VN], fd[VN];
          Vec<Tin>::unpack(ut, ft);
          Vec<Tin>::unpack(ud, fd);
#pragma unroll
          for (int q = 0; q < VN; ++q) { ft[q] *= kLog2e; fd[q] *= kLog2e; }
          online_update<VN>(mt, ssum_t, ft);
          online_update<VN>(md, ssum_d, fd);
        }
        for (int e = e0 + nv * VN + tid; e < e1; e += kTVThreads) {  // ragged tail
          float xt = Elt<Tin>::to_f(st[e]) * kLog2e;
          float xd = Elt<Tin>::to_f(sd[e]) * kLog2e;
          online_update<1>(mt, ssum_t, &xt);
          online_update<1>(md, ssum_d, &xd);
        }
      }
      block_lse2(mt, ssum_t, sh.wred);
      block_lse2(md, ssum_d, sh.wred);
      if (tid == 0) sh.cl_red1 = make_float4(mt, ssum_t, md, ssum_d);
      cluster.sync();
      mt = -INFINITY; ssum_t = 0.f; md = -INFINITY; ssum_d = 0.f;
      for (int r = 0; r < A.CL; ++r) {
        const float4 v = *cluster.map_shared_rank(&sh.cl_red1, r);
        lse2_combine(mt, ssum_t, v.x, v.y);
        lse2_combine(md, ssum_d, v.z, v.w);
      }
      const float lse2_t = mt + log2f(ssum_t);
      const float lse2_d = md + log2f(ssum_d);
      // pass 2: overlap and masked draft mass, from shared memory
      float pa = 0.f, ps = 0.f;
      {
        const int nv = len / VN;
        for (int vi = tid; vi < nv; vi += kTVThreads) {
          const uint4 ut = *reinterpret_cast<const uint4*>(st + vi * VN);
          const uint4 ud = *reinterpret_cast<const uint4*>(sd + vi * VN);
          float ft[VN], fd[VN];
          Vec<Tin>::unpack(ut, ft);
          Vec<Tin>::unpack(ud, fd);
#pragma unroll
          for (int q = 0; q < VN; ++q) {
            const float lt = __fmaf_rn(ft[q], kLog2e, -lse2_t);
            const float ld = __fmaf_rn(fd[q], kLog2e, -lse2_d);
            const float e = exp2f(fminf(lt, ld));
            pa += e;
            ps += (ld < lt) ? e : 0.f;
          }
        }
        for (int e = nv * VN + tid; e < len; e += kTVThreads) {
          const float lt = __fmaf_rn(Elt<Tin>::to_f(st[e]), kLog2e, -lse2_t);
          const float ld = __fmaf_rn(Elt<Tin>::to_f(sd[e]), kLog2e, -lse2_d);
          const float ex = exp2f(fminf(lt, ld));
          pa += ex;
          ps += (ld < lt) ? ex : 0.f;
        }
      }
      pa = block_sum(pa, sh.fred);
      ps = block_sum(ps, sh.fred2);
      if (tid == 0) sh.cl_red2 = make_float2(pa, ps);
      cluster.sync();
      if (rank == 0) {
        float a_val = 0.f, s_val = 0.f;
        for (int r = 0; r < A.CL; ++r) {
          const float2 v = *cluster.map_shared_rank(&sh.cl_red2, r);
          a_val += v.x;
          s_val += v.y;
        }
        int last_all = 0;
        if (tid == 0) {
          const bool finite = (mt != -INFINITY) && (md != -INFINITY);
          if (!tr.row_ok) set_status(SPECOPD_DEV_ROW_RANGE);
          if (!finite) set_status(SPECOPD_DEV_ALL_NEG_INF);
          if (!tr.row_ok || !finite) { a_val = __int_as_float(0x7fc00000); s_val = a_val; }
          A.rec[pos] = make_float4(lse2_t, lse2_d, s_val, 0.f);
          A.a_out[pos] = a_val;
          __threadfence();
          const unsigned old = atomicAdd(&A.cnt[b], 1u);
          if (old == (unsigned)A.W - 1u) {
            // This task completes branch b: prefix scan + gradient coefficients.
            __threadfence();
            const int base = b * A.W;
            float P = 1.f;
            double sumP = 0.0;
            for (int i = 0; i < A.W; ++i) {
              P *= __ldcg(&A.a_out[base + i]);
              A.prefix[base + i] = P;
              sumP += (double)P;
            }
            float S = 1.f;
            for (int i = A.W - 1; i >= 0; --i) {
              const float Pprev = (i == 0) ? 1.f : A.prefix[base + i - 1];
              reinterpret_cast<float*>(&A.rec[base + i])[3] = -A.inv_norm * Pprev * S;
              S = fmaf(__ldcg(&A.a_out[base + i]), S, 1.f);
            }
            A.bsum[b] = sumP;
            __threadfence();
            st_release_gpu(&A.ready[b], 1u);
            const unsigned done = atomicAdd(&A.ctl[1], 1u);
            if (done == (unsigned)A.nbranch - 1u) { __threadfence(); last_all = 1; }
          }
          sh.flag = last_all;
        }
        __syncthreads();
        if (sh.flag) {
          // Last branch: loss = 1 - sum_b bsum[b] / norm, fixed summation order.
          double acc = 0.0;
          for (int i = tid; i < A.nbranch; i += kTVThreads) acc += __ldcg(&A.bsum[i]);
          acc = warp_sum_d(acc);
          __syncthreads();
          if ((tid & 31) == 0) sh.dred[tid >> 5] = acc;
          __syncthreads();
          if (tid == 0) {
            double tot = 0.0;
            for (int w = 0; w < kTVWarps; ++w) tot += sh.dred[w];
            A.loss[0] = (float)(1.0 - tot / A.norm);
            if (A.numer) A.numer[0] = tot;
          }
        }
      }
    } else {
      // ---------------------------------------------------------- G-task
      if (A.aligned) {
        for (int c = 0; c < kTVChunks; ++c)
          if (!mbar_wait(&sh.bar[bb][c], parity) && tid == 0) atomicExch(&A.ctl[2], 1u);
      }
      if (tid == 0) {
        const bool ok = wait_flag_geq(&A.ready[b], 1u);
        if (!ok) atomicExch(&A.ctl[2], 1u);
        sh.flag = ok ? 1 : 0;
      }
      __syncthreads();
      const int ok = sh.flag;
      if (ok && len > 0) {
        const float4 r = __ldcg(&A.rec[pos]);
        const float lse2_t = r.x, lse2_d = r.y, s_val = r.z, g = r.w;
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
    }
  }
  // Rank 0 may still be reading a peer's shared memory (DSMEM) from the last
  // task; no CTA of the cluster may exit before every peer is done with it.
  cluster.sync();
}

// ------------------------------------------------------------------ host
namespace {

struct TVLayout {
  size_t rec, bsum, cnt, ready, ctl, total, zero_begin, zero_bytes;
};

TVLayout tv_layout(const TVProblem& p) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  TVLayout L;
  size_t off = 0;
  L.rec = off;   off = up(off + sizeof(float4) * (size_t)p.N);
  L.bsum = off;  off = up(off + sizeof(double) * (size_t)p.nbranch);
  L.cnt = off;   off += sizeof(unsigned) * (size_t)p.nbranch;
  L.ready = off; off += sizeof(unsigned) * (size_t)p.nbranch;
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
  const int es = elt_size(p.logit_dtype);
  const int gs = elt_size(p.grad_dtype);
  // Cluster size: smallest CL whose per-CTA slice of both rows fits the budget.
  int CL = (int)((4ll * p.V * es + kTVSmemBudget - 1) / kTVSmemBudget);
  if (CL < 1) CL = 1;
  int Lc = (p.V + CL - 1) / CL;
  Lc = (Lc + 15) / 16 * 16;
  CL = (p.V + Lc - 1) / Lc;
  if (CL > 16) return cudaErrorInvalidConfiguration;
  const size_t smem = ((sizeof(TVShared) + 127) / 128) * 128 + 4ull * Lc * es;

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
  A.ready = reinterpret_cast<unsigned*>(w + L.ready);
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
  A.total_tasks = p.N * (A.compute_grad ? 2 : 1);
  if (nclusters > A.total_tasks) nclusters = A.total_tasks;
  A.lag = (nclusters + p.W - 1) / p.W + 1;
  cfg.gridDim = dim3(CL * nclusters);
  void* args[] = {&A};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace specopd
