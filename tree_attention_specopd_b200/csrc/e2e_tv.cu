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
// B200 design.  The work is HBM-bound: its algorithmic traffic is one read
// of both logit rows and one write of the gradient.  Two schedules, picked
// by the host code at the end of this file:
//  - whole-row (e2e_tv_row.cuh, the default for 16-byte aligned rows and W
//    up to the SM count): one position per task, its rows streamed through
//    a shared-memory ring three times with the passes of consecutive tasks
//    pipelined;
//  - slice (this file's kernel, the fallback): a position's rows cut into
//    slices that stay in shared memory for all three passes, so it moves
//    exactly the algorithmic bytes, at the price of a cross-CTA handshake
//    per position and per branch.
// The slice schedule:
//  * Task = (position n, vocabulary slice c), NS slices per row.  A CTA
//    (128 threads) holds one task: both rows' slice arrive by 1-D bulk copy
//    (TMA) into its shared memory and stay there for all three passes.  Four
//    CTAs share an SM, so one CTA's copy and handshake waits overlap the
//    others' math.
//  * pass 1: one sweep for row maxima (packed bf16x2 compares) and sums of
//    2^(x - max) under a running maximum; the slice publishes (max, sum) of
//    both rows and waits (bounded) until the NS slices of its position have
//    published; every slice combines the NS statistics in the same fixed
//    order -> identical lse everywhere.
//  * pass 2: partial overlap a and masked draft mass s; publish, then wait
//    until the W*NS tasks of its branch have published; combine per
//    position in fixed order -> a_{b,j}, s_n; g_n from the branch.
//  * pass 3: dz from the slice still in shared memory, chunk by chunk; as
//    each chunk is done the next task's copy of that chunk starts.
//  * Static schedule in rounds: CTA g of a grid of G resident CTAs runs
//    tasks g, g + G, g + 2G, ...  G is a multiple of W*NS when that idles
//    few slots: a round (G consecutive tasks) then holds whole branches,
//    all of whose tasks start together, so the handshake waits only absorb
//    the spread of task durations.  Deadlock freedom needs only G >= W*NS
//    (checked on the host): a task waits for tasks of its own branch, less
//    than W*NS ids away, and a task not yet started is held by a CTA busy
//    with the task G ids before it, so a cycle of waits would have to gain
//    G ids per step while moving fewer than W*NS.  Every wait is bounded.
//  * The (i = 1, c = 0) task of each branch writes its overlaps and prefix
//    products; the last branch to finish reduces the loss in a fixed order.
//  * All math in the log2 domain with packed fp32x2 FMAs: x2 = z*log2(e) -
//    lse2, one ex2 per element per pass.  Passes 2 and 3 decide [q < p] from
//    the same FMA, so s_n and the gradient's mask always agree.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace specopd {

constexpr int kTVThreads = 128;
constexpr int kTVWarps = kTVThreads / 32;
constexpr int kTVCtasPerSm = 4;            // independent CTAs per SM hide each other's waits
constexpr int kTVChunks = 4;               // bulk copies per row slice (pipelined)
constexpr int kTVSmemBudget = 52 * 1024;   // bytes of row slices per CTA
constexpr int kTVMaxW = 256;               // positions per branch held in shared memory
constexpr int kTVMaxParts = 256;           // (a, s) partials staged in shared memory per round
constexpr int kTVMaxSlices = 64;           // slices per row (two per lane in one warp)
constexpr float kLog2e = 1.4426950408889634f;

struct TVArgs {
  int nbranch, W, V, N, rows_target, compute_grad;
  int NS, Lc, aligned, total_tasks;
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
  float4* stats;     // [N][NS] (max_t, sum_t, max_d, sum_d), log2 units
  float2* part;      // [N][NS] (a, s) partials
  double* bsum;      // [nbranch]
  unsigned* pos_cnt; // [N]      slices of the position with statistics published
  unsigned* br_cnt;  // [nbranch] tasks of the branch with partials published
  unsigned* ctl;     // [1] branches done, [2] abort
};

// bf16x2 / fp32 vectors of 16 bytes as packed fp32x2 pairs.
template <typename Tin> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;      // elements per 16 bytes
  static constexpr int kPairs = 4;
  static __device__ __forceinline__ void pairs(const uint4& u, float2* f) {
    f[0] = make_float2(bf16lo(u.x), bf16hi(u.x));
    f[1] = make_float2(bf16lo(u.y), bf16hi(u.y));
    f[2] = make_float2(bf16lo(u.z), bf16hi(u.z));
    f[3] = make_float2(bf16lo(u.w), bf16hi(u.w));
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
  static constexpr int kPairs = 2;
  static __device__ __forceinline__ void pairs(const uint4& u, float2* f) {
    f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    f[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
  static __device__ __forceinline__ float vmax(const uint4& u) {
    return fmaxf(fmaxf(__uint_as_float(u.x), __uint_as_float(u.y)),
                 fmaxf(__uint_as_float(u.z), __uint_as_float(u.w)));
  }
};

__device__ __forceinline__ float2 ex2_pair(float2 x) { return make_float2(ex2_fast(x.x), ex2_fast(x.y)); }

__device__ __forceinline__ void warp_lse2(float& m, float& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse2_combine(m, s, m2, s2);
  }
}

struct TVShared {
  uint64_t bar[kTVChunks];  // bulk-copy completion, one phase per task
  int next;                 // next task of this CTA
  int flag;
  float2 lse;               // (lse2_t, lse2_d) of the current position
  float g, s_own;           // gradient coefficient and s_n of the current position
  float4 red_stats[kTVWarps];
  float2 red_as[kTVWarps];
  double dred[kTVWarps];
  float sa[kTVMaxW];        // overlaps of the current branch
  float2 parts[kTVMaxParts];  // (a, s) partials of the current branch's tasks
};
// kTVCtasPerSm CTAs must fit the SM's 228 KB of shared memory (1 KB of it
// reserved per CTA): header + both rows' slices + alignment.
static_assert(kTVCtasPerSm * (sizeof(TVShared) + 128 + kTVSmemBudget + 1024) <= 228 * 1024,
              "E2E-TV shared memory does not fit kTVCtasPerSm CTAs per SM");

template <typename Tin, typename Tg>
__global__ void __launch_bounds__(kTVThreads, kTVCtasPerSm) e2e_tv_kernel(const TVArgs A) {
  extern __shared__ __align__(128) unsigned char tv_smem_raw[];
  TVShared& sh = *reinterpret_cast<TVShared*>(tv_smem_raw);
  Tin* st = reinterpret_cast<Tin*>(tv_smem_raw + ((sizeof(TVShared) + 127) / 128) * 128);
  Tin* sd = st + A.Lc;  // Lc is a multiple of 16 elements: 16-byte aligned
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int VN = Vec<Tin>::kN;
  constexpr int VP = Vec<Tin>::kPairs;
  const int V = A.V, W = A.W, NS = A.NS;
  const int chunk_elems = ((A.Lc / kTVChunks) + 15) / 16 * 16;
  const Tin* zt = reinterpret_cast<const Tin*>(A.zt);
  const Tin* zd = reinterpret_cast<const Tin*>(A.zd);
  const float2 L2E = make_float2(kLog2e, kLog2e);
  const float qnan = __int_as_float(0x7fc00000);

  if (tid == 0) {
    for (int c = 0; c < kTVChunks; ++c) mbar_init(&sh.bar[c], 1);
    fence_mbar_init();
  }

  // Next task of this CTA (static rounds); after a wait anywhere ran out,
  // stop.
  auto next_task = [&](int t) -> int {
    if (__ldcg(&A.ctl[2]) != 0u) return A.total_tasks;
    const long long n = (long long)t + gridDim.x;
    return n < A.total_tasks ? (int)n : A.total_tasks;
  };
  auto target_row = [&](int n, bool& ok) -> int {
    const int row = A.trow ? A.trow[n] : n;
    ok = (row >= 0 && row < A.rows_target);
    return ok ? row : 0;
  };
  // Bulk copy of chunk ch of task t into the slice buffers (thread 0; every
  // chunk barrier completes exactly one phase per task, empty chunks too).
  int cp_row = 0, cp_n = 0, cp_v0 = 0, cp_len = 0;
  auto prepare_copy = [&](int t) {
    bool ok;
    cp_n = t / NS;
    cp_v0 = (t % NS) * A.Lc;
    cp_len = max(0, min(V, cp_v0 + A.Lc) - cp_v0);
    cp_row = target_row(cp_n, ok);
  };
  auto issue_chunk = [&](int ch) {
    // The block barrier before this call ended every thread's generic reads
    // of the chunk; order them before the async-proxy writes of the copy.
    fence_proxy_async_smem();
    const uint64_t pol = l2_policy_evict_first();  // every logit is read once
    const int e0 = ch * chunk_elems;
    const int e1 = min(cp_len, e0 + chunk_elems);
    const unsigned bytes = e1 > e0 ? (unsigned)((e1 - e0) * sizeof(Tin)) : 0u;
    mbar_arrive_expect_tx(&sh.bar[ch], 2u * bytes);
    if (bytes) {
      bulk_g2s_hint(st + e0, zt + (long long)cp_row * V + cp_v0 + e0, bytes, &sh.bar[ch], pol);
      bulk_g2s_hint(sd + e0, zd + (long long)cp_n * V + cp_v0 + e0, bytes, &sh.bar[ch], pol);
    }
  };

  if (tid == 0) {
    sh.next = (int)blockIdx.x < A.total_tasks ? (int)blockIdx.x : A.total_tasks;
    if (sh.next < A.total_tasks && A.aligned) {
      prepare_copy(sh.next);
      for (int ch = 0; ch < kTVChunks; ++ch) issue_chunk(ch);
    }
  }
  __syncthreads();
  int t = sh.next;
  unsigned phase = 0;

  while (t < A.total_tasks) {
    const int n = t / NS, c = t % NS, b = n / W, i = n % W;
    const int v0 = c * A.Lc;
    const int len = max(0, min(V, v0 + A.Lc) - v0);
    const unsigned par = phase & 1u;
    ++phase;
    if (!A.aligned) {
      bool ok;
      const Tin* rt = zt + (long long)target_row(n, ok) * V + v0;
      const Tin* rd = zd + (long long)n * V + v0;
      for (int e = tid; e < len; e += kTVThreads) {
        st[e] = rt[e];
        sd[e] = rd[e];
      }
      __syncthreads();
    }

    // ------------------------------------------------ pass 1: statistics
    // One sweep over the slice as the copies land, with the element-to-thread
    // mapping of passes 2 and 3: per 16-byte group the running maxima (log2
    // units) move up when the group's maximum exceeds them, and the partial
    // sums of 2^(x - max) are rescaled then (rarely after the first groups).
    float mt = -INFINITY, md = -INFINITY;
    float sum_t = 0.f, sum_d = 0.f;
    {
      float2 at0 = make_float2(0.f, 0.f), at1 = at0, ad0 = at0, ad1 = at0;
      // Raise a running maximum; a sum formed under a -inf maximum holds only
      // NaNs from -inf entries and is reset, not rescaled.
      auto raise = [](float g, float& m, float2& s0, float2& s1) {
        if (g > m) {
          const float f = (m == -INFINITY) ? 0.f : ex2_fast(m - g);
          s0 = (m == -INFINITY) ? make_float2(0.f, 0.f) : __fmul2_rn(s0, make_float2(f, f));
          s1 = (m == -INFINITY) ? make_float2(0.f, 0.f) : __fmul2_rn(s1, make_float2(f, f));
          m = g;
        }
      };
      for (int ch = 0; ch < kTVChunks; ++ch) {
        const int e0 = ch * chunk_elems;
        const int e1 = min(len, e0 + chunk_elems);
        if (A.aligned && !mbar_wait(&sh.bar[ch], par) && tid == 0) atomicExch(&A.ctl[2], 1u);
        if (e1 <= e0) continue;
        const int nv = (e1 - e0) / VN;
        for (int vi = tid; vi < nv; vi += kTVThreads) {
          const uint4 ut = *reinterpret_cast<const uint4*>(st + e0 + vi * VN);
          const uint4 ud = *reinterpret_cast<const uint4*>(sd + e0 + vi * VN);
          raise(Vec<Tin>::vmax(ut) * kLog2e, mt, at0, at1);
          raise(Vec<Tin>::vmax(ud) * kLog2e, md, ad0, ad1);
          float2 ft[VP], fd[VP];
          Vec<Tin>::pairs(ut, ft);
          Vec<Tin>::pairs(ud, fd);
          const float2 nmt = make_float2(-mt, -mt), nmd = make_float2(-md, -md);
#pragma unroll
          for (int p = 0; p < VP; p += 2) {
            at0 = __fadd2_rn(at0, ex2_pair(__ffma2_rn(ft[p], L2E, nmt)));
            ad0 = __fadd2_rn(ad0, ex2_pair(__ffma2_rn(fd[p], L2E, nmd)));
            at1 = __fadd2_rn(at1, ex2_pair(__ffma2_rn(ft[p + 1], L2E, nmt)));
            ad1 = __fadd2_rn(ad1, ex2_pair(__ffma2_rn(fd[p + 1], L2E, nmd)));
          }
        }
        for (int e = e0 + nv * VN + tid; e < e1; e += kTVThreads) {
          const float xt = Elt<Tin>::to_f(st[e]) * kLog2e;
          const float xd = Elt<Tin>::to_f(sd[e]) * kLog2e;
          raise(xt, mt, at0, at1);
          raise(xd, md, ad0, ad1);
          at0.x += ex2_fast(xt - mt);
          ad0.x += ex2_fast(xd - md);
        }
      }
      sum_t = (at0.x + at0.y) + (at1.x + at1.y);
      sum_d = (ad0.x + ad0.y) + (ad1.x + ad1.y);
      // -inf maximum: this thread saw no finite entry of that row, no mass
      // (the NaNs formed above are dropped; the combine skips -inf)
      if (mt == -INFINITY) sum_t = 0.f;
      if (md == -INFINITY) sum_d = 0.f;
    }
    warp_lse2(mt, sum_t);
    warp_lse2(md, sum_d);
    if (lane == 0) sh.red_stats[warp] = make_float4(mt, sum_t, md, sum_d);
    __syncthreads();
    if (tid == 0) {
      float4 v = sh.red_stats[0];
      for (int w = 1; w < kTVWarps; ++w) {
        const float4 u = sh.red_stats[w];
        lse2_combine(v.x, v.y, u.x, u.y);
        lse2_combine(v.z, v.w, u.z, u.w);
      }
      bool row_ok;
      target_row(n, row_ok);
      if (!row_ok) {
        set_status(SPECOPD_DEV_ROW_RANGE);
        v.x = qnan;  // poisons this position's statistics
      }
      A.stats[(size_t)n * NS + c] = v;
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&A.pos_cnt[n]) : "memory");
      const bool ok = wait_flag_geq(&A.pos_cnt[n], (unsigned)NS);
      if (!ok) atomicExch(&A.ctl[2], 1u);
      sh.flag = ok ? 1 : 0;
    }
    __syncthreads();
    if (warp == 0) {
      // The position's NS slice statistics, combined in one fixed order in
      // every slice: lane j holds slices j and j + 32.
      float4 v = make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
      if (lane < NS) v = __ldcg(&A.stats[(size_t)n * NS + lane]);
      if (lane + 32 < NS) {
        const float4 u = __ldcg(&A.stats[(size_t)n * NS + lane + 32]);
        lse2_combine(v.x, v.y, u.x, u.y);
        lse2_combine(v.z, v.w, u.z, u.w);
      }
      warp_lse2(v.x, v.y);
      warp_lse2(v.z, v.w);
      if (lane == 0) {
        float2 L = make_float2(v.x + log2f(v.y), v.z + log2f(v.w));
        if (v.x == -INFINITY || v.z == -INFINITY) {
          if (c == 0) set_status(SPECOPD_DEV_ALL_NEG_INF);
          L = make_float2(qnan, qnan);
        }
        if (!sh.flag) L = make_float2(qnan, qnan);
        sh.lse = L;
      }
    }
    __syncthreads();
    const float lse2_t = sh.lse.x, lse2_d = sh.lse.y;
    const float2 nLt = make_float2(-lse2_t, -lse2_t), nLd = make_float2(-lse2_d, -lse2_d);

    // ------------------------------------------------ pass 2: overlap partials
    float pa = 0.f, ps = 0.f;
    {
      float2 pa2 = make_float2(0.f, 0.f), ps2 = pa2;
      for (int ch = 0; ch < kTVChunks; ++ch) {
        const int e0 = ch * chunk_elems;
        const int e1 = min(len, e0 + chunk_elems);
        if (e1 <= e0) continue;
        const int nv = (e1 - e0) / VN;
        for (int vi = tid; vi < nv; vi += kTVThreads) {
          float2 ft[VP], fd[VP];
          Vec<Tin>::pairs(*reinterpret_cast<const uint4*>(st + e0 + vi * VN), ft);
          Vec<Tin>::pairs(*reinterpret_cast<const uint4*>(sd + e0 + vi * VN), fd);
#pragma unroll
          for (int p = 0; p < VP; ++p) {
            const float2 lt = __ffma2_rn(ft[p], L2E, nLt);
            const float2 ld = __ffma2_rn(fd[p], L2E, nLd);
            const float2 e = make_float2(ex2_fast(fminf(lt.x, ld.x)), ex2_fast(fminf(lt.y, ld.y)));
            pa2 = __fadd2_rn(pa2, e);
            ps2 = __fadd2_rn(ps2, make_float2(ld.x < lt.x ? e.x : 0.f, ld.y < lt.y ? e.y : 0.f));
          }
        }
        for (int e = e0 + nv * VN + tid; e < e1; e += kTVThreads) {
          const float lt = __fmaf_rn(Elt<Tin>::to_f(st[e]), kLog2e, -lse2_t);
          const float ld = __fmaf_rn(Elt<Tin>::to_f(sd[e]), kLog2e, -lse2_d);
          const float ex = ex2_fast(fminf(lt, ld));
          pa2.x += ex;
          ps2.x += (ld < lt) ? ex : 0.f;
        }
      }
      pa = warp_sum(pa2.x + pa2.y);
      ps = warp_sum(ps2.x + ps2.y);
    }
    if (lane == 0) sh.red_as[warp] = make_float2(pa, ps);
    __syncthreads();
    const bool owner = (i == 0 && c == 0);  // writes the branch's overlaps and prefix products
    const bool need_branch = A.compute_grad || owner;
    if (tid == 0) {
      float2 v = sh.red_as[0];
      for (int w = 1; w < kTVWarps; ++w) {
        v.x += sh.red_as[w].x;
        v.y += sh.red_as[w].y;
      }
      A.part[(size_t)n * NS + c] = v;
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&A.br_cnt[b]) : "memory");
      int ok = 1;
      if (need_branch) {
        ok = wait_flag_geq(&A.br_cnt[b], (unsigned)(W * NS)) ? 1 : 0;
        if (!ok) atomicExch(&A.ctl[2], 1u);
      }
      sh.flag = ok;
    }
    __syncthreads();
    if (need_branch) {
      // Overlap (and this position's s) of every position of the branch,
      // each summed over its NS slices in a fixed order.  The partials of up
      // to kTVMaxParts / NS positions are loaded in one parallel round trip
      // into shared memory, then summed there.
      const bool ok = sh.flag != 0;
      const int pw = kTVMaxParts / NS;  // positions per round (NS <= kTVMaxSlices)
      for (int j0 = 0; j0 < W; j0 += pw) {
        const int j1 = min(W, j0 + pw);
        for (int k = tid; k < (j1 - j0) * NS; k += kTVThreads)
          sh.parts[k] = __ldcg(&A.part[((size_t)b * W + j0) * NS + k]);
        __syncthreads();
        for (int j = j0 + tid; j < j1; j += kTVThreads) {
          float av = 0.f, sv = 0.f;
          for (int cc = 0; cc < NS; ++cc) {
            const float2 u = sh.parts[(j - j0) * NS + cc];
            av += u.x;
            sv += u.y;
          }
          sh.sa[j] = ok ? av : qnan;
          if (j == i) sh.s_own = ok ? sv : qnan;
        }
        __syncthreads();
      }
      if (tid == 0) {
        // g_n = -(1/norm) P_{i-1} S_i, with no division by any overlap
        float P = 1.f;
        for (int j = 0; j < i; ++j) P *= sh.sa[j];
        float S = 1.f;
        for (int j = W - 1; j > i; --j) S = fmaf(sh.sa[j], S, 1.f);
        sh.g = -A.inv_norm * P * S;
        int last = 0;
        if (owner) {
          float Pp = 1.f;
          double sumP = 0.0;
          for (int j = 0; j < W; ++j) {
            Pp *= sh.sa[j];
            A.a_out[b * W + j] = sh.sa[j];
            A.prefix[b * W + j] = Pp;
            sumP += (double)Pp;
          }
          A.bsum[b] = sumP;
          __threadfence();
          const unsigned done = atomicAdd(&A.ctl[1], 1u);
          if (done == (unsigned)A.nbranch - 1u) {
            __threadfence();
            last = 1;
          }
        }
        sh.flag = last;
      }
      __syncthreads();
      if (sh.flag) {
        // Last branch: loss = 1 - sum_b bsum[b] / norm, fixed summation order.
        double acc = 0.0;
        for (int j = tid; j < A.nbranch; j += kTVThreads) acc += __ldcg(&A.bsum[j]);
        acc = warp_sum_d(acc);
        if (lane == 0) sh.dred[warp] = acc;
        __syncthreads();
        if (tid == 0) {
          double tot = 0.0;
          for (int w = 0; w < kTVWarps; ++w) tot += sh.dred[w];
          A.loss[0] = (float)(1.0 - tot / A.norm);
          if (A.numer) A.numer[0] = tot;
        }
      }
    }
    // This task's waits are over: set up the next one, whose copy streams in
    // chunk by chunk behind the gradient pass.
    if (tid == 0) {
      sh.next = next_task(t);
      if (sh.next < A.total_tasks && A.aligned) prepare_copy(sh.next);
    }
    __syncthreads();
    const int tn = sh.next;

    // ------------------------------------------------ pass 3: gradient
    if (A.compute_grad) {
      const float g = sh.g, s_val = sh.s_own;
      const float c1 = g * (1.f - s_val), c0 = -g * s_val;  // coefficient for [q<p] = 1 / 0
      Tg* gout = reinterpret_cast<Tg*>(A.grad) + (long long)n * V + v0;
      for (int ch = 0; ch < kTVChunks; ++ch) {
        const int e0 = ch * chunk_elems;
        const int e1 = min(len, e0 + chunk_elems);
        if (e1 > e0) {
          // Vector stores need 16-byte aligned gradient rows (aligned path);
          // otherwise every element goes through the scalar loop below.
          const int nv = A.aligned ? (e1 - e0) / VN : 0;
          for (int vi = tid; vi < nv; vi += kTVThreads) {
            float2 ft[VP], fd[VP], o[VP];
            Vec<Tin>::pairs(*reinterpret_cast<const uint4*>(st + e0 + vi * VN), ft);
            Vec<Tin>::pairs(*reinterpret_cast<const uint4*>(sd + e0 + vi * VN), fd);
#pragma unroll
            for (int p = 0; p < VP; ++p) {
              const float2 lt = __ffma2_rn(ft[p], L2E, nLt);
              const float2 ld = __ffma2_rn(fd[p], L2E, nLd);
              const float2 coef = make_float2(ld.x < lt.x ? c1 : c0, ld.y < lt.y ? c1 : c0);
              o[p] = __fmul2_rn(ex2_pair(ld), coef);
            }
            Tg* dst = gout + e0 + vi * VN;
            if constexpr (sizeof(Tg) == 4) {
#pragma unroll
              for (int p = 0; p < VP; p += 2)
                __stcs(reinterpret_cast<float4*>(dst + 2 * p),
                       make_float4(o[p].x, o[p].y, o[p + 1].x, o[p + 1].y));
            } else if constexpr (VP == 4) {
              uint4 u;
              u.x = pack_bf16x2(o[0].x, o[0].y);
              u.y = pack_bf16x2(o[1].x, o[1].y);
              u.z = pack_bf16x2(o[2].x, o[2].y);
              u.w = pack_bf16x2(o[3].x, o[3].y);
              __stcs(reinterpret_cast<uint4*>(dst), u);
            } else {
              uint2 u;
              u.x = pack_bf16x2(o[0].x, o[0].y);
              u.y = pack_bf16x2(o[1].x, o[1].y);
              __stcs(reinterpret_cast<uint2*>(dst), u);
            }
          }
          for (int e = e0 + nv * VN + tid; e < e1; e += kTVThreads) {
            const float lt = __fmaf_rn(Elt<Tin>::to_f(st[e]), kLog2e, -lse2_t);
            const float ld = __fmaf_rn(Elt<Tin>::to_f(sd[e]), kLog2e, -lse2_d);
            gout[e] = Elt<Tg>::from_f(ex2_fast(ld) * ((ld < lt) ? c1 : c0));
          }
        }
        // Chunk ch is done by every thread: the next task's copy of it starts.
        __syncthreads();
        if (tid == 0 && tn < A.total_tasks && A.aligned) issue_chunk(ch);
      }
    } else {
      if (tid == 0 && tn < A.total_tasks && A.aligned)
        for (int ch = 0; ch < kTVChunks; ++ch) issue_chunk(ch);
    }
    if (!A.aligned) __syncthreads();  // the next task's synchronous copy overwrites the slice
    t = tn;
  }
}

#include "e2e_tv_row.cuh"

// ------------------------------------------------------------------ host
namespace {

struct TVLayout {
  size_t stats, part, bsum, pos_cnt, br_cnt, ctl, total, zero_begin, zero_bytes;
};

// Slice geometry: the fewest slices per row, NS slices of Lc elements (a
// multiple of 16), whose two rows fit the shared-memory budget.
void tv_min_slices(const TVProblem& p, int& NS, int& Lc) {
  const int es = p.logit_dtype == SPECOPD_BF16 ? 2 : 4;
  NS = (int)((2ll * p.V * es + kTVSmemBudget - 1) / kTVSmemBudget);
  if (NS < 1) NS = 1;
  while (true) {
    Lc = (p.V + NS - 1) / NS;
    Lc = (Lc + 15) / 16 * 16;
    if (2ll * Lc * es <= kTVSmemBudget || Lc == 16) break;
    ++NS;  // rounding Lc up overshot the budget
  }
  NS = (p.V + Lc - 1) / Lc;
}

// Slice count for `resident` co-resident CTAs: from the budget's count up,
// the first for which rounds of whole branches (multiples of W*NS CTAs)
// idle under 5 % of the resident CTAs; the budget's count if none does.  A
// round then holds whole branches (see the kernel's schedule); a branch that
// straddles two rounds makes its early tasks wait about a whole task.
void tv_slices(const TVProblem& p, long long resident, int& NS, int& Lc) {
  tv_min_slices(p, NS, Lc);
  for (int want = NS; want <= kTVMaxSlices; ++want) {
    int lc = (p.V + want - 1) / want;
    lc = (lc + 15) / 16 * 16;
    const int ns = (p.V + lc - 1) / lc;
    const long long wns = (long long)p.W * ns;
    if (ns > kTVMaxSlices || wns > resident) break;
    if ((resident % wns) * 20 <= resident) {
      NS = ns;
      Lc = lc;
      return;
    }
  }
}

// Resident CTAs assumed for host-side sizing: the current device's SMs (148
// without one) times kTVCtasPerSm.
long long nominal_resident() {
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    nsm = 148;
  return (long long)nsm * kTVCtasPerSm;
}

TVLayout tv_layout(const TVProblem& p, int NS) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  TVLayout L;
  size_t off = 0;
  L.stats = off;   off = up(off + sizeof(float4) * (size_t)p.N * NS);
  L.part = off;    off = up(off + sizeof(float2) * (size_t)p.N * NS);
  L.bsum = off;    off = up(off + sizeof(double) * (size_t)p.nbranch);
  L.pos_cnt = off; off += sizeof(unsigned) * (size_t)p.N;
  L.br_cnt = off;  off += sizeof(unsigned) * (size_t)p.nbranch;
  L.ctl = off;     off = up(off + 4 * sizeof(unsigned));
  L.zero_begin = L.pos_cnt;
  L.zero_bytes = off - L.pos_cnt;
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
std::map<std::tuple<int, void*, int>, int> g_occ_cache;  // (dev, fn, smem) -> resident CTAs

}  // namespace

size_t tv_workspace(const TVProblem& p) {
  int NS, Lc;
  tv_slices(p, nominal_resident(), NS, Lc);
  return std::max(tv_layout(p, NS).total, tvrow::row_layout(p).total);
}

// The fewest slices per row this problem needs (the kernel needs W * NS
// resident CTAs).
int tv_slice_count(const TVProblem& p) {
  int NS, Lc;
  tv_min_slices(p, NS, Lc);
  return NS;
}

namespace {

template <typename Tin, typename Tg>
void* row_kernel_ptr() {
  return reinterpret_cast<void*>(&e2e_tv_row_kernel<Tin, Tg>);
}

void* pick_row_kernel(specopd_dtype in, specopd_dtype g) {
  if (in == SPECOPD_BF16)
    return g == SPECOPD_BF16 ? row_kernel_ptr<__nv_bfloat16, __nv_bfloat16>()
                             : row_kernel_ptr<__nv_bfloat16, float>();
  return g == SPECOPD_BF16 ? row_kernel_ptr<float, __nv_bfloat16>() : row_kernel_ptr<float, float>();
}

// Whole-row schedule (e2e_tv_row.cuh).  Returns cudaErrorNotSupported when
// it does not apply (the slice schedule takes over).
cudaError_t launch_row(const TVProblem& p, bool aligned, const void* z_target,
                       const int32_t* target_row, const void* z_draft, float* a, float* prefix,
                       float* loss, double* numer, void* grad, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  using namespace tvrow;
  if (!aligned) return cudaErrorNotSupported;
  const tvrow::RowLayout L = row_layout(p);
  if (ws_bytes < L.total) return cudaErrorNotSupported;
  void* fn = pick_row_kernel(p.logit_dtype, p.grad_dtype);
  int dev = 0, per_sm = 0, nsm = 148, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  // Pass B's [q < p] bits stay in shared memory after the ring when they
  // fit (one byte per chunk, vector and consumer thread): pass C then reads
  // the draft row only.
  const long long ce_b = (long long)kConsumers * kVPT * (16 / elt_size(p.logit_dtype));
  const size_t bits_bytes = (size_t)((p.V + ce_b - 1) / ce_b) * kVPT * kConsumers;
  size_t smem = ((sizeof(tvrow::Shared) + 127) / 128) * 128 + (size_t)kStages * 2 * kChunkBytes;
  const bool use_bits = p.compute_grad && grad != nullptr && smem + bits_bytes <= (size_t)optin;
  if (use_bits) smem += (bits_bytes + 15) / 16 * 16;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // Two CTAs per SM (the kernel's geometry).
  const long long resident = (long long)std::min(per_sm, 2) * nsm;
  if (p.W > resident) return cudaErrorNotSupported;
  // Whole branches per round, at most the resident CTAs; the rounds that
  // takes are then spread evenly (N = 512 at 296 slots: two rounds of 256
  // instead of 296 + 216; measured 180 against 184 us, bit-identical).
  const long long G0 = resident / p.W * p.W;
  const long long rounds = (p.N + G0 - 1) / G0;
  const long long G = std::min(G0, ((p.N + rounds - 1) / rounds + p.W - 1) / p.W * p.W);
  const int grid = (int)std::min<long long>(G, p.N);
  // The ring's chunk counter is 32-bit: keep a CTA's chunks below 2^32.
  const long long ce = (long long)kConsumers * kVPT * (16 / elt_size(p.logit_dtype));
  if ((long long)((p.N + G - 1) / G) * 3 * ((p.V + ce - 1) / ce) >= (1LL << 32))
    return cudaErrorNotSupported;

  RowArgs A;
  A.nbranch = p.nbranch; A.W = p.W; A.V = p.V; A.N = p.N; A.rows_target = p.rows_target;
  A.compute_grad = p.compute_grad && grad != nullptr;
  A.bits = use_bits ? 1 : 0;
  A.norm = p.norm_count;
  A.inv_norm = (float)(1.0 / p.norm_count);
  A.zt = z_target; A.trow = target_row; A.zd = z_draft;
  A.a_out = a; A.prefix = prefix; A.loss = loss; A.numer = numer; A.grad = grad;
  char* w = reinterpret_cast<char*>(ws);
  A.part = reinterpret_cast<float2*>(w + L.part);
  A.bsum = reinterpret_cast<double*>(w + L.bsum);
  A.br_cnt = reinterpret_cast<unsigned*>(w + L.br_cnt);
  A.ctl = reinterpret_cast<unsigned*>(w + L.ctl);
  e = cudaMemsetAsync(w + L.zero_begin, 0, L.zero_bytes, stream);
  if (e != cudaSuccess) return e;
  void* args[] = {&A};
  return cudaLaunchKernel(fn, dim3(grid), dim3(kThreads), args, smem, stream);
}

}  // namespace

// loss = 1 - numer_sum / norm (distributed normalisation, one thread).
__global__ void tv_finalize_kernel(const double* numer_sum, double norm, float* loss,
                                   double* loss64) {
  const double l = 1.0 - numer_sum[0] / norm;
  loss[0] = (float)l;
  if (loss64) loss64[0] = l;
}

cudaError_t launch_tv_finalize(const double* numer_sum, double norm, float* loss, double* loss64,
                               cudaStream_t st) {
  tv_finalize_kernel<<<1, 1, 0, st>>>(numer_sum, norm, loss, loss64);
  return cudaGetLastError();
}

namespace {

// Rows and pointers that the vector and bulk-copy paths of the whole-row
// schedule need: 16-byte aligned bases and row strides.
bool rows_aligned(const TVProblem& p, const void* z_target, const void* z_draft, const void* grad) {
  const int es = elt_size(p.logit_dtype);
  const int gs = elt_size(p.grad_dtype);
  const bool cg = p.compute_grad && grad != nullptr;
  return ((uintptr_t)z_target % 16 == 0) && ((uintptr_t)z_draft % 16 == 0) &&
         (!cg || (uintptr_t)grad % 16 == 0) && ((size_t)p.V * es % 16 == 0) &&
         (!cg || (size_t)p.V * gs % 16 == 0);
}

// Whether the whole-row schedule runs this problem (two CTAs per SM, rounds
// of whole branches).
bool row_applies(const TVProblem& p) {
  void* fn = pick_row_kernel(p.logit_dtype, p.grad_dtype);
  const size_t smem = ((sizeof(tvrow::Shared) + 127) / 128) * 128 +
                      (size_t)tvrow::kStages * 2 * tvrow::kChunkBytes;
  int dev = 0, per_sm = 0, nsm = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, tvrow::kThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  return p.W <= (long long)std::min(per_sm, 2) * nsm;
}

}  // namespace

size_t tv_workspace_for_call(const TVProblem& p, const void* z_target, const void* z_draft,
                             const void* grad) {
  if (rows_aligned(p, z_target, z_draft, grad) && row_applies(p)) return tvrow::row_layout(p).total;
  return tv_workspace(p);
}

cudaError_t launch_e2e_tv(const TVProblem& p, const void* z_target, const int32_t* target_row,
                          const void* z_draft, float* a, float* prefix, float* loss, double* numer,
                          void* grad, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (p.W > kTVMaxW) return cudaErrorInvalidConfiguration;
  const int es = elt_size(p.logit_dtype);
  const int gs = elt_size(p.grad_dtype);
  {
    const bool aligned = rows_aligned(p, z_target, z_draft, grad);
    const cudaError_t e = launch_row(p, aligned, z_target, target_row, z_draft, a, prefix, loss,
                                     numer, grad, ws, ws_bytes, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  void* fn = pick_kernel(p.logit_dtype, p.grad_dtype);
  // Resident CTAs at the budget's shared memory, the most any slice count
  // uses: every CTA of the grid is then co-resident whatever NS is chosen.
  const size_t smem_max = ((sizeof(TVShared) + 127) / 128) * 128 + (size_t)kTVSmemBudget;
  int dev = 0;
  cudaGetDevice(&dev);
  int resident = 0;
  cudaError_t e;
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    // The attribute is per function: set it on every launch (another problem
    // size may have lowered it since).
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    auto key = std::make_tuple(dev, fn, (int)smem_max);
    auto it = g_occ_cache.find(key);
    if (it != g_occ_cache.end()) {
      resident = it->second;
    } else {
      int per_sm = 0, nsm = 148;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kTVThreads, smem_max);
      if (e != cudaSuccess) return e;
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
      resident = per_sm * nsm;
      g_occ_cache[key] = resident;
    }
  }
  int NS, Lc;
  tv_slices(p, resident, NS, Lc);
  TVLayout L = tv_layout(p, NS);
  if (ws_bytes < L.total) {  // sized for another device: the budget's slices
    tv_min_slices(p, NS, Lc);
    L = tv_layout(p, NS);
  }
  if (ws_bytes < L.total) return cudaErrorInvalidValue;
  if (NS > kTVMaxSlices) return cudaErrorInvalidConfiguration;
  const size_t smem = ((sizeof(TVShared) + 127) / 128) * 128 + 2ull * Lc * es;

  TVArgs A;
  A.nbranch = p.nbranch; A.W = p.W; A.V = p.V; A.N = p.N; A.rows_target = p.rows_target;
  A.compute_grad = p.compute_grad && grad != nullptr;
  A.NS = NS; A.Lc = Lc;
  const bool ptr_ok = ((uintptr_t)z_target % 16 == 0) && ((uintptr_t)z_draft % 16 == 0) &&
                      (!A.compute_grad || (uintptr_t)grad % 16 == 0);
  A.aligned = ptr_ok && ((size_t)p.V * es % 16 == 0) && (!A.compute_grad || (size_t)p.V * gs % 16 == 0);
  A.norm = p.norm_count;
  A.inv_norm = (float)(1.0 / p.norm_count);
  A.zt = z_target; A.trow = target_row; A.zd = z_draft;
  A.a_out = a; A.prefix = prefix; A.loss = loss; A.numer = numer; A.grad = grad;
  char* w = reinterpret_cast<char*>(ws);
  A.stats = reinterpret_cast<float4*>(w + L.stats);
  A.part = reinterpret_cast<float2*>(w + L.part);
  A.bsum = reinterpret_cast<double*>(w + L.bsum);
  A.pos_cnt = reinterpret_cast<unsigned*>(w + L.pos_cnt);
  A.br_cnt = reinterpret_cast<unsigned*>(w + L.br_cnt);
  A.ctl = reinterpret_cast<unsigned*>(w + L.ctl);
  A.total_tasks = p.N * NS;

  e = cudaMemsetAsync(w + L.zero_begin, 0, L.zero_bytes, stream);
  if (e != cudaSuccess) return e;
  // Every task of a branch must be able to be resident at once.  The grid is
  // a whole number of branches' worth of tasks when that idles under 5 % of
  // the resident slots, else every slot (see the kernel's schedule).
  const long long wns = (long long)p.W * NS;
  if (wns > resident) return cudaErrorInvalidConfiguration;
  const long long spare = resident % wns;
  const long long G = spare * 20 <= resident ? resident - spare : resident;
  const int grid = (int)std::min<long long>(G, A.total_tasks);
  void* args[] = {&A};
  return cudaLaunchKernel(fn, dim3(grid), dim3(kTVThreads), args, smem, stream);
}

}  // namespace specopd
