// E2E-TV, one whole position per task (the default schedule for aligned
// rows).  Included by e2e_tv.cu after its kernel: shares TVArgs, Vec and the
// reduction helpers; the host side there picks the schedule.
//
// Same quantities as e2e_tv.cu (SpecOPD review (jaehun.me) §1.1, §3.3;
// paper summary (rustineverything.app) §2.3).
//
// A task is one supervised position n.  A CTA streams both logit rows of
// its positions through a ring of shared-memory chunks, three passes per
// position:
//   A: the row statistics (maxima, sums of 2^(x - max)) -> lse of both rows
//      (no other CTA is involved);
//   B: the overlap a_n = sum_v min(p_v, q_v) and s_n = sum_{q<p} q_v;
//      a_n and s_n are published for the branch;
//   C: after the branch's W overlaps are in, the gradient row.  Pass B keeps
//      [q < p] of every element in shared memory (one byte per chunk,
//      vector and consumer thread, beside the ring) when it fits, and pass C
//      then copies the draft row only: five row reads per entry instead of
//      six, which is what the kernel is bound by (the latency of the
//      ring's copies, not instruction issue or DRAM bandwidth).
// The passes of consecutive tasks are pipelined: phase k interleaves pass A
// of task k with pass C of task k - 1 chunk by chunk (A leads by kLag
// chunks), then runs pass B of task k.  So each phase reads new rows from
// DRAM while it writes the previous gradient row, and the branch handshake
// of task k - 1 has pass B of that task and the first chunks of pass A of
// task k to complete in.  The price is L2 reuse distance: between pass A
// of a task and its pass B the L2 also serves pass C of the previous task,
// so part of pass B's and pass C's re-reads come from DRAM.
//
// Roles: one producer warp issues the 1-D bulk copies (TMA) of every chunk
// ahead of the consumers (pass A at normal L2 priority, pass B evict-last
// for what pass C reads again -- the draft row only when pass B keeps the
// bits -- and evict-first otherwise, pass C evict-first); 12 consumer warps
// do the arithmetic; one scorer warp
// publishes each task's (a_n, s_n) from the consumer warps' partials, waits
// for the branch, computes g_n and the owner's outputs, and hands g_n to the
// consumers through an mbarrier.
//
// Schedule: CTA g runs positions g, g + G, g + 2G, ... with G a multiple of
// W and at most the resident CTAs, so every round holds whole branches.  A
// task's handshake waits only for the other positions of its branch, which
// run on resident CTAs of the same round and publish after pass B, which
// needs only earlier handshakes of the same CTAs: no deadlock.  Two CTAs
// share an SM (12 consumer warps, a 72 KB ring and the pass-B bits each):
// two positions in flight per SM, each ring coupling fewer warps (measured
// 3 % faster at 8B than one CTA of 24 warps with a 192 KB ring).  Every wait
// is bounded.

namespace tvrow {

constexpr int kConsumers = 384;              // 12 consumer warps (two CTAs per SM)
constexpr int kCWarps = kConsumers / 32;
constexpr int kProducerWarp = kCWarps;       // issues the bulk copies
constexpr int kScorerWarp = kCWarps + 1;     // branch handshake, g_n, owner outputs, loss
constexpr int kThreads = kConsumers + 64;
constexpr int kVPT = 1;                      // 16-byte vectors per consumer per row per chunk
constexpr int kStages = 6;                   // ring depth (6 x 12 KB)
constexpr int kChunkBytes = kConsumers * 16 * kVPT;  // bytes of one row per chunk
constexpr int kMaxW = 256;
constexpr int kLag = 8;                      // pass-A chunks ahead of pass C in a phase

struct Shared {
  uint64_t full[kStages], empty[kStages];
  uint64_t bdone;            // one phase per task: every consumer warp's pass-B partials are in
  uint64_t gfull;            // one phase per task: g_n and s_n are in
  uint64_t lsebar;           // one phase per task: every consumer warp's pass-A record is in
  float4 red[2][kCWarps];    // per-warp (max, sum) of both rows after pass A, by task parity
  float2 redB[kCWarps];      // per-warp (a, s) partials after pass B
  float g, s_own;            // written by the scorer warp
  float sa[kMaxW];           // the branch's overlaps (scorer warp)
};

// Row-task workspace: per-position (a, s) records, per-branch prefix-product
// sums, per-branch arrival counters, control words.
struct RowLayout {
  size_t part, bsum, br_cnt, ctl, total, zero_begin, zero_bytes;
};

inline RowLayout row_layout(const TVProblem& p) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  RowLayout L;
  size_t off = 0;
  L.part = off;   off = up(off + sizeof(float2) * (size_t)p.N);
  L.bsum = off;   off = up(off + sizeof(double) * (size_t)p.nbranch);
  L.br_cnt = off; off += sizeof(unsigned) * (size_t)p.nbranch;
  L.ctl = off;    off = up(off + 4 * sizeof(unsigned));
  L.zero_begin = L.br_cnt;
  L.zero_bytes = off - L.br_cnt;
  L.total = off;
  return L;
}

struct RowArgs {
  int nbranch, W, V, N, rows_target, compute_grad;
  int bits;  // 1: pass B keeps [q < p] per element in shared memory; pass C reads the draft row only
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
  float2* part;      // [N] (a, s)
  double* bsum;      // [nbranch]
  unsigned* br_cnt;  // [nbranch] positions of the branch with (a, s) published
  unsigned* ctl;     // [1] branches done, [2] abort
};

__device__ __forceinline__ uint64_t l2_policy_evict_last_full() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// (max, sum) pair of log2-domain statistics: combine two, branch-free.  An
// empty side (max = -inf) contributes nothing; the result is symmetric in
// the two operands bit for bit.
__device__ __forceinline__ void lse2_merge(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  const float a = (m == -INFINITY) ? 0.f : s * ex2_fast(m - mn);
  const float b = (m2 == -INFINITY) ? 0.f : s2 * ex2_fast(m2 - mn);
  m = mn;
  s = a + b;
}
__device__ __forceinline__ void warp_lse2_merge(float& m, float& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse2_merge(m, s, m2, s2);
  }
}

}  // namespace tvrow

template <typename Tin, typename Tg>
__global__ void __launch_bounds__(tvrow::kThreads, 2) e2e_tv_row_kernel(const tvrow::RowArgs A) {
  using namespace tvrow;
  extern __shared__ __align__(128) unsigned char row_smem[];
  Shared& sh = *reinterpret_cast<Shared*>(row_smem);
  uint8_t* ring = row_smem + ((sizeof(Shared) + 127) / 128) * 128;  // [stage][target | draft]
  // [q < p] of this task's elements, one byte per (chunk, vector, consumer
  // thread), written by pass B and read by pass C of the same thread (when
  // A.bits; the buffer follows the ring)
  uint8_t* bitbuf = ring + (size_t)kStages * 2 * kChunkBytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int VN = Vec<Tin>::kN;  // elements per 16-byte vector
  constexpr int VP = Vec<Tin>::kPairs;
  constexpr int CE = kConsumers * VN * kVPT;  // elements of a row per chunk
  const int V = A.V, W = A.W;
  const int nch = (V + CE - 1) / CE;   // chunks per row
  const int G = gridDim.x;
  const int ntask = (int)blockIdx.x < A.N ? (A.N - 1 - (int)blockIdx.x) / G + 1 : 0;
  const bool grad = A.compute_grad != 0;
  const float2 L2E = make_float2(kLog2e, kLog2e);
  const float qnan = __int_as_float(0x7fc00000);
  auto target_row = [&](int n, bool& ok) -> int {
    const int row = A.trow ? A.trow[n] : n;
    ok = (row >= 0 && row < A.rows_target);
    return ok ? row : 0;
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kCWarps);
    }
    mbar_init(&sh.bdone, kCWarps);
    mbar_init(&sh.gfull, 1);
    mbar_init(&sh.lsebar, kCWarps);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    // ================================================================ producer
    // Chunk order, shared with the consumers: for k = 0 .. ntask, phase k
    // interleaves pass A of task k with pass C of task k - 1 (A leads by
    // kLag chunks), then pass B of task k; phase ntask holds only the last C.
    if (lane == 0) {
      // Pass A loads at normal priority: between pass A of a task and its
      // pass B the L2 also serves the previous task's pass C, and an
      // evict-last hint on pass A as well left more of pass B's re-reads to
      // DRAM (measured).
      const uint64_t load = l2_policy_evict_normal();     // pass A
      const uint64_t keep = l2_policy_evict_last_full();  // pass B: read again by pass C
      const uint64_t drop = l2_policy_evict_first();      // pass C: last use
      // With the [q < p] bits pass C reads the draft row only: pass B keeps
      // just the draft in L2 (one row of one model per CTA, about 90 MB over
      // the grid, which fits where both rows did not).
      const uint64_t keep_t = A.bits ? drop : keep;
      const Tin* zt = reinterpret_cast<const Tin*>(A.zt);
      const Tin* zd = reinterpret_cast<const Tin*>(A.zd);
      unsigned q = 0;  // chunk sequence number over all tasks and passes (mod 2^32)
      bool live = true;
      auto issue = [&](const Tin* rt, const Tin* rd, int c, uint64_t pol_t, uint64_t pol) {
        if (!live) return;
        const int st = (int)(q % kStages);
        const unsigned use = q / kStages;
        if (use > 0u && !mbar_wait(&sh.empty[st], (use - 1u) & 1u)) {
          atomicExch(&A.ctl[2], 1u);
          live = false;  // the consumers' waits run out in turn
          return;
        }
        const int e0 = c * CE;
        const unsigned bytes = (unsigned)(min(CE, V - e0) * (int)sizeof(Tin));
        uint8_t* dst = ring + (size_t)st * 2 * kChunkBytes;
        mbar_arrive_expect_tx(&sh.full[st], 2u * bytes);
        bulk_g2s_hint(dst, rt + e0, bytes, &sh.full[st], pol_t);
        bulk_g2s_hint(dst + kChunkBytes, rd + e0, bytes, &sh.full[st], pol);
        ++q;
      };
      // pass C with the [q < p] bits: the draft row's chunk only
      auto issue_d = [&](const Tin* rd, int c, uint64_t pol) {
        if (!live) return;
        const int st = (int)(q % kStages);
        const unsigned use = q / kStages;
        if (use > 0u && !mbar_wait(&sh.empty[st], (use - 1u) & 1u)) {
          atomicExch(&A.ctl[2], 1u);
          live = false;
          return;
        }
        const int e0 = c * CE;
        const unsigned bytes = (unsigned)(min(CE, V - e0) * (int)sizeof(Tin));
        uint8_t* dst = ring + (size_t)st * 2 * kChunkBytes;
        mbar_arrive_expect_tx(&sh.full[st], bytes);
        bulk_g2s_hint(dst + kChunkBytes, rd + e0, bytes, &sh.full[st], pol);
        ++q;
      };
      const Tin *rt_prev = zt, *rd_prev = zd;
      for (int k = 0; k <= ntask && live; ++k) {
        // Another warp's wait ran out (abort): issue nothing more.
        if (__ldcg(&A.ctl[2]) != 0u) break;
        const bool hasA = k < ntask, hasC = grad && k > 0;
        const Tin *rt = zt, *rd = zd;
        if (hasA) {
          const int n = (int)blockIdx.x + k * G;
          bool ok;
          rt = zt + (long long)target_row(n, ok) * V;
          rd = zd + (long long)n * V;
        }
        for (int i = -kLag; i < nch; ++i) {
          if (hasC && i >= 0) {
            if (A.bits) issue_d(rd_prev, i, drop); else issue(rt_prev, rd_prev, i, drop, drop);
          }
          if (hasA && i + kLag < nch) issue(rt, rd, i + kLag, load, load);
        }
        if (hasA)
          for (int c = 0; c < nch; ++c) issue(rt, rd, c, keep_t, keep);
        rt_prev = rt;
        rd_prev = rd;
      }
      // No copy may still be landing when this warp -- the last user of the
      // CTA's shared memory that can start one -- returns: wait (bounded)
      // for the last phase issued into every stage.  In a normal run the
      // consumers have waited for each already and these return at once.
      for (unsigned j = (q > (unsigned)kStages ? q - (unsigned)kStages : 0u); j < q; ++j)
        mbar_wait(&sh.full[j % kStages], (j / kStages) & 1u);
    }
    return;
  }

  if (warp == kScorerWarp) {
    // ================================================================ scorer
    // Per task, after the W positions of its branch have published (a, s):
    // g_n for pass C, the owner's outputs, and the loss once every branch is
    // in.  Runs beside the consumers, which need g_n only a few chunks into
    // the next phase.
    for (int k = 0; k < ntask; ++k) {
      const int n = (int)blockIdx.x + k * G;
      const int b = n / W, i = n % W;
      const bool owner = (i == 0);  // writes the branch's overlaps and prefix products
      int last = 0;
      int ok_branch = 0;
      if (lane == 0) {
        // publish (a_n, s_n) once every consumer warp's partials are in
        const bool in = mbar_wait(&sh.bdone, (unsigned)(k & 1));
        float2 v = make_float2(qnan, qnan);
        if (in) {
          v = make_float2(0.f, 0.f);
          for (int w = 0; w < kCWarps; ++w) {
            v.x += sh.redB[w].x;
            v.y += sh.redB[w].y;
          }
        } else {
          atomicExch(&A.ctl[2], 1u);
        }
        if ((long long)n != g_inject.withhold_position) {  // test hook: off by default
          A.part[n] = v;
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&A.br_cnt[b]) : "memory");
        }
        if (grad || owner) {
          // A branch wait that runs out makes this task's outputs NaN; it
          // does not abort the copy ring (the other tasks go on).
          const unsigned long long lim =
              g_inject.branch_wait_ns ? g_inject.branch_wait_ns : kWaitLimitNs;
          ok_branch = (in && __ldcg(&A.ctl[2]) == 0u &&
                       wait_flag_geq_limit(&A.br_cnt[b], (unsigned)W, lim)) ? 1 : 0;
        }
      }
      // The branch's W overlaps, one load per lane, each lane ordered after
      // its own acquire of the (complete) counter.
      ok_branch = __shfl_sync(0xffffffffu, ok_branch, 0);
      if (grad || owner) {
        if (ok_branch) ld_acquire_gpu(&A.br_cnt[b]);
        for (int j = lane; j < W; j += 32)
          sh.sa[j] = ok_branch ? __ldcg(&A.part[(size_t)b * W + j]).x : qnan;
      }
      __syncwarp();
      if (lane == 0) {
        if (grad || owner) {
          const float s_own = ok_branch ? __ldcg(&A.part[n]).y : qnan;
          // g_n = -(1/norm) P_{i-1} S_i, with no division by any overlap
          float P = 1.f;
          for (int j = 0; j < i; ++j) P *= sh.sa[j];
          float S = 1.f;
          for (int j = W - 1; j > i; --j) S = fmaf(sh.sa[j], S, 1.f);
          sh.g = -A.inv_norm * P * S;
          sh.s_own = s_own;
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
            if (atomicAdd(&A.ctl[1], 1u) == (unsigned)A.nbranch - 1u) {
              __threadfence();
              last = 1;
            }
          }
        }
        mbar_arrive(&sh.gfull);  // releases sh.g and sh.s_own to the consumers
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        // Last branch: loss = 1 - sum_b bsum[b] / norm, fixed summation order.
        double acc = 0.0;
        for (int j = lane; j < A.nbranch; j += 32) acc += __ldcg(&A.bsum[j]);
        acc = warp_sum_d(acc);
        if (lane == 0) {
          A.loss[0] = (float)(1.0 - acc / A.norm);
          if (A.numer) A.numer[0] = acc;
        }
      }
    }
    return;
  }

  // ================================================================== consumers
  unsigned q = 0;
  bool dead = false;  // a wait ran out: skip the remaining waits
  // Wait for chunk q, return its two row vectors of this thread (valid when
  // the element index is below V).
  // Vector v of this thread in chunk c: elements c*CE + (v*kConsumers + tid)*VN.
  auto wait_chunk = [&]() {
    const int st = (int)(q % kStages);
    if (!dead && !mbar_wait(&sh.full[st], (q / kStages) & 1u)) {
      dead = true;
      atomicExch(&A.ctl[2], 1u);
    }
  };
  // `full` (std::true_type / std::false_type): chunk c lies wholly inside
  // the row, so no vector of it needs the bounds check (the common case: only
  // the last chunk of a row is ragged).
  const int nfull = V / CE;
  auto take = [&](int c, int v, uint4& ut, uint4& ud, auto full) -> bool {
    const int st = (int)(q % kStages);
    const int vec = v * kConsumers + tid;
    const bool in = decltype(full)::value || (c * CE + vec * VN < V);
    if (in) {
      const uint8_t* src = ring + (size_t)st * 2 * kChunkBytes + vec * 16;
      ut = *reinterpret_cast<const uint4*>(src);
      ud = *reinterpret_cast<const uint4*>(src + kChunkBytes);
    }
    return in;
  };
  // The draft row's vector only (pass C with the [q < p] bits).
  auto take_d = [&](int c, int v, uint4& ud, auto full) -> bool {
    const int st = (int)(q % kStages);
    const int vec = v * kConsumers + tid;
    const bool in = decltype(full)::value || (c * CE + vec * VN < V);
    if (in) ud = *reinterpret_cast<const uint4*>(ring + (size_t)st * 2 * kChunkBytes + kChunkBytes + vec * 16);
    return in;
  };
  // Release chunk q (one arrive per consumer warp) and advance.
  auto give = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[(int)(q % kStages)]);
    ++q;
  };

  // lse (log2 units) of the position whose gradient the next phase writes
  float lseC_t = 0.f, lseC_d = 0.f;
  for (int k = 0; k <= ntask; ++k) {
    const bool hasA = k < ntask, hasC = grad && k > 0;
    const int n = (int)blockIdx.x + k * G;  // task k (pass A, B); n - G is task k - 1

    // ------------------------------ phase k: pass A of task k, pass C of task k - 1
    float mt = -INFINITY, md = -INFINITY;
    float2 at0 = make_float2(0.f, 0.f), at1 = at0, ad0 = at0, ad1 = at0;
    auto raise = [](float gm, float& m, float2& s0, float2& s1) {
      if (gm > m) {
        const float f = (m == -INFINITY) ? 0.f : ex2_fast(m - gm);
        s0 = (m == -INFINITY) ? make_float2(0.f, 0.f) : __fmul2_rn(s0, make_float2(f, f));
        s1 = (m == -INFINITY) ? make_float2(0.f, 0.f) : __fmul2_rn(s1, make_float2(f, f));
        m = gm;
      }
    };
    const float2 nLtC = make_float2(-lseC_t, -lseC_t), nLdC = make_float2(-lseC_d, -lseC_d);
    float c1 = 0.f, c0 = 0.f;  // gradient coefficient for [q<p] = 1 / 0
    Tg* gout = reinterpret_cast<Tg*>(A.grad) + (hasC ? (long long)(n - G) * V : 0LL);
    if (!grad && k > 0 && !dead && !mbar_wait(&sh.gfull, (unsigned)((k - 1) & 1))) {
      // Without pass C the consumers still keep within one task of the
      // scorer, which reads sh.redB of the previous task.
      dead = true;
      atomicExch(&A.ctl[2], 1u);
    }
    // ---- pass C, chunk i: the gradient row of task k - 1
    auto chunkC = [&](int i, auto full) {
        wait_chunk();
#pragma unroll
        for (int v = 0; v < kVPT; ++v) {
          uint4 ut, ud;
          if (A.bits ? take_d(i, v, ud, full) : take(i, v, ut, ud, full)) {
            float2 fd[VP], o[VP];
            Vec<Tin>::pairs(ud, fd);
            if (A.bits) {
              const unsigned bm = bitbuf[(i * kVPT + v) * kConsumers + tid];
#pragma unroll
              for (int p = 0; p < VP; ++p) {
                const float2 ld = __ffma2_rn(fd[p], L2E, nLdC);
                const float2 coef = make_float2((bm >> (2 * p)) & 1u ? c1 : c0,
                                                (bm >> (2 * p + 1)) & 1u ? c1 : c0);
                o[p] = __fmul2_rn(ex2_pair(ld), coef);
              }
            } else {
              float2 ft[VP];
              Vec<Tin>::pairs(ut, ft);
#pragma unroll
              for (int p = 0; p < VP; ++p) {
                const float2 lt = __ffma2_rn(ft[p], L2E, nLtC);
                const float2 ld = __ffma2_rn(fd[p], L2E, nLdC);
                const float2 coef = make_float2(ld.x < lt.x ? c1 : c0, ld.y < lt.y ? c1 : c0);
                o[p] = __fmul2_rn(ex2_pair(ld), coef);
              }
            }
            Tg* dst = gout + i * CE + (v * kConsumers + tid) * VN;
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
        }
        give();
    };
        // ---- pass A, chunk c: row sums under a running maximum.
        // From the second chunk on, the chunk is summed under the current
        // maxima first and accepted when both partial sums stay at most
        // 2^64 (no term overflowed, none was -inf - -inf); otherwise, and
        // for the first chunk, every vector raises the maxima before it is
        // summed.  Either way the sums are of 2^(x - m) for the m they are
        // kept under, so the lse below is the same quantity.
    auto chunkA = [&](int c, auto full) {
        wait_chunk();
        uint4 ut[kVPT], ud[kVPT];
        bool in[kVPT];
#pragma unroll
        for (int v = 0; v < kVPT; ++v) in[v] = take(c, v, ut[v], ud[v], full);
        bool exact = (c == 0);
        if (!exact) {
          float2 ct0 = make_float2(0.f, 0.f), ct1 = ct0, cd0 = ct0, cd1 = ct0;
          const float2 nmt = make_float2(-mt, -mt), nmd = make_float2(-md, -md);
#pragma unroll
          for (int v = 0; v < kVPT; ++v) {
            if (in[v]) {
              float2 ft[VP], fd[VP];
              Vec<Tin>::pairs(ut[v], ft);
              Vec<Tin>::pairs(ud[v], fd);
#pragma unroll
              for (int p = 0; p < VP; p += 2) {
                ct0 = __fadd2_rn(ct0, ex2_pair(__ffma2_rn(ft[p], L2E, nmt)));
                cd0 = __fadd2_rn(cd0, ex2_pair(__ffma2_rn(fd[p], L2E, nmd)));
                ct1 = __fadd2_rn(ct1, ex2_pair(__ffma2_rn(ft[p + 1], L2E, nmt)));
                cd1 = __fadd2_rn(cd1, ex2_pair(__ffma2_rn(fd[p + 1], L2E, nmd)));
              }
            }
          }
          const float st = (ct0.x + ct0.y) + (ct1.x + ct1.y);
          const float sd = (cd0.x + cd0.y) + (cd1.x + cd1.y);
          if (st <= 0x1p64f && sd <= 0x1p64f) {
            at0 = __fadd2_rn(at0, ct0);
            at1 = __fadd2_rn(at1, ct1);
            ad0 = __fadd2_rn(ad0, cd0);
            ad1 = __fadd2_rn(ad1, cd1);
          } else {
            exact = true;
          }
        }
        if (exact) {
#pragma unroll
          for (int v = 0; v < kVPT; ++v) {
            if (in[v]) {
              raise(Vec<Tin>::vmax(ut[v]) * kLog2e, mt, at0, at1);
              raise(Vec<Tin>::vmax(ud[v]) * kLog2e, md, ad0, ad1);
              float2 ft[VP], fd[VP];
              Vec<Tin>::pairs(ut[v], ft);
              Vec<Tin>::pairs(ud[v], fd);
              const float2 nmt = make_float2(-mt, -mt), nmd = make_float2(-md, -md);
#pragma unroll
              for (int p = 0; p < VP; p += 2) {
                at0 = __fadd2_rn(at0, ex2_pair(__ffma2_rn(ft[p], L2E, nmt)));
                ad0 = __fadd2_rn(ad0, ex2_pair(__ffma2_rn(fd[p], L2E, nmd)));
                at1 = __fadd2_rn(at1, ex2_pair(__ffma2_rn(ft[p + 1], L2E, nmt)));
                ad1 = __fadd2_rn(ad1, ex2_pair(__ffma2_rn(fd[p + 1], L2E, nmd)));
              }
            }
          }
        }
        give();
    };
    for (int i = -kLag; i < nch; ++i) {
      if (hasC && i >= 0) {
        if (i == 0) {
          if (!dead && !mbar_wait(&sh.gfull, (unsigned)((k - 1) & 1))) {
            dead = true;
            atomicExch(&A.ctl[2], 1u);
          }
          const float g = sh.g, s_val = sh.s_own;
          c1 = g * (1.f - s_val);
          c0 = -g * s_val;
        }
        if (i < nfull) chunkC(i, std::true_type{}); else chunkC(i, std::false_type{});
      }
      if (hasA && i + kLag < nch) {
        const int c = i + kLag;
        if (c < nfull) chunkA(c, std::true_type{}); else chunkA(c, std::false_type{});
        if (c == nch - 1) {
          // Pass A of this warp is complete: its record of the row
          // statistics goes in now, and the warp waits for the others'
          // only after the C chunks that follow (the last kLag of pass C),
          // so those absorb the warps' skew.
          float sum_t = (at0.x + at0.y) + (at1.x + at1.y);
          float sum_d = (ad0.x + ad0.y) + (ad1.x + ad1.y);
          // -inf maximum: this thread saw no finite entry of that row, no mass
          if (mt == -INFINITY) sum_t = 0.f;
          if (md == -INFINITY) sum_d = 0.f;
          warp_lse2_merge(mt, sum_t);
          warp_lse2_merge(md, sum_d);
          if (lane == 0) {
            sh.red[k & 1][warp] = make_float4(mt, sum_t, md, sum_d);
            mbar_arrive(&sh.lsebar);
          }
        }
      }
    }
    if (!hasA) break;  // the last phase held only the last gradient row

    // ------------------------------ lse of task k
    // Every warp waits for the kCWarps records (bounded), then combines them
    // itself.  The combination is symmetric in its two operands, so the
    // butterfly leaves the same bits in every lane, and every warp computes
    // the same L.  The records alternate between two buffers by task parity:
    // a warp writes this buffer again (task k + 2) only after waiting for
    // task k + 1's records, which every warp writes after reading these.
    if (!dead && !mbar_wait(&sh.lsebar, (unsigned)(k & 1))) {
      dead = true;
      atomicExch(&A.ctl[2], 1u);
    }
    float2 L;
    {
      float4 v = lane < kCWarps ? sh.red[k & 1][lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
      warp_lse2_merge(v.x, v.y);
      warp_lse2_merge(v.z, v.w);
      L = make_float2(v.x + log2f(v.y), v.z + log2f(v.w));
      bool row_ok;
      target_row(n, row_ok);
      if (!row_ok) {
        if (tid == 0) set_status(SPECOPD_DEV_ROW_RANGE);
        L = make_float2(qnan, qnan);
      } else if (v.x == -INFINITY || v.z == -INFINITY) {
        if (tid == 0) set_status(SPECOPD_DEV_ALL_NEG_INF);
        L = make_float2(qnan, qnan);
      }
      if (dead) L = make_float2(qnan, qnan);
    }
    lseC_t = L.x;
    lseC_d = L.y;
    const float2 nLt = make_float2(-L.x, -L.x), nLd = make_float2(-L.y, -L.y);

    // ------------------------------ pass B of task k: a_n and s_n
    float2 pa2 = make_float2(0.f, 0.f), ps2 = pa2;
    auto chunkB = [&](int c, auto full) {
      wait_chunk();
#pragma unroll
      for (int v = 0; v < kVPT; ++v) {
        uint4 ut, ud;
        if (take(c, v, ut, ud, full)) {
          float2 ft[VP], fd[VP];
          Vec<Tin>::pairs(ut, ft);
          Vec<Tin>::pairs(ud, fd);
          unsigned bm = 0u;
#pragma unroll
          for (int p = 0; p < VP; ++p) {
            const float2 lt = __ffma2_rn(ft[p], L2E, nLt);
            const float2 ld = __ffma2_rn(fd[p], L2E, nLd);
            const float2 e = make_float2(ex2_fast(fminf(lt.x, ld.x)), ex2_fast(fminf(lt.y, ld.y)));
            const bool bx = ld.x < lt.x, by = ld.y < lt.y;
            pa2 = __fadd2_rn(pa2, e);
            ps2 = __fadd2_rn(ps2, make_float2(bx ? e.x : 0.f, by ? e.y : 0.f));
            bm |= (bx ? 1u : 0u) << (2 * p);
            bm |= (by ? 1u : 0u) << (2 * p + 1);
          }
          if (A.bits) bitbuf[(c * kVPT + v) * kConsumers + tid] = (uint8_t)bm;
        }
      }
      give();
    };
    for (int c = 0; c < nch; ++c) {
      if (c < nfull) chunkB(c, std::true_type{}); else chunkB(c, std::false_type{});
    }
    // Partials to the scorer warp, which publishes them; no consumer waits.
    // sh.redB is written again only after the scorer's gfull arrival for
    // this task, which follows its read of sh.redB.
    {
      const float pa = warp_sum(pa2.x + pa2.y);
      const float ps = warp_sum(ps2.x + ps2.y);
      if (lane == 0) {
        sh.redB[warp] = make_float2(pa, ps);
        mbar_arrive(&sh.bdone);
      }
    }
  }
}
