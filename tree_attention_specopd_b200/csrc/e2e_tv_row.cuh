// E2E-TV, one whole position per task (the default schedule for aligned
// rows).  Included by e2e_tv.cu after its kernel: shares TVArgs, Vec and the
// reduction helpers; the host side there picks the schedule.
//
// Same quantities as e2e_tv.cu (SpecOPD review (jaehun.me) §1.1, §3.3;
// paper summary (rustineverything.app) §2.3).
//
// A CTA owns one supervised position n at a time and streams both logit
// rows through a ring of shared-memory chunks three times:
//   A: the row statistics (maxima, sums of 2^(x - max)) -> lse of both rows
//      (no other CTA is involved);
//   B: the overlap a_n = sum_v min(p_v, q_v) and s_n = sum_{q<p} q_v;
//      a_n and s_n are published for the branch;
//   C: after the branch's W overlaps are in, the gradient row.
// One producer warp issues the 1-D bulk copies (TMA) of every chunk of every
// pass ahead of the consumers (24 warps); chunks of passes A and B are
// fetched with an L2 evict-last hint, so passes B and C mostly re-read the
// rows from L2, and pass C with evict-first.  The only cross-CTA wait is the
// branch's, after pass B: the W positions of a branch are processed at the
// same time by W CTAs.
//
// Schedule: CTA g runs positions g, g + G, g + 2G, ... with G a multiple of
// W and at most the resident CTAs, so every round holds whole branches and a
// task waits only for tasks of its own round, each the current task of a
// resident CTA: no deadlock.  One CTA per SM keeps the rows in flight
// (G x 2 rows) within the L2.  Every wait is bounded.

namespace tvrow {

constexpr int kConsumers = 768;              // 24 consumer warps
constexpr int kThreads = kConsumers + 32;    // + the producer warp
constexpr int kCWarps = kConsumers / 32;
constexpr int kVPT = 2;                      // 16-byte vectors per consumer per row per chunk
constexpr int kStages = 4;                   // ring depth (4 x 48 KB)
constexpr int kChunkBytes = kConsumers * 16 * kVPT;  // bytes of one row per chunk
constexpr int kMaxW = 256;

struct Shared {
  uint64_t full[kStages], empty[kStages];
  float4 red[kCWarps];
  double dred[kCWarps];
  float2 lse;
  float g, s_own;
  int flag;
  float sa[kMaxW];
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

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

}  // namespace tvrow

template <typename Tin, typename Tg>
__global__ void __launch_bounds__(tvrow::kThreads, 1) e2e_tv_row_kernel(const tvrow::RowArgs A) {
  using namespace tvrow;
  extern __shared__ __align__(128) unsigned char row_smem[];
  Shared& sh = *reinterpret_cast<Shared*>(row_smem);
  uint8_t* ring = row_smem + ((sizeof(Shared) + 127) / 128) * 128;  // [stage][target | draft]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int VN = Vec<Tin>::kN;  // elements per 16-byte vector
  constexpr int VP = Vec<Tin>::kPairs;
  constexpr int CE = kConsumers * VN * kVPT;  // elements of a row per chunk
  const int V = A.V, W = A.W;
  const int nch = (V + CE - 1) / CE;   // chunks per row
  const int G = gridDim.x;
  const int ntask = (int)blockIdx.x < A.N ? (A.N - 1 - (int)blockIdx.x) / G + 1 : 0;
  const int npass = A.compute_grad ? 3 : 2;
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
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCWarps) {
    // ================================================================ producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last_full();  // passes A, B: read again soon
      const uint64_t drop = l2_policy_evict_first();      // pass C: last use
      const Tin* zt = reinterpret_cast<const Tin*>(A.zt);
      const Tin* zd = reinterpret_cast<const Tin*>(A.zd);
      long long q = 0;  // chunk sequence number over all tasks and passes
      for (int k = 0; k < ntask; ++k) {
        const int n = (int)blockIdx.x + k * G;
        bool ok;
        const Tin* rt = zt + (long long)target_row(n, ok) * V;
        const Tin* rd = zd + (long long)n * V;
        for (int pass = 0; pass < npass; ++pass) {
          for (int c = 0; c < nch; ++c, ++q) {
            const int st = (int)(q % kStages);
            const long long use = q / kStages;
            if (use > 0 && !mbar_wait(&sh.empty[st], (unsigned)((use - 1) & 1))) {
              atomicExch(&A.ctl[2], 1u);
              return;  // the consumers' waits run out in turn
            }
            const int e0 = c * CE;
            const unsigned bytes = (unsigned)(min(CE, V - e0) * (int)sizeof(Tin));
            uint8_t* dst = ring + (size_t)st * 2 * kChunkBytes;
            mbar_arrive_expect_tx(&sh.full[st], 2u * bytes);
            bulk_g2s_hint(dst, rt + e0, bytes, &sh.full[st], pass < 2 ? keep : drop);
            bulk_g2s_hint(dst + kChunkBytes, rd + e0, bytes, &sh.full[st], pass < 2 ? keep : drop);
          }
        }
      }
    }
    return;
  }

  // ================================================================== consumers
  long long q = 0;
  bool dead = false;  // a wait ran out: skip the remaining waits
  // Wait for chunk q, return its two row vectors of this thread (valid when
  // the element index is below V).
  // Vector v of this thread in chunk c: elements c*CE + (v*kConsumers + tid)*VN.
  auto wait_chunk = [&]() {
    const int st = (int)(q % kStages);
    if (!dead && !mbar_wait(&sh.full[st], (unsigned)((q / kStages) & 1))) {
      dead = true;
      atomicExch(&A.ctl[2], 1u);
    }
  };
  auto take = [&](int c, int v, uint4& ut, uint4& ud) -> bool {
    const int st = (int)(q % kStages);
    const int vec = v * kConsumers + tid;
    const bool in = c * CE + vec * VN < V;
    if (in) {
      const uint8_t* src = ring + (size_t)st * 2 * kChunkBytes + vec * 16;
      ut = *reinterpret_cast<const uint4*>(src);
      ud = *reinterpret_cast<const uint4*>(src + kChunkBytes);
    }
    return in;
  };
  // Release chunk q (one arrive per consumer warp) and advance.
  auto give = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[(int)(q % kStages)]);
    ++q;
  };

  for (int k = 0; k < ntask; ++k) {
    const int n = (int)blockIdx.x + k * G;
    const int b = n / W, i = n % W;

    // ---------------------------------------------- pass A: row statistics
    float mt = -INFINITY, md = -INFINITY, sum_t, sum_d;
    {
      float2 at0 = make_float2(0.f, 0.f), at1 = at0, ad0 = at0, ad1 = at0;
      auto raise = [](float gm, float& m, float2& s0, float2& s1) {
        if (gm > m) {
          const float f = (m == -INFINITY) ? 0.f : ex2_fast(m - gm);
          s0 = (m == -INFINITY) ? make_float2(0.f, 0.f) : __fmul2_rn(s0, make_float2(f, f));
          s1 = (m == -INFINITY) ? make_float2(0.f, 0.f) : __fmul2_rn(s1, make_float2(f, f));
          m = gm;
        }
      };
      for (int c = 0; c < nch; ++c) {
        wait_chunk();
#pragma unroll
        for (int v = 0; v < kVPT; ++v) {
        uint4 ut, ud;
        if (take(c, v, ut, ud)) {
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
        }
        give();
      }
      sum_t = (at0.x + at0.y) + (at1.x + at1.y);
      sum_d = (ad0.x + ad0.y) + (ad1.x + ad1.y);
      // -inf maximum: this thread saw no finite entry of that row, no mass
      if (mt == -INFINITY) sum_t = 0.f;
      if (md == -INFINITY) sum_d = 0.f;
    }
    warp_lse2(mt, sum_t);
    warp_lse2(md, sum_d);
    if (lane == 0) sh.red[warp] = make_float4(mt, sum_t, md, sum_d);
    named_sync(1, kConsumers);
    if (tid == 0) {
      float4 v = sh.red[0];
      for (int w = 1; w < kCWarps; ++w) {
        lse2_combine(v.x, v.y, sh.red[w].x, sh.red[w].y);
        lse2_combine(v.z, v.w, sh.red[w].z, sh.red[w].w);
      }
      float2 L = make_float2(v.x + log2f(v.y), v.z + log2f(v.w));
      bool row_ok;
      target_row(n, row_ok);
      if (!row_ok) {
        set_status(SPECOPD_DEV_ROW_RANGE);
        L = make_float2(qnan, qnan);
      } else if (v.x == -INFINITY || v.z == -INFINITY) {
        set_status(SPECOPD_DEV_ALL_NEG_INF);
        L = make_float2(qnan, qnan);
      }
      if (dead) L = make_float2(qnan, qnan);
      sh.lse = L;
    }
    named_sync(1, kConsumers);
    const float lse2_t = sh.lse.x, lse2_d = sh.lse.y;
    const float2 nLt = make_float2(-lse2_t, -lse2_t), nLd = make_float2(-lse2_d, -lse2_d);

    // ---------------------------------------------- pass B: a_n and s_n
    {
      float2 pa2 = make_float2(0.f, 0.f), ps2 = pa2;
      for (int c = 0; c < nch; ++c) {
        wait_chunk();
#pragma unroll
        for (int v = 0; v < kVPT; ++v) {
        uint4 ut, ud;
        if (take(c, v, ut, ud)) {
          float2 ft[VP], fd[VP];
          Vec<Tin>::pairs(ut, ft);
          Vec<Tin>::pairs(ud, fd);
#pragma unroll
          for (int p = 0; p < VP; ++p) {
            const float2 lt = __ffma2_rn(ft[p], L2E, nLt);
            const float2 ld = __ffma2_rn(fd[p], L2E, nLd);
            const float2 e = make_float2(ex2_fast(fminf(lt.x, ld.x)), ex2_fast(fminf(lt.y, ld.y)));
            pa2 = __fadd2_rn(pa2, e);
            ps2 = __fadd2_rn(ps2, make_float2(ld.x < lt.x ? e.x : 0.f, ld.y < lt.y ? e.y : 0.f));
          }
        }
        }
        give();
      }
      const float pa = warp_sum(pa2.x + pa2.y);
      const float ps = warp_sum(ps2.x + ps2.y);
      if (lane == 0) sh.red[warp] = make_float4(pa, ps, 0.f, 0.f);
    }
    named_sync(1, kConsumers);
    const bool owner = (i == 0);  // writes the branch's overlaps and prefix products
    const bool need_branch = A.compute_grad || owner;
    if (tid == 0) {
      float2 v = make_float2(0.f, 0.f);
      for (int w = 0; w < kCWarps; ++w) {
        v.x += sh.red[w].x;
        v.y += sh.red[w].y;
      }
      A.part[n] = v;
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&A.br_cnt[b]) : "memory");
      int last = 0;
      if (need_branch) {
        // The W positions of the branch run in this round on W CTAs.
        bool ok = !dead && __ldcg(&A.ctl[2]) == 0u;
        if (ok) ok = wait_flag_geq(&A.br_cnt[b], (unsigned)W);
        if (!ok) atomicExch(&A.ctl[2], 1u);
        for (int j = 0; j < W; ++j) {
          const float2 u = __ldcg(&A.part[(size_t)b * W + j]);
          sh.sa[j] = ok ? u.x : qnan;
          if (j == i) sh.s_own = ok ? u.y : qnan;
        }
        // g_n = -(1/norm) P_{i-1} S_i, with no division by any overlap
        float P = 1.f;
        for (int j = 0; j < i; ++j) P *= sh.sa[j];
        float S = 1.f;
        for (int j = W - 1; j > i; --j) S = fmaf(sh.sa[j], S, 1.f);
        sh.g = -A.inv_norm * P * S;
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
      sh.flag = last;
    }
    named_sync(1, kConsumers);
    if (sh.flag) {
      // Last branch: loss = 1 - sum_b bsum[b] / norm, fixed summation order.
      double acc = 0.0;
      for (int j = tid; j < A.nbranch; j += kConsumers) acc += __ldcg(&A.bsum[j]);
      acc = warp_sum_d(acc);
      if (lane == 0) sh.dred[warp] = acc;
      named_sync(1, kConsumers);
      if (tid == 0) {
        double tot = 0.0;
        for (int w = 0; w < kCWarps; ++w) tot += sh.dred[w];
        A.loss[0] = (float)(1.0 - tot / A.norm);
        if (A.numer) A.numer[0] = tot;
      }
    }

    // ---------------------------------------------- pass C: gradient row
    if (A.compute_grad) {
      const float g = sh.g, s_val = sh.s_own;
      const float c1 = g * (1.f - s_val), c0 = -g * s_val;  // coefficient for [q<p] = 1 / 0
      Tg* gout = reinterpret_cast<Tg*>(A.grad) + (long long)n * V;
      for (int c = 0; c < nch; ++c) {
        wait_chunk();
#pragma unroll
        for (int v = 0; v < kVPT; ++v) {
        uint4 ut, ud;
        if (take(c, v, ut, ud)) {
          float2 ft[VP], fd[VP], o[VP];
          Vec<Tin>::pairs(ut, ft);
          Vec<Tin>::pairs(ud, fd);
#pragma unroll
          for (int p = 0; p < VP; ++p) {
            const float2 lt = __ffma2_rn(ft[p], L2E, nLt);
            const float2 ld = __ffma2_rn(fd[p], L2E, nLd);
            const float2 coef = make_float2(ld.x < lt.x ? c1 : c0, ld.y < lt.y ? c1 : c0);
            o[p] = __fmul2_rn(ex2_pair(ld), coef);
          }
          Tg* dst = gout + c * CE + (v * kConsumers + tid) * VN;
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
      }
    }
    // sh.lse, sh.g, sh.s_own and sh.red are rewritten by the next task only
    // after its pass A, which every consumer reaches past this point.
    named_sync(1, kConsumers);
  }
}
