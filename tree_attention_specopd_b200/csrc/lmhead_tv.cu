// E2E-TV with the two LM heads fused in front: the N x V logits are formed
// tile by tile on the tensor cores and never written to HBM.
//
// Sources: SpecOPD review (jaehun.me) §3.2(a), the score-row reading rule
// (the target logits of position n are read from the output of its
// predictor row, target_row[n]); review §3.3 and §1.1 (E2E-TV on those
// logits, the same quantities as e2e_tv.cu); paper summary
// (rustineverything.app) §2.3 (the loss).  The LM head is the linear map
// z = W h, W [V, d] (row v scores token v); no bias, norm or temperature.
//
//   z_t[n] = W_t h_t[target_row[n]],   z_d[n] = W_d h_d[n]      (fp32 accumulation)
//   then a_n, prefix products, loss and dz_d exactly as specopd_e2e_tv.
//
// B200 design.  Two or three passes of one tcgen05 GEMM kernel over tiles of
// 128 positions x 128 vocabulary entries, each tile holding both models'
// logits in TMEM (fp32, 2 x 128 columns, double-buffered: 512 columns, one
// CTA per SM; pass 2 the draft's only), with a per-pass epilogue:
//   pass 0: per row, running (max, sum of 2^(x - max)) of both rows over the
//           CTA's vocabulary chunk -> one record per (chunk, row);
//   (combine: the chunks' records in chunk order -> lse of both rows)
//   pass 1: per row, sum_v 2^min(lt, ld) and the [ld < lt] part of it over
//           the chunk -> one (a, s) record per (chunk, row);
//   (branch: a_n, s_n in chunk order, prefix products, g_n, the loss)
//   then the gradient dz_d[n, v] = g_n q_v ([q_v < p_v] - s_n), whose two
//   values per row, g (1 - s) and -g s, are known only after the branch:
//   - fp32 gradient: pass 1 (as MODE 3) writes q_v into the gradient row with
//     [q_v < p_v] in its sign, and an elementwise kernel multiplies in place
//     (four GEMMs per call);
//   - bf16 gradient: pass 1 stores [q_v < p_v] as one bit (N V / 8 bytes) and
//     pass 2 forms the draft tiles again and writes the gradient as its
//     epilogue (a rounded q would be rounded twice).
//   Either way s_n and the gradient's mask are the same decisions.
//  * Warp 0 drives TMA: per stage a 64-column slice (one 128-byte swizzled
//    row) of the 128 target rows, of 128 rows of the target head, of the
//    128 draft rows and of the draft head (4 x 16 KB, 3 stages; pass 2: two
//    consecutive slices of the draft's rows and head).  Rows past N or V and
//    columns past d arrive as zeros.
//  * Warp 1 issues tcgen05.mma (M = N = 128, K = 16, both operands K-major
//    from shared memory) from one thread, commits each stage back to the
//    producer and each finished tile to the epilogue.
//  * Warps 2-5 own one TMEM lane (= one position) each and read the tile 32
//    columns at a time.
//  * Grid: vocabulary chunks x row tiles, row tiles innermost so the CTAs
//    that share a head tile run together and read it from L2.
//  * Every wait is bounded (%globaltimer); expiry sets the status word and
//    makes the affected records NaN.
//
// Included by api.cu after tree_attn_sm100.cu: the tcgen05/TMA helpers of
// namespace sm100 are reused here.

namespace specopd {
namespace lmtv {

using sm100::idesc_bf16;
using sm100::mma_ss;
using sm100::sdesc;
using sm100::tc_commit;
using sm100::tc_fence_after;
using sm100::tc_fence_before;
using sm100::tmem_ld32;
using sm100::tmem_wait_ld;

constexpr int kThreads = 192;           // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int kBM = 128;                // positions per tile (TMEM lanes)
constexpr int kBN = 128;                // vocabulary entries per tile (MMA N)
constexpr int kBK = 64;                 // hidden columns per stage (one 128-byte swizzled row)
constexpr int kTile = kBM * kBK * 2;    // 16 KB: one operand slice of one stage
constexpr int kRing = 12 * kTile;       // 192 KB of stages: 3 of both models, 6 of the draft only
constexpr int kMaxStages = 6;
constexpr int kTmemCols = 512;          // buffer b: target [256b, 256b+128), draft [256b+128, 256b+256)
constexpr int kMaxW = 256;
constexpr float kLog2e = 1.4426950408889634f;

struct Hdr {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t acc_full[2];  // by tile parity: both logit tiles are in TMEM
  uint64_t acc_free[2];  // by tile parity: the epilogue warps have read them
  uint64_t mma_done;     // one phase: every MMA the CTA issued has completed
  uint32_t tmem_base;
  int abort;
};

struct Params {
  int N, V, d, nvt, nchunk, mtiles;
  const float2* lse;   // [N] (target, draft) log-sum-exp in log2 units (passes 1, 2)
  const float2* coef;  // [N] (g (1 - s), -g s): the gradient's two values per q (pass 2)
  float4* stats;       // [nchunk][N] (max_t, sum_t, max_d, sum_d), log2 units (pass 0)
  float2* partB;       // [nchunk][N] (a, s) (pass 1)
  uint4* bits;         // [nvt][N] [q < p] of the tile's 128 entries (pass 1 writes, pass 2 reads)
  void* grad;          // [N][V] (pass 2)
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, unsigned parity, Hdr* hdr) {
  if (*reinterpret_cast<volatile int*>(&hdr->abort)) return false;
  if (mbar_wait(bar, parity)) return true;
  hdr->abort = 1;
  return false;
}
// Warp-uniform result (the tcgen05.ld that follow are warp-collective).
__device__ __forceinline__ bool warp_wait_or_abort(uint64_t* bar, unsigned parity, Hdr* hdr) {
  const bool live = !*reinterpret_cast<volatile int*>(&hdr->abort);
  const bool ok = __all_sync(0xffffffffu, live && mbar_wait(bar, parity));
  if (!ok) hdr->abort = 1;
  return ok;
}

// Vocabulary tiles [vt0, vt1) of chunk c (balanced split of nvt tiles).
__device__ __forceinline__ void chunk_tiles(const Params& P, int c, int& vt0, int& vt1) {
  vt0 = (int)((long long)c * P.nvt / P.nchunk);
  vt1 = (int)((long long)(c + 1) * P.nvt / P.nchunk);
}

// One pass over the CTA's (row tile, vocabulary chunk): MODE 0 statistics,
// 1 overlap partials and the [q < p] bits, 2 gradient tiles from the bits
// (Tg = the gradient's element type), 3 overlap partials and, for an fp32
// gradient, q_v written in place with [q_v < p_v] in its sign (negative:
// false), which lmtv_scale_kernel turns into the gradient.
template <int MODE, typename Tg>
__global__ void __launch_bounds__(kThreads, 1)
lmtv_kernel(const __grid_constant__ CUtensorMap tm_ht, const __grid_constant__ CUtensorMap tm_wt,
            const __grid_constant__ CUtensorMap tm_hd, const __grid_constant__ CUtensorMap tm_wd,
            const Params P) {
  // 128-byte swizzled slices need 1024-byte aligned shared memory (the
  // dynamic region starts at the CTA's shared-memory base).
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // A stage is 64 KB, 8 MMAs: passes 0 and 1 stage one 64-column slice of
  // both models (rows and head of each), pass 2 two consecutive slices of
  // the draft only (its [q < p] decisions come from pass 1).  Stages of 4
  // MMAs (one model per stage, 32 KB) were measured slower: the cost per
  // stage, not the copy latency, sets the rate.
  constexpr int NM = MODE == 2 ? 1 : 2;  // models formed
  constexpr int KPS = 3 - NM;            // 64-column slices per stage
  constexpr int kStageBytes = 4 * kTile;
  constexpr int kStages = kRing / kStageBytes;
  Hdr* hdr = reinterpret_cast<Hdr*>(smem_raw + kRing);
  if (smem_u32(smem_raw) & 1023u) {  // uniform over the CTA; nothing touched yet
    if (threadIdx.x == 0) set_status(SPECOPD_DEV_LAYOUT);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = (int)blockIdx.x % P.mtiles;
  const int c = (int)blockIdx.x / P.mtiles;
  int vt0, vt1;
  chunk_tiles(P, c, vt0, vt1);
  const int nkb = (P.d + kBK - 1) / kBK;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&hdr->full[s], 1);
      mbar_init(&hdr->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&hdr->acc_full[b], 1);
      mbar_init(&hdr->acc_free[b], 4);
    }
    mbar_init(&hdr->mma_done, 1);
    hdr->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&hdr->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = hdr->tmem_base;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      unsigned q = 0;  // stage sequence number
      bool live = true;
      for (int vt = vt0; vt < vt1 && live; ++vt) {
        for (int kb = 0; kb < nkb; kb += KPS) {
          const int st = (int)(q % kStages);
          const unsigned use = q / kStages;
          if (use > 0u && !wait_or_abort(&hdr->empty[st], (use - 1u) & 1u, hdr)) {
            live = false;
            break;
          }
          uint8_t* base = smem_raw + st * kStageBytes;
          if constexpr (NM == 2) {
            mbar_arrive_expect_tx(&hdr->full[st], (unsigned)kStageBytes);
            tma_load_2d(base, &tm_ht, kb * kBK, m * kBM, &hdr->full[st]);
            tma_load_2d(base + kTile, &tm_wt, kb * kBK, vt * kBN, &hdr->full[st]);
            tma_load_2d(base + 2 * kTile, &tm_hd, kb * kBK, m * kBM, &hdr->full[st]);
            tma_load_2d(base + 3 * kTile, &tm_wd, kb * kBK, vt * kBN, &hdr->full[st]);
          } else {
            const int nsub = min(2, nkb - kb);  // the last stage may hold one slice
            mbar_arrive_expect_tx(&hdr->full[st], (unsigned)(nsub * 2 * kTile));
            for (int sub = 0; sub < nsub; ++sub) {
              tma_load_2d(base + sub * 2 * kTile, &tm_hd, (kb + sub) * kBK, m * kBM, &hdr->full[st]);
              tma_load_2d(base + sub * 2 * kTile + kTile, &tm_wd, (kb + sub) * kBK, vt * kBN,
                          &hdr->full[st]);
            }
          }
          ++q;
        }
      }
      // No copy may land after the CTA exits: wait (bounded) for the last
      // phase issued into every stage (already complete in a normal run).
      for (unsigned j = (q > (unsigned)kStages ? q - (unsigned)kStages : 0u); j < q; ++j)
        mbar_wait(&hdr->full[j % kStages], (j / kStages) & 1u);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(kBN, false);  // M = N = 128, B K-major
      unsigned q = 0;
      bool ok = true;
      for (int i = 0, vt = vt0; vt < vt1 && ok; ++vt, ++i) {
        const int b = i & 1;
        // buffer b last held tile i - 2: the epilogue warps have read it
        if (i >= 2 && !wait_or_abort(&hdr->acc_free[b], ((i >> 1) - 1) & 1, hdr)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tT = tmem + b * 2 * kBN, tD = tT + kBN;
        for (int kb = 0; kb < nkb; kb += KPS) {
          const int st = (int)(q % kStages);
          if (!wait_or_abort(&hdr->full[st], (q / kStages) & 1u, hdr)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem_raw + st * kStageBytes);
          // K-major slices: 16 columns = 32 B inside each 128-byte swizzled row
          if constexpr (NM == 2) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
              mma_ss(tT, sdesc(base + kk * 32, 16, 1024), sdesc(base + kTile + kk * 32, 16, 1024),
                     kId, acc);
              mma_ss(tD, sdesc(base + 2 * kTile + kk * 32, 16, 1024),
                     sdesc(base + 3 * kTile + kk * 32, 16, 1024), kId, acc);
            }
          } else {
            const int nsub = min(2, nkb - kb);
            for (int sub = 0; sub < nsub; ++sub) {
              const uint32_t bs = base + sub * 2 * kTile;
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk) {
                const uint32_t acc = (kb + sub > 0 || kk > 0) ? 1u : 0u;
                mma_ss(tD, sdesc(bs + kk * 32, 16, 1024), sdesc(bs + kTile + kk * 32, 16, 1024),
                       kId, acc);
              }
            }
          }
          tc_commit(&hdr->empty[st]);
          ++q;
        }
        if (ok) tc_commit(&hdr->acc_full[b]);
      }
      // tracks every MMA issued above, abort or not
      tc_commit(&hdr->mma_done);
    }
  } else {
    // ================================================================ epilogue
    const int q4 = warp & 3;  // TMEM lane quadrant of this warp
    const int rl = q4 * 32 + lane;
    const int n = m * kBM + rl;
    const bool row = n < P.N;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float mt = -INFINITY, sT = 0.f, md = -INFINITY, sD = 0.f;  // pass 0
    float pa = 0.f, ps = 0.f;                                   // pass 1
    float Lt = 0.f, Ld = 0.f, c1 = 0.f, c0 = 0.f;               // passes 1, 2
    if (MODE >= 1 && row) {
      const float2 L = P.lse[n];
      Lt = L.x;
      Ld = L.y;
    }
    if (MODE == 2 && row) {
      const float2 cf = P.coef[n];
      c1 = cf.x;
      c0 = cf.y;
    }
    bool dead = false;
    for (int i = 0, vt = vt0; vt < vt1; ++vt, ++i) {
      const int b = i & 1;
      dead = !warp_wait_or_abort(&hdr->acc_full[b], (i >> 1) & 1, hdr);
      if (dead) break;
      tc_fence_after();
      __syncwarp();
      const uint32_t tT = tmem + lane_off + b * 2 * kBN, tD = tT + kBN;
      // pass 1 writes, pass 2 reads the tile's [q < p] bits: word ch holds
      // entries 32 ch .. 32 ch + 31 of the row
      uint4 bw = make_uint4(0u, 0u, 0u, 0u);
      if (MODE == 2 && row) bw = P.bits[(size_t)vt * P.N + n];
#pragma unroll 1
      for (int ch = 0; ch < kBN / 32; ++ch) {
        uint32_t xt[32], xd[32];
        if constexpr (NM == 2) tmem_ld32(tT + ch * 32, xt);
        tmem_ld32(tD + ch * 32, xd);
        tmem_wait_ld();
        if (ch == kBN / 32 - 1) {
          // the whole tile has been read: the MMA may reuse this buffer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&hdr->acc_free[b]);
        }
        const int v0 = vt * kBN + ch * 32;
        const int nv = min(32, P.V - v0);  // columns of this chunk inside the vocabulary
        if (nv <= 0) continue;
        if constexpr (MODE == 0) {
          float cmt = -INFINITY, cmd = -INFINITY;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e < nv) {
              cmt = fmaxf(cmt, __uint_as_float(xt[e]));
              cmd = fmaxf(cmd, __uint_as_float(xd[e]));
            }
          cmt *= kLog2e;
          cmd *= kLog2e;
          if (cmt > mt) {
            sT = (mt == -INFINITY) ? 0.f : sT * ex2_fast(mt - cmt);
            mt = cmt;
          }
          if (cmd > md) {
            sD = (md == -INFINITY) ? 0.f : sD * ex2_fast(md - cmd);
            md = cmd;
          }
          float at = 0.f, ad = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e < nv) {
              at += ex2_fast(fmaf(__uint_as_float(xt[e]), kLog2e, -mt));
              ad += ex2_fast(fmaf(__uint_as_float(xd[e]), kLog2e, -md));
            }
          sT += at;
          sD += ad;
        } else if constexpr (MODE == 1 || MODE == 3) {
          uint32_t mask = 0u;
          float o[32];  // pass 3: q_v, negated where [q_v < p_v] is false
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            o[e] = 0.f;
            if (e < nv) {
              const float lt = fmaf(__uint_as_float(xt[e]), kLog2e, -Lt);
              const float ld = fmaf(__uint_as_float(xd[e]), kLog2e, -Ld);
              const float w = ex2_fast(fminf(lt, ld));
              pa += w;
              ps += (ld < lt) ? w : 0.f;
              mask |= (ld < lt ? 1u : 0u) << e;
              if constexpr (MODE == 3) o[e] = (ld < lt) ? w : -ex2_fast(ld);
            }
          }
          if constexpr (MODE == 1) {
            if (ch == 0) bw.x = mask; else if (ch == 1) bw.y = mask; else if (ch == 2) bw.z = mask; else bw.w = mask;
          } else if (row) {
            float* dst = reinterpret_cast<float*>(P.grad) + (long long)n * P.V + v0;
            if (nv == 32) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e < nv) dst[e] = o[e];
            }
          }
        } else {
          const uint32_t mask = ch == 0 ? bw.x : ch == 1 ? bw.y : ch == 2 ? bw.z : bw.w;
          float o[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float ld = fmaf(__uint_as_float(xd[e]), kLog2e, -Ld);
            o[e] = ex2_fast(ld) * (((mask >> e) & 1u) ? c1 : c0);
          }
          if (row) {
            Tg* dst = reinterpret_cast<Tg*>(P.grad) + (long long)n * P.V + v0;
            if (nv == 32) {
              if constexpr (sizeof(Tg) == 4) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                  __stcs(reinterpret_cast<float4*>(dst + e), make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]));
              } else {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                  uint4 u;
                  u.x = pack_bf16x2(o[e], o[e + 1]);
                  u.y = pack_bf16x2(o[e + 2], o[e + 3]);
                  u.z = pack_bf16x2(o[e + 4], o[e + 5]);
                  u.w = pack_bf16x2(o[e + 6], o[e + 7]);
                  __stcs(reinterpret_cast<uint4*>(dst + e), u);
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e < nv) dst[e] = Elt<Tg>::from_f(o[e]);
            }
          }
        }
      }
      if (MODE == 1 && row) P.bits[(size_t)vt * P.N + n] = bw;
    }
    if (row) {
      const float qnan = __int_as_float(0x7fc00000);
      if constexpr (MODE == 0)
        P.stats[(size_t)c * P.N + n] = dead ? make_float4(qnan, qnan, qnan, qnan) : make_float4(mt, sT, md, sD);
      if constexpr (MODE == 1 || MODE == 3)
        P.partB[(size_t)c * P.N + n] = dead ? make_float2(qnan, qnan) : make_float2(pa, ps);
    }
  }

  // ---- teardown: every MMA has completed before TMEM is released
  __syncthreads();
  if (warp == 1) {
    mbar_wait(&hdr->mma_done, 0);
    tc_fence_after();
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// Target hidden rows in position order: out[n] = h_t[target_row[n]] (zeros,
// and SPECOPD_DEV_ROW_RANGE, for a row outside [0, rows_target)).  One
// 16-byte vector per thread; d8 = d / 8 vectors per row.
__global__ void lmtv_gather_kernel(const uint4* h, const int32_t* trow, int rows_target, int N,
                                   int d8, uint4* out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)N * d8) return;
  const int n = (int)(i / d8), k = (int)(i % d8);
  const int r = trow ? trow[n] : n;
  const bool ok = r >= 0 && r < rows_target;
  if (!ok && k == 0) set_status(SPECOPD_DEV_ROW_RANGE);
  out[i] = ok ? h[(long long)r * d8 + k] : make_uint4(0u, 0u, 0u, 0u);
}

// lse of both rows from the chunks' records: one warp per row, lane l
// combining chunks l, l + 32, ... in order, then a fixed butterfly over the
// lanes (the same combination order on every call).  A row whose target row
// is out of range, or whose records carry a NaN (a wait ran out), gets NaN.
__global__ void lmtv_stats_kernel(const float4* stats, int nchunk, int N, const int32_t* trow,
                                  int rows_target, float2* lse) {
  const int n = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;  // uniform over the warp
  float mt = -INFINITY, st = 0.f, md = -INFINITY, sd = 0.f;
  bool bad = false;
  for (int c = lane; c < nchunk; c += 32) {
    const float4 r = stats[(size_t)c * N + n];
    bad |= isnan(r.x) || isnan(r.y) || isnan(r.z) || isnan(r.w);
    lse2_combine(mt, st, r.x, r.y);
    lse2_combine(md, sd, r.z, r.w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lse2_combine(mt, st, __shfl_xor_sync(0xffffffffu, mt, o), __shfl_xor_sync(0xffffffffu, st, o));
    lse2_combine(md, sd, __shfl_xor_sync(0xffffffffu, md, o), __shfl_xor_sync(0xffffffffu, sd, o));
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane != 0) return;
  const int row = trow ? trow[n] : n;
  const float qnan = __int_as_float(0x7fc00000);
  if (row < 0 || row >= rows_target || bad || mt == -INFINITY || md == -INFINITY) {
    lse[n] = make_float2(qnan, qnan);
  } else {
    lse[n] = make_float2(mt + log2f(st), md + log2f(sd));
  }
}

// Per branch: a_n and s_n from the chunks' (a, s) records (one warp per
// branch: lane l sums chunks l, l + 32, ... in order, then a fixed butterfly
// over the lanes), then on lane 0 the prefix products, g_n and the
// gradient's two values per q, and the branch's sum of prefix products.
__global__ void lmtv_branch_kernel(const float2* partB, int nchunk, int N, int nbranch, int W,
                                   const float2* lse, float inv_norm, float* a_out, float* prefix,
                                   float2* coef, double* bsum) {
  const int b = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= nbranch) return;  // uniform over the warp
  const float qnan = __int_as_float(0x7fc00000);
  float sa[kMaxW], ss[kMaxW];
  for (int i = 0; i < W; ++i) {
    const int n = b * W + i;
    float a = 0.f, s = 0.f;
    for (int c = lane; c < nchunk; c += 32) {
      const float2 r = partB[(size_t)c * N + n];
      a += r.x;
      s += r.y;
    }
    a = warp_sum(a);
    s = warp_sum(s);
    const float2 L = lse[n];
    if (isnan(L.x) || isnan(L.y)) a = s = qnan;
    sa[i] = a;
    ss[i] = s;
  }
  if (lane != 0) return;
  float P = 1.f;
  double sumP = 0.0;
  for (int i = 0; i < W; ++i) {
    const int n = b * W + i;
    // g = -(1/norm) P_{i-1} S_i, with no division by any overlap
    float S = 1.f;
    for (int j = W - 1; j > i; --j) S = fmaf(sa[j], S, 1.f);
    const float g = -inv_norm * P * S;
    coef[n] = make_float2(g * (1.f - ss[i]), -g * ss[i]);
    P *= sa[i];
    a_out[n] = sa[i];
    prefix[n] = P;
    sumP += (double)P;
  }
  bsum[b] = sumP;
}

// fp32 gradient in place from pass 3's signed q_v: dz = |v| * (v >= 0 ? c1 : c0)
// with (c1, c0) = (g (1 - s), -g s) of its row; the same product pass 2 forms.
// Columns in float4 (V % 4 == 0), rows strided over gridDim.y.
__global__ void lmtv_scale_kernel(float* grad, const float2* coef, int N, int V) {
  const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
  if (c4 >= V / 4) return;
  for (int n = blockIdx.y; n < N; n += gridDim.y) {
    float4* p = reinterpret_cast<float4*>(grad + (size_t)n * V) + c4;
    const float2 cf = coef[n];
    float4 v = __ldcs(p);
    v.x = fabsf(v.x) * (signbit(v.x) ? cf.y : cf.x);
    v.y = fabsf(v.y) * (signbit(v.y) ? cf.y : cf.x);
    v.z = fabsf(v.z) * (signbit(v.z) ? cf.y : cf.x);
    v.w = fabsf(v.w) * (signbit(v.w) ? cf.y : cf.x);
    __stcs(p, v);
  }
}

// loss = 1 - sum_b bsum[b] / norm, in a fixed summation order (one block).
__global__ void lmtv_loss_kernel(const double* bsum, int nbranch, double norm, float* loss,
                                 double* numer) {
  __shared__ double red[256];
  double acc = 0.0;
  for (int j = threadIdx.x; j < nbranch; j += blockDim.x) acc += bsum[j];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    loss[0] = (float)(1.0 - red[0] / norm);
    if (numer) numer[0] = red[0];
  }
}

}  // namespace lmtv

// ------------------------------------------------------------------ host
namespace lmtv {
namespace {

struct Plan {
  int mtiles, nvt, nchunk;
};

// Row tiles x vocabulary chunks (one CTA per SM): the fewest chunks whose
// CTAs fill at least 95 % of the SM slots of their waves (each chunk adds a
// record per row and re-reads the hidden rows), else the best filling found;
// never more chunks than vocabulary tiles.
Plan make_plan(int N, int V, int nsm) {
  Plan pl;
  pl.mtiles = (N + kBM - 1) / kBM;
  pl.nvt = (V + kBN - 1) / kBN;
  nsm = std::max(1, nsm);
  const int cap = std::min(pl.nvt, 8 * nsm);
  int best = 1;
  double best_fill = 0.0;
  for (int nc = 1; nc <= cap; ++nc) {
    const long long ctas = (long long)pl.mtiles * nc;
    const double fill = (double)ctas / ((double)((ctas + nsm - 1) / nsm) * nsm);
    if (fill > best_fill + 1e-9) {
      best_fill = fill;
      best = nc;
    }
    if (fill >= 0.95) break;
  }
  pl.nchunk = best;
  return pl;
}

struct Layout {
  size_t ht, stats, lse, partB, bits, coef, bsum, total;
};

Layout layout(const LmtvProblem& p, const Plan& pl) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  Layout L;
  size_t off = 0;
  L.ht = off;    off = up(off + (size_t)p.N * p.d * 2);
  L.stats = off; off = up(off + sizeof(float4) * (size_t)pl.nchunk * p.N);
  L.lse = off;   off = up(off + sizeof(float2) * (size_t)p.N);
  L.partB = off; off = up(off + sizeof(float2) * (size_t)pl.nchunk * p.N);
  L.bits = off;  off = up(off + sizeof(uint4) * (size_t)pl.nvt * p.N);
  L.coef = off;  off = up(off + sizeof(float2) * (size_t)p.N);
  L.bsum = off;  off = up(off + sizeof(double) * (size_t)p.nbranch);
  L.total = off;
  return L;
}

// 2-D view [rows, cols] of a row-major bf16 matrix, box 64 columns x 128
// rows, 128-byte swizzle; reads past either edge return zeros.
bool make_map2d(CUtensorMap* m, const void* ptr, int cols, long long rows) {
  auto enc = sm100::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kSmem = (size_t)kRing + sizeof(Hdr);

template <int MODE, typename Tg>
cudaError_t launch_pass(const CUtensorMap* maps, const Params& P, int grid, cudaStream_t st) {
  auto fn = lmtv_kernel<MODE, Tg>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  fn<<<grid, kThreads, kSmem, st>>>(maps[0], maps[1], maps[2], maps[3], P);
  return cudaGetLastError();
}

}  // namespace
}  // namespace lmtv

size_t lmtv_workspace(const LmtvProblem& p) {
  const lmtv::Plan pl = lmtv::make_plan(p.N, p.V, sm100::sm_count());
  return lmtv::layout(p, pl).total;
}

cudaError_t launch_lmtv(const LmtvProblem& p, const void* h_target, const int32_t* target_row,
                        const void* w_target, const void* h_draft, const void* w_draft, float* a,
                        float* prefix, float* loss, double* numer, void* grad, void* ws,
                        size_t ws_bytes, cudaStream_t st) {
  using namespace lmtv;
  const Plan pl = make_plan(p.N, p.V, sm100::sm_count());
  const Layout L = layout(p, pl);
  if (ws_bytes < L.total) return cudaErrorInvalidValue;
  // An fp32 gradient is formed in place: pass 3 writes q_v with its [q < p]
  // sign, the scale kernel applies the row's two values once g_n is known.
  // A bf16 gradient needs pass 1's bits and pass 2 (a rounded q would be
  // rounded twice).  The in-place path moves whole float4 of a row.
  const bool inplace = p.compute_grad && grad && p.grad_dtype == SPECOPD_F32;
  if (inplace && (p.V % 4 != 0 || reinterpret_cast<uintptr_t>(grad) % 16 != 0))
    return cudaErrorInvalidValue;
  char* w = reinterpret_cast<char*>(ws);
  void* ht = w + L.ht;
  CUtensorMap maps[4];
  if (!make_map2d(&maps[0], ht, p.d, p.N) || !make_map2d(&maps[1], w_target, p.d, p.V) ||
      !make_map2d(&maps[2], h_draft, p.d, p.N) || !make_map2d(&maps[3], w_draft, p.d, p.V))
    return cudaErrorInvalidValue;
  Params P;
  P.N = p.N; P.V = p.V; P.d = p.d;
  P.nvt = pl.nvt; P.nchunk = pl.nchunk; P.mtiles = pl.mtiles;
  P.lse = reinterpret_cast<const float2*>(w + L.lse);
  P.coef = reinterpret_cast<const float2*>(w + L.coef);
  P.stats = reinterpret_cast<float4*>(w + L.stats);
  P.partB = reinterpret_cast<float2*>(w + L.partB);
  P.bits = reinterpret_cast<uint4*>(w + L.bits);
  P.grad = grad;
  const int grid = pl.mtiles * pl.nchunk;
  const long long nvec = (long long)p.N * (p.d / 8);
  lmtv_gather_kernel<<<(unsigned)((nvec + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(h_target), target_row, p.rows_target, p.N, p.d / 8,
      reinterpret_cast<uint4*>(ht));
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = launch_pass<0, float>(maps, P, grid, st);
  if (e != cudaSuccess) return e;
  lmtv_stats_kernel<<<(unsigned)(((size_t)p.N * 32 + 255) / 256), 256, 0, st>>>(P.stats, pl.nchunk, p.N, target_row,
                                                       p.rows_target, reinterpret_cast<float2*>(w + L.lse));
  e = cudaGetLastError();
  if (e == cudaSuccess) e = inplace ? launch_pass<3, float>(maps, P, grid, st)
                                    : launch_pass<1, float>(maps, P, grid, st);
  if (e != cudaSuccess) return e;
  lmtv_branch_kernel<<<(unsigned)(((size_t)p.nbranch * 32 + 127) / 128), 128, 0, st>>>(
      P.partB, pl.nchunk, p.N, p.nbranch, p.W, P.lse, (float)(1.0 / p.norm_count), a, prefix,
      reinterpret_cast<float2*>(w + L.coef), reinterpret_cast<double*>(w + L.bsum));
  lmtv_loss_kernel<<<1, 256, 0, st>>>(reinterpret_cast<const double*>(w + L.bsum), p.nbranch,
                                      p.norm_count, loss, numer);
  e = cudaGetLastError();
  if (e != cudaSuccess || !p.compute_grad || !grad) return e;
  if (inplace) {
    const dim3 sg((unsigned)((p.V / 4 + 255) / 256), (unsigned)std::min(p.N, 64));
    lmtv_scale_kernel<<<sg, 256, 0, st>>>(reinterpret_cast<float*>(grad), P.coef, p.N, p.V);
    return cudaGetLastError();
  }
  return launch_pass<2, __nv_bfloat16>(maps, P, grid, st);
}

}  // namespace specopd
