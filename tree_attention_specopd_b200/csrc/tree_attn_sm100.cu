// Tree-masked GQA attention of branch rows, bf16, tcgen05 / TMEM / TMA (sm_100a).
//
// SpecOPD review (jaehun.me) §3.2(a): the trunk K/V is computed once and
// cached; the branch queries attach to that cache and each reads only itself
// and its ancestors.  For branch row r = (s, b, i) the visible keys are the
// trunk positions 0..a_b of sequence s and the branch nodes (s, b, 1..i);
// siblings and later trunk tokens are masked.  Review §3.1: the condition of
// position i is (x_{<=a_b}, y_{b,<i}).
//
// Tensor-core formulation (B200):
//  * A work unit is (query tile, kv head, key chunk).  A query tile stacks
//    RT = floor(128 / G) consecutive branch rows of one sequence times the G
//    query heads of one kv head: M = RT*G <= 128 rows of the MMA.  The rows
//    of a tile have nearby anchors (anchors are sorted per sequence), so the
//    trunk keys a tile needs are [0, max anchor]; whole 64-key tiles beyond
//    the tile's largest anchor are never loaded (masked-tile skipping), and
//    each row masks only the ragged end of the last tile.
//  * The branch keys are the tile's own branch nodes (plus the earlier nodes
//    of its first branch): one or two extra 64-key tiles with the per-row
//    mask first(branch) <= node <= row.  No dense T x T mask exists anywhere.
//  * Long trunks are split into key chunks over several CTAs (split-KV);
//    partial (O, max, sum) go to the workspace and the last CTA of a tile to
//    finish merges them in a fixed order (no spin-wait, deterministic).
//  * Two CTAs share an SM (TMEM: 256 of the 512 columns each; shared memory
//    under half), so one CTA's softmax overlaps the other's MMAs, and one
//    CTA's prologue and epilogue overlap the other's main loop.
//  * RoPE of the branch rows is fused: the query tile and the branch key
//    tiles arrive unrotated by TMA, and the softmax warps rotate them in
//    shared memory at each row's semantic position (review §3.2(a)) before
//    the first MMA reads them; the branch key tiles come first in the key
//    order of the leading chunk, so this happens in the prologue.
//  * Per unit, warp 0 drives TMA (Q once, then 64-key K/V tiles in a 2-stage
//    ring, 128-byte swizzle), warp 1 issues tcgen05.mma from one thread:
//    S = Q K^T into TMEM (two S buffers, so QK^T of tile j+1 overlaps the
//    softmax of tile j), and O += P V with P read from TMEM (P overwrites
//    its S buffer as bf16).  Warps 2-5 own one TMEM lane (= one query row)
//    each and a full 64-key row of S per tile: tcgen05.ld, mask, online
//    softmax in the log2 domain with a lazy rescale (O is rescaled in TMEM
//    only when the running max grows by more than 2^8), tcgen05.st of P.
//    The epilogue reads O from TMEM 32 columns at a time.
//  * Every wait is bounded (%globaltimer); expiry sets the status word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace specopd {
namespace sm100 {

constexpr int kThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2..5: softmax + epilogue
constexpr int kBN = 64;        // keys per tile
constexpr int kKStages = 3;    // K ring depth (K tiles run ahead of V tiles)
constexpr int kVStages = 2;    // V ring depth
constexpr int kCtasPerSm = 2;
// Key tiles that chunk 0 of a split (tile, kv head) pair is counted heavier
// when its trunk keys are shared out (it also scores and rotates the branch
// tiles and is usually the one that merges).
constexpr int kChunk0Extra = 4;
constexpr int kTmemCols = 256;              // S0 [0,64), S1 [64,128), O [128, 128+D)
constexpr int kQHalf = 128 * 128;           // Q box: 128 rows x 64 bf16 (swizzled)
constexpr int kKVHalf = kBN * 128;          // K/V box: 64 rows x 64 bf16 (swizzled)
constexpr float kRescaleThreshold = 8.f;    // log2 units

struct Params {
  int S, B, W, Hq, Hkv, G, R;
  int prefill;         // 1: trunk prefill (query rows = trunk rows, causal within a sequence)
  int T_tot;
  int RT;              // branch rows per query tile
  int ntile_per_seq, ntile;
  int nsplit, C;       // key chunks per (tile, kv head), keys per chunk (multiple of kBN)
  int s_lo, n_hi;      // s_lo > 0: the heaviest n_hi tiles split in s_lo + 1 chunks, the
                       // others in s_lo, each pair's chunks sized from its own key span
  float scale_log2;    // softmax scale * log2(e)
  const int32_t* cu_trunk;
  const int32_t* anchors;
  const int32_t* pos_br;  // semantic position of every branch row (sem_pos of the branch nodes)
  double theta[64];       // RoPE frequencies base^(-2k/D), k < D/2 (double: angles reach ~3e4 rad)
  __nv_bfloat16* out;
  float* lse;
  float* part;         // split-KV partials
  unsigned* cnt;       // [ntile * Hkv] arrival counters
};

struct Hdr {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done;   // one phase per P.V tile (used by the lazy rescale)
  uint64_t o_final;  // single phase: every MMA of the unit has completed
  uint64_t rot_done; // single phase: Q and the branch key tiles are rotated (softmax warps)
  uint32_t tmem_base;
  int wmax[4];       // per-warp maxima of the tile's anchors
  int last;
  int abort;
};

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

#define SPECOPD_R32(r)                                                                       \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),        \
      "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
      "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),           \
      "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),           \
      "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define SPECOPD_W32(r)                                                                      \
  "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),    \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),       \
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),     \
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),     \
      "r"(r[29]), "r"(r[30]), "r"(r[31])

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : SPECOPD_R32(r)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      SPECOPD_W32(r)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100
// version bits = 1.  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int N, bool b_mn_major) {
  return (1u << 4)                      // D format f32
         | (1u << 7)                    // A format bf16
         | (1u << 10)                   // B format bf16
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Bounded wait; once any wait of the CTA has run out (hdr->abort), later
// waits return false at once, so an aborting CTA finishes quickly.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, unsigned parity, Hdr* hdr) {
  if (*reinterpret_cast<volatile int*>(&hdr->abort)) return false;
  if (mbar_wait(bar, parity)) return true;
  hdr->abort = 1;
  return false;
}

// Same, for the softmax warps: the result is uniform over the warp, because
// the tcgen05.ld/st that follow are warp-collective (.sync.aligned).
__device__ __forceinline__ bool warp_wait_or_abort(uint64_t* bar, unsigned parity, Hdr* hdr) {
  const bool live = !*reinterpret_cast<volatile int*>(&hdr->abort);
  const bool ok = __all_sync(0xffffffffu, live && mbar_wait(bar, parity));
  if (!ok) hdr->abort = 1;
  return ok;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// RoPE of one row held in shared memory as 128-byte swizzled lines (the
// layout TMA writes with SWIZZLE_128B): pairs (d, d + D/2) for the pair
// chunks c in [c0, c1), chunk c holding d = 8c .. 8c + 7.  For D = 128 the
// two halves of the row are the same line of two 64-column boxes (same
// swizzle), for D = 64 they are chunks c and c + 4 of one line.  The angle
// pos * theta_d is formed and reduced to [-pi, pi] in double precision, as in
// specopd_rope_apply, then evaluated in fp32; results are rounded to bf16.
template <int D>
__device__ __forceinline__ void rope_row_smem(uint8_t* lo_line, uint8_t* hi_line, int line, int pos,
                                              const double* theta, int c0, int c1) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  const int sw = line & 7;
  for (int c = c0; c < c1; ++c) {
    uint4* pa = reinterpret_cast<uint4*>(lo_line + ((c ^ sw) << 4));
    uint4* pb = reinterpret_cast<uint4*>(hi_line + (((D == 128 ? c : c + 4) ^ sw) << 4));
    const uint4 a = *pa, b = *pb;
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    uint32_t ra[4], rb[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      float ya[2], yb[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const double ang = (double)pos * theta[8 * c + 2 * e2 + h];
        const float red = (float)(ang - two_pi * rint(ang * inv_two_pi));
        float sn, cs;
        __sincosf(red, &sn, &cs);
        const float xa = h ? bf16hi(wa[e2]) : bf16lo(wa[e2]);
        const float xb = h ? bf16hi(wb[e2]) : bf16lo(wb[e2]);
        ya[h] = xa * cs - xb * sn;
        yb[h] = xb * cs + xa * sn;
      }
      ra[e2] = pack_bf16x2(ya[0], ya[1]);
      rb[e2] = pack_bf16x2(yb[0], yb[1]);
    }
    *pa = make_uint4(ra[0], ra[1], ra[2], ra[3]);
    *pb = make_uint4(rb[0], rb[1], rb[2], rb[3]);
  }
}

// ------------------------------------------------------------------ kernel
template <int D>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
tree_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ktr,
                 const __grid_constant__ CUtensorMap tm_vtr,
                 const __grid_constant__ CUtensorMap tm_kbr,
                 const __grid_constant__ CUtensorMap tm_vbr, const Params P) {
  constexpr int NH = D / 64;      // 64-column halves of a row
  constexpr int KSTEPS = D / 16;  // MMA K steps of QK^T
  constexpr int DC = D / 32;      // 32-column chunks of O
  // 128-byte swizzled tiles need 1024-byte aligned shared memory; the
  // dynamic region starts at the CTA's shared-memory base (no static shared
  // memory), and two CTAs per SM leave no room for alignment slack.
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  uint8_t* sQ = smem_raw;
  uint8_t* sK = sQ + NH * kQHalf;
  uint8_t* sV = sK + kKStages * NH * kKVHalf;
  Hdr* hdr = reinterpret_cast<Hdr*>(sV + kVStages * NH * kKVHalf);
  if (smem_u32(smem_raw) & 1023u) {  // uniform over the CTA; nothing touched yet
    if (threadIdx.x == 0) set_status(SPECOPD_DEV_LAYOUT);
    return;
  }

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // ---- work unit: (query tile, kv head, key chunk), chunk-major so that the
  // full leading chunks start first and the partial or empty trailing ones
  // fill in last; within a chunk, heavier tiles (larger anchors) first.
  //
  // Branch pass: a query tile is RT branch rows of one sequence s; its keys
  // are trunk rows t0 + 0 .. t0 + a (t0 = start of s, a = the row's anchor)
  // and its branch nodes.  Trunk prefill: a query tile is RT consecutive
  // packed trunk rows (it may span a sequence boundary); its keys are the
  // packed trunk rows t0 .. r, t0 = start of the sequence of the tile's
  // first row, and row r sees the rows of its own sequence up to itself.
  // In both cases row r sees the keys t0 + vlo_r .. t0 + vhi_r.
  const int u = blockIdx.x;
  int c, tile, h, nsp = 0;  // nsp > 0: this pair's chunk count (chunk size from its span)
  if (P.s_lo > 0) {
    // One wave of units: the n_hi heaviest tiles (the last ones) in s_lo + 1
    // chunks, the others in s_lo; heavier tiles first within each group.
    const int heavy = P.n_hi * P.Hkv;
    const int u_hi = heavy * (P.s_lo + 1);
    int rem;
    if (u < u_hi) {
      c = u / heavy;
      rem = u % heavy;
      tile = P.ntile - 1 - rem / P.Hkv;
      nsp = P.s_lo + 1;
    } else {
      const int light = (P.ntile - P.n_hi) * P.Hkv;
      c = (u - u_hi) / light;
      rem = (u - u_hi) % light;
      tile = P.ntile - P.n_hi - 1 - rem / P.Hkv;
      nsp = P.s_lo;
    }
    h = rem % P.Hkv;
  } else {
    const int per_c = P.ntile * P.Hkv;
    c = u / per_c;
    tile = P.ntile - 1 - (u % per_c) / P.Hkv;
    h = (u % per_c) % P.Hkv;
  }
  const int Wm1 = P.W - 1;
  int s, r0, r1;
  if (P.prefill) {
    r0 = tile * P.RT;
    r1 = min(r0 + P.RT, P.T_tot);
    int lo = 0, hi = P.S - 1;  // sequence of row r0: cu[s] <= r0 < cu[s+1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P.cu_trunk[mid] <= r0) lo = mid; else hi = mid - 1;
    }
    s = lo;
  } else {
    s = tile / P.ntile_per_seq;
    const int rows_seq = P.B * Wm1;
    r0 = s * rows_seq + (tile % P.ntile_per_seq) * P.RT;
    r1 = min(r0 + P.RT, (s + 1) * rows_seq);
  }
  const int t0 = P.cu_trunk[s];
  const int Ts = P.cu_trunk[s + 1] - t0;
  const int G = P.G;
  const int MT = P.RT * G;

  // ---- prologue: barriers and the Q copy (thread 0), the tile's largest
  // valid anchor (warps 0-3), TMEM (warp 1), then one block barrier.
  if (tid == 0) {
    mbar_init(&hdr->q_full, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&hdr->k_full[i], 1);
      mbar_init(&hdr->k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&hdr->v_full[i], 1);
      mbar_init(&hdr->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&hdr->s_full[i], 1);
      mbar_init(&hdr->p_full[i], 128);
    }
    mbar_init(&hdr->o_done, 1);
    mbar_init(&hdr->o_final, 1);
    mbar_init(&hdr->rot_done, 128);
    hdr->abort = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(&hdr->q_full, (unsigned)(NH * MT * 128));
    for (int hh = 0; hh < NH; ++hh)
      tma_load_3d(sQ + hh * kQHalf, &tm_q, hh * 64, h * G, r0, &hdr->q_full);
  }
  if (warp < 4) {
    // RT <= 128: warp w covers rows r0 + 32w .. r0 + 32w + 31
    const int r = r0 + warp * 32 + lane;
    int a = -1;
    if (r < r1) {
      if (P.prefill) {
        a = r - t0;
      } else {
        a = P.anchors[r / Wm1];
        if (a < 0 || a >= Ts) a = -1;
      }
    }
    a = __reduce_max_sync(0xffffffffu, a);
    if (lane == 0) hdr->wmax[warp] = a;
  }
  // Q rows beyond the tile (M = RT*G < 128) are never written by TMA: zero them.
  for (int idx = tid; idx < NH * (128 - MT) * 8; idx += kThreads) {
    const int hh = idx / ((128 - MT) * 8);
    const int rem = idx % ((128 - MT) * 8);
    reinterpret_cast<uint4*>(sQ + hh * kQHalf + (MT + rem / 8) * 128)[rem % 8] =
        make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
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
  const int kmax = max(max(hdr->wmax[0], hdr->wmax[1]), max(hdr->wmax[2], hdr->wmax[3]));
  // Trunk keys of this chunk.  Fixed chunks of P.C keys, or (nsp > 0) this
  // pair's key tiles split over its nsp chunks with chunk 0 -- which also
  // scores and rotates the branch tiles and usually merges -- counted
  // kChunk0Extra tiles heavier.  Either way the chunks that hold keys are
  // 0 .. nact - 1, the same on every unit of the pair.
  int nact, k_begin, k_end;
  if (nsp > 0) {
    const int ntk = kmax < 0 ? 0 : (kmax + 1 + kBN - 1) / kBN;  // trunk key tiles
    int t0n = ntk, per = 1;  // trunk tiles of chunk 0, of the others
    if (nsp > 1) {
      t0n = min(ntk, max(0, (ntk + kChunk0Extra + nsp - 1) / nsp - kChunk0Extra));
      per = max(1, (ntk - t0n + nsp - 2) / (nsp - 1));
    }
    nact = 1 + (ntk > t0n ? (ntk - t0n + per - 1) / per : 0);
    const int tb = c == 0 ? 0 : t0n + (c - 1) * per;
    const int te = c == 0 ? t0n : min(ntk, t0n + c * per);
    k_begin = tb * kBN;
    k_end = min(te * kBN, kmax + 1);
  } else {
    nact = kmax < 0 ? 1 : (kmax + P.C) / P.C;  // chunks with trunk keys (>= 1)
    k_begin = c * P.C;
    k_end = min(k_begin + P.C, kmax + 1);
  }
  const int nt = k_end > k_begin ? (k_end - k_begin + kBN - 1) / kBN : 0;
  if (c > 0 && nt == 0) {
    // Nothing for this chunk (uniform over the CTA).  The Q copy must land
    // before the CTA's shared memory is released.
    if (tid == 0 && !mbar_wait(&hdr->q_full, 0)) set_status(SPECOPD_DEV_TIMEOUT);
    if (warp == 1) {
      __syncwarp();
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    }
    return;
  }
  const int kb0 = P.prefill ? 0 : (r0 / Wm1) * Wm1;  // first branch node the tile needs
  const int nbt = (c == 0 && !P.prefill) ? (r1 - kb0 + kBN - 1) / kBN : 0;
  const int nk = nt + nbt;
  const uint32_t tS[2] = {tmem, tmem + kBN};
  const uint32_t tO = tmem + 2 * kBN;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      // K tiles run kKStages - kVStages tiles ahead of V tiles: the QK^T that
      // frees a K slot completes before the P.V that frees the V slot of the
      // same tile, so a blocked V copy never holds back the next K copy.
      // Key order: the branch tiles (leading chunk only) first, so that the
      // softmax warps can rotate them in the prologue, then the trunk tiles.
      auto row_of = [&](int j) { return j < nbt ? kb0 + j * kBN : t0 + k_begin + (j - nbt) * kBN; };
      constexpr int kLead = kKStages - kVStages;
      int nk_issued = 0, nv_issued = 0;
      for (int i = 0; i < nk + kLead && !hdr->abort; ++i) {
        if (i < nk) {
          const int j = i, st = j % kKStages;
          if (j >= kKStages && !wait_or_abort(&hdr->k_empty[st], ((j / kKStages) - 1) & 1, hdr)) break;
          mbar_arrive_expect_tx(&hdr->k_full[st], NH * kKVHalf);
          for (int hh = 0; hh < NH; ++hh)
            tma_load_3d(sK + (st * NH + hh) * kKVHalf, j < nbt ? &tm_kbr : &tm_ktr, hh * 64, h,
                        row_of(j), &hdr->k_full[st]);
          nk_issued = j + 1;
        }
        if (i >= kLead) {
          const int j = i - kLead, st = j % kVStages;
          if (j >= kVStages && !wait_or_abort(&hdr->v_empty[st], ((j / kVStages) - 1) & 1, hdr)) break;
          mbar_arrive_expect_tx(&hdr->v_full[st], NH * kKVHalf);
          for (int hh = 0; hh < NH; ++hh)
            tma_load_3d(sV + (st * NH + hh) * kKVHalf, j < nbt ? &tm_vbr : &tm_vtr, hh * 64, h,
                        row_of(j), &hdr->v_full[st]);
          nv_issued = j + 1;
        }
      }
      // No copy may still be landing when the CTA's shared memory is
      // released: wait (bounded, whatever the abort flag says) for the Q copy
      // and the last phase issued into every K and V stage.  In a normal run
      // the MMA warp has waited for each already and these return at once.
      mbar_wait(&hdr->q_full, 0);
      for (int j = max(0, nk_issued - kKStages); j < nk_issued; ++j)
        mbar_wait(&hdr->k_full[j % kKStages], (j / kKStages) & 1);
      for (int j = max(0, nv_issued - kVStages); j < nv_issued; ++j)
        mbar_wait(&hdr->v_full[j % kVStages], (j / kVStages) & 1);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = idesc_bf16(kBN, false);
      constexpr uint32_t kIdPV = idesc_bf16(D, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      auto pv = [&](int jj) -> bool {
        const int b = jj & 1;
        const int st = jj % kVStages;
        if (!wait_or_abort(&hdr->p_full[b], (jj >> 1) & 1, hdr)) return false;
        if (!wait_or_abort(&hdr->v_full[st], (jj / kVStages) & 1, hdr)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // B = V tile, MN-major: 16 keys = two 8-row groups of 1024 B; the
          // 64-column halves of D are kKVHalf apart.
          const uint64_t bd = sdesc(v_addr + st * NH * kKVHalf + kk * 2048, kKVHalf, 1024);
          mma_ts(tO, tS[b] + kk * 8, bd, kIdPV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&hdr->v_empty[st]);
        tc_commit(&hdr->o_done);
        return true;
      };
      // Q (and the leading branch key tiles) are rotated in shared memory
      // by the softmax warps before the first MMA reads them.
      bool ok = wait_or_abort(&hdr->rot_done, 0, hdr);
      tc_fence_after();
      for (int j = 0; j < nk && ok; ++j) {
        const int st = j % kKStages;
        const int b = j & 1;
        if (!wait_or_abort(&hdr->k_full[st], (j / kKStages) & 1, hdr)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          // K-major operands: 16 columns = 32 B inside a 128-byte swizzled row.
          const int hh = kk >> 2, w = kk & 3;
          const uint64_t ad = sdesc(q_addr + hh * kQHalf + w * 32, 16, 1024);
          const uint64_t bd = sdesc(k_addr + (st * NH + hh) * kKVHalf + w * 32, 16, 1024);
          mma_ss(tS[b], ad, bd, kIdQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&hdr->k_empty[st]);
        tc_commit(&hdr->s_full[b]);
        if (j >= 1 && !pv(j - 1)) { ok = false; break; }
      }
      if (ok && nk > 0) pv(nk - 1);
      // A commit tracks every MMA issued before it: the epilogue waits on this
      // one barrier instead of a phase of o_done, which can be two phases
      // behind there (P.V of tile nk-2 is issued after the last S commit).
      tc_commit(&hdr->o_final);
    }
  } else {
    // ================================================================ softmax / epilogue
    // Warp w accesses TMEM lanes 32*(w%4) .. +31; each thread owns one query
    // row of the tile (TMEM lane) and all kBN columns of its S tiles.
    const int q4 = warp & 3;
    const int mrow = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int lr = mrow / G, g = mrow % G;
    const int r = r0 + lr;
    const bool in_tile = (lr < P.RT) && (r < r1);
    int a_r = -1, kfirst = 0, vlo = 0, qpos = 0;
    bool bad = false;
    if (in_tile) {
      if (P.prefill) {
        int sr = s;  // the row's own sequence (a tile spans few sequences)
        while (sr + 1 < P.S && P.cu_trunk[sr + 1] <= r) ++sr;
        vlo = P.cu_trunk[sr] - t0;
        a_r = r - t0;
        qpos = r - P.cu_trunk[sr];
      } else {
        const int bid = r / Wm1;
        a_r = P.anchors[bid];
        bad = (a_r < 0 || a_r >= Ts);
        kfirst = bid * Wm1;
        qpos = P.pos_br[r];
      }
    }
    const bool live = in_tile && !bad;
    const float sl2 = P.scale_log2;
    {
      // ---- RoPE in shared memory: this thread's query row (TMEM lane =
      // Q line), then half a line of each leading branch key tile.  The
      // async proxy (tcgen05.mma) reads them after the fence and rot_done.
      bool okr = warp_wait_or_abort(&hdr->q_full, 0, hdr);
      if (okr && in_tile)
        rope_row_smem<D>(sQ + mrow * 128, sQ + (D == 128 ? kQHalf : 0) + mrow * 128, mrow, qpos,
                         P.theta, 0, D / 16);
      const int t128 = tid - 64;  // 0..127
      for (int j = 0; j < nbt; ++j) {
        // branch tile j sits in K stage j (nbt <= 2 < kKStages), first use
        okr = okr && warp_wait_or_abort(&hdr->k_full[j], 0, hdr);
        const int line = t128 >> 1;
        const int node = kb0 + j * kBN + line;
        if (okr && node < P.R) {
          uint8_t* base = sK + (j * NH) * kKVHalf + line * 128;
          const int half = D / 32;  // pair chunks per thread
          rope_row_smem<D>(base, base + (D == 128 ? kKVHalf : 0), line, P.pos_br[node], P.theta,
                           (t128 & 1) * half, (t128 & 1) * half + half);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&hdr->rot_done);
    }
    float m = -INFINITY, l = 0.f;  // running max (log2 units) and sum
    uint32_t sv[kBN];
    // After a wait runs out the warp keeps stepping through the loop with its
    // TMEM work skipped (dead).
    bool dead = false;
    for (int j = 0; j < nk; ++j) {
      const int b = j & 1;
      if (!dead) dead = !warp_wait_or_abort(&hdr->s_full[b], (j >> 1) & 1, hdr);
      if (!dead) {
        tc_fence_after();
        __syncwarp();  // tcgen05.ld/st are warp-collective (.sync.aligned)
        tmem_ld32(tS[b] + lane_off, sv);
        tmem_ld32(tS[b] + lane_off + 32, sv + 32);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < kBN; ++e) sv[e] = 0u;
      }
      // visible columns of the tile: lo <= col <= hi
      int lo, hi;
      if (j >= nbt) {
        lo = vlo - (k_begin + (j - nbt) * kBN);
        hi = a_r - (k_begin + (j - nbt) * kBN);
      } else {
        const int node0 = kb0 + j * kBN;
        lo = kfirst - node0;
        hi = r - node0;
      }
      if (!live) hi = -1;
      // raw-score maximum (the scale is positive, so it commutes with max)
      float mx3[3] = {-INFINITY, -INFINITY, -INFINITY};
      if (__all_sync(0xffffffffu, lo <= 0 && hi >= kBN - 1)) {
        // every column is visible to every row of the warp
#pragma unroll
        for (int e = 0; e + 1 < kBN; e += 2)
          mx3[(e >> 1) % 3] = fmax3(mx3[(e >> 1) % 3], __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
      } else {
#pragma unroll
        for (int e = 0; e < kBN; ++e) {
          const float x = (e >= lo && e <= hi) ? __uint_as_float(sv[e]) : -INFINITY;
          sv[e] = __float_as_uint(x);
        }
#pragma unroll
        for (int e = 0; e + 1 < kBN; e += 2)
          mx3[(e >> 1) % 3] = fmax3(mx3[(e >> 1) % 3], __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
      }
      const float mx = fmax3(mx3[0], mx3[1], mx3[2]) * sl2;
      const float m_new = fmaxf(m, mx);
      // Lazy rescale: keep the stale max unless it grew by more than 2^8.
      const bool need = (m != -INFINITY) && (m_new > m + kRescaleThreshold);
      if (m == -INFINITY) m = m_new;  // first visible keys: O and l are still zero
      if (__any_sync(0xffffffffu, need)) {
        // Warp-uniform branch (the TMEM accesses are warp-collective); rows
        // that need no rescale multiply by 1.
        const float f = need ? exp2f(m - m_new) : 1.f;
        if (need) {
          l *= f;
          m = m_new;
        }
        if (j > 0 && !dead) dead = !warp_wait_or_abort(&hdr->o_done, (j - 1) & 1, hdr);
        if (j > 0 && !dead) {
          // O holds PV of tiles < j; PV of tile j-1 must be complete.
          tc_fence_after();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < DC; ++q) {
            uint32_t ov[32];
            tmem_ld32(tO + lane_off + q * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
            tmem_st32(tO + lane_off + q * 32, ov);
          }
        }
      }
      // p = 2^(s*scale*log2e - m); masked entries are -inf -> 0
      // (packed fp32x2 arithmetic: one FFMA2 and one FADD2 per key pair; P
      // as bf16 pairs overwrites sv in place, sv[e] having been read at step
      // e / 2)
      const float nm = (m == -INFINITY) ? 0.f : -m;
      const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(nm, nm);
      float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int e = 0; e < kBN / 2; ++e) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                                    sl2v, nmv);
        const float2 p = make_float2(ex2_fast(x.x), ex2_fast(x.y));
        rs2[e & 1] = __fadd2_rn(rs2[e & 1], p);
        sv[e] = pack_bf16x2(p.x, p.y);
      }
      l += (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
      if (!dead) {
        __syncwarp();
        tmem_st32(tS[b] + lane_off, sv);  // P of the tile's kBN keys as bf16 pairs
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&hdr->p_full[b]);
      }
    }
    // ---- epilogue
    // o_final is committed by the MMA thread in every case, abort or not,
    // and tracks every MMA it issued: wait for it (bounded) even after an
    // abort, so no MMA still writes TMEM when it is read or deallocated.
    const bool fin = __all_sync(0xffffffffu, mbar_wait(&hdr->o_final, 0));
    const bool ok = fin && !hdr->abort;
    tc_fence_after();
    __syncwarp();
    const int hq = h * G + g;
    const float qnan = __int_as_float(0x7fc00000);
    __nv_bfloat16* dst = P.out + ((size_t)r * P.Hq + hq) * D;
    // 32 columns of the output row as four 16-byte stores
    auto write_chunk = [&](int q, const float* acc, float inv) {
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v;
        v.x = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
        v.y = pack_bf16x2(acc[e + 2] * inv, acc[e + 3] * inv);
        v.z = pack_bf16x2(acc[e + 4] * inv, acc[e + 5] * inv);
        v.w = pack_bf16x2(acc[e + 6] * inv, acc[e + 7] * inv);
        *reinterpret_cast<uint4*>(dst + q * 32 + e) = v;
      }
    };
    auto write_lse = [&](float mm, float ll) {
      if (P.lse) P.lse[(size_t)r * P.Hq + hq] = (bad || !ok) ? qnan : (mm + log2f(ll)) * 0.6931471805599453f;
      if (bad && g == 0) set_status(SPECOPD_DEV_ANCHOR_RANGE);
    };
    if (nact == 1) {
      const float inv = (bad || !ok) ? qnan : 1.f / l;
#pragma unroll
      for (int q = 0; q < DC; ++q) {
        uint32_t ov[32];
        tmem_ld32(tO + lane_off + q * 32, ov);
        tmem_wait_ld();
        if (in_tile) write_chunk(q, reinterpret_cast<const float*>(ov), inv);
      }
      if (in_tile) write_lse(m, l);
    } else {
      // split-KV: publish this chunk's partial, the last chunk to arrive merges.
      // Partial layout: float4 k of row mrow at index k * 128 + mrow, so the
      // 32 rows of a warp store and load 512 contiguous bytes.
      const size_t slot = ((size_t)tile * P.Hkv + h) * P.nsplit;
      const size_t slot_floats = (size_t)128 * D + 256;
      float* pbase = P.part + slot * slot_floats;
      float4* mine4 = reinterpret_cast<float4*>(pbase + c * slot_floats);
#pragma unroll
      for (int q = 0; q < DC; ++q) {
        uint32_t ov[32];
        tmem_ld32(tO + lane_off + q * 32, ov);
        tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4)
          __stcg(mine4 + (q * 8 + e4) * 128 + mrow,
                 make_float4(__uint_as_float(ov[4 * e4]), __uint_as_float(ov[4 * e4 + 1]),
                             __uint_as_float(ov[4 * e4 + 2]), __uint_as_float(ov[4 * e4 + 3])));
      }
      pbase[c * slot_floats + 128 * D + mrow] = m;
      pbase[c * slot_floats + 128 * D + 128 + mrow] = l;
      __threadfence();
      named_bar_sync(1, 128);
      if (tid == 64) {
        const unsigned old = atomicAdd(&P.cnt[tile * P.Hkv + h], 1u);
        hdr->last = (old == (unsigned)nact - 1u) ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (hdr->last) {
        __threadfence();
        float mm = -INFINITY;
        for (int cc = 0; cc < nact; ++cc)
          mm = fmaxf(mm, __ldcg(pbase + cc * slot_floats + 128 * D + mrow));
        // Fixed chunk order 0 .. nact-1 whichever chunk merges: the result
        // does not depend on the arrival order (bit for bit).
        float ll = 0.f;
        float acc[D];
#pragma unroll
        for (int e = 0; e < D; ++e) acc[e] = 0.f;
        for (int cc = 0; cc < nact; ++cc) {
          const float* pc = pbase + cc * slot_floats;
          const float mc = __ldcg(pc + 128 * D + mrow);
          const float wgt = (mc == -INFINITY) ? 0.f : exp2f(mc - mm);
          ll += wgt * __ldcg(pc + 128 * D + 128 + mrow);
          const float4* pc4 = reinterpret_cast<const float4*>(pc);
#pragma unroll
          for (int k = 0; k < D / 4; ++k) {
            const float4 v = __ldcg(pc4 + k * 128 + mrow);
            acc[4 * k] += wgt * v.x;
            acc[4 * k + 1] += wgt * v.y;
            acc[4 * k + 2] += wgt * v.z;
            acc[4 * k + 3] += wgt * v.w;
          }
        }
        if (in_tile) {
          const float inv = (bad || !ok) ? qnan : 1.f / ll;
#pragma unroll
          for (int q = 0; q < DC; ++q) write_chunk(q, acc + q * 32, inv);
          write_lse(mm, ll);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D view [rows, H, D] (bf16, contiguous) with box (64, box_h, box_rows).
bool make_map(CUtensorMap* m, const void* ptr, int D, int H, int rows, int box_h, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_h, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
  int RT, ntile_per_seq, ntile, nsplit, C;
  int s_lo, n_hi;  // one-wave split of the branch pass (s_lo > 0), see make_plan
  long long units;
  size_t part_bytes, cnt_bytes;
};

// Work decomposition.  base = (query tile, kv head) pairs; each splits into
// key chunks.  Branch pass with fewer pairs than resident CTA slots (SMs x
// 2): one wave of units (the s_lo / n_hi split below, chunk sizes per pair
// on the device).  Otherwise nsplit chunks of C keys: with one to eight
// waves of pairs two chunks halve the tail of the last wave; the prefill
// keeps one.
Plan make_plan(const AttnProblem& p, int num_sms, bool prefill) {
  Plan pl;
  pl.RT = 128 / p.G;
  if (prefill) {
    // Tiles of RT packed trunk rows; a tile's keys start at the first
    // sequence it touches, so a key range is at most T_max + RT long.
    pl.ntile_per_seq = 0;
    pl.ntile = (p.T_tot + pl.RT - 1) / pl.RT;
  } else {
    const int rows_seq = p.B * (p.W - 1);
    pl.ntile_per_seq = (rows_seq + pl.RT - 1) / pl.RT;
    pl.ntile = pl.ntile_per_seq * p.S;
  }
  const int key_span = prefill ? p.T_max + pl.RT : p.T_max;
  const long long base = (long long)pl.ntile * p.Hkv;
  const long long slots = (long long)std::max(1, num_sms) * kCtasPerSm;
  // (The prefill keeps one chunk per pair once the pairs fill the slots:
  // its tiles' key ranges grow row by row, the tiles are ordered longest
  // first, and every extra chunk adds a unit's prologue and epilogue; 180
  // against 216 us on the 8B trunk.)
  long long want = base < slots ? (slots + base - 1) / base : (base < 8 * slots && !prefill ? 2 : 1);
  const int max_split = std::max(1, key_span / (4 * kBN));  // chunks of at least 4 key tiles
  const int best = (int)std::min<long long>(std::min<long long>(want, max_split), 64);
  int C = (key_span + best - 1) / best;
  C = (C + kBN - 1) / kBN * kBN;
  pl.nsplit = (key_span + C - 1) / C;
  pl.C = C;
  pl.s_lo = 0;
  pl.n_hi = 0;
  pl.units = base * pl.nsplit;
  if (!prefill && base < slots) {
    // Fewer (tile, kv head) pairs than CTA slots: split so that the units
    // fit one wave exactly -- s_lo chunks per pair, one more for the
    // heaviest tiles while slots remain -- each pair's chunks sized on the
    // device from its own key span.  A fixed chunk size left units for a
    // second wave (8B: 304 of 336 non-empty on 296 slots).
    const int cap = std::min(max_split, 64);
    const int s_lo = (int)std::min<long long>(std::max<long long>(1, slots / base), cap);
    const int n_hi = s_lo < cap ? (int)std::min<long long>(pl.ntile, (slots - base * s_lo) / p.Hkv) : 0;
    pl.s_lo = s_lo;
    pl.n_hi = n_hi;
    pl.nsplit = s_lo + (n_hi > 0 ? 1 : 0);
    pl.units = (long long)n_hi * p.Hkv * (s_lo + 1) + (long long)(pl.ntile - n_hi) * p.Hkv * s_lo;
  }
  pl.part_bytes = pl.nsplit > 1 ? (size_t)pl.ntile * p.Hkv * pl.nsplit * ((size_t)128 * p.D + 256) * 4 : 0;
  pl.cnt_bytes = (size_t)pl.ntile * p.Hkv * 4;
  return pl;
}

size_t smem_bytes(int D) {
  const int NH = D / 64;
  size_t b = (size_t)NH * kQHalf + (size_t)(kKStages + kVStages) * NH * kKVHalf + sizeof(Hdr);
  // Each CTA allocates half of the SM's TMEM: at most two may be resident.
  if (b < 80 * 1024) b = 80 * 1024;
  return b;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    return n;
  return 148;
}

}  // namespace
}  // namespace sm100

size_t attn_sm100_workspace(const AttnProblem& p, bool prefill) {
  const sm100::Plan pl = sm100::make_plan(p, sm100::sm_count(), prefill);
  return ((pl.part_bytes + 255) & ~size_t(255)) + pl.cnt_bytes;
}

cudaError_t launch_attn_sm100(const AttnProblem& p, const void* q_br, const void* k_br,
                              const void* v_br, const void* k_tr, const void* v_tr,
                              const int32_t* cu_trunk, const int32_t* anchors,
                              const int32_t* pos_br, const double* theta, void* out,
                              float* lse, void* ws, size_t ws_bytes, cudaStream_t st,
                              bool prefill) {
  using namespace sm100;
  const int nq = prefill ? p.T_tot : p.R;  // query rows
  if (nq == 0) return cudaSuccess;
  if (p.D != 64 && p.D != 128) return cudaErrorInvalidValue;
  const Plan pl = make_plan(p, sm_count(), prefill);
  const size_t part_off = 0;
  const size_t cnt_off = (pl.part_bytes + 255) & ~size_t(255);
  if (ws_bytes < cnt_off + pl.cnt_bytes) return cudaErrorInvalidValue;
  CUtensorMap tq, tktr, tvtr, tkbr, tvbr;
  // Prefill has no branch keys: the branch maps repeat the trunk ones.
  if (!make_map(&tq, q_br, p.D, p.Hq, nq, p.G, pl.RT) ||
      !make_map(&tktr, k_tr, p.D, p.Hkv, p.T_tot, 1, kBN) ||
      !make_map(&tvtr, v_tr, p.D, p.Hkv, p.T_tot, 1, kBN) ||
      !make_map(&tkbr, prefill ? k_tr : k_br, p.D, p.Hkv, prefill ? p.T_tot : p.R, 1, kBN) ||
      !make_map(&tvbr, prefill ? v_tr : v_br, p.D, p.Hkv, prefill ? p.T_tot : p.R, 1, kBN))
    return cudaErrorInvalidValue;
  Params P;
  P.S = p.S; P.B = p.B; P.W = p.W; P.Hq = p.Hq; P.Hkv = p.Hkv; P.G = p.G; P.R = p.R;
  P.prefill = prefill ? 1 : 0;
  P.T_tot = p.T_tot;
  P.RT = pl.RT; P.ntile_per_seq = pl.ntile_per_seq; P.ntile = pl.ntile;
  P.nsplit = pl.nsplit; P.C = pl.C;
  P.s_lo = pl.s_lo; P.n_hi = pl.n_hi;
  P.scale_log2 = p.scale * 1.4426950408889634f;
  P.cu_trunk = cu_trunk;
  P.anchors = anchors;
  P.pos_br = pos_br;
  for (int k = 0; k < 64; ++k) P.theta[k] = k < p.D / 2 ? theta[k] : 0.0;
  P.out = reinterpret_cast<__nv_bfloat16*>(out);
  P.lse = lse;
  char* w = reinterpret_cast<char*>(ws);
  P.part = reinterpret_cast<float*>(w + part_off);
  P.cnt = reinterpret_cast<unsigned*>(w + cnt_off);
  cudaError_t e = cudaMemsetAsync(w + cnt_off, 0, pl.cnt_bytes, st);
  if (e != cudaSuccess) return e;
  const size_t smem = smem_bytes(p.D);
  const dim3 grid((unsigned)pl.units);
  if (p.D == 128) {
    e = cudaFuncSetAttribute(tree_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_attn_kernel<128>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    tree_attn_kernel<128><<<grid, kThreads, smem, st>>>(tq, tktr, tvtr, tkbr, tvbr, P);
  } else {
    e = cudaFuncSetAttribute(tree_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_attn_kernel<64>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    tree_attn_kernel<64><<<grid, kThreads, smem, st>>>(tq, tktr, tvtr, tkbr, tvbr, P);
  }
  return cudaGetLastError();
}

}  // namespace specopd
