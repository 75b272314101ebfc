/*
 * specopd.h -- C ABI of the SpecOPD branch-scoring library for B200 (sm_100a).
 *
 * SpecOPD scores B anchor-rooted, W-token draft branches in one shared-prefix
 * target pass and trains the drafter with the E2E-TV acceptance-length loss.
 * This library holds the hot path of that pass:
 *
 *   specopd_tree_build  parent map, semantic positions and score-row map of
 *                       the proposal tree
 *   specopd_rope_apply  rotary embedding at given positions (trunk K cache)
 *   specopd_tree_attn   GQA attention of the B(W-1) branch rows over the
 *                       cached trunk K/V and their own branch history
 *   specopd_e2e_tv      per-position overlap a = sum_v min(p_v, q_v), branch
 *                       prefix products, loss and d loss / d draft logits
 *   specopd_e2e_tv_lmhead  the same from hidden rows and the two LM heads,
 *                       the logits formed on chip and never stored
 *
 * Sources (web pages on arXiv 2611.02846, cited by title and section):
 *   [review]  "SpecOPD: Branch-Parallel On-Policy Distillation for
 *             Speculative Decoding", paper review (jaehun.me), sections
 *             1.1, 3.1, 3.2(a), 3.3, 3.4.
 *   [summary] "SpecOPD: 面向投机解码的分支并行在线策略蒸馏", paper summary
 *             (rustineverything.app), paragraphs tagged §2.1, §2.2, §2.3.
 *
 * Conventions shared by every call
 *   - Pointers are DEVICE pointers unless the name ends in _host.
 *   - The caller owns every buffer.  No call allocates device memory: calls
 *     that need scratch take a caller-provided workspace whose size the
 *     matching *_workspace_size function returns.
 *   - Every call enqueues its work on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream) and returns without
 *     synchronising, except specopd_get_device_status.
 *   - Shapes, dtypes, alignment and workspace size are checked on the host
 *     before anything is launched; a failed check returns an error status and
 *     launches nothing.  Errors that only the device can see (an anchor
 *     outside its trunk, a target row out of range, a row whose logits are all
 *     -inf, a bounded wait that ran out) never trap: the kernel sets a bit in
 *     a per-device status word, writes NaN to the affected outputs and
 *     returns.  specopd_get_device_status reads and clears that word.
 *   - Tensors are dense and row-major with the shapes given; rows are
 *     contiguous (row stride = product of the trailing dims).  bf16 tensors
 *     must start on a 16-byte boundary.
 *   - Packed node order of the proposal tree (used by every call):
 *       trunk nodes  : n = cu_trunk[s] + j            (j = 0 .. T_s - 1)
 *       branch nodes : n = T_tot + (s*B + b)*(W-1) + (i-1)   (i = 1 .. W-1)
 *     Branch node (s,b,i) is the i-th drafted token after anchor a_{s,b}.
 *     Branch rows (inputs/outputs of specopd_tree_attn) are indexed by
 *     r = n - T_tot, i.e. r = (s*B + b)*(W-1) + (i-1), R = S*B*(W-1) rows.
 *     Supervised positions (inputs/outputs of specopd_e2e_tv) are indexed by
 *     (s*B + b)*W + (i-1), i = 1 .. W, N = S*B*W positions.
 */
#ifndef SPECOPD_H
#define SPECOPD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPECOPD_OK = 0,
  SPECOPD_ERR_INVALID_ARG = 1, /* a pointer, size or shape argument is invalid  */
  SPECOPD_ERR_UNSUPPORTED = 2, /* valid but not supported (dtype, head_dim, alignment, size) */
  SPECOPD_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than *_workspace_size */
  SPECOPD_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, attribute, ...) */
  SPECOPD_ERR_TIMEOUT = 5,     /* reported through the device status word only */
  SPECOPD_ERR_NO_DEVICE = 6    /* no sm_100 device is current */
} specopd_status;

typedef enum { SPECOPD_F32 = 0, SPECOPD_BF16 = 1 } specopd_dtype;

/* Bits of the per-device status word (specopd_get_device_status). */
#define SPECOPD_DEV_ANCHOR_RANGE 0x1u  /* an anchor outside [0, T_s)            */
#define SPECOPD_DEV_ROW_RANGE 0x2u     /* a target_row outside [0, rows_target) */
#define SPECOPD_DEV_ALL_NEG_INF 0x4u   /* a logit row with no finite entry      */
#define SPECOPD_DEV_TIMEOUT 0x8u       /* a bounded wait ran out                */
#define SPECOPD_DEV_LAYOUT 0x10u       /* shared memory not laid out as the kernel
                                          requires; the kernel wrote nothing    */

/* Human-readable name of a status code.  Never NULL. */
const char* specopd_status_string(int status);

/* Library ABI version (major*10000 + minor*100 + patch). */
int specopd_version(void);

/*
 * Reads the status word of the current device into *host_out and clears it.
 * Synchronises `stream` first.  Returns SPECOPD_OK, or SPECOPD_ERR_CUDA if
 * the copy failed.  The word is one per device, shared by every call
 * whatever its stream: with calls in flight on several streams a set bit
 * says that one of them met the condition (their outputs carry the NaN);
 * to attribute it to a call, synchronise the other streams first.
 */
specopd_status specopd_get_device_status(uint32_t* host_out, void* stream);

/* ------------------------------------------------------------------------ */
/* Proposal tree: [review §3.1] (trunk, anchors, branches attached to the
 * anchors), [summary §2.1] (the first branch token's parent is the anchor
 * token, later tokens' parent is the previous sampled token, the semantic
 * position is the anchor position plus the offset), [review §3.2(a)] and
 * [summary §2.2] (score-row reading rule: the anchor row scores branch token
 * 1, branch row i scores token i+1, so B branches add B(W-1) rows).
 *
 * Inputs
 *   S              number of independent reference sequences (>= 1)
 *   cu_trunk_host  host int32[S+1], prefix sums of trunk lengths,
 *                  cu_trunk_host[0] = 0, every T_s = cu[s+1]-cu[s] >= 1
 *   anchors        device int32[S*B], LOCAL anchor positions, 0 <= a < T_s
 *                  (any order, duplicates allowed)
 *   B, W           anchors per sequence (>= 1) and branch width (>= 1)
 * Outputs (device, caller-allocated)
 *   parent     int32[T_tot + R]: trunk node j>0 -> its predecessor, j=0 -> -1;
 *              branch node i=1 -> the anchor's trunk node, i>=2 -> node i-1
 *   sem_pos    int32[T_tot + R]: trunk node -> j; branch node -> a + i
 *   score_row  int32[S*B*W]: packed node whose target output scores supervised
 *              position (s,b,i): i=1 -> anchor's trunk node, i>=2 -> branch
 *              node i-1.  Any of the three outputs may be NULL (skipped).
 * An anchor outside its trunk sets SPECOPD_DEV_ANCHOR_RANGE and that
 * branch's entries are written as -1.
 */
specopd_status specopd_tree_build(int S, const int32_t* cu_trunk_host,
                                  const int32_t* anchors, int B, int W,
                                  int32_t* parent, int32_t* sem_pos,
                                  int32_t* score_row, void* stream);

/* ------------------------------------------------------------------------ */
/* Rotary position embedding at logical positions: [review §3.2(a)] (RoPE
 * uses each token's logical position, not its packing order).  The pages do
 * not fix the convention; this library uses the half-split pairing
 * (d, d + D/2), angle pos * base^(-2k/D) for k < D/2:
 *   y[k]       = x[k] cos - x[k+D/2] sin
 *   y[k+D/2]   = x[k+D/2] cos + x[k] sin
 * Angles are reduced in double precision, then evaluated in fp32.
 */
typedef struct {
  int D;               /* head dim, even, 2..256                           */
  specopd_dtype dtype; /* of x                                             */
  float rope_base;     /* > 0, e.g. 10000                                  */
} specopd_rope_desc;

/*
 * In place: x [n, H, D] (dtype), row t rotated at position pos[t].
 * pos: device int32[n], any value >= 0.  bf16 results are rounded to nearest
 * even.  Used to write the trunk K cache at trunk positions (sem_pos of the
 * trunk nodes).
 */
specopd_status specopd_rope_apply(const specopd_rope_desc* desc, void* x,
                                  const int32_t* pos, int n, int H,
                                  void* stream);

/* ------------------------------------------------------------------------ */
/* Tree-masked GQA attention of the branch rows: [review §3.2(a)] (trunk K/V
 * computed once and cached; each query reads only itself and its
 * ancestors; sibling branches and future reference tokens are masked) and
 * [review §3.1] (the condition of position i is the reference prefix up to
 * the anchor and the earlier samples of the same branch).
 *
 * For branch row r = (s,b,i) and query head h (kv head h / (Hq/Hkv)):
 *   keys  = trunk nodes cu_trunk[s] + 0 .. cu_trunk[s] + a_{s,b}   (a+1 keys)
 *         + branch nodes (s,b,1) .. (s,b,i)                       (i keys)
 *   out[r,h,:] = softmax(scale * q' . k'^T) v,   scale = 1/sqrt(D) unless set
 * where q' (and the branch k') are the inputs rotated at the branch node's
 * semantic position (sem_pos), and trunk K is taken as already rotated
 * (specopd_rope_apply at trunk positions).  Nothing else is visible; no
 * dense mask is built.
 */
typedef struct {
  int S, B, W;          /* sequences, anchors per sequence, branch width     */
  int Hq, Hkv, D;       /* query heads, kv heads (Hq % Hkv == 0), head dim   */
  specopd_dtype dtype;  /* F32: any D in {64,128}; BF16: D in {64,128}      */
  float rope_base;      /* RoPE base for the branch rows                     */
  float softmax_scale;  /* 0 -> 1/sqrt(D)                                    */
} specopd_attn_desc;

/* Bytes of workspace specopd_tree_attn needs for this problem (>= 256). */
size_t specopd_tree_attn_workspace_size(const specopd_attn_desc* desc,
                                        const int32_t* cu_trunk_host);

/*
 * q_br   [R, Hq, D]  branch queries, NOT rotated
 * k_br   [R, Hkv, D] branch keys,    NOT rotated
 * v_br   [R, Hkv, D] branch values
 * k_tr   [T_tot, Hkv, D] trunk keys, rotated at trunk positions
 * v_tr   [T_tot, Hkv, D] trunk values
 * cu_trunk       device int32[S+1] (same values as cu_trunk_host)
 * cu_trunk_host  host   int32[S+1]
 * anchors        device int32[S*B], local, 0 <= a < T_s
 * sem_pos        device int32[T_tot + R] from specopd_tree_build
 * out    [R, Hq, D] (dtype)
 * lse    optional fp32 [R, Hq] natural-log sum-exp of the scaled scores, or NULL
 * All tensors of one call share `dtype`.  R = S*B*(W-1); W = 1 is valid and
 * launches nothing.  An anchor outside its trunk sets
 * SPECOPD_DEV_ANCHOR_RANGE and that branch's rows are written as NaN.
 * BF16 returns SPECOPD_ERR_UNSUPPORTED when floor(128 / (Hq/Hkv)) + W - 2 >
 * 192 (a query tile's branch keys must fit three 64-key tiles).
 */
specopd_status specopd_tree_attn(const specopd_attn_desc* desc,
                                 const void* q_br, const void* k_br,
                                 const void* v_br, const void* k_tr,
                                 const void* v_tr, const int32_t* cu_trunk,
                                 const int32_t* cu_trunk_host,
                                 const int32_t* anchors, const int32_t* sem_pos,
                                 void* out, float* lse, void* workspace,
                                 size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Trunk prefill: [review §3.2(a)] (the trunk -- prompt plus reference
 * response -- is computed once and its K/V cached; every branch then reads
 * that cache) and the aimodeling.com news page (the trunk is prefilled once
 * and shared by all of its branches).  The step before specopd_tree_attn:
 * plain causal self-attention of every trunk token over its own sequence.
 *
 * For trunk row t of sequence s (position p = t - cu_trunk[s]) and query
 * head h (kv head h / (Hq/Hkv)):
 *   keys      = trunk rows cu_trunk[s] .. t            (p + 1 keys)
 *   out[t,h,:] = softmax(scale * q' . k'^T) v,   scale = 1/sqrt(D) unless set
 * with q' and k' rotated at their positions within their sequence (the RoPE
 * convention of specopd_rope_apply).  Sequences never see each other.
 *
 * desc       the same descriptor as specopd_tree_attn (B and W are not used)
 * q_tr       [T_tot, Hq, D] trunk queries, NOT rotated
 * k_tr       [T_tot, Hkv, D] IN: trunk keys, not rotated.  OUT: the K cache,
 *            rotated in place -- the k_tr argument of specopd_tree_attn.
 * v_tr       [T_tot, Hkv, D] trunk values (the V cache as it is)
 * cu_trunk / cu_trunk_host  device / host int32[S+1]
 * out        [T_tot, Hq, D] (dtype); row cu_trunk[s] + a is the anchor row
 *            whose target output scores the first token of a branch at a
 * lse        optional fp32 [T_tot, Hq] natural-log sum-exp, or NULL
 * The bf16 path runs on the tensor cores (the kernel of specopd_tree_attn
 * with the trunk rows as queries); fp32 uses the SIMT kernel.
 */
size_t specopd_trunk_prefill_workspace_size(const specopd_attn_desc* desc,
                                            const int32_t* cu_trunk_host);

specopd_status specopd_trunk_prefill(const specopd_attn_desc* desc,
                                     const void* q_tr, void* k_tr,
                                     const void* v_tr, const int32_t* cu_trunk,
                                     const int32_t* cu_trunk_host, void* out,
                                     float* lse, void* workspace, size_t ws_bytes,
                                     void* stream);

/* ------------------------------------------------------------------------ */
/* E2E-TV loss: [review §1.1] and [review §3.3] (single-draft acceptance
 * probability = overlap of the two distributions = 1 - TV(p, q); the loss is
 * built from prefix products of the overlaps within each branch; target mass
 * outside the drafter's support is kept, p is never renormalised; the
 * gradient treats the sampled tokens and the target as fixed and has no
 * score-function term) and [summary §2.3] (loss = 1 - mean over the B*W
 * proposed tokens of the prefix product).
 *
 * For supervised position n = (b, i), b < nbranch, i = 1..W:
 *   p = softmax(z_target[target_row[n]]),  q = softmax(z_draft[n])   (fp32)
 *   a[n]      = sum_v min(p_v, q_v)
 *   prefix[n] = P_{b,i} = prod_{j<=i} a[(b,j)]
 *   numer     = sum_n prefix[n]
 *   loss      = 1 - numer / norm_count
 *   grad[n,u] = g_n * q_u * ([q_u < p_u] - s_n),  s_n = sum_{v: q_v<p_v} q_v,
 *   g_{b,j}   = d loss / d a_{b,j} = -(1/norm_count) * P_{b,j-1} * S_{b,j},
 *   S_{b,W} = 1,  S_{b,j} = 1 + a_{b,j+1} S_{b,j+1},  P_{b,0} = 1.
 */
typedef struct {
  int nbranch;               /* S*B branches                                 */
  int W;                     /* positions per branch (>= 1)                  */
  int V;                     /* vocabulary size (>= 1)                       */
  int rows_target;           /* rows of z_target (bounds for target_row)     */
  specopd_dtype logit_dtype; /* z_target and z_draft                         */
  specopd_dtype grad_dtype;  /* grad_draft                                   */
  int compute_grad;          /* 0: skip grad_draft                           */
  int64_t norm_count;        /* divisor of the loss; 0 -> nbranch*W.  Set to
                                the global count when positions are sharded
                                over ranks ([review §3.2] distributed
                                normalisation: numerators and counts are
                                gathered separately).                        */
} specopd_tv_desc;

/* Bytes of workspace specopd_e2e_tv needs (>= 256). */
size_t specopd_e2e_tv_workspace_size(const specopd_tv_desc* desc);

/*
 * z_target    [rows_target, V] target logits (logit_dtype)
 * target_row  device int32[N] row of z_target scoring position n, or NULL for
 *             the identity (rows_target must then be >= N).  score_row from
 *             specopd_tree_build is the intended argument.
 * z_draft     [N, V] draft logits, branch-major (b, i)
 * a, prefix   device fp32[N]        (required)
 * loss        device fp32[1]        (required)
 * numer       device fp64[1] or NULL (sum of prefix, for cross-rank sums)
 * grad_draft  [N, V] (grad_dtype) or NULL; required when compute_grad != 0
 * A row whose logits are all -inf sets SPECOPD_DEV_ALL_NEG_INF and makes the
 * outputs of its branch NaN.
 */
specopd_status specopd_e2e_tv(const specopd_tv_desc* desc,
                              const void* z_target, const int32_t* target_row,
                              const void* z_draft, float* a, float* prefix,
                              float* loss, double* numer, void* grad_draft,
                              void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Distributed normalisation of the E2E-TV loss: [review §3.2], its paragraph
 * on numerical consistency (numerators and counts are gathered separately
 * over the ranks and the loss normalised once, so the weight of a position
 * does not depend on how many positions its rank scored).
 *
 * When the branches of a batch are sharded over ranks, every rank calls
 * specopd_e2e_tv on its own branches with norm_count = the GLOBAL position
 * count (its gradient then already carries the global 1/N), the ranks sum
 * their `numer` outputs (one all-reduce of one double), and this call
 * finishes the loss on the device:
 *   loss = 1 - numer_sum / norm_count
 * numer_sum   device fp64[1]: the sum over ranks of specopd_e2e_tv's numer
 * norm_count  the global position count, > 0 (the one every rank passed)
 * loss        device fp32[1] (out)
 * loss64      device fp64[1] (out), or NULL
 */
specopd_status specopd_e2e_tv_finalize(const double* numer_sum, int64_t norm_count,
                                       float* loss, double* loss64, void* stream);

/* ------------------------------------------------------------------------ */
/* E2E-TV with the LM heads fused in front: [review §3.2(a)] (score-row
 * reading rule: the logits that score position n come from the output of
 * its predictor row, target_row[n]) and [review §3.3] (E2E-TV on those
 * logits).  The logits are formed tile by tile on the tensor cores from the
 * hidden rows and the two heads and never stored:
 *   z_t[n] = W_target h_target[target_row[n]],   z_d[n] = W_draft h_draft[n]
 * (fp32 accumulation of bf16 products; no bias, norm or temperature), then
 * a, prefix, numer, loss and grad_draft = d loss / d z_d exactly as
 * specopd_e2e_tv defines them.  Two passes over both heads (statistics,
 * overlaps); an fp32 gradient is then finished in place by one elementwise
 * pass, a bf16 gradient by a third pass over the draft head.
 */
typedef struct {
  int nbranch;               /* S*B branches                                 */
  int W;                     /* positions per branch, 1 .. 256               */
  int V;                     /* vocabulary size (rows of each head)          */
  int d_model;               /* hidden size, a multiple of 8                 */
  int rows_target;           /* rows of h_target (bounds for target_row)     */
  specopd_dtype grad_dtype;  /* grad_draft                                   */
  int compute_grad;          /* 0: skip grad_draft                           */
  int64_t norm_count;        /* divisor of the loss; 0 -> nbranch*W          */
} specopd_lmhead_tv_desc;

/* Bytes of workspace specopd_e2e_tv_lmhead needs (>= 256; depends on the
 * current device's SM count). */
size_t specopd_e2e_tv_lmhead_workspace_size(const specopd_lmhead_tv_desc* desc);

/*
 * h_target    bf16 [rows_target, d_model] target hidden rows
 * target_row  device int32[N] row of h_target scoring position n, or NULL for
 *             the identity (rows_target must then be >= N)
 * w_target    bf16 [V, d_model] target LM head (row v scores token v)
 * h_draft     bf16 [N, d_model] draft hidden rows, branch-major (b, i)
 * w_draft     bf16 [V, d_model] draft LM head
 * a, prefix   device fp32[N]; loss device fp32[1]; numer fp64[1] or NULL
 * grad_draft  [N, V] (grad_dtype) or NULL; required when compute_grad != 0;
 *             16-byte aligned with V * element size a multiple of 16
 * The four bf16 matrices must start on 16-byte boundaries.  A target_row
 * outside [0, rows_target) sets SPECOPD_DEV_ROW_RANGE and makes NaN that
 * position's a, its branch's prefix products from it on, its branch's
 * gradient rows and the loss; a bounded wait that runs out sets
 * SPECOPD_DEV_TIMEOUT.
 */
specopd_status specopd_e2e_tv_lmhead(const specopd_lmhead_tv_desc* desc,
                                     const void* h_target, const int32_t* target_row,
                                     const void* w_target, const void* h_draft,
                                     const void* w_draft, float* a, float* prefix,
                                     float* loss, double* numer, void* grad_draft,
                                     void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* E2E-TV for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is an interface addition of this library.
 *
 * Some callers cannot call cudaMalloc: code that runs inside another
 * framework's memory pool (which owns the device memory and forbids
 * allocations outside it), or code on a path where cudaMalloc's implicit
 * device-wide synchronisation is not allowed.  specopd_e2e_tv_noalloc
 * computes exactly what specopd_e2e_tv computes (same arguments, minus the
 * workspace) and allocates nothing: its scratch is a fixed array of
 * SPECOPD_E2E_TV_STATIC_SCRATCH_BYTES in the library's device image, held by
 * every GPU that loads the library until the process exits.
 *   - Size limit: returns SPECOPD_ERR_WORKSPACE, launching nothing, when the
 *     scratch of the schedule this call runs exceeds the array (8 MiB).  With
 *     16-byte aligned rows and W up to the SM count (the whole-row schedule)
 *     that is about 10 bytes per position plus a few per branch: any problem
 *     up to about 800,000 positions fits.  The slice fallback (unaligned rows) needs about
 *     24 bytes per position and vocabulary slice: about 29,000 positions at a
 *     151,936-token bf16 vocabulary.
 *   - The first call on each device resolves the array's device address
 *     (cudaGetSymbolAddress) and keeps it for the life of the process; make
 *     that first call before any stream capture, and do not use this entry
 *     point across a reset of the device (cudaDeviceReset), which can move
 *     the array.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents (each call clears what must start at zero).  Calls that
 *     overlap on the GPU -- other streams, other host threads -- race on it:
 *     serialise them.
 */
#define SPECOPD_E2E_TV_STATIC_SCRATCH_BYTES (8u << 20)

specopd_status specopd_e2e_tv_noalloc(const specopd_tv_desc* desc,
                                      const void* z_target,
                                      const int32_t* target_row,
                                      const void* z_draft, float* a, float* prefix,
                                      float* loss, double* numer, void* grad_draft,
                                      void* stream);

/* ------------------------------------------------------------------------ */
/* Testing hook: host-driven fault injection.  The paper has no counterpart.
 *
 * Lets a test make a bounded device-side wait run out on purpose, without
 * faulting, trapping or hanging the GPU, to check the library's wind-down:
 *   withhold_position  >= 0: in E2E-TV calls that use the whole-row schedule
 *                      (the default for 16-byte aligned rows and W up to the
 *                      SM count), the scorer of that supervised position never
 *                      publishes its overlap, so every position of its branch
 *                      waits for it in vain; -1 (the default) turns this off.
 *   branch_wait_limit_ns  limit of those branch waits; 0 (the default) keeps
 *                      the normal limit of 2 s.
 * When such a wait runs out the kernel sets SPECOPD_DEV_TIMEOUT, writes NaN
 * to the outputs of the affected branch (and the loss), finishes every other
 * branch normally and returns.  The setting is per device (the current one),
 * applies to calls launched after it, and stays until changed: reset it with
 * (-1, 0).  Call it only while no E2E-TV call is running on the device.
 * Returns SPECOPD_ERR_CUDA if the setting could not be written.
 */
specopd_status specopd_debug_fault_injection(int64_t withhold_position,
                                             uint64_t branch_wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* SPECOPD_H */
