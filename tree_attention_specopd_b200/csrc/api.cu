// C ABI of the SpecOPD B200 library: argument validation and dispatch.
//
// Single translation unit (the kernel sources are included below) so that
// the per-device status word is one symbol.  No function here allocates
// device memory; scratch comes from the caller's workspace.
#include <math.h>
#include <string.h>

#include <vector>

#include "common.cuh"
#include "kernels.h"

#include "e2e_tv.cu"
#include "rope.cu"
#include "tree_attn_simt.cu"
#include "tree_attn_sm100.cu"
#include "lmhead_tv.cu"
#include "tree_build.cu"

using namespace specopd;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The library's kernels are built for sm_100a only.
specopd_status check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SPECOPD_ERR_NO_DEVICE; }
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return SPECOPD_ERR_NO_DEVICE;
  return SPECOPD_OK;
}

specopd_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPECOPD_OK;
  cudaGetLastError();
  return SPECOPD_ERR_CUDA;
}

// Validates cu_trunk_host and fills the kernel-parameter copy.
specopd_status read_cu(int S, const int32_t* cu_host, CuTrunk& cu) {
  if (S < 1 || S > kMaxSeq || !cu_host) return SPECOPD_ERR_INVALID_ARG;
  if (cu_host[0] != 0) return SPECOPD_ERR_INVALID_ARG;
  cu.S = S;
  cu.T_max = 0;
  for (int s = 0; s <= S; ++s) cu.cu[s] = cu_host[s];
  for (int s = 0; s < S; ++s) {
    const long long T = (long long)cu_host[s + 1] - cu_host[s];
    if (T < 1) return SPECOPD_ERR_INVALID_ARG;
    if (T > cu.T_max) cu.T_max = (int)T;
  }
  cu.T_tot = cu_host[S];
  return SPECOPD_OK;
}

void rope_theta(int D, float base, double* theta) {
  for (int k = 0; k < D / 2; ++k) theta[k] = pow((double)base, -2.0 * k / (double)D);
}

size_t elt(specopd_dtype d) { return d == SPECOPD_BF16 ? 2 : 4; }

struct AttnWs {
  size_t q_off, k_off, tail_off, total;
};

// fp32 (SIMT kernel): rotated copies of the branch q and k, rotated once by
// a RoPE launch.  bf16 (tensor-core kernel): the split-KV partials only (the
// kernel rotates q and k in shared memory).
// Trunk prefill: fp32 keeps the rotated trunk queries, bf16 the split-KV
// partials.
AttnWs attn_ws_layout(const AttnProblem& p, bool prefill = false) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  AttnWs w;
  w.q_off = 0;
  if (p.dtype == SPECOPD_BF16) {
    w.k_off = 0;
    w.tail_off = 0;
    w.total = up(attn_sm100_workspace(p, prefill));
  } else if (prefill) {
    w.k_off = 0;
    w.tail_off = up((size_t)p.T_tot * p.Hq * p.D * elt(p.dtype));
    w.total = w.tail_off;
  } else {
    w.k_off = up((size_t)p.R * p.Hq * p.D * elt(p.dtype));
    w.tail_off = up(w.k_off + (size_t)p.R * p.Hkv * p.D * elt(p.dtype));
    w.total = w.tail_off;
  }
  if (w.total < 256) w.total = 256;
  return w;
}

specopd_status attn_problem(const specopd_attn_desc* d, const CuTrunk& cu, AttnProblem& p) {
  if (!d) return SPECOPD_ERR_INVALID_ARG;
  if (d->S != cu.S || d->B < 1 || d->W < 1 || d->Hq < 1 || d->Hkv < 1 || d->D < 2)
    return SPECOPD_ERR_INVALID_ARG;
  if (d->Hq % d->Hkv) return SPECOPD_ERR_INVALID_ARG;
  if (!(d->rope_base > 0.f) || d->softmax_scale < 0.f) return SPECOPD_ERR_INVALID_ARG;
  if (d->dtype != SPECOPD_F32 && d->dtype != SPECOPD_BF16) return SPECOPD_ERR_INVALID_ARG;
  if (d->D != 64 && d->D != 128) return SPECOPD_ERR_UNSUPPORTED;
  const int G = d->Hq / d->Hkv;
  if (d->dtype == SPECOPD_F32 && G > 32) return SPECOPD_ERR_UNSUPPORTED;
  if (d->dtype == SPECOPD_BF16 && G > 128) return SPECOPD_ERR_UNSUPPORTED;
  const long long R = (long long)d->S * d->B * (d->W - 1);
  if (R > (1ll << 30)) return SPECOPD_ERR_UNSUPPORTED;
  p.S = d->S; p.B = d->B; p.W = d->W; p.Hq = d->Hq; p.Hkv = d->Hkv; p.D = d->D; p.G = G;
  p.R = (int)R; p.T_tot = cu.T_tot; p.T_max = cu.T_max;
  p.scale = d->softmax_scale > 0.f ? d->softmax_scale : (float)(1.0 / sqrt((double)d->D));
  p.dtype = d->dtype;
  return SPECOPD_OK;
}

specopd_status tv_problem(const specopd_tv_desc* d, TVProblem& p) {
  if (!d) return SPECOPD_ERR_INVALID_ARG;
  if (d->nbranch < 1 || d->W < 1 || d->V < 1 || d->rows_target < 1) return SPECOPD_ERR_INVALID_ARG;
  if (d->logit_dtype != SPECOPD_F32 && d->logit_dtype != SPECOPD_BF16) return SPECOPD_ERR_INVALID_ARG;
  if (d->grad_dtype != SPECOPD_F32 && d->grad_dtype != SPECOPD_BF16) return SPECOPD_ERR_INVALID_ARG;
  if (d->norm_count < 0) return SPECOPD_ERR_INVALID_ARG;
  const long long N = (long long)d->nbranch * d->W;
  if (N > (1ll << 30)) return SPECOPD_ERR_UNSUPPORTED;
  p.nbranch = d->nbranch; p.W = d->W; p.V = d->V; p.N = (int)N; p.rows_target = d->rows_target;
  p.logit_dtype = d->logit_dtype; p.grad_dtype = d->grad_dtype;
  p.compute_grad = d->compute_grad ? 1 : 0;
  p.norm_count = d->norm_count > 0 ? (double)d->norm_count : (double)N;
  // Slices per row (each CTA holds one slice of both rows in shared memory).
  if (tv_slice_count(p) > kTVMaxSlices || d->W > kTVMaxW) return SPECOPD_ERR_UNSUPPORTED;
  return SPECOPD_OK;
}

// E2E-TV after host validation.  The workspace must hold
// specopd_e2e_tv_workspace_size bytes, or, with exact_need, what the schedule
// picked for these pointers needs (the allocation-free entry point, whose
// scratch is fixed).
specopd_status e2e_tv_checked(const specopd_tv_desc* d, const void* z_target,
                              const int32_t* target_row, const void* z_draft, float* a,
                              float* prefix, float* loss, double* numer, void* grad_draft,
                              void* workspace, size_t ws_bytes, void* stream, bool exact_need) {
  TVProblem p;
  specopd_status s = tv_problem(d, p);
  if (s != SPECOPD_OK) return s;
  if (!z_target || !z_draft || !a || !prefix || !loss) return SPECOPD_ERR_INVALID_ARG;
  if (p.compute_grad && !grad_draft) return SPECOPD_ERR_INVALID_ARG;
  if (!target_row && p.rows_target < p.N) return SPECOPD_ERR_INVALID_ARG;
  if (!workspace) return SPECOPD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SPECOPD_ERR_UNSUPPORTED;
  s = check_device();
  if (s != SPECOPD_OK) return s;
  void* grad = p.compute_grad ? grad_draft : nullptr;
  const size_t need = exact_need ? tv_workspace_for_call(p, z_target, z_draft, grad) : tv_workspace(p);
  if (ws_bytes < need) return SPECOPD_ERR_WORKSPACE;
  cudaError_t e = launch_e2e_tv(p, z_target, target_row, z_draft, a, prefix, loss, numer, grad,
                                workspace, ws_bytes, as_stream(stream));
  if (e == cudaErrorInvalidConfiguration) { cudaGetLastError(); return SPECOPD_ERR_UNSUPPORTED; }
  return cuda_status(e);
}

specopd_status lmtv_problem(const specopd_lmhead_tv_desc* d, LmtvProblem& p) {
  if (!d) return SPECOPD_ERR_INVALID_ARG;
  if (d->nbranch < 1 || d->W < 1 || d->V < 1 || d->d_model < 1 || d->rows_target < 1)
    return SPECOPD_ERR_INVALID_ARG;
  if (d->grad_dtype != SPECOPD_F32 && d->grad_dtype != SPECOPD_BF16) return SPECOPD_ERR_INVALID_ARG;
  if (d->norm_count < 0) return SPECOPD_ERR_INVALID_ARG;
  // rows of the hidden states and heads must be whole 16-byte units (TMA)
  if (d->d_model % 8 != 0 || d->W > 256) return SPECOPD_ERR_UNSUPPORTED;
  const long long N = (long long)d->nbranch * d->W;
  if (N > (1ll << 30)) return SPECOPD_ERR_UNSUPPORTED;
  p.nbranch = d->nbranch; p.W = d->W; p.V = d->V; p.N = (int)N; p.d = d->d_model;
  p.rows_target = d->rows_target;
  p.grad_dtype = d->grad_dtype;
  p.compute_grad = d->compute_grad ? 1 : 0;
  p.norm_count = d->norm_count > 0 ? (double)d->norm_count : (double)N;
  return SPECOPD_OK;
}

}  // namespace

extern "C" {

const char* specopd_status_string(int s) {
  switch (s) {
    case SPECOPD_OK: return "SPECOPD_OK";
    case SPECOPD_ERR_INVALID_ARG: return "SPECOPD_ERR_INVALID_ARG";
    case SPECOPD_ERR_UNSUPPORTED: return "SPECOPD_ERR_UNSUPPORTED";
    case SPECOPD_ERR_WORKSPACE: return "SPECOPD_ERR_WORKSPACE";
    case SPECOPD_ERR_CUDA: return "SPECOPD_ERR_CUDA";
    case SPECOPD_ERR_TIMEOUT: return "SPECOPD_ERR_TIMEOUT";
    case SPECOPD_ERR_NO_DEVICE: return "SPECOPD_ERR_NO_DEVICE";
    default: return "SPECOPD_ERR_UNKNOWN";
  }
}

int specopd_version(void) { return 10000; }

specopd_status specopd_get_device_status(uint32_t* host_out, void* stream) {
  if (!host_out) return SPECOPD_ERR_INVALID_ARG;
  specopd_status ds = check_device();
  if (ds != SPECOPD_OK) return ds;
  cudaStream_t st = as_stream(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_status(cudaErrorUnknown);
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, specopd::g_status, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_status(e);
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(specopd::g_status, &zero, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_status(e);
  *host_out = v;
  return SPECOPD_OK;
}

specopd_status specopd_tree_build(int S, const int32_t* cu_trunk_host, const int32_t* anchors,
                                  int B, int W, int32_t* parent, int32_t* sem_pos,
                                  int32_t* score_row, void* stream) {
  CuTrunk cu;
  specopd_status s = read_cu(S, cu_trunk_host, cu);
  if (s != SPECOPD_OK) return s;
  if (B < 1 || W < 1 || !anchors) return SPECOPD_ERR_INVALID_ARG;
  if ((long long)S * B * W > (1ll << 30)) return SPECOPD_ERR_UNSUPPORTED;
  if (!parent && !sem_pos && !score_row) return SPECOPD_OK;
  s = check_device();
  if (s != SPECOPD_OK) return s;
  return cuda_status(launch_tree_build(cu, anchors, B, W, parent, sem_pos, score_row, as_stream(stream)));
}

specopd_status specopd_rope_apply(const specopd_rope_desc* d, void* x, const int32_t* pos, int n,
                                  int H, void* stream) {
  if (!d || n < 0 || H < 1) return SPECOPD_ERR_INVALID_ARG;
  if (d->D < 2 || d->D > 256 || (d->D & 1)) return SPECOPD_ERR_INVALID_ARG;
  if (!(d->rope_base > 0.f)) return SPECOPD_ERR_INVALID_ARG;
  if (d->dtype != SPECOPD_F32 && d->dtype != SPECOPD_BF16) return SPECOPD_ERR_INVALID_ARG;
  if (n == 0) return SPECOPD_OK;
  if (!x || !pos) return SPECOPD_ERR_INVALID_ARG;
  specopd_status s = check_device();
  if (s != SPECOPD_OK) return s;
  double theta[128];
  rope_theta(d->D, d->rope_base, theta);
  return cuda_status(launch_rope(d->dtype, x, x, pos, n, H, d->D, theta, as_stream(stream)));
}

size_t specopd_tree_attn_workspace_size(const specopd_attn_desc* d, const int32_t* cu_trunk_host) {
  if (!d) return 0;
  CuTrunk cu;
  if (read_cu(d->S, cu_trunk_host, cu) != SPECOPD_OK) return 0;
  AttnProblem p;
  if (attn_problem(d, cu, p) != SPECOPD_OK) return 0;
  return attn_ws_layout(p).total;
}

specopd_status specopd_tree_attn(const specopd_attn_desc* d, const void* q_br, const void* k_br,
                                 const void* v_br, const void* k_tr, const void* v_tr,
                                 const int32_t* cu_trunk, const int32_t* cu_trunk_host,
                                 const int32_t* anchors, const int32_t* sem_pos, void* out,
                                 float* lse, void* workspace, size_t ws_bytes, void* stream) {
  if (!d) return SPECOPD_ERR_INVALID_ARG;
  CuTrunk cu;
  specopd_status s = read_cu(d->S, cu_trunk_host, cu);
  if (s != SPECOPD_OK) return s;
  AttnProblem p;
  s = attn_problem(d, cu, p);
  if (s != SPECOPD_OK) return s;
  if (p.R == 0) return SPECOPD_OK;
  // bf16: the branch keys of a query tile (its rows and the earlier nodes of
  // its first branch, floor(128 / G) + W - 2 rows at most) are rotated in the
  // kernel's K ring before the first MMA reads them: three 64-key tiles at most.
  if (p.dtype == SPECOPD_BF16 && (128 / p.G + p.W - 2 + 63) / 64 > 3) return SPECOPD_ERR_UNSUPPORTED;
  if (!q_br || !k_br || !v_br || !k_tr || !v_tr || !cu_trunk || !anchors || !sem_pos || !out)
    return SPECOPD_ERR_INVALID_ARG;
  const AttnWs L = attn_ws_layout(p);
  if (!workspace || ws_bytes < L.total) return SPECOPD_ERR_WORKSPACE;
  if (p.dtype == SPECOPD_BF16) {
    if (!aligned16(q_br) || !aligned16(k_br) || !aligned16(v_br) || !aligned16(k_tr) ||
        !aligned16(v_tr) || !aligned16(out) || !aligned16(workspace))
      return SPECOPD_ERR_UNSUPPORTED;
  }
  s = check_device();
  if (s != SPECOPD_OK) return s;
  cudaStream_t st = as_stream(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  double theta[128];
  rope_theta(p.D, d->rope_base, theta);
  cudaError_t e;
  if (p.dtype == SPECOPD_F32) {
    // Branch q/k rotated once at their semantic positions (sem_pos of the
    // branch nodes); every key block of a row reuses the rotated copy.
    void* q_rot = ws + L.q_off;
    void* k_rot = ws + L.k_off;
    e = launch_rope2(p.dtype, q_br, q_rot, p.Hq, k_br, k_rot, p.Hkv, sem_pos + p.T_tot, p.R, p.D,
                     theta, st);
    if (e != cudaSuccess) return cuda_status(e);
    e = launch_attn_simt_f32(p, (const float*)q_rot, (const float*)k_rot, (const float*)v_br,
                             (const float*)k_tr, (const float*)v_tr, cu_trunk, anchors,
                             (float*)out, lse, st, false);
  } else {
    e = launch_attn_sm100(p, q_br, k_br, v_br, k_tr, v_tr, cu_trunk, anchors, sem_pos + p.T_tot,
                          theta, out, lse, ws + L.tail_off, L.total - L.tail_off, st, false);
  }
  return cuda_status(e);
}

size_t specopd_trunk_prefill_workspace_size(const specopd_attn_desc* d,
                                            const int32_t* cu_trunk_host) {
  if (!d) return 0;
  CuTrunk cu;
  if (read_cu(d->S, cu_trunk_host, cu) != SPECOPD_OK) return 0;
  AttnProblem p;
  if (attn_problem(d, cu, p) != SPECOPD_OK) return 0;
  return attn_ws_layout(p, true).total;
}

specopd_status specopd_trunk_prefill(const specopd_attn_desc* d, const void* q_tr, void* k_tr,
                                     const void* v_tr, const int32_t* cu_trunk,
                                     const int32_t* cu_trunk_host, void* out, float* lse,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (!d) return SPECOPD_ERR_INVALID_ARG;
  CuTrunk cu;
  specopd_status s = read_cu(d->S, cu_trunk_host, cu);
  if (s != SPECOPD_OK) return s;
  AttnProblem p;
  s = attn_problem(d, cu, p);
  if (s != SPECOPD_OK) return s;
  if (!q_tr || !k_tr || !v_tr || !cu_trunk || !out) return SPECOPD_ERR_INVALID_ARG;
  const AttnWs L = attn_ws_layout(p, true);
  if (!workspace || ws_bytes < L.total) return SPECOPD_ERR_WORKSPACE;
  if (p.dtype == SPECOPD_BF16) {
    if (!aligned16(q_tr) || !aligned16(k_tr) || !aligned16(v_tr) || !aligned16(out) ||
        !aligned16(workspace))
      return SPECOPD_ERR_UNSUPPORTED;
  }
  s = check_device();
  if (s != SPECOPD_OK) return s;
  cudaStream_t st = as_stream(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  double theta[128];
  rope_theta(p.D, d->rope_base, theta);
  // The K cache: trunk keys rotated in place at their positions.
  cudaError_t e = launch_rope_trunk(p.dtype, k_tr, k_tr, cu_trunk, p.S, p.T_tot, p.Hkv, p.D,
                                    theta, st);
  if (e != cudaSuccess) return cuda_status(e);
  if (p.dtype == SPECOPD_F32) {
    void* q_rot = ws + L.q_off;
    e = launch_rope_trunk(p.dtype, q_tr, q_rot, cu_trunk, p.S, p.T_tot, p.Hq, p.D, theta, st);
    if (e != cudaSuccess) return cuda_status(e);
    e = launch_attn_simt_f32(p, (const float*)q_rot, nullptr, nullptr, (const float*)k_tr,
                             (const float*)v_tr, cu_trunk, nullptr, (float*)out, lse, st, true);
  } else {
    e = launch_attn_sm100(p, q_tr, k_tr, v_tr, k_tr, v_tr, cu_trunk, nullptr, nullptr, theta, out,
                          lse, ws + L.tail_off, L.total - L.tail_off, st, true);
  }
  return cuda_status(e);
}

size_t specopd_e2e_tv_workspace_size(const specopd_tv_desc* d) {
  TVProblem p;
  if (tv_problem(d, p) != SPECOPD_OK) return 0;
  size_t w = tv_workspace(p);
  return w < 256 ? 256 : w;
}

specopd_status specopd_e2e_tv(const specopd_tv_desc* d, const void* z_target,
                              const int32_t* target_row, const void* z_draft, float* a,
                              float* prefix, float* loss, double* numer, void* grad_draft,
                              void* workspace, size_t ws_bytes, void* stream) {
  return e2e_tv_checked(d, z_target, target_row, z_draft, a, prefix, loss, numer, grad_draft,
                        workspace, ws_bytes, stream, false);
}

specopd_status specopd_e2e_tv_finalize(const double* numer_sum, int64_t norm_count,
                                       float* loss, double* loss64, void* stream) {
  if (!numer_sum || !loss || norm_count <= 0) return SPECOPD_ERR_INVALID_ARG;
  specopd_status s = check_device();
  if (s != SPECOPD_OK) return s;
  return cuda_status(launch_tv_finalize(numer_sum, (double)norm_count, loss, loss64,
                                        as_stream(stream)));
}

specopd_status specopd_debug_fault_injection(int64_t withhold_position,
                                             uint64_t branch_wait_limit_ns) {
  if (withhold_position < -1) return SPECOPD_ERR_INVALID_ARG;
  specopd_status s = check_device();
  if (s != SPECOPD_OK) return s;
  const FaultInject f = {(long long)withhold_position, (unsigned long long)branch_wait_limit_ns};
  return cuda_status(cudaMemcpyToSymbol(specopd::g_inject, &f, sizeof(f)));
}

size_t specopd_e2e_tv_lmhead_workspace_size(const specopd_lmhead_tv_desc* d) {
  LmtvProblem p;
  if (lmtv_problem(d, p) != SPECOPD_OK) return 0;
  const size_t w = lmtv_workspace(p);
  return w < 256 ? 256 : w;
}

specopd_status specopd_e2e_tv_lmhead(const specopd_lmhead_tv_desc* d, const void* h_target,
                                     const int32_t* target_row, const void* w_target,
                                     const void* h_draft, const void* w_draft, float* a,
                                     float* prefix, float* loss, double* numer, void* grad_draft,
                                     void* workspace, size_t ws_bytes, void* stream) {
  LmtvProblem p;
  specopd_status s = lmtv_problem(d, p);
  if (s != SPECOPD_OK) return s;
  if (!h_target || !w_target || !h_draft || !w_draft || !a || !prefix || !loss)
    return SPECOPD_ERR_INVALID_ARG;
  if (p.compute_grad && !grad_draft) return SPECOPD_ERR_INVALID_ARG;
  if (!target_row && p.rows_target < p.N) return SPECOPD_ERR_INVALID_ARG;
  if (!aligned16(h_target) || !aligned16(w_target) || !aligned16(h_draft) || !aligned16(w_draft))
    return SPECOPD_ERR_UNSUPPORTED;
  const size_t gs = p.grad_dtype == SPECOPD_BF16 ? 2 : 4;
  if (p.compute_grad && (!aligned16(grad_draft) || ((size_t)p.V * gs) % 16 != 0))
    return SPECOPD_ERR_UNSUPPORTED;
  if (!workspace) return SPECOPD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SPECOPD_ERR_UNSUPPORTED;
  s = check_device();
  if (s != SPECOPD_OK) return s;
  if (ws_bytes < lmtv_workspace(p)) return SPECOPD_ERR_WORKSPACE;
  return cuda_status(launch_lmtv(p, h_target, target_row, w_target, h_draft, w_draft, a, prefix,
                                 loss, numer, p.compute_grad ? grad_draft : nullptr, workspace,
                                 ws_bytes, as_stream(stream)));
}

}  // extern "C"

// Entry point without a workspace argument (library-owned scratch).
#include "e2e_tv_noalloc.cu"
