// Internal launchers of the SpecOPD B200 library (host side, C++ linkage).
// The exported C ABI lives in api.cu; these are the per-kernel launch
// routines it dispatches to after validating arguments.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/specopd.h"

namespace specopd {

constexpr int kMaxSeq = 1024;  // sequences per call (cu_trunk travels as a kernel parameter)

struct CuTrunk {
  int S;
  int T_tot;
  int T_max;
  int cu[kMaxSeq + 1];
};

// ---- tree build
cudaError_t launch_tree_build(const CuTrunk& cu, const int32_t* anchors, int B, int W,
                              int32_t* parent, int32_t* sem_pos, int32_t* score_row,
                              cudaStream_t st);

// ---- RoPE: y[t,h,:] = rope(x[t,h,:], pos[t]) for t < n (x may equal y).
// theta: host array of D/2 frequencies base^(-2k/D) in double precision.
cudaError_t launch_rope(specopd_dtype dt, const void* x, void* y, const int32_t* pos, int n, int H,
                        int D, const double* theta_host, cudaStream_t st);
// Trunk rows rotated at their position within their sequence (row t of
// sequence s sits at t - cu[s]); cu_trunk is the device copy.
cudaError_t launch_rope_trunk(specopd_dtype dt, const void* x, void* y, const int32_t* cu_trunk,
                              int S, int n, int H, int D, const double* theta_host,
                              cudaStream_t st);
// Two tensors (H0 and H1 heads) rotated at the same positions in one launch.
cudaError_t launch_rope2(specopd_dtype dt, const void* x0, void* y0, int H0, const void* x1,
                         void* y1, int H1, const int32_t* pos, int n, int D,
                         const double* theta_host, cudaStream_t st);

// ---- tree attention, SIMT (fp32 workloads)
struct AttnProblem {
  int S, B, W, Hq, Hkv, D, G, R, T_tot, T_max;
  float scale;  // softmax scale
  specopd_dtype dtype;
};
// prefill: q_rot is the rotated trunk queries [T_tot, Hq, D] and every trunk
// row attends causally within its sequence (k_rot, v_br, anchors unused).
cudaError_t launch_attn_simt_f32(const AttnProblem& p, const float* q_rot, const float* k_rot,
                                 const float* v_br, const float* k_tr, const float* v_tr,
                                 const int32_t* cu_trunk, const int32_t* anchors, float* out,
                                 float* lse, cudaStream_t st, bool prefill);

// ---- tree attention, tcgen05/TMEM/TMA (bf16 workloads)
size_t attn_sm100_workspace(const AttnProblem& p, bool prefill);
// q_br / k_br are NOT rotated: the kernel rotates them at pos_br (the
// semantic positions of the branch rows) with frequencies theta[D/2].
// prefill: q_br is the trunk queries [T_tot, Hq, D] (rotated in the kernel at
// their positions within their sequence), k_tr the rotated K cache, and the
// output covers every trunk row (causal within each sequence); k_br, v_br,
// anchors and pos_br are unused.
cudaError_t launch_attn_sm100(const AttnProblem& p, const void* q_br, const void* k_br,
                              const void* v_br, const void* k_tr, const void* v_tr,
                              const int32_t* cu_trunk, const int32_t* anchors,
                              const int32_t* pos_br, const double* theta, void* out,
                              float* lse, void* ws, size_t ws_bytes, cudaStream_t st,
                              bool prefill);

// ---- E2E-TV
struct TVProblem {
  int nbranch, W, V, N, rows_target;
  specopd_dtype logit_dtype, grad_dtype;
  int compute_grad;
  double norm_count;
};
size_t tv_workspace(const TVProblem& p);
// Workspace bytes of the schedule launch_e2e_tv picks for these pointers on
// the current device (at most tv_workspace(p)).
size_t tv_workspace_for_call(const TVProblem& p, const void* z_target, const void* z_draft,
                             const void* grad);
int tv_slice_count(const TVProblem& p);
cudaError_t launch_tv_finalize(const double* numer_sum, double norm, float* loss, double* loss64,
                               cudaStream_t st);
cudaError_t launch_e2e_tv(const TVProblem& p, const void* z_target, const int32_t* target_row,
                          const void* z_draft, float* a, float* prefix, float* loss, double* numer,
                          void* grad, void* ws, size_t ws_bytes, cudaStream_t st);

// E2E-TV with the LM heads fused in front (lmhead_tv.cu): hidden rows and
// heads in bf16, N = nbranch * W positions, d = hidden size.
struct LmtvProblem {
  int nbranch, W, V, N, d, rows_target;
  specopd_dtype grad_dtype;
  int compute_grad;
  double norm_count;
};
size_t lmtv_workspace(const LmtvProblem& p);
cudaError_t launch_lmtv(const LmtvProblem& p, const void* h_target, const int32_t* target_row,
                        const void* w_target, const void* h_draft, const void* w_draft, float* a,
                        float* prefix, float* loss, double* numer, void* grad, void* ws,
                        size_t ws_bytes, cudaStream_t st);

}  // namespace specopd
