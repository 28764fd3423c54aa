// Backward pass on tensor cores (tc_bwd.cu): declarations shared with bwd.cu.
#pragma once

#include "tc.h"

namespace mlstm {

// Backward gradients on tensor cores (tc_bwd.cu), for a problem chunked in
// 128-token chunks (pb.L = 128) with bf16 Q, K, V.  From du~ (bf16, dU16), da~,
// the forward's chunk states (bf16 operand copy Cb, fp32 n_states) and the
// reverse states (G~ as a bf16 operand copy Gb in the same block layout,
// indexed bh (NC + 1) + k, and fp32 g~) it writes dQ, dK, dV (bf16) and adds
// q.dq and k.dk into qdq and kdk.  sq: tc_bwd_square_elems(pb) bf16 scratch.
bool tc_bwd_supported(const Problem& pb);
size_t tc_bwd_square_elems(const Problem& pb);
cudaError_t launch_tc_bwd(const Problem& pb, const void* Q, const void* K, const void* V,
                          const __nv_bfloat16* dU16, Gates g, const float* dA,
                          const float* n_states, const float* g_states, const __nv_bfloat16* Cb,
                          const __nv_bfloat16* Gb, __nv_bfloat16* sq, void* dQ, void* dK,
                          void* dV, float* qdq, float* kdk, cudaStream_t st);
constexpr int kTcBwdLaunches = 4;
// Reverse states on tensor cores (tc_bwd.cu): the per-chunk g~ increments u
// (scratch [BH, NC, DK] fp32), then the recurrence G~_k = decay_k G~_{k+1} +
// Q_k^T dUr_k (dUr16: du~ with rows scaled by e^{m_k - mu_t}, bf16) writing Gb
// (bf16 operand copy of every G~_k, NC + 1 per head), g_states (fp32) and
// dC0 = G~_0 (fp32).
cudaError_t launch_tc_bwd_states(const Problem& pb, const void* Q, const __nv_bfloat16* dUr16,
                                 Gates g, const float* dA, float* u, __nv_bfloat16* Gb,
                                 float* g_states, float* dC0, cudaStream_t st);
constexpr int kTcBwdStateLaunches = 2;

// Training pair (bwd.cu), for the shapes of the tensor-core backward
// (train_supported): a forward at 128-token chunks that keeps, in a caller
// buffer of train_saved_bytes, the bf16 chunk states, the n states and per
// token the signed denominator and the stabiliser; and the backward that
// takes that buffer and the forward's H instead of recomputing them.
bool train_supported(const Problem& p, mlstm_dtype dt);
size_t train_saved_bytes(const Problem& p);
size_t fw_train_workspace_bytes(const Problem& p);
size_t bw_saved_workspace_bytes(const Problem& p);
int fw_train_launches(const Problem& p);
int bw_saved_launches(const Problem& p);
cudaError_t launch_fw_train(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* i_pre, const float* f_pre, const float* C0,
                            const float* n0, const float* m0, void* H, float* C_T, float* n_T,
                            float* m_T, void* saved, void* ws, cudaStream_t st);
cudaError_t launch_bw_saved(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* i_pre, const float* f_pre, const float* C0,
                            const float* n0, const float* m0, const void* H, const void* saved,
                            const void* dH, void* dQ, void* dK, void* dV, float* di, float* df,
                            float* dC0, float* dn0, float* dm0, void* ws, cudaStream_t st);

}  // namespace mlstm
