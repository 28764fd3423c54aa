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

}  // namespace mlstm
