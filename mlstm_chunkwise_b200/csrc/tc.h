// Tensor-core (tcgen05 / TMEM / TMA) kernels of the mLSTM forward pass.
#pragma once

#include "common.cuh"

namespace mlstm {

// Whether the tensor-core kernels support this problem (bf16 inputs assumed).
bool tc_unfused_supported(const Problem& p);
bool tc_fused_supported(const Problem& p);

// Chunk states on tensor cores: same outputs as launch_simt_states.
cudaError_t launch_tc_states(const Problem& p, const void* K, const void* V, const float* C0,
                             const float* n0, Gates g, float* C_states, float* n_states,
                             float* C_T, float* n_T, float* m_T, cudaStream_t st);

// Intra-chunk TFLA kernel + inter-chunk term: same outputs as launch_simt_parallel.
cudaError_t launch_tc_parallel(const Problem& p, const void* Q, const void* K, const void* V,
                               Gates g, const float* C_states, const float* n_states, void* H,
                               float* n_out, float* m_out, cudaStream_t st);

// Fused kernel: chunk state carried on chip; H and the final state.
cudaError_t launch_tc_fused(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* C0, const float* n0, Gates g, void* H, float* C_T,
                            float* n_T, float* m_T, cudaStream_t st);

}  // namespace mlstm
