// Tensor-core (tcgen05 / TMEM / TMA) kernels of the mLSTM forward pass.
#pragma once

#include "common.cuh"

namespace mlstm {

// Support predicates (bf16 inputs assumed).
bool tc_states_supported(const Problem& p);
bool tc_parallel_supported(const Problem& p);
bool tc_unfused_supported(const Problem& p);
bool tc_fused_supported(const Problem& p);

// Chunk states on tensor cores.  Writes the state entering every chunk as fp32
// (C_states, nullable) and/or as the bf16 operand copy read by the parallel
// kernel (Cb, nullable), the fp32 n states, and the optional final state.
cudaError_t launch_tc_states(const Problem& p, const void* K, const void* V, const float* C0,
                             const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                             float* n_states, float* C_T, float* n_T, float* m_T, cudaStream_t st);

// Intra-chunk TFLA kernel + inter-chunk term, reading bf16 chunk states.
cudaError_t launch_tc_parallel(const Problem& p, const void* Q, const void* K, const void* V,
                               Gates g, const __nv_bfloat16* Cb, const float* n_states, void* H,
                               float* n_out, float* m_out, cudaStream_t st);

// fp32 -> bf16 copy of caller-provided chunk states (n elements).
cudaError_t launch_states_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t st);

// Fused kernel: chunk state carried on chip; H and the final state.
cudaError_t launch_tc_fused(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* C0, const float* n0, Gates g, void* H, float* C_T,
                            float* n_T, float* m_T, cudaStream_t st);

// Implementations (one per kernel file).
cudaError_t launch_tc_states_impl(const Problem& p, const void* K, const void* V, const float* C0,
                                  const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                                  float* n_states, float* C_T, float* n_T, float* m_T,
                                  cudaStream_t st);
bool tc_parallel_wide_supported(const Problem& p);
cudaError_t launch_tc_parallel_wide(const Problem& p, const void* Q, const void* K, const void* V,
                                    Gates g, const __nv_bfloat16* Cb, const float* n_states,
                                    void* H, float* n_out, float* m_out, cudaStream_t st);
cudaError_t launch_tc_parallel_bf16states(const Problem& p, const void* Q, const void* K,
                                          const void* V, Gates g, const __nv_bfloat16* Cb,
                                          const float* n_states, void* H, float* n_out,
                                          float* m_out, cudaStream_t st);

}  // namespace mlstm
