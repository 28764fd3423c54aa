// Tensor-core (tcgen05 / TMEM / TMA) kernels of the mLSTM forward pass.
#pragma once

#include "common.cuh"

namespace mlstm {

// Layout of the bf16 operand copy of the chunk states (internal to the
// tensor-core path).  For every (b, h, chunk) index bhk and every 64-column
// block vb of DV there is a [DK][64] block of 128-byte rows, and row dk holds
// its 16-byte chunk j at position j ^ (dk & 7): byte for byte the shared-memory
// image of an MN-major operand tile with the 128-byte swizzle.  A run of rows
// that starts at a multiple of 8 therefore moves between global and shared
// memory with one untiled bulk copy, in either direction.
__host__ __device__ inline size_t cb_block_row(long bhk, int vb, int dk, int DK, int n_vb) {
  return (((size_t)bhk * n_vb + vb) * DK + dk) * 64;  // element offset of row dk of the block
}

// Support predicates (bf16 inputs assumed).
bool tc_states_supported(const Problem& p);
bool tc_parallel_supported(const Problem& p);
bool tc_unfused_supported(const Problem& p);
bool tc_fused_supported(const Problem& p);

// Chunk states on tensor cores.  Writes the state entering every chunk as fp32
// (C_states, nullable) and/or as the bf16 operand copy read by the parallel
// kernel (Cb, nullable), the fp32 n states, and the optional final state.
// With too few (b, h, d_v tile) units to fill the GPU the chunk sequences are
// split into tc_states_segments(p) segments; seg_ws (tc_states_segment_floats(p)
// floats, nullable when that is 0) holds the segments' end states between the
// recurrence and the fix-up launch.
cudaError_t launch_tc_states(const Problem& p, const void* K, const void* V, const float* C0,
                             const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                             float* n_states, float* C_T, float* n_T, float* m_T, float* seg_ws,
                             cudaStream_t st);
int tc_states_dvt(const Problem& p);
int tc_states_segments(const Problem& p);
size_t tc_states_segment_floats(const Problem& p);
inline int tc_states_launches(const Problem& p) { return tc_states_segments(p) > 1 ? 2 : 1; }

// Intra-chunk TFLA kernel + inter-chunk term, reading bf16 chunk states.
cudaError_t launch_tc_parallel(const Problem& p, const void* Q, const void* K, const void* V,
                               Gates g, const __nv_bfloat16* Cb, const float* n_states, void* H,
                               float* n_out, float* m_out, cudaStream_t st);

// Caller-provided fp32 chunk states [BH * NC][DK][DV] -> the bf16 operand copy
// in the swizzled block layout above (DV a multiple of 64).
cudaError_t launch_states_to_operand(const float* src, __nv_bfloat16* dst, long n_bhk, int DK,
                                     int DV, cudaStream_t st);

// Fused kernel: chunk state carried on chip; H and the final state.
cudaError_t launch_tc_fused(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* C0, const float* n0, Gates g, void* H, float* C_T,
                            float* n_T, float* m_T, cudaStream_t st);

// Failure-detection self-test (selftest.cu): one bounded wait that nothing
// satisfies; it sets the watchdog bit and its site in *err and returns.
cudaError_t launch_watchdog_selftest(uint32_t* err, unsigned long long max_polls,
                                     cudaStream_t st);

// Implementations (one per kernel file).
cudaError_t launch_tc_states_impl(const Problem& p, const void* K, const void* V, const float* C0,
                                  const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                                  float* n_states, float* C_T, float* n_T, float* m_T,
                                  float* seg_ws, cudaStream_t st);
bool tc_parallel_wide_supported(const Problem& p);
cudaError_t launch_tc_parallel_wide(const Problem& p, const void* Q, const void* K, const void* V,
                                    Gates g, const __nv_bfloat16* Cb, const float* n_states,
                                    void* H, float* n_out, float* m_out, cudaStream_t st);
cudaError_t launch_tc_parallel_bf16states(const Problem& p, const void* Q, const void* K,
                                          const void* V, Gates g, const __nv_bfloat16* Cb,
                                          const float* n_states, void* H, float* n_out,
                                          float* m_out, cudaStream_t st);

}  // namespace mlstm
