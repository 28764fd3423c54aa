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
// Where the gate kernels mark the state entering chunk k as dominated by one
// token t* (Gates::dom), the operand copy of that chunk holds
// R_k = C_k - n*_k v_{t*}^T instead of C_k (formed in fp32, then rounded), the
// n handed to the output kernel is n*_k, and the output kernels add
// (n*_k^T q~) v_{t*} back in fp32.  Near rank one, h = C^T q / |n^T q| cancels
// in both numerator and denominator on rows where n^T q is small; the rank-one
// part then goes through the same fp32 product n*^T q that the denominator
// uses, and only the small remainder through bf16.
// n*_k = n_k - d_k: the state's MMA input is the bf16-rounded weighted key
// bf16(w k_{t*}) while n accumulates the unrounded w k_{t*}; d_k is that
// rounding residual of t*'s row, carried to chunk k's frame
// (dom_residual), so that numerator and denominator see the same key.
__device__ __forceinline__ float dom_residual(const Gates& g, const Problem& p, int bh, int k,
                                              int td, int i, const __nv_bfloat16* __restrict__ K) {
  const long tpad = (long)p.NC * p.L;
  const int kp = td / p.L;  // the chunk that added t* to the state
  // the weight the state kernels gave t* (same fp32 operations)
  const float w = p.key_scale * expf(g.gtot[(long)bh * p.NC + kp] + g.acol[(long)bh * tpad + td] -
                                     g.mchk[(long)bh * (p.NC + 1) + kp + 1]);
  if (!(w > 0.f)) return 0.f;
  const float x = __bfloat162float(K[((long)bh * p.T + td) * p.DK + i]) * w;
  const float r = x - __bfloat162float(__float2bfloat16_rn(x));
  // decays since: s e^{M_k - m_k} / w
  return (r / w) * p.key_scale *
         expf(g.mdom[(long)bh * p.NC + k] - g.mchk[(long)bh * (p.NC + 1) + k]);
}

// v[j] += c * x[j] for 32 consecutive value columns (v: fp32 bits from
// TMEM, x: a bf16 row, 16-byte aligned): the rank-one part (n^T q~) v_{t*} of
// a dominated chunk's inter-chunk term.
__device__ __forceinline__ void add_rank1_32(uint32_t (&v)[32], float c,
                                             const __nv_bfloat16* __restrict__ x) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x) + j);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      v[8 * j + 2 * e] = __float_as_uint(fmaf(c, f.x, __uint_as_float(v[8 * j + 2 * e])));
      v[8 * j + 2 * e + 1] =
          __float_as_uint(fmaf(c, f.y, __uint_as_float(v[8 * j + 2 * e + 1])));
    }
  }
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
// in the swizzled block layout above (DV a multiple of 64).  With `dom` (and
// the fp32 n states, the bf16 V and the problem), dominated chunks are written
// as R_k = C_k - n_k v_{t*}^T.
cudaError_t launch_states_to_operand(const float* src, __nv_bfloat16* dst, long n_bhk, int DK,
                                     int DV, cudaStream_t st, const float* n_states = nullptr,
                                     const void* V = nullptr, const int* dom = nullptr,
                                     const Problem& p = Problem{});

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
