// Shared device/host helpers for the mLSTM forward kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mlstm_fw.h"

namespace mlstm {

// ---------------------------------------------------------------------------
// Device error word.  Kernels OR a bit in here instead of trapping; the host
// reads and clears it in mlstm_last_device_error().
// ---------------------------------------------------------------------------
enum : uint32_t {
  kErrWatchdog = 1u << 0,   // a bounded wait (mbarrier / flag) ran out
  kErrBounds = 1u << 1,     // a debug bounds check failed
  kErrTmem = 1u << 2,       // TMEM allocation returned an unexpected address
};
__device__ __forceinline__ void raise_error(uint32_t* word, uint32_t bit) {
  if (word) atomicOr(word, bit);
}

// Debug bounds checks.  In a build with -DMLSTM_DEBUG_BOUNDS=1,
// MLSTM_IN_BOUNDS(p, cond) sets kErrBounds in the device error word when cond
// is false and returns cond; the caller then skips a store, or redirects a
// load to the start of its buffer, so that every barrier still completes and
// nothing traps.  In a normal build it is `true` and cond is not evaluated.
__device__ __forceinline__ bool bounds_check(uint32_t* err, bool ok) {
  if (!ok) raise_error(err, kErrBounds);
  return ok;
}
#ifdef MLSTM_DEBUG_BOUNDS
#define MLSTM_IN_BOUNDS(p, cond) ::mlstm::bounds_check((p).err, (cond))
#else
#define MLSTM_IN_BOUNDS(p, cond) true
#endif

// ---------------------------------------------------------------------------
// Problem description passed by value to every kernel.
// ---------------------------------------------------------------------------
struct Problem {
  int B, NH, T, DK, DV, L;  // L = chunk size
  int NC;                   // number of chunks = ceil(T / L)
  int BH;                   // B * NH
  int gate_sigmoid;         // 0: log i = i_pre; 1: log i = logsigmoid(i_pre)
  int no_norm;              // sigmoid variant without normaliser: h = e^{m} O (else O / max(|den|, e^{-m}))
  float key_scale;          // 1 / sqrt(DK)
  int signed_den;           // output kernels: n_out = copysign(max(|den|, e^{-m}), den)
  uint32_t* err;            // device error word (see raise_error)
  unsigned long long max_polls;  // spin limit of every bounded wait
};

// Gate workspace (all fp32, written by the gate kernels).
//   bcum [BH, NC*L]  inclusive cumulative log forget gate inside each chunk
//   acol [BH, NC*L]  column log-weight  a_s = log i_s - bcum_s (-inf on padding)
//   amax [BH, NC*L]  running max of acol inside the chunk (prefix max)
//   gtot [BH, NC]    chunk total of log forget gates (= bcum at the chunk end)
//   mchk [BH, NC+1]  state stabiliser entering chunk k (k = NC: final m)
// Dominance of the state entering each chunk (forward paths only; null
// elsewhere):
//   csum [BH, NC]    sum_s e^{acol_s - amax_{L-1}} over the chunk's tokens
//   cidx [BH, NC]    index (within the chunk) of the chunk's largest acol
//   dom  [BH, NC]    the token t* (0 <= t* < T) that holds more than half of
//                    the total gate weight of the state entering chunk k, or
//                    -1.  Such a state is close to rank one, C_k ~ n_k v_{t*}^T,
//                    and the tensor-core paths then hand it on as
//                    R_k = C_k - n*_k v_{t*}^T (see tc.h).
//   mdom [BH, NC]    the log-weight of the largest term of that state (t*'s
//                    when dom >= 0), in the unstabilised frame
//   hdom [BH]        1 if some chunk of the (b, h) has dom >= 0, else 0
struct Gates {
  float* bcum = nullptr;
  float* acol = nullptr;
  float* amax = nullptr;
  float* gtot = nullptr;
  float* mchk = nullptr;
  float* csum = nullptr;
  int* cidx = nullptr;
  int* dom = nullptr;
  float* mdom = nullptr;
  int* hdom = nullptr;  // [BH]: 1 if any chunk of the (b, h) has dom >= 0
};

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ float from_float<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// log(sigmoid(x)) without overflow in either branch.
__device__ __forceinline__ float logsigmoidf(float x) {
  return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace mlstm

// Launchers implemented in the individual .cu files.
namespace mlstm {
cudaError_t launch_gates(const Problem& p, const float* i_pre, const float* f_pre,
                         const float* m0, Gates g, cudaStream_t st);
// Backward pass (bwd.cu).  dH in the input dtype; dQ, dK, dV in the input
// dtype; di, df [BH, T], dC0 [BH, DK, DV], dn0 [BH, DK], dm0 [BH] fp32
// (the last three nullable).  `ws` holds bwd_workspace_bytes(p) bytes.
size_t bwd_workspace_bytes(const Problem& p, mlstm_dtype dt);
int bwd_launches(const Problem& p, mlstm_dtype dt);
cudaError_t launch_backward(const Problem& p, mlstm_dtype dt, const void* Q, const void* K,
                            const void* V, const float* i_pre, const float* f_pre,
                            const float* C0, const float* n0, const float* m0, const void* dH,
                            void* dQ, void* dK, void* dV, float* di, float* df, float* dC0,
                            float* dn0, float* dm0, void* ws, cudaStream_t st);
int step_launches(const Problem& p);
cudaError_t launch_step(const Problem& p, mlstm_dtype dt, const void* q, const void* k,
                        const void* v, const float* i_pre, const float* f_pre, float* C,
                        float* n, float* m, void* h, cudaStream_t st);
cudaError_t launch_simt_states(const Problem& p, mlstm_dtype dt, const void* K, const void* V,
                               const float* C0, const float* n0, Gates g, float* C_states,
                               float* n_states, float* C_T, float* n_T, float* m_T,
                               cudaStream_t st);
cudaError_t launch_simt_parallel(const Problem& p, mlstm_dtype dt, const void* Q, const void* K,
                                 const void* V, Gates g, const float* C_states,
                                 const float* n_states, void* H, float* n_out, float* m_out,
                                 cudaStream_t st, float* H32 = nullptr);
}  // namespace mlstm
