// SIMT (CUDA-core, fp32 FFMA) kernels for the chunkwise mLSTM forward pass.
//
// This is the fp32-input path (fp32 arithmetic throughout, tight tolerance)
// and a second, independent GPU implementation for the bf16 tensor-core
// kernels to be compared against.  It follows the same chunkwise split as
// "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
// (abstract): an inter-chunk state recurrence plus an intra-chunk parallel
// part, and the two-launch structure of flash-xlstm-exp 0.1.0 ("Upgrade
// roadmap" item 2: chunk states materialised in HBM between a recurrent and a
// parallel kernel; "Usage": the parallel kernel consumes matC_states,
// vecN_states, scaMinter_states).
//
// States kernel, per (b, h) and 64x64 tile of C = [DK, DV]:
//   C_states[k] = state entering chunk k (frame mchk[k]);
//   C_{k+1} = e^{g_k + m_k - m_{k+1}} C_k
//           + sum_r (s k_r e^{g_k + acol_r - m_{k+1}}) v_r^T,  n likewise.
// Parallel kernel, per (b, h), 64 query rows and 64 value columns:
//   mu_r  = max(m_k, amax_r)            (row stabiliser minus bcum_r)
//   num_r = e^{m_k - mu_r} C_k^T q_r + sum_{s<=r} e^{acol_s - mu_r} (s q_r.k_s) v_s
//   den_r = e^{m_k - mu_r} n_k.q_r   + sum_{s<=r} e^{acol_s - mu_r} (s q_r.k_s)
//   h_r   = num_r / max(|den_r|, e^{-(bcum_r + mu_r)})
// Every exponent above is <= 0 by construction of the stabilisers.
#include <math.h>

#include "common.cuh"

namespace mlstm {
namespace {

constexpr int kTile = 64;
constexpr int kThreads = 256;

template <typename TIn>
__device__ __forceinline__ float load_or_zero(const TIn* base, long idx, bool ok) {
  return ok ? to_float(base[idx]) : 0.f;
}

template <typename TIn>
__global__ void __launch_bounds__(kThreads)
simt_states_kernel(Problem p, const TIn* __restrict__ K, const TIn* __restrict__ V,
                   const float* __restrict__ C0, const float* __restrict__ n0, Gates g,
                   float* __restrict__ C_states, float* __restrict__ n_states,
                   float* __restrict__ C_T, float* __restrict__ n_T, float* __restrict__ m_T) {
  __shared__ float Ks[kTile][kTile + 1];
  __shared__ float Vs[kTile][kTile + 1];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int dv0 = blockIdx.x * kTile, dk0 = blockIdx.y * kTile, bh = blockIdx.z;
  const int DK = p.DK, DV = p.DV, T = p.T, L = p.L;
  const bool n_owner = blockIdx.x == 0 && tid < kTile && dk0 + tid < DK;
  const long tpad = (long)p.NC * L;

  float acc[4][4];
  float nacc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int a = dk0 + ty * 4 + i, c = dv0 + tx * 4 + j;
      acc[i][j] = (C0 && a < DK && c < DV) ? C0[((long)bh * DK + a) * DV + c] : 0.f;
    }
  if (n_owner && n0) nacc = n0[(long)bh * DK + dk0 + tid];

  for (int k = 0; k < p.NC; ++k) {
    float* Cs = C_states + ((long)bh * p.NC + k) * DK * DV;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int a = dk0 + ty * 4 + i, c = dv0 + tx * 4 + j;
        if (a < DK && c < DV) Cs[(long)a * DV + c] = acc[i][j];
      }
    if (n_owner) n_states[((long)bh * p.NC + k) * DK + dk0 + tid] = nacc;

    const float m_in = g.mchk[(long)bh * (p.NC + 1) + k];
    const float m_out = g.mchk[(long)bh * (p.NC + 1) + k + 1];
    const float gk = g.gtot[(long)bh * p.NC + k];
    const float decay = expf(gk + m_in - m_out);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= decay;
    nacc *= decay;

    for (int r0 = 0; r0 < L; r0 += kTile) {
      for (int e = tid; e < kTile * kTile; e += kThreads) {
        const int r = e / kTile, c = e % kTile;
        const long t = (long)k * L + r0 + r;
        const bool tok = (r0 + r < L) && t < T;
        float w = 0.f;
        if (tok) w = p.key_scale * expf(gk + g.acol[(long)bh * tpad + t] - m_out);
        Ks[r][c] = w * load_or_zero(K, ((long)bh * T + t) * DK + dk0 + c, tok && dk0 + c < DK);
        Vs[r][c] = load_or_zero(V, ((long)bh * T + t) * DV + dv0 + c, tok && dv0 + c < DV);
      }
      __syncthreads();
#pragma unroll 4
      for (int r = 0; r < kTile; ++r) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = Ks[r][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Vs[r][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        if (n_owner) nacc += Ks[r][tid];
      }
      __syncthreads();
    }
  }
  if (C_T) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int a = dk0 + ty * 4 + i, c = dv0 + tx * 4 + j;
        if (a < DK && c < DV) C_T[((long)bh * DK + a) * DV + c] = acc[i][j];
      }
  }
  if (n_T && n_owner) n_T[(long)bh * DK + dk0 + tid] = nacc;
  if (m_T && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0)
    m_T[bh] = g.mchk[(long)bh * (p.NC + 1) + p.NC];
}

// Reduction over the 16 lanes that share a row group (lanes tx = 0..15).
__device__ __forceinline__ float sum16(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename TIn>
__global__ void __launch_bounds__(kThreads)
simt_parallel_kernel(Problem p, const TIn* __restrict__ Q, const TIn* __restrict__ K,
                     const TIn* __restrict__ V, Gates g, const float* __restrict__ C_states,
                     const float* __restrict__ n_states, TIn* __restrict__ H,
                     float* __restrict__ n_out, float* __restrict__ m_out,
                     float* __restrict__ H32) {
  constexpr int kSlab = 32;
  // Phase buffers alias one another: {Qs, Ks} or {Qs, Cs} during the
  // contractions over DK, {Ps, Vs} during P.V.
  __shared__ float buf[kTile * (kTile + 1) + kTile * kTile];
  __shared__ float mu_s[kTile], bc_s[kTile], acol_s[kTile], ns[kSlab];
  float (*Qs)[kSlab + 1] = reinterpret_cast<float (*)[kSlab + 1]>(buf);
  float (*Ks)[kSlab + 1] = reinterpret_cast<float (*)[kSlab + 1]>(buf + kTile * (kSlab + 1));
  float (*Cs)[kTile] = reinterpret_cast<float (*)[kTile]>(buf + kTile * (kSlab + 1));
  float (*Ps)[kTile + 1] = reinterpret_cast<float (*)[kTile + 1]>(buf);
  float (*Vs)[kTile] = reinterpret_cast<float (*)[kTile]>(buf + kTile * (kTile + 1));

  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int dv0 = blockIdx.x * kTile, bh = blockIdx.z;
  const int DK = p.DK, DV = p.DV, T = p.T, L = p.L;
  const long t0 = (long)blockIdx.y * kTile;  // first query token of this block
  const int k = (int)(t0 / L);
  const long tpad = (long)p.NC * L;
  const float m_in = g.mchk[(long)bh * (p.NC + 1) + k];

  if (tid < kTile) {
    const long t = t0 + tid;
    mu_s[tid] = fmaxf(m_in, g.amax[(long)bh * tpad + t]);
    bc_s[tid] = g.bcum[(long)bh * tpad + t];
  }
  __syncthreads();

  float acc[4][4] = {};
  float den[4] = {};

  // Inter-chunk term: q_r . C_k and q_r . n_k.
  const float* Ck = C_states + ((long)bh * p.NC + k) * DK * DV;
  const float* nk = n_states + ((long)bh * p.NC + k) * DK;
  for (int c0 = 0; c0 < DK; c0 += kSlab) {
    for (int e = tid; e < kTile * kSlab; e += kThreads) {
      const int r = e / kSlab, c = e % kSlab;
      const long t = t0 + r;
      Qs[r][c] = load_or_zero(Q, ((long)bh * T + t) * DK + c0 + c, t < T && c0 + c < DK);
    }
    for (int e = tid; e < kSlab * kTile; e += kThreads) {
      const int c = e / kTile, j = e % kTile;
      Cs[c][j] = (c0 + c < DK && dv0 + j < DV) ? Ck[(long)(c0 + c) * DV + dv0 + j] : 0.f;
    }
    if (tid < kSlab) ns[tid] = c0 + tid < DK ? nk[c0 + tid] : 0.f;
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kSlab; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Qs[ty * 4 + i][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Cs[c][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float part = Qs[ty * 4 + i][2 * tx] * ns[2 * tx] + Qs[ty * 4 + i][2 * tx + 1] * ns[2 * tx + 1];
      den[i] += sum16(part);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float f = expf(m_in - mu_s[ty * 4 + i]);
    den[i] *= f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] *= f;
  }

  // Intra-chunk term over key blocks up to and including the diagonal block.
  const long chunk0 = (long)k * L;
  for (long s0 = chunk0; s0 <= t0; s0 += kTile) {
    float S[4][4] = {};
    for (int c0 = 0; c0 < DK; c0 += kSlab) {
      for (int e = tid; e < kTile * kSlab; e += kThreads) {
        const int r = e / kSlab, c = e % kSlab;
        const bool okc = c0 + c < DK;
        Qs[r][c] = load_or_zero(Q, ((long)bh * T + t0 + r) * DK + c0 + c, t0 + r < T && okc);
        Ks[r][c] = load_or_zero(K, ((long)bh * T + s0 + r) * DK + c0 + c, s0 + r < T && okc);
      }
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < kSlab; ++c) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = Qs[ty * 4 + i][c];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Ks[tx * 4 + j][c];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) S[i][j] = fmaf(a[i], b[j], S[i][j]);
      }
      __syncthreads();
    }
    if (tid < kTile) acol_s[tid] = g.acol[(long)bh * tpad + s0 + tid];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const long tr = t0 + ty * 4 + i;
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const long ts = s0 + tx * 4 + j;
        float pv = 0.f;
        if (ts <= tr) pv = S[i][j] * p.key_scale * expf(acol_s[tx * 4 + j] - mu_s[ty * 4 + i]);
        Ps[ty * 4 + i][tx * 4 + j] = pv;
        rs += pv;
      }
      den[i] += sum16(rs);
    }
    for (int e = tid; e < kTile * kTile; e += kThreads) {
      const int r = e / kTile, j = e % kTile;
      Vs[r][j] = load_or_zero(V, ((long)bh * T + s0 + r) * DV + dv0 + j, s0 + r < T && dv0 + j < DV);
    }
    __syncthreads();
#pragma unroll 4
    for (int s = 0; s < kTile; ++s) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Ps[ty * 4 + i][s];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Vs[s][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    const long t = t0 + r;
    if (t >= T) continue;
    const float mr = bc_s[r] + mu_s[r];
    // the plain sigmoid variant has no normaliser: h = e^{m} O
    const float denom = p.no_norm ? expf(-mr) : fmaxf(fabsf(den[i]), expf(-mr));
    const float inv = p.no_norm ? expf(mr) : 1.f / denom;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = dv0 + tx * 4 + j;
      if (c >= DV) continue;
      if (H32) H32[((long)bh * T + t) * DV + c] = acc[i][j] * inv;
      else H[((long)bh * T + t) * DV + c] = from_float<TIn>(acc[i][j] * inv);
    }
    if (blockIdx.x == 0 && tx == 0) {
      if (n_out) n_out[(long)bh * T + t] = p.signed_den ? copysignf(denom, den[i]) : denom;
      if (m_out) m_out[(long)bh * T + t] = mr;
    }
  }
}

}  // namespace

cudaError_t launch_simt_states(const Problem& p, mlstm_dtype dt, const void* K, const void* V,
                               const float* C0, const float* n0, Gates g, float* C_states,
                               float* n_states, float* C_T, float* n_T, float* m_T,
                               cudaStream_t st) {
  dim3 grid((p.DV + kTile - 1) / kTile, (p.DK + kTile - 1) / kTile, p.BH);
  if (dt == MLSTM_DT_F32)
    simt_states_kernel<float><<<grid, kThreads, 0, st>>>(
        p, (const float*)K, (const float*)V, C0, n0, g, C_states, n_states, C_T, n_T, m_T);
  else
    simt_states_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
        p, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, C0, n0, g, C_states, n_states,
        C_T, n_T, m_T);
  return cudaGetLastError();
}

cudaError_t launch_simt_parallel(const Problem& p, mlstm_dtype dt, const void* Q, const void* K,
                                 const void* V, Gates g, const float* C_states,
                                 const float* n_states, void* H, float* n_out, float* m_out,
                                 cudaStream_t st, float* H32) {
  if (p.T == 0) return cudaSuccess;
  const int qblocks = (p.T + kTile - 1) / kTile;
  dim3 grid((p.DV + kTile - 1) / kTile, qblocks, p.BH);
  if (dt == MLSTM_DT_F32)
    simt_parallel_kernel<float><<<grid, kThreads, 0, st>>>(
        p, (const float*)Q, (const float*)K, (const float*)V, g, C_states, n_states, (float*)H,
        n_out, m_out, H32);
  else
    simt_parallel_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
        p, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, g,
        C_states, n_states, (__nv_bfloat16*)H, n_out, m_out, H32);
  return cudaGetLastError();
}

}  // namespace mlstm
