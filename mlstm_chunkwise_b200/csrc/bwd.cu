// Backward pass of the chunkwise mLSTM: host orchestration and the fp32
// CUDA-core gradient kernels.
//
// The forward ("Tiled Flash Linear Attention: More Efficient Linear RNN and
// xLSTM Kernels", abstract: the mLSTM as an inter-chunk recurrence plus an
// intra-chunk parallel part) is h_t = C-bar_t^T q_t / max(|n-bar_t . q_t|, 1)
// in the unstabilised frame, where C-bar_t = sum_{s<=t} W_ts (s k_s) v_s^T
// (plus the decayed initial state) and W_ts = e^{log i_s + sum_{s<l<=t} log f_l}.
// For a loss L(H) with dh_t = dL/dh_t, writing D_t = max(|a_t|, 1),
// a_t = n-bar_t . q_t, du_t = dh_t / D_t and
// da_t = -(dh_t . h_t) / D_t sign(a_t) [|a_t| > 1]:
//
//   dq_t  = sum_{s<=t} W_ts (v_s . du_t + da_t) k^_s      (k^ = s k)
//   dk^_s = sum_{t>=s} W_ts (du_t . v_s + da_t) q_t
//   dv_s  = sum_{t>=s} W_ts (q_t . k^_s) du_t
//   dL/d log i_s = k_s . dk_s,   dL/d log f_l = sum_{t>=l} (q_t . dq_t - k_t . dk_t)
//
// (the last two identities, and these three sums, are checked against an
// fp64 autograd oracle).  In the stabilised frame of the forward every weight
// becomes a factor <= 1 that the forward already uses:
//   intra-chunk   W_ts e^{-m_t} = e^{acol_s - mu_t}            (the gate factor of P)
//   query side    e^{m_k + bcum_t - m_t} = e^{m_k - mu_t}       (the Q~ scaling)
//   key side      e^{g_k + acol_s - m_{k+1}}                    (the state-update weight)
// and with du~_t = dh_t / den_t, da~_t = -(dh_t . h_t) / den_t sign(a_t)
// [|a_t| > e^{-m_t}] (den_t = max(|a_t|, e^{-m_t}) in the stabilised frame):
//
//   G~_k = e^{g_k + m_k - m_{k+1}} G~_{k+1} + sum_{t in k} e^{m_k - mu_t} q_t du~_t^T
//   g~_k = (the same with du~ -> da~)                      G~_NC = 0, g~_NC = 0
//   dq_t  = e^{m_k - mu_t} (C_k du~_t + da~_t n_k) + sum_{s<=t in k} e^{acol_s - mu_t} dP_ts k^_s
//   dk^_s = w_s (G~_{k+1} v_s + g~_{k+1}) + sum_{t>=s in k} e^{acol_s - mu_t} dP_ts q_t
//   dv_s  = w_s G~_{k+1}^T k^_s + sum_{t>=s in k} e^{acol_s - mu_t} S_ts du~_t
//   dP_ts = du~_t . v_s + da~_t,  S_ts = q_t . k^_s,  w_s = e^{g_k + acol_s - m_{k+1}}
//
// G~_k is the gradient with respect to the state entering chunk k, in that
// state's frame, so dC0 = G~_0, dn0 = g~_0 and dm0 = <C0, dC0> + n0 . dn0.
//
// Two paths.  bf16 inputs with d_qk of 128 or 256 (and a d_v the tensor-core
// forward takes), at least 128 tokens: everything on 128-token chunks, the
// forward recomputed on the tensor cores, the reverse states and dq, dk, dv as
// tcgen05 GEMMs (tc_bwd.cu; launch_bwd_tc below).  Otherwise, in this file:
// the forward's gates, chunk states and outputs (h and the signed denominator
// kept), a per-token pass forming du~ and da~, the reverse state recurrence,
// dq, dk, dv, and the gate gradients (dot products and a reverse scan), on
// fp32 CUDA-core kernels (the forward recomputed on the tensor cores for bf16
// shapes the unfused tensor-core forward supports: fp32 chunk states, their
// bf16 operand copy, h in bf16).  The gradient kernels own 64 rows and up to
// 256 output columns (8 x 8 accumulators per thread).
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "tc.h"
#include "tc_bwd.h"

namespace mlstm {
namespace {

constexpr int kT = 64;        // tile edge
constexpr int kS = 32;        // contraction slab
constexpr int kThr = 256;

template <typename TIn>
__device__ __forceinline__ float ld(const TIn* base, long idx, bool ok) {
  return ok ? to_float(base[idx]) : 0.f;
}

// Two floats as one packed bf16 pair (round to nearest even).
__device__ __forceinline__ uint32_t tc_pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// du~ [BH, T, DV] (fp32) and da~ [BH, T]: one warp per token.
// ---------------------------------------------------------------------------
// den_s holds copysign(max(|a|, e^{-m}), a) of the forward (signed_den mode).
template <typename TIn, typename TH>
__global__ void __launch_bounds__(kThr)
bwd_prep_kernel(Problem p, const TIn* __restrict__ dH, const TH* __restrict__ Hf,
                const float* __restrict__ den_s, const float* __restrict__ mr,
                float* __restrict__ dU, float* __restrict__ dA) {
  const long tok = (long)blockIdx.x * (kThr / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= (long)p.BH * p.T) return;
  const float ds = den_s[tok];
  const float inv = 1.f / fabsf(ds);
  float dot = 0.f;
  for (int c = lane; c < p.DV; c += 32) {
    const float g = to_float(dH[tok * p.DV + c]);
    dU[tok * p.DV + c] = g * inv;
    dot = fmaf(g, to_float(Hf[tok * p.DV + c]), dot);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if (lane == 0) {
    const bool on_n = fabsf(ds) > expf(-mr[tok]);  // the max picked |n.q|
    dA[tok] = on_n ? -dot * inv * (ds >= 0.f ? 1.f : -1.f) : 0.f;
  }
}

// The tensor-core path's per-token pass (bf16 dH and h, d_v a multiple of
// 8): du~ in bf16, plain and with the row factor e^{m_k - mu_t}, and da~.  One
// warp per token, each lane 8 consecutive values per step (16-byte accesses).
__global__ void __launch_bounds__(kThr)
bwd_prep_tc_kernel(Problem p, const __nv_bfloat16* __restrict__ dH,
                   const __nv_bfloat16* __restrict__ Hf, const float* __restrict__ den_s,
                   const float* __restrict__ mr, Gates gt, float* __restrict__ dA,
                   __nv_bfloat16* __restrict__ dU16, __nv_bfloat16* __restrict__ dUr16) {
  const long tok = (long)blockIdx.x * (kThr / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= (long)p.BH * p.T) return;
  const float ds = den_s[tok];
  const float inv = 1.f / fabsf(ds);
  const long bh = tok / p.T, t = tok % p.T;
  const float m_in = gt.mchk[bh * (p.NC + 1) + t / p.L];
  const float r = expf(m_in - fmaxf(m_in, gt.amax[bh * (long)p.NC * p.L + t]));
  const uint4* g4 = reinterpret_cast<const uint4*>(dH + tok * p.DV);
  const uint4* h4 = reinterpret_cast<const uint4*>(Hf + tok * p.DV);
  uint4* u4 = reinterpret_cast<uint4*>(dU16 + tok * p.DV);
  uint4* ur4 = reinterpret_cast<uint4*>(dUr16 + tok * p.DV);
  float dot = 0.f;
  for (int c = lane; c < p.DV / 8; c += 32) {
    const uint4 gv = g4[c], hv = h4[c];
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, hw[4] = {hv.x, hv.y, hv.z, hv.w};
    uint32_t uw[4], urw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
      const float2 h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[e]));
      dot = fmaf(g.x, h.x, fmaf(g.y, h.y, dot));
      uw[e] = tc_pack_bf16x2(g.x * inv, g.y * inv);
      urw[e] = tc_pack_bf16x2(r * g.x * inv, r * g.y * inv);
    }
    u4[c] = make_uint4(uw[0], uw[1], uw[2], uw[3]);
    ur4[c] = make_uint4(urw[0], urw[1], urw[2], urw[3]);
  }
  dot = warp_sum(dot);
  if (lane == 0) {
    const bool on_n = fabsf(ds) > expf(-mr[tok]);  // the max picked |n.q|
    dA[tok] = on_n ? -dot * inv * (ds >= 0.f ? 1.f : -1.f) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Reverse recurrence: G~_k [BH, NC+1, DK, DV], g~_k [BH, NC+1, DK].  One block
// per (b, h, 64 x 64 tile of [DK, DV], segment); blocks with blockIdx.x == 0
// carry g~.  With n_seg > 1 the chunks are cut into segments (as the forward
// state kernel does) that each run from a zero state at their end;
// bwd_states_fixup_kernel then adds the state carried in from the segments
// after them: G~_k += e^{sum_{j in [k, k1)} (g_j + m_j - m_{j+1})} G~_{k1}.
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kThr)
bwd_states_kernel(Problem p, const TIn* __restrict__ Q, const float* __restrict__ dU,
                  const float* __restrict__ dA, Gates g, float* __restrict__ G_states,
                  float* __restrict__ g_states, int n_seg) {
  __shared__ float Qs[kT][kT + 1];
  __shared__ float Us[kT][kT + 1];
  __shared__ float das[kT];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int dv0 = blockIdx.x * kT, dk0 = blockIdx.y * kT;
  const int bh = blockIdx.z / n_seg, seg = blockIdx.z % n_seg;
  const int DK = p.DK, DV = p.DV, T = p.T, L = p.L, NC = p.NC;
  const int ncs = (NC + n_seg - 1) / n_seg;
  const int k0 = seg * ncs, k1 = k0 + ncs < NC ? k0 + ncs : NC;
  const bool g_owner = blockIdx.x == 0 && tid < kT && dk0 + tid < DK;
  const long tpad = (long)NC * L;
  float acc[4][4] = {};
  float gacc = 0.f;
  auto store = [&](int k) {
    float* Gk = G_states + ((long)bh * (NC + 1) + k) * DK * DV;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int a = dk0 + ty * 4 + i, c = dv0 + tx * 4 + j;
        if (a < DK && c < DV) Gk[(long)a * DV + c] = acc[i][j];
      }
    if (g_owner) g_states[((long)bh * (NC + 1) + k) * DK + dk0 + tid] = gacc;
  };
  if (seg == n_seg - 1) store(NC);  // G~_NC = 0; other segment ends belong to the next segment
  for (int k = k1 - 1; k >= k0; --k) {
    const float m_in = g.mchk[(long)bh * (NC + 1) + k];
    const float m_out = g.mchk[(long)bh * (NC + 1) + k + 1];
    const float decay = expf(g.gtot[(long)bh * NC + k] + m_in - m_out);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= decay;
    gacc *= decay;
    for (int r0 = 0; r0 < L; r0 += kT) {
      for (int e = tid; e < kT * kT; e += kThr) {
        const int r = e / kT, c = e % kT;
        const long t = (long)k * L + r0 + r;
        const bool tok = t < T;
        float f = 0.f;
        if (tok) f = expf(m_in - fmaxf(m_in, g.amax[(long)bh * tpad + t]));  // e^{m_k - mu_t}
        Qs[r][c] = f * ld(Q, ((long)bh * T + t) * DK + dk0 + c, tok && dk0 + c < DK);
        Us[r][c] = (tok && dv0 + c < DV) ? dU[((long)bh * T + t) * DV + dv0 + c] : 0.f;
      }
      if (tid < kT) {
        const long t = (long)k * L + r0 + tid;
        das[tid] = t < T ? dA[(long)bh * T + t] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int r = 0; r < kT; ++r) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = Qs[r][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Us[r][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        if (g_owner) gacc = fmaf(Qs[r][tid], das[r], gacc);
      }
      __syncthreads();
    }
    store(k);
  }
}

// Adds the carried-in state to the segments before the last one.  One thread
// per element of [DK, DV] (then of g~'s DK) and (b, h); walks the segments
// from the end, so each segment's end value is final when it is used.
__global__ void __launch_bounds__(kThr)
bwd_states_fixup_kernel(Problem p, Gates g, float* __restrict__ G_states,
                        float* __restrict__ g_states, int n_seg) {
  const long per = (long)p.DK * p.DV;
  const long e = (long)blockIdx.x * kThr + threadIdx.x;
  const int bh = blockIdx.y, NC = p.NC;
  if (e >= per + p.DK) return;
  float* base;
  long stride;
  if (e < per) {
    base = G_states + (long)bh * (NC + 1) * per + e;
    stride = per;
  } else {
    base = g_states + (long)bh * (NC + 1) * p.DK + (e - per);
    stride = p.DK;
  }
  const float* gt = g.gtot + (long)bh * NC;
  const float* mc = g.mchk + (long)bh * (NC + 1);
  const int ncs = (NC + n_seg - 1) / n_seg;
  for (int s = n_seg - 2; s >= 0; --s) {
    const int k0 = s * ncs, k1 = k0 + ncs < NC ? k0 + ncs : NC;
    const float carried = base[(long)k1 * stride];  // final: its segment was fixed before
    float lg = 0.f;
    for (int k = k1 - 1; k >= k0; --k) {
      lg += gt[k] + mc[k] - mc[k + 1];
      base[(long)k * stride] = fmaf(expf(lg), carried, base[(long)k * stride]);
    }
  }
}

// ---------------------------------------------------------------------------
// dq, dk, dv.  A block owns 64 rows (queries for dq, keys for dk and dv) and a
// range of kW <= 256 output columns, so the 64 x 64 products it needs per
// pair of row tiles (dP = dU V^T, or S = K^ Q^T) are formed once for the whole
// range rather than once per 64 columns.  Layouts (all in shared memory,
// contraction index first so that every inner-loop read is a float4):
//   At[c][r]  A operand: 64 rows, slab of 32 along the contraction
//   Bw[c][j]  B operand: kW columns (or 64 for the square products)
//   Pt[s][r]  the gated 64 x 64 tile, contraction index (s or t) first
// Square products use a 16 x 16 thread grid with 4 x 4 outputs per thread;
// the wide accumulators a grid of 8 row groups (warps) x 32 lanes with 8 rows x
// kW/32 columns per thread (columns 4 lane + {0..3} and 128 + 4 lane + {0..3}
// for kW = 256, so every float4 read of a warp is contiguous).
// ---------------------------------------------------------------------------
constexpr int kTP = kT + 4;  // row stride of At and Pt (keeps float4 alignment)

template <int kW>
struct WideSmem {
  float At[kS][kTP];
  float Bw[kS][kW];
  float Pt[kT][kTP];
  float mu[kT], da[kT], acol[kT], fw[kT];
};

template <int kW>
__device__ __forceinline__ int wide_col(int lane, int j) {
  constexpr int kC = kW / 32;
  return kC >= 4 ? (j >> 2) * 128 + 4 * lane + (j & 3) : kC * lane + j;
}

// acc[i][j] += sum_{c < kS} A[c][wy*8 + i] * B[c][wide_col(wx, j)]
template <int kW>
__device__ __forceinline__ void mac_wide(float (&acc)[8][kW / 32], const float (*A)[kTP],
                                         const float (*B)[kW], int wy, int wx) {
  constexpr int kC = kW / 32;
#pragma unroll 4
  for (int c = 0; c < kS; ++c) {
    const float4 a0 = *reinterpret_cast<const float4*>(&A[c][wy * 8]);
    const float4 a1 = *reinterpret_cast<const float4*>(&A[c][wy * 8 + 4]);
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    float b[kC];
    if (kC >= 4) {
#pragma unroll
      for (int h = 0; h < kC / 4; ++h) {
        const float4 bv = *reinterpret_cast<const float4*>(&B[c][h * 128 + 4 * wx]);
        b[4 * h] = bv.x; b[4 * h + 1] = bv.y; b[4 * h + 2] = bv.z; b[4 * h + 3] = bv.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kC; ++j) b[j] = B[c][kC * wx + j];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < kC; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

// acc[i][j] += sum_{c < kS} A[c][ty*4 + i] * B[c][tx*4 + j]   (64 x 64 product)
template <int kW>
__device__ __forceinline__ void mac_square(float (&acc)[4][4], const float (*A)[kTP],
                                           const float (*B)[kW], int ty, int tx) {
#pragma unroll 4
  for (int c = 0; c < kS; ++c) {
    const float4 av = *reinterpret_cast<const float4*>(&A[c][ty * 4]);
    const float4 bv = *reinterpret_cast<const float4*>(&B[c][tx * 4]);
    const float a[4] = {av.x, av.y, av.z, av.w}, b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

// dst[c][r] = scale * X[(row0 + r) * ld + c0 + c] for r < nrows (<= width of
// dst rows), c < kS; zero outside [0, rows_valid) x [0, cols_valid).  Lanes
// take consecutive rows (conflict-free shared stores).
template <typename TX, int kLd>
__device__ __forceinline__ void load_cmajor(float (*dst)[kLd], const TX* X, long row0, int nrows,
                                            long rows_valid, long ld, int c0, int cols_valid,
                                            float scale) {
  for (int e = threadIdx.x; e < nrows * (kS / 4); e += kThr) {
    const int r = e % nrows, grp = e / nrows;
    const long row = row0 + r;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + grp * 4 + q;
      dst[grp * 4 + q][r] = (row < rows_valid && c < cols_valid) ? scale * to_float(X[row * ld + c]) : 0.f;
    }
  }
}

// dst[s][j] = scale * X[(row0 + s) * ld + col0 + j] for s < kS, j < kW: the
// contraction runs along X's rows, the wide index along its columns.
template <typename TX, int kW>
__device__ __forceinline__ void load_rmajor(float (*dst)[kW], const TX* X, long row0,
                                            long rows_valid, long ld, int col0, int cols_valid,
                                            float scale) {
  for (int e = threadIdx.x; e < kS * (kW / 4); e += kThr) {
    const int j4 = e % (kW / 4), s = e / (kW / 4);
    const long row = row0 + s;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = col0 + 4 * j4 + q;
      dst[s][4 * j4 + q] = (row < rows_valid && col < cols_valid) ? scale * to_float(X[row * ld + col]) : 0.f;
    }
  }
}

// dq for 64 queries and kW columns of d_qk; adds q_t . dq_t into qdq.
template <typename TIn, int kW>
__global__ void __launch_bounds__(kThr)
bwd_dq_kernel(Problem p, const TIn* __restrict__ Q, const TIn* __restrict__ K,
              const TIn* __restrict__ V, Gates g, const float* __restrict__ C_states,
              const float* __restrict__ n_states, const float* __restrict__ dU,
              const float* __restrict__ dA, TIn* __restrict__ dQ, float* __restrict__ qdq) {
  constexpr int kC = kW / 32;
  extern __shared__ __align__(16) unsigned char dsm[];
  WideSmem<kW>& sm = *reinterpret_cast<WideSmem<kW>*>(dsm);
  const int tid = threadIdx.x, wy = tid >> 5, wx = tid & 31, ty = tid >> 4, tx = tid & 15;
  const int d0 = blockIdx.x * kW, bh = blockIdx.z;
  const long t0 = (long)blockIdx.y * kT;
  const int DK = p.DK, DV = p.DV, T = p.T, L = p.L, NC = p.NC;
  const int k = (int)(t0 / L);
  const long tpad = (long)NC * L, base = (long)bh * T;
  const float m_in = g.mchk[(long)bh * (NC + 1) + k];
  if (tid < kT) {
    const long t = t0 + tid;
    sm.mu[tid] = fmaxf(m_in, g.amax[(long)bh * tpad + t]);
    sm.da[tid] = t < T ? dA[base + t] : 0.f;
    sm.fw[tid] = expf(m_in - sm.mu[tid]);
  }
  float acc[8][kC] = {};
  // inter: sum_c du~[t][c] C_k[d][c]
  const float* Ck = C_states + ((long)bh * NC + k) * DK * DV;
  for (int c0 = 0; c0 < DV; c0 += kS) {
    load_cmajor<float, kTP>(sm.At, dU + base * DV, t0, kT, T, DV, c0, DV, 1.f);
    load_cmajor<float, kW>(sm.Bw, Ck, d0, kW, DK, DV, c0, DV, 1.f);
    __syncthreads();
    mac_wide<kW>(acc, sm.At, sm.Bw, wy, wx);
    __syncthreads();
  }
  const float* nk = n_states + ((long)bh * NC + k) * DK;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = wy * 8 + i;
#pragma unroll
    for (int j = 0; j < kC; ++j) {
      const int d = d0 + wide_col<kW>(wx, j);
      acc[i][j] = sm.fw[r] * (acc[i][j] + sm.da[r] * (d < DK ? nk[d] : 0.f));
    }
  }
  // intra: key tiles of the chunk up to the diagonal
  for (long s0 = (long)k * L; s0 <= t0; s0 += kT) {
    if (tid < kT) sm.acol[tid] = g.acol[(long)bh * tpad + s0 + tid];
    float dP[4][4] = {};
    for (int c0 = 0; c0 < DV; c0 += kS) {
      load_cmajor<float, kTP>(sm.At, dU + base * DV, t0, kT, T, DV, c0, DV, 1.f);
      load_cmajor<TIn, kW>(sm.Bw, V + base * DV, s0, kT, T, DV, c0, DV, 1.f);
      __syncthreads();
      mac_square<kW>(dP, sm.At, sm.Bw, ty, tx);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = ty * 4 + i, sc = tx * 4 + j;
        const bool ok = s0 + sc <= t0 + r && t0 + r < T;
        sm.Pt[sc][r] = ok ? expf(sm.acol[sc] - sm.mu[r]) * (dP[i][j] + sm.da[r]) : 0.f;
      }
    for (int half = 0; half < 2; ++half) {
      load_rmajor<TIn, kW>(sm.Bw, K + base * DK, s0 + half * kS, T, DK, d0, DK, p.key_scale);
      __syncthreads();
      mac_wide<kW>(acc, sm.Pt + half * kS, sm.Bw, wy, wx);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long t = t0 + wy * 8 + i;
    float part = 0.f;
#pragma unroll
    for (int j = 0; j < kC; ++j) {
      const int d = d0 + wide_col<kW>(wx, j);
      if (t < T && d < DK) {
        dQ[(base + t) * DK + d] = from_float<TIn>(acc[i][j]);
        part = fmaf(to_float(Q[(base + t) * DK + d]), acc[i][j], part);
      }
    }
    part = warp_sum(part);
    if (wx == 0 && t < T) atomicAdd(&qdq[base + t], part);
  }
}

// dk for 64 keys and kW columns of d_qk; adds k_s . dk_s into kdk.
template <typename TIn, int kW>
__global__ void __launch_bounds__(kThr)
bwd_dk_kernel(Problem p, const TIn* __restrict__ Q, const TIn* __restrict__ K,
              const TIn* __restrict__ V, Gates g, const float* __restrict__ G_states,
              const float* __restrict__ g_states, const float* __restrict__ dU,
              const float* __restrict__ dA, TIn* __restrict__ dK, float* __restrict__ kdk) {
  constexpr int kC = kW / 32;
  extern __shared__ __align__(16) unsigned char dsm[];
  WideSmem<kW>& sm = *reinterpret_cast<WideSmem<kW>*>(dsm);
  const int tid = threadIdx.x, wy = tid >> 5, wx = tid & 31, ty = tid >> 4, tx = tid & 15;
  const int d0 = blockIdx.x * kW, bh = blockIdx.z;
  const long s0 = (long)blockIdx.y * kT;
  const int DK = p.DK, DV = p.DV, T = p.T, L = p.L, NC = p.NC;
  const int k = (int)(s0 / L);
  const long tpad = (long)NC * L, base = (long)bh * T;
  const float m_in = g.mchk[(long)bh * (NC + 1) + k];
  const float m_out = g.mchk[(long)bh * (NC + 1) + k + 1];
  const float gk = g.gtot[(long)bh * NC + k];
  if (tid < kT) {
    sm.acol[tid] = g.acol[(long)bh * tpad + s0 + tid];
    sm.fw[tid] = expf(gk + sm.acol[tid] - m_out);  // 0 on padding (acol = -inf)
  }
  float acc[8][kC] = {};
  // inter: sum_c v_s[c] G~_{k+1}[d][c] + g~_{k+1}[d], times w_s
  const float* Gk = G_states + ((long)bh * (NC + 1) + k + 1) * DK * DV;
  const float* gk1 = g_states + ((long)bh * (NC + 1) + k + 1) * DK;
  for (int c0 = 0; c0 < DV; c0 += kS) {
    load_cmajor<TIn, kTP>(sm.At, V + base * DV, s0, kT, T, DV, c0, DV, 1.f);
    load_cmajor<float, kW>(sm.Bw, Gk, d0, kW, DK, DV, c0, DV, 1.f);
    __syncthreads();
    mac_wide<kW>(acc, sm.At, sm.Bw, wy, wx);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = wy * 8 + i;
#pragma unroll
    for (int j = 0; j < kC; ++j) {
      const int d = d0 + wide_col<kW>(wx, j);
      acc[i][j] = sm.fw[r] * (acc[i][j] + (d < DK ? gk1[d] : 0.f));
    }
  }
  // intra: query tiles of the chunk from the diagonal on
  const long chunk_end = (long)(k + 1) * L;
  for (long q0 = s0; q0 < chunk_end && q0 < T; q0 += kT) {
    if (tid < kT) {
      const long t = q0 + tid;
      sm.mu[tid] = fmaxf(m_in, g.amax[(long)bh * tpad + t]);
      sm.da[tid] = t < T ? dA[base + t] : 0.f;
    }
    float dP[4][4] = {};  // [key s][query t]
    for (int c0 = 0; c0 < DV; c0 += kS) {
      load_cmajor<TIn, kTP>(sm.At, V + base * DV, s0, kT, T, DV, c0, DV, 1.f);
      load_cmajor<float, kW>(sm.Bw, dU + base * DV, q0, kT, T, DV, c0, DV, 1.f);
      __syncthreads();
      mac_square<kW>(dP, sm.At, sm.Bw, ty, tx);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sr = ty * 4 + i, tq = tx * 4 + j;
        const bool ok = q0 + tq >= s0 + sr && q0 + tq < T;
        sm.Pt[tq][sr] = ok ? expf(sm.acol[sr] - sm.mu[tq]) * (dP[i][j] + sm.da[tq]) : 0.f;
      }
    for (int half = 0; half < 2; ++half) {
      load_rmajor<TIn, kW>(sm.Bw, Q + base * DK, q0 + half * kS, T, DK, d0, DK, 1.f);
      __syncthreads();
      mac_wide<kW>(acc, sm.Pt + half * kS, sm.Bw, wy, wx);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long sr = s0 + wy * 8 + i;
    float part = 0.f;
#pragma unroll
    for (int j = 0; j < kC; ++j) {
      const int d = d0 + wide_col<kW>(wx, j);
      if (sr < T && d < DK) {
        const float v = p.key_scale * acc[i][j];
        dK[(base + sr) * DK + d] = from_float<TIn>(v);
        part = fmaf(to_float(K[(base + sr) * DK + d]), v, part);
      }
    }
    part = warp_sum(part);
    if (wx == 0 && sr < T) atomicAdd(&kdk[base + sr], part);
  }
}

// dv for 64 keys and kW columns of d_v.
template <typename TIn, int kW>
__global__ void __launch_bounds__(kThr)
bwd_dv_kernel(Problem p, const TIn* __restrict__ Q, const TIn* __restrict__ K, Gates g,
              const float* __restrict__ G_states, const float* __restrict__ dU,
              TIn* __restrict__ dV) {
  constexpr int kC = kW / 32;
  extern __shared__ __align__(16) unsigned char dsm[];
  WideSmem<kW>& sm = *reinterpret_cast<WideSmem<kW>*>(dsm);
  const int tid = threadIdx.x, wy = tid >> 5, wx = tid & 31, ty = tid >> 4, tx = tid & 15;
  const int c0w = blockIdx.x * kW, bh = blockIdx.z;
  const long s0 = (long)blockIdx.y * kT;
  const int DK = p.DK, DV = p.DV, T = p.T, L = p.L, NC = p.NC;
  const int k = (int)(s0 / L);
  const long tpad = (long)NC * L, base = (long)bh * T;
  const float m_in = g.mchk[(long)bh * (NC + 1) + k];
  const float m_out = g.mchk[(long)bh * (NC + 1) + k + 1];
  const float gk = g.gtot[(long)bh * NC + k];
  if (tid < kT) {
    sm.acol[tid] = g.acol[(long)bh * tpad + s0 + tid];
    sm.fw[tid] = expf(gk + sm.acol[tid] - m_out);
  }
  float acc[8][kC] = {};
  // inter: sum_d k^_s[d] G~_{k+1}[d][c], times w_s
  const float* Gk = G_states + ((long)bh * (NC + 1) + k + 1) * DK * DV;
  for (int dd = 0; dd < DK; dd += kS) {
    load_cmajor<TIn, kTP>(sm.At, K + base * DK, s0, kT, T, DK, dd, DK, p.key_scale);
    load_rmajor<float, kW>(sm.Bw, Gk, dd, DK, DV, c0w, DV, 1.f);
    __syncthreads();
    mac_wide<kW>(acc, sm.At, sm.Bw, wy, wx);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < kC; ++j) acc[i][j] *= sm.fw[wy * 8 + i];
  const long chunk_end = (long)(k + 1) * L;
  for (long q0 = s0; q0 < chunk_end && q0 < T; q0 += kT) {
    if (tid < kT) sm.mu[tid] = fmaxf(m_in, g.amax[(long)bh * tpad + q0 + tid]);
    float S[4][4] = {};  // [key s][query t] = k^_s . q_t
    for (int dd = 0; dd < DK; dd += kS) {
      load_cmajor<TIn, kTP>(sm.At, K + base * DK, s0, kT, T, DK, dd, DK, p.key_scale);
      load_cmajor<TIn, kW>(sm.Bw, Q + base * DK, q0, kT, T, DK, dd, DK, 1.f);
      __syncthreads();
      mac_square<kW>(S, sm.At, sm.Bw, ty, tx);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sr = ty * 4 + i, tq = tx * 4 + j;
        const bool ok = q0 + tq >= s0 + sr && q0 + tq < T;
        sm.Pt[tq][sr] = ok ? expf(sm.acol[sr] - sm.mu[tq]) * S[i][j] : 0.f;
      }
    for (int half = 0; half < 2; ++half) {
      load_rmajor<float, kW>(sm.Bw, dU + base * DV, q0 + half * kS, T, DV, c0w, DV, 1.f);
      __syncthreads();
      mac_wide<kW>(acc, sm.Pt + half * kS, sm.Bw, wy, wx);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long sr = s0 + wy * 8 + i;
#pragma unroll
    for (int j = 0; j < kC; ++j) {
      const int c = c0w + wide_col<kW>(wx, j);
      if (sr < T && c < DV) dV[(base + sr) * DV + c] = from_float<TIn>(acc[i][j]);
    }
  }
}

// ---------------------------------------------------------------------------
// Gate gradients, one block per (b, h): di from k.dk, df from the reverse
// scan of q.dq - k.dk, and dm0 = <C0, dC0> + n0 . dn0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThr)
bwd_gates_kernel(Problem p, const float* __restrict__ i_pre, const float* __restrict__ f_pre,
                 const float* __restrict__ qdq, const float* __restrict__ kdk,
                 float* __restrict__ di, float* __restrict__ df, const float* __restrict__ C0,
                 const float* __restrict__ n0, const float* __restrict__ dC0,
                 const float* __restrict__ dn0, float* __restrict__ dm0) {
  __shared__ float seg[kThr];
  const int bh = blockIdx.x, tid = threadIdx.x;
  const long T = p.T, base = (long)bh * T;
  // thread tid owns tokens [lo, hi)
  const long per = (T + kThr - 1) / kThr;
  const long lo = tid * per < T ? tid * per : T, hi = lo + per < T ? lo + per : T;
  float sum = 0.f;
  for (long t = lo; t < hi; ++t) {
    const float i = i_pre[base + t];
    const float dli = kdk[base + t];
    di[base + t] = p.gate_sigmoid ? dli / (1.f + expf(i)) : dli;  // 1 - sigmoid(i) = 1/(1+e^i)
    sum += qdq[base + t] - kdk[base + t];
  }
  seg[tid] = sum;
  __syncthreads();
  // suffix sums of the segment totals (inclusive, from the right)
  for (int o = 1; o < kThr; o <<= 1) {
    const float add = tid + o < kThr ? seg[tid + o] : 0.f;
    __syncthreads();
    seg[tid] += add;
    __syncthreads();
  }
  float run = tid + 1 < kThr ? seg[tid + 1] : 0.f;  // everything right of this segment
  for (long t = hi - 1; t >= lo; --t) {
    run += qdq[base + t] - kdk[base + t];
    df[base + t] = run / (1.f + expf(f_pre[base + t]));  // d log f / d f~ = 1 - sigmoid(f~)
  }
  if (dm0) {
    float acc = 0.f;
    if (C0) {
      const long n = (long)p.DK * p.DV;
      for (long e = tid; e < n; e += kThr) acc = fmaf(C0[bh * n + e], dC0[bh * n + e], acc);
      for (int e = tid; e < p.DK; e += kThr)
        acc = fmaf(n0[(long)bh * p.DK + e], dn0[(long)bh * p.DK + e], acc);
    }
    __syncthreads();
    seg[tid] = acc;
    __syncthreads();
    for (int o = kThr / 2; o > 0; o >>= 1) {
      if (tid < o) seg[tid] += seg[tid + o];
      __syncthreads();
    }
    if (tid == 0) dm0[bh] = seg[0];
  }
}

// Segments of the reverse recurrence: enough (b, h, tile, segment) blocks
// for about four per SM of a 148-SM B200, at most 8 segments, each at least
// two chunks and none empty.
int bwd_segments(const Problem& p) {
  const int units = p.BH * ((p.DK + kT - 1) / kT) * ((p.DV + kT - 1) / kT);
  int s = 4 * 148 / units;
  if (s > 8) s = 8;
  if (s > p.NC / 2) s = p.NC / 2;
  while (s > 1 && (s - 1) * ((p.NC + s - 1) / s) >= p.NC) --s;
  return s < 1 ? 1 : s;
}

// Picks the column range of the wide gradient kernels for an output of D
// columns and calls fn(std::integral_constant<int, W>, grid, shared bytes).
template <typename TIn, typename Fn>
cudaError_t launch_wide(const Problem& p, int D, Fn&& fn) {
  const dim3 g64((D + 63) / 64, (p.T + kT - 1) / kT, p.BH);
  const dim3 g128((D + 127) / 128, g64.y, p.BH), g256((D + 255) / 256, g64.y, p.BH);
  if (D > 128) return fn(std::integral_constant<int, 256>{}, g256, sizeof(WideSmem<256>));
  if (D > 64) return fn(std::integral_constant<int, 128>{}, g128, sizeof(WideSmem<128>));
  return fn(std::integral_constant<int, 64>{}, g64, sizeof(WideSmem<64>));
}

// Workspace carve (all fp32): see bwd_workspace_bytes.
struct BwdWs {
  Gates g;
  float *C_states, *n_states, *H32, *den, *mr, *dU, *dA, *G_states, *g_states, *qdq, *kdk, *dC0,
      *dn0, *seg;
  __nv_bfloat16 *Cb, *H16;  // tensor-core recompute: operand copy of the states, bf16 h
  // tensor-core gradients: du~ (plain and row-scaled), reverse states, squares,
  // per-chunk increments of g~
  __nv_bfloat16 *dU16, *dUr16, *Gb, *sq;
  float* uvec;
};

// Whether the forward is recomputed on the tensor cores.
bool tc_recompute(const Problem& p, mlstm_dtype dt) {
  return dt == MLSTM_DT_BF16 && tc_unfused_supported(p);
}

// The tensor-core gradients work in chunks of 128 tokens (one MMA tile of
// rows) whatever the caller's chunk size: the gradients do not depend on the
// chunking (up to rounding), and the whole backward, recomputed forward
// included, then runs on that chunking.
Problem tc_bwd_problem(const Problem& p) {
  Problem pb = p;
  pb.L = 128;
  pb.NC = (p.T + 127) / 128;
  return pb;
}
// Sequences shorter than one such chunk stay on the fp32 kernels: they cost
// nothing there, and with a handful of tokens the terms of the forget-gate
// gradient (sums of q.dq - k.dk) cancel far below the bf16 operands' rounding.
bool tc_backward(const Problem& p, mlstm_dtype dt) {
  return dt == MLSTM_DT_BF16 && p.T >= 128 && tc_bwd_supported(tc_bwd_problem(p));
}

constexpr size_t kAlign = 256;
inline size_t al(size_t b) { return (b + kAlign - 1) / kAlign * kAlign; }

// saved: the tensor-core backward given the training forward's saved buffers
// (no room for the recomputed forward: chunk states, h, denominators).
size_t carve(const Problem& p_in, mlstm_dtype dt, char* base, BwdWs* w, bool saved = false) {
  const bool tcb = tc_backward(p_in, dt);
  const Problem p = tcb ? tc_bwd_problem(p_in) : p_in;
  const size_t BH = p.BH, T = p.T, NC = p.NC, tpad = NC * p.L, DK = p.DK, DV = p.DV;
  const bool tc = tcb || tc_recompute(p, dt);
  const bool rec = !(tcb && saved);  // room for the recomputed forward
  size_t off = 0;
  auto take = [&](size_t n) -> float* {
    float* ptr = base ? reinterpret_cast<float*>(base + off) : nullptr;
    off += al(n * sizeof(float));
    return ptr;
  };
  auto take16 = [&](size_t n) -> __nv_bfloat16* {
    __nv_bfloat16* ptr = base ? reinterpret_cast<__nv_bfloat16*>(base + off) : nullptr;
    off += al(n * sizeof(__nv_bfloat16));
    return ptr;
  };
  Gates g;
  g.bcum = take(BH * tpad);
  g.acol = take(BH * tpad);
  g.amax = take(BH * tpad);
  g.gtot = take(BH * NC);
  g.mchk = take(BH * (NC + 1));
  BwdWs x = {};
  x.g = g;
  x.C_states = tcb ? nullptr : take(BH * NC * DK * DV);
  x.n_states = rec ? take(BH * NC * DK) : nullptr;
  x.H32 = tc ? nullptr : take(BH * T * DV);
  x.Cb = tc && rec ? take16(BH * NC * DK * DV) : nullptr;
  x.H16 = tc && rec ? take16(BH * T * DV) : nullptr;
  x.seg = tc && rec ? take(tc_states_segment_floats(p)) : nullptr;
  x.den = rec ? take(BH * T) : nullptr;
  x.mr = rec ? take(BH * T) : nullptr;
  x.dU = tcb ? nullptr : take(BH * T * DV);
  x.dA = take(BH * T);
  x.G_states = tcb ? nullptr : take(BH * (NC + 1) * DK * DV);
  x.g_states = take(BH * (NC + 1) * DK);
  x.qdq = take(BH * T);
  x.kdk = take(BH * T);
  x.dC0 = take(BH * DK * DV);
  x.dn0 = take(BH * DK);
  if (tcb) {
    x.dU16 = take16(BH * T * DV);
    x.dUr16 = take16(BH * T * DV);
    x.Gb = take16(BH * (NC + 1) * DK * DV);
    x.sq = take16(tc_bwd_square_elems(p));
    x.uvec = take(BH * NC * DK);
  }
  if (w) *w = x;
  return off;
}

// The backward on the tensor cores (bf16, 128-token chunks): the forward
// recomputed on the tensor cores (gates, chunk states as the bf16 operand
// copy, h and the signed denominator), the per-token pass (du~ in bf16, plain
// and row-scaled), the reverse states (per-chunk updates on the tensor cores,
// then a reverse scan), the squares and dq, dk, dv (tc_bwd.cu), and the gate
// gradients.
// The gradients of the tensor-core backward from the forward's chunk states
// (bf16 operand copy Cb, fp32 n_states), h (bf16), signed denominators and
// per-token stabilisers, all at 128-token chunks.
cudaError_t bwd_tc_grads(const Problem& p, BwdWs& w, const void* Q, const void* K, const void* V,
                         const float* i_pre, const float* f_pre, const float* C0, const float* n0,
                         const __nv_bfloat16* Cb, const float* n_states, const __nv_bfloat16* H,
                         const float* den, const float* mr, const void* dH, void* dQ, void* dK,
                         void* dV, float* di, float* df, float* dC0, float* dn0, float* dm0,
                         cudaStream_t st) {
  const long toks = (long)p.BH * p.T;
  bwd_prep_tc_kernel<<<(unsigned)((toks + 7) / 8), kThr, 0, st>>>(
      p, static_cast<const __nv_bfloat16*>(dH), H, den, mr, w.g, w.dA, w.dU16, w.dUr16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_tc_bwd_states(p, Q, w.dUr16, w.g, w.dA, w.uvec, w.Gb, w.g_states, w.dC0, st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpy2DAsync(w.dn0, sizeof(float) * p.DK, w.g_states, sizeof(float) * (p.NC + 1) * p.DK,
                        sizeof(float) * p.DK, p.BH, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(w.qdq, 0, sizeof(float) * toks, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(w.kdk, 0, sizeof(float) * toks, st);
  if (e != cudaSuccess) return e;
  e = launch_tc_bwd(p, Q, K, V, w.dU16, w.g, w.dA, n_states, w.g_states, Cb, w.Gb, w.sq, dQ, dK,
                    dV, w.qdq, w.kdk, st);
  if (e != cudaSuccess) return e;
  bwd_gates_kernel<<<p.BH, kThr, 0, st>>>(p, i_pre, f_pre, w.qdq, w.kdk, di, df, C0, n0, w.dC0,
                                          w.dn0, dm0);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (dC0) {
    e = cudaMemcpyAsync(dC0, w.dC0, sizeof(float) * p.BH * p.DK * p.DV,
                        cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  if (dn0)
    e = cudaMemcpyAsync(dn0, w.dn0, sizeof(float) * p.BH * p.DK, cudaMemcpyDeviceToDevice, st);
  return e;
}

// The forward on the tensor cores at 128-token chunks, keeping what the
// gradients need: chunk states (Cb, n_states), h in H, signed denominators
// and stabilisers (den, mr); the final state when C_T is given.
cudaError_t fw_tc_keep(const Problem& p, Gates g, float* seg, const void* Q, const void* K,
                       const void* V, const float* i_pre, const float* f_pre, const float* C0,
                       const float* n0, const float* m0, __nv_bfloat16* Cb, float* n_states,
                       void* H, float* den, float* mr, float* C_T, float* n_T, float* m_T,
                       cudaStream_t st) {
  cudaError_t e = launch_gates(p, i_pre, f_pre, m0, g, st);
  if (e != cudaSuccess) return e;
  e = launch_tc_states(p, K, V, C0, n0, g, nullptr, Cb, n_states, C_T, n_T, m_T, seg, st);
  if (e != cudaSuccess) return e;
  Problem ps = p;
  ps.signed_den = 1;  // the outputs keep the sign of the denominator
  return launch_tc_parallel(ps, Q, K, V, g, Cb, n_states, H, den, mr, st);
}

// The backward on the tensor cores (bf16, 128-token chunks): the forward
// recomputed on the tensor cores (gates, chunk states as the bf16 operand
// copy, h and the signed denominator), the per-token pass (du~ in bf16, plain
// and row-scaled), the reverse states (g~ increments, then the recurrence),
// the squares and dq, dk, dv (tc_bwd.cu), and the gate gradients.
cudaError_t launch_bwd_tc(const Problem& p_in, const void* Q, const void* K, const void* V,
                          const float* i_pre, const float* f_pre, const float* C0,
                          const float* n0, const float* m0, const void* dH, void* dQ, void* dK,
                          void* dV, float* di, float* df, float* dC0, float* dn0, float* dm0,
                          void* ws, cudaStream_t st) {
  const Problem p = tc_bwd_problem(p_in);
  BwdWs w;
  carve(p_in, MLSTM_DT_BF16, static_cast<char*>(ws), &w);
  cudaError_t e = fw_tc_keep(p, w.g, w.seg, Q, K, V, i_pre, f_pre, C0, n0, m0, w.Cb, w.n_states,
                             w.H16, w.den, w.mr, nullptr, nullptr, nullptr, st);
  if (e != cudaSuccess) return e;
  return bwd_tc_grads(p, w, Q, K, V, i_pre, f_pre, C0, n0, w.Cb, w.n_states, w.H16, w.den, w.mr,
                      dH, dQ, dK, dV, di, df, dC0, dn0, dm0, st);
}

template <typename TIn>
cudaError_t launch_bwd_t(const Problem& p, mlstm_dtype dt, const void* Q, const void* K,
                         const void* V, const float* i_pre, const float* f_pre, const float* C0,
                         const float* n0, const float* m0, const void* dH, void* dQ, void* dK,
                         void* dV, float* di, float* df, float* dC0, float* dn0, float* dm0,
                         void* ws, cudaStream_t st) {
  BwdWs w;
  carve(p, dt, static_cast<char*>(ws), &w);
  const TIn* q = static_cast<const TIn*>(Q);
  const TIn* k = static_cast<const TIn*>(K);
  const TIn* v = static_cast<const TIn*>(V);
  Problem ps = p;
  ps.signed_den = 1;  // the forward outputs keep the sign of the denominator
  const bool tc = tc_recompute(p, dt);
  cudaError_t e = launch_gates(p, i_pre, f_pre, m0, w.g, st);
  if (e != cudaSuccess) return e;
  if (tc) {
    e = launch_tc_states(p, K, V, C0, n0, w.g, w.C_states, nullptr, w.n_states, nullptr, nullptr,
                         nullptr, w.seg, st);
    if (e != cudaSuccess) return e;
    e = launch_states_to_operand(w.C_states, w.Cb, (long)p.BH * p.NC, p.DK, p.DV, st);
    if (e != cudaSuccess) return e;
    e = launch_tc_parallel(ps, Q, K, V, w.g, w.Cb, w.n_states, w.H16, w.den, w.mr, st);
  } else {
    e = launch_simt_states(p, dt, K, V, C0, n0, w.g, w.C_states, w.n_states, nullptr, nullptr,
                           nullptr, st);
    if (e != cudaSuccess) return e;
    e = launch_simt_parallel(ps, dt, Q, K, V, w.g, w.C_states, w.n_states, nullptr, w.den, w.mr,
                             st, w.H32);
  }
  if (e != cudaSuccess) return e;
  const long toks = (long)p.BH * p.T;
  const unsigned prep_blocks = (unsigned)((toks + 7) / 8);
  if (tc)
    bwd_prep_kernel<TIn, __nv_bfloat16><<<prep_blocks, kThr, 0, st>>>(
        p, static_cast<const TIn*>(dH), w.H16, w.den, w.mr, w.dU, w.dA);
  else
    bwd_prep_kernel<TIn, float><<<prep_blocks, kThr, 0, st>>>(
        p, static_cast<const TIn*>(dH), w.H32, w.den, w.mr, w.dU, w.dA);
  const int nk = (p.DK + kT - 1) / kT, nv = (p.DV + kT - 1) / kT;
  const int n_seg = bwd_segments(p);
  bwd_states_kernel<TIn><<<dim3(nv, nk, p.BH * n_seg), kThr, 0, st>>>(p, q, w.dU, w.dA, w.g,
                                                                     w.G_states, w.g_states, n_seg);
  if (n_seg > 1) {
    const long n_el = (long)p.DK * p.DV + p.DK;
    bwd_states_fixup_kernel<<<dim3((unsigned)((n_el + kThr - 1) / kThr), p.BH), kThr, 0, st>>>(
        p, w.g, w.G_states, w.g_states, n_seg);
  }
  // dC0 = G~_0, dn0 = g~_0 (index 0 of every head's states)
  e = cudaMemcpy2DAsync(w.dC0, sizeof(float) * p.DK * p.DV, w.G_states,
                        sizeof(float) * (p.NC + 1) * p.DK * p.DV, sizeof(float) * p.DK * p.DV,
                        p.BH, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpy2DAsync(w.dn0, sizeof(float) * p.DK, w.g_states, sizeof(float) * (p.NC + 1) * p.DK,
                        sizeof(float) * p.DK, p.BH, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(w.qdq, 0, sizeof(float) * toks, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(w.kdk, 0, sizeof(float) * toks, st);
  if (e != cudaSuccess) return e;
  e = launch_wide<TIn>(p, p.DK, [&](auto wtag, dim3 grid, size_t smem) {
    constexpr int W = decltype(wtag)::value;
    const cudaError_t ea = cudaFuncSetAttribute(bwd_dq_kernel<TIn, W>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
    if (ea != cudaSuccess) return ea;
    bwd_dq_kernel<TIn, W><<<grid, kThr, smem, st>>>(p, q, k, v, w.g, w.C_states, w.n_states,
                                                    w.dU, w.dA, static_cast<TIn*>(dQ), w.qdq);
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  e = launch_wide<TIn>(p, p.DK, [&](auto wtag, dim3 grid, size_t smem) {
    constexpr int W = decltype(wtag)::value;
    const cudaError_t ea = cudaFuncSetAttribute(bwd_dk_kernel<TIn, W>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
    if (ea != cudaSuccess) return ea;
    bwd_dk_kernel<TIn, W><<<grid, kThr, smem, st>>>(p, q, k, v, w.g, w.G_states, w.g_states,
                                                    w.dU, w.dA, static_cast<TIn*>(dK), w.kdk);
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  e = launch_wide<TIn>(p, p.DV, [&](auto wtag, dim3 grid, size_t smem) {
    constexpr int W = decltype(wtag)::value;
    const cudaError_t ea = cudaFuncSetAttribute(bwd_dv_kernel<TIn, W>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
    if (ea != cudaSuccess) return ea;
    bwd_dv_kernel<TIn, W><<<grid, kThr, smem, st>>>(p, q, k, w.g, w.G_states, w.dU,
                                                    static_cast<TIn*>(dV));
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  bwd_gates_kernel<<<p.BH, kThr, 0, st>>>(p, i_pre, f_pre, w.qdq, w.kdk, di, df, C0, n0, w.dC0,
                                          w.dn0, dm0);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (dC0) {
    e = cudaMemcpyAsync(dC0, w.dC0, sizeof(float) * p.BH * p.DK * p.DV,
                        cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  if (dn0)
    e = cudaMemcpyAsync(dn0, w.dn0, sizeof(float) * p.BH * p.DK, cudaMemcpyDeviceToDevice, st);
  return e;
}

}  // namespace

size_t bwd_workspace_bytes(const Problem& p, mlstm_dtype dt) { return carve(p, dt, nullptr, nullptr); }

int bwd_launches(const Problem& p, mlstm_dtype dt) {
  // gates (2) + recompute (simt: 2; tensor cores: states [+ fix-up] + operand copy + outputs)
  // + prep, reverse states [+ fix-up], dq, dk, dv, gate gradients (6 or 7)
  if (tc_backward(p, dt)) {
    // gates (2), chunk states [+ fix-up], outputs, prep, reverse states
    // (g~ increments, recurrence), squares + dq + dk + dv, gate gradients
    const Problem pb = tc_bwd_problem(p);
    return 2 + tc_states_launches(pb) + 1 + 1 + kTcBwdStateLaunches + kTcBwdLaunches + 1;
  }
  return 2 + (tc_recompute(p, dt) ? 2 + tc_states_launches(p) : 2) + 6 +
         (bwd_segments(p) > 1 ? 1 : 0);
}

cudaError_t launch_backward(const Problem& p, mlstm_dtype dt, const void* Q, const void* K,
                            const void* V, const float* i_pre, const float* f_pre,
                            const float* C0, const float* n0, const float* m0, const void* dH,
                            void* dQ, void* dK, void* dV, float* di, float* df, float* dC0,
                            float* dn0, float* dm0, void* ws, cudaStream_t st) {
  if (tc_backward(p, dt))
    return launch_bwd_tc(p, Q, K, V, i_pre, f_pre, C0, n0, m0, dH, dQ, dK, dV, di, df, dC0, dn0,
                         dm0, ws, st);
  if (dt == MLSTM_DT_BF16)
    return launch_bwd_t<__nv_bfloat16>(p, dt, Q, K, V, i_pre, f_pre, C0, n0, m0, dH, dQ, dK, dV,
                                       di, df, dC0, dn0, dm0, ws, st);
  return launch_bwd_t<float>(p, dt, Q, K, V, i_pre, f_pre, C0, n0, m0, dH, dQ, dK, dV, di, df,
                             dC0, dn0, dm0, ws, st);
}


// ---------------------------------------------------------------------------
// Training pair: the forward that keeps what the tensor-core backward needs,
// and that backward without the recomputation.
// ---------------------------------------------------------------------------
namespace {

struct Saved {
  __nv_bfloat16* Cb;
  float *n_states, *den, *mr;
};

// Saved buffer: the bf16 chunk states and n states entering every 128-token
// chunk, then per token the signed denominator and the stabiliser.
size_t saved_carve(const Problem& p_in, char* base, Saved* out) {
  const Problem p = tc_bwd_problem(p_in);
  const size_t BH = p.BH, T = p.T, NC = p.NC, DK = p.DK, DV = p.DV;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* ptr = base ? base + off : nullptr;
    off += al(bytes);
    return ptr;
  };
  Saved x;
  x.Cb = reinterpret_cast<__nv_bfloat16*>(take(BH * NC * DK * DV * 2));
  x.n_states = reinterpret_cast<float*>(take(BH * NC * DK * 4));
  x.den = reinterpret_cast<float*>(take(BH * T * 4));
  x.mr = reinterpret_cast<float*>(take(BH * T * 4));
  if (out) *out = x;
  return off;
}

// Training forward workspace: the gates and the segment end states.
size_t fw_train_carve(const Problem& p_in, char* base, Gates* g, float** seg) {
  const Problem p = tc_bwd_problem(p_in);
  const size_t BH = p.BH, NC = p.NC, tpad = NC * p.L;
  size_t off = 0;
  auto take = [&](size_t n) -> float* {
    float* ptr = base ? reinterpret_cast<float*>(base + off) : nullptr;
    off += al(n * sizeof(float));
    return ptr;
  };
  Gates x;
  x.bcum = take(BH * tpad);
  x.acol = take(BH * tpad);
  x.amax = take(BH * tpad);
  x.gtot = take(BH * NC);
  x.mchk = take(BH * (NC + 1));
  float* sg = take(tc_states_segment_floats(p));
  if (g) *g = x;
  if (seg) *seg = sg;
  return off;
}

}  // namespace

bool train_supported(const Problem& p, mlstm_dtype dt) { return tc_backward(p, dt); }
size_t train_saved_bytes(const Problem& p) { return saved_carve(p, nullptr, nullptr); }
size_t fw_train_workspace_bytes(const Problem& p) { return fw_train_carve(p, nullptr, nullptr, nullptr); }
size_t bw_saved_workspace_bytes(const Problem& p) {
  return carve(p, MLSTM_DT_BF16, nullptr, nullptr, true);
}
int fw_train_launches(const Problem& p) { return 2 + tc_states_launches(tc_bwd_problem(p)) + 1; }
int bw_saved_launches(const Problem&) { return 2 + 1 + kTcBwdStateLaunches + kTcBwdLaunches + 1; }

cudaError_t launch_fw_train(const Problem& p_in, const void* Q, const void* K, const void* V,
                            const float* i_pre, const float* f_pre, const float* C0,
                            const float* n0, const float* m0, void* H, float* C_T, float* n_T,
                            float* m_T, void* saved, void* ws, cudaStream_t st) {
  const Problem p = tc_bwd_problem(p_in);
  Saved sv;
  saved_carve(p_in, static_cast<char*>(saved), &sv);
  Gates g;
  float* seg = nullptr;
  fw_train_carve(p_in, static_cast<char*>(ws), &g, &seg);
  return fw_tc_keep(p, g, seg, Q, K, V, i_pre, f_pre, C0, n0, m0, sv.Cb, sv.n_states, H, sv.den,
                    sv.mr, C_T, n_T, m_T, st);
}

cudaError_t launch_bw_saved(const Problem& p_in, const void* Q, const void* K, const void* V,
                            const float* i_pre, const float* f_pre, const float* C0,
                            const float* n0, const float* m0, const void* H, const void* saved,
                            const void* dH, void* dQ, void* dK, void* dV, float* di, float* df,
                            float* dC0, float* dn0, float* dm0, void* ws, cudaStream_t st) {
  const Problem p = tc_bwd_problem(p_in);
  Saved sv;
  saved_carve(p_in, static_cast<char*>(const_cast<void*>(saved)), &sv);
  BwdWs w;
  carve(p_in, MLSTM_DT_BF16, static_cast<char*>(ws), &w, true);
  // the same gates as the training forward (a function of the gate inputs)
  cudaError_t e = launch_gates(p, i_pre, f_pre, m0, w.g, st);
  if (e != cudaSuccess) return e;
  return bwd_tc_grads(p, w, Q, K, V, i_pre, f_pre, C0, n0, sv.Cb, sv.n_states,
                      static_cast<const __nv_bfloat16*>(H), sv.den, sv.mr, dH, dQ, dK, dV, di, df,
                      dC0, dn0, dm0, st);
}

}  // namespace mlstm
