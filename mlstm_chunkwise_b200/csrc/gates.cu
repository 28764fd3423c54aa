// G1: gate preprocessing for the chunkwise mLSTM forward pass.
//
// Chunkwise form ("Tiled Flash Linear Attention: More Efficient Linear RNN
// and xLSTM Kernels", abstract: the chunkwise-parallel formulation that
// parallelises over chunks).  Inside chunk k with local index r:
//   lf_r = logsigmoid(f~_r)                forget gate in log space
//   li_r = i~_r | logsigmoid(i~_r)         input gate (exp | sigmoid mode)
//   bcum_r = sum_{s<=r} lf_s               inclusive scan inside the chunk
//   acol_r = li_r - bcum_r                 column log-weight
//   amax_r = max_{s<=r} acol_s             running max inside the chunk
//   g_k    = bcum_{L-1}
//   m_k+1  = max(g_k + m_k, g_k + amax_{L-1})   state stabiliser (sequential
//            over chunks; an associative (max,+) recurrence, scanned by a warp)
// Tokens past T in a ragged last chunk get lf = 0 and li = -inf: they neither
// decay the state nor contribute to it.
//
// Kernel 1 (gates_chunk_kernel): one CTA per (chunk, b*h); block-wide scans.
// Kernel 2 (gates_state_kernel): one warp per b*h; warp scan of the (max,+)
// maps over chunks.
//
// Dominance (when g.dom is given).  The state entering chunk k is a sum of
// per-token terms with log-weights lw_j = li_j + (sum of lf after j), plus the
// initial state with log-weight m0 + (sum of lf) when one is given.  Let M_k
// be the largest of them (the same (max,+) recurrence as m, started from m0
// with an initial state and from -inf without one, and carrying the index of
// the token that attains it) and z_k = sum_j e^{lw_j - M_k} >= 1 (an affine
// recurrence over chunks, z_{k+1} = e^{g_k + M_k - M_{k+1}} z_k +
// e^{g_k + amax_{L-1} - M_{k+1}} csum_k).  When z_k < 2 one term holds more than
// half of the weight: then dom_k is that token (or -1 if it is the initial
// state).
#include <math.h>

#include "common.cuh"

namespace mlstm {

namespace {

constexpr int kGateThreads = 256;
constexpr int kMaxPerThread = 16;  // chunk sizes up to 4096

template <bool kMax>
__device__ __forceinline__ float combine(float a, float b) {
  return kMax ? fmaxf(a, b) : a + b;
}

// Exclusive block scan (sum or max) of one value per thread.
template <bool kMax>
__device__ float block_exclusive_scan(float v, float identity, float* smem) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl = combine<kMax>(incl, y);
  }
  if (lane == 31) smem[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    float w = lane < kGateThreads / 32 ? smem[lane] : identity;
    float wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      float y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi = combine<kMax>(wi, y);
    }
    if (lane < kGateThreads / 32) smem[32 + lane] = wi;  // inclusive warp totals
  }
  __syncthreads();
  float warp_off = warp == 0 ? identity : smem[32 + warp - 1];
  float excl_in_warp = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl_in_warp = identity;
  float r = combine<kMax>(warp_off, excl_in_warp);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kGateThreads)
gates_chunk_kernel(Problem p, const float* __restrict__ i_pre, const float* __restrict__ f_pre,
                   Gates g) {
  __shared__ float smem[64];
  const int k = blockIdx.x, bh = blockIdx.y;
  const int L = p.L;
  const int per = (L + kGateThreads - 1) / kGateThreads;
  const long tpad = (long)p.NC * L;
  const int first = threadIdx.x * per;

  float lcum[kMaxPerThread], li[kMaxPerThread];
  float run = 0.f;
#pragma unroll
  for (int e = 0; e < kMaxPerThread; ++e) {
    if (e >= per) break;
    const int r = first + e;
    const long t = (long)k * L + r;
    float lf = 0.f, l_i = -INFINITY;
    if (r < L && t < p.T) {
      lf = logsigmoidf(f_pre[(long)bh * p.T + t]);
      const float x = i_pre[(long)bh * p.T + t];
      l_i = p.gate_sigmoid ? logsigmoidf(x) : x;
    }
    run += lf;
    lcum[e] = run;
    li[e] = l_i;
  }
  const float off = block_exclusive_scan<false>(run, 0.f, smem);

  float pmax = -INFINITY;
  float acol[kMaxPerThread];
#pragma unroll
  for (int e = 0; e < kMaxPerThread; ++e) {
    if (e >= per) break;
    lcum[e] += off;
    acol[e] = li[e] - lcum[e];  // -inf on padding
    pmax = fmaxf(pmax, acol[e]);
    li[e] = pmax;               // reuse: local running max
  }
  const float moff = block_exclusive_scan<true>(pmax, -INFINITY, smem);

  const long base = (long)bh * tpad + (long)k * L;
#pragma unroll
  for (int e = 0; e < kMaxPerThread; ++e) {
    if (e >= per) break;
    const int r = first + e;
    if (r < L) {
      g.bcum[base + r] = lcum[e];
      g.acol[base + r] = acol[e];
      g.amax[base + r] = fmaxf(li[e], moff);
      if (r == L - 1) g.gtot[(long)bh * p.NC + k] = lcum[e];
    }
  }
  if (!g.dom) return;
  // The chunk's largest column log-weight (the inclusive max at its end), the
  // first token that attains it, and sum_s e^{acol_s - max}.
  __shared__ float cmax_s;
  __shared__ float sum_s[kGateThreads / 32];
  __shared__ int idx_s[kGateThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int e = 0; e < kMaxPerThread; ++e) {
    if (e >= per) break;
    if (first + e == L - 1) cmax_s = fmaxf(li[e], moff);  // amax is a running max
  }
  __syncthreads();
  const float cmax = cmax_s;
  float sum = 0.f;
  int idx = L;
#pragma unroll
  for (int e = 0; e < kMaxPerThread; ++e) {
    if (e >= per) break;
    const int r = first + e;
    if (r < L) {
      sum += expf(acol[e] - cmax);  // -inf (padding) -> 0
      if (acol[e] == cmax && r < idx) idx = r;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    idx = min(idx, __shfl_xor_sync(0xffffffffu, idx, o));
  }
  if (lane == 0) {
    sum_s[warp] = sum;
    idx_s[warp] = idx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    int best = L;
    for (int w = 0; w < kGateThreads / 32; ++w) {
      tot += sum_s[w];
      best = min(best, idx_s[w]);
    }
    g.csum[(long)bh * p.NC + k] = tot;
    g.cidx[(long)bh * p.NC + k] = best < L ? best : 0;
  }
}

// One warp per (b, h): m_{k+1} = max(m_k + g_k, c_k) with c_k = g_k + amax at
// the chunk end.  The maps x -> max(x + G, C) compose associatively:
// (later o earlier) has G = G_l + G_e and C = max(C_e + G_l, C_l).
__global__ void gates_state_kernel(Problem p, const float* __restrict__ m0, Gates g) {
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (bh >= p.BH) return;
  float carry = m0 ? m0[bh] : 0.f;
  float* mchk = g.mchk + (long)bh * (p.NC + 1);
  if (lane == 0) mchk[0] = carry;
  const long tpad = (long)p.NC * p.L;
  for (int k0 = 0; k0 < p.NC; k0 += 32) {
    const int k = k0 + lane;
    float G = 0.f, C = -INFINITY;  // identity map
    if (k < p.NC) {
      G = g.gtot[(long)bh * p.NC + k];
      C = G + g.amax[(long)bh * tpad + (long)k * p.L + p.L - 1];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float Ge = __shfl_up_sync(0xffffffffu, G, o);
      const float Ce = __shfl_up_sync(0xffffffffu, C, o);
      if (lane >= o) {
        C = fmaxf(Ce + G, C);
        G = G + Ge;
      }
    }
    const float m = fmaxf(carry + G, C);
    if (k < p.NC) mchk[k + 1] = m;
    carry = __shfl_sync(0xffffffffu, m, 31);
  }
  if (!g.dom) return;

  // Dominance: M_k with the index of the term that attains it (-1: the
  // initial state), then z_k.  dom_0 = -1: the state entering the first chunk
  // is the initial state alone (or zero).
  int* dom = g.dom + (long)bh * p.NC;
  float* mdom = g.mdom + (long)bh * p.NC;
  if (lane == 0 && p.NC > 0) {
    dom[0] = -1;
    mdom[0] = m0 ? m0[bh] : -INFINITY;
  }
  float cM = m0 ? m0[bh] : -INFINITY, cz = m0 ? 1.f : 0.f;
  int cI = -1;
  for (int k0 = 0; k0 < p.NC; k0 += 32) {
    const int k = k0 + lane;
    float gk = 0.f, G = 0.f, C = -INFINITY, amx = -INFINITY, cs = 0.f;
    int I = -1;
    if (k < p.NC) {
      gk = G = g.gtot[(long)bh * p.NC + k];
      amx = g.amax[(long)bh * tpad + (long)k * p.L + p.L - 1];
      C = G + amx;
      I = k * p.L + g.cidx[(long)bh * p.NC + k];
      cs = g.csum[(long)bh * p.NC + k];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float Ge = __shfl_up_sync(0xffffffffu, G, o);
      const float Ce = __shfl_up_sync(0xffffffffu, C, o);
      const int Ie = __shfl_up_sync(0xffffffffu, I, o);
      if (lane >= o) {
        if (Ce + G > C) {
          C = Ce + G;
          I = Ie;
        }
        G = G + Ge;
      }
    }
    // M_{k+1} and its index; M_k is the previous lane's (or the carry)
    float Mo = C;
    int Io = I;
    if (cM + G >= C) {
      Mo = cM + G;
      Io = cI;
    }
    float Mi = __shfl_up_sync(0xffffffffu, Mo, 1);
    if (lane == 0) Mi = cM;
    // z_{k+1} = a z_k + b, scanned as affine maps
    float a = 1.f, b = 0.f;
    if (k < p.NC) {
      a = Mi == -INFINITY ? 0.f : expf(gk + Mi - Mo);
      b = expf(gk + amx - Mo) * cs;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float ae = __shfl_up_sync(0xffffffffu, a, o);
      const float be = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) {
        b = fmaf(a, be, b);
        a = a * ae;
      }
    }
    const float z = fmaf(a, cz, b);
    if (k + 1 < p.NC) {
      dom[k + 1] = (z < 2.f) ? Io : -1;
      mdom[k + 1] = Mo;
    }
    cM = __shfl_sync(0xffffffffu, Mo, 31);
    cI = __shfl_sync(0xffffffffu, Io, 31);
    cz = __shfl_sync(0xffffffffu, z, 31);
  }
}

}  // namespace

cudaError_t launch_gates(const Problem& p, const float* i_pre, const float* f_pre,
                         const float* m0, Gates g, cudaStream_t st) {
  if (p.NC > 0) {
    dim3 grid(p.NC, p.BH);
    gates_chunk_kernel<<<grid, kGateThreads, 0, st>>>(p, i_pre, f_pre, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int warps = 8;
  gates_state_kernel<<<(p.BH + warps - 1) / warps, warps * 32, 0, st>>>(p, m0, g);
  return cudaGetLastError();
}

}  // namespace mlstm
