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
// Kernel 1: gates_chunk_kernel, one CTA per (chunk, b*h) with block-wide
// scans (the backward pass and every call without the dominance marks use
// it; with the marks, chunks of more than 128 tokens); gates_chunk_warp_kernel,
// one warp per (chunk, b*h) with warp scans (the forward tensor-core paths at
// chunks of at most 128 tokens, where a CTA per chunk leaves most threads
// idle).  Both write the same arrays; with the marks, also the per-chunk
// dominance statistics below.
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
constexpr int kChunksPerBlock = kGateThreads / 32;  // warp-per-chunk kernel

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

template <bool kDominance>
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
  if constexpr (kDominance) {
    // The max scan left the inclusive warp totals in smem[32..]: the last is
    // the chunk's largest acol.  Then sum_s e^{acol_s - max} and the first
    // token attaining the max, by a block reduction.
    __shared__ float sum_s[kGateThreads / 32];
    __shared__ int idx_s[kGateThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float cmax = smem[32 + kGateThreads / 32 - 1];
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
}

// One warp per (chunk, b*h), 32 tokens per round: warp scans of lf (sum) and
// acol (max) carried from round to round.  The sum runs in fp64, so bcum and
// acol are the fp32 roundings of the exact partial sums.  It also keeps,
// online, the chunk's largest acol, sum_s e^{acol_s - max} (rescaled when the
// max grows) and the first token that attains the max.
__global__ void __launch_bounds__(kGateThreads)
gates_chunk_warp_kernel(Problem p, const float* __restrict__ i_pre, const float* __restrict__ f_pre,
                        Gates g) {
  const int lane = threadIdx.x & 31;
  const long cid = (long)blockIdx.x * kChunksPerBlock + (threadIdx.x >> 5);
  if (cid >= (long)p.BH * p.NC) return;
  const int bh = (int)(cid / p.NC), k = (int)(cid % p.NC);
  const int L = p.L;
  const long tpad = (long)p.NC * L;
  const long base = (long)bh * tpad + (long)k * L;
  const bool dominance = g.dom != nullptr;
  double run_b = 0.0;
  float run_m = -INFINITY;
  float dmax = -INFINITY, dsum = 0.f;
  int didx = 0;
  for (int r0 = 0; r0 < L; r0 += 32) {
    const int r = r0 + lane;
    const long t = (long)k * L + r;
    float lf = 0.f, li = -INFINITY;
    if (t < p.T) {
      lf = logsigmoidf(f_pre[(long)bh * p.T + t]);
      const float x = i_pre[(long)bh * p.T + t];
      li = p.gate_sigmoid ? logsigmoidf(x) : x;
    }
    double bd = lf;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, bd, o);
      if (lane >= o) bd += y;
    }
    bd += run_b;
    run_b = __shfl_sync(0xffffffffu, bd, 31);
    const float b = (float)bd;
    const float a = (float)((double)li - bd);  // -inf on padding
    float am = a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, am, o);
      if (lane >= o) am = fmaxf(am, y);
    }
    am = fmaxf(am, run_m);
    run_m = __shfl_sync(0xffffffffu, am, 31);
    g.bcum[base + r] = b;
    g.acol[base + r] = a;
    g.amax[base + r] = am;
    if (dominance) {
      float e = expf(a - run_m);  // -inf (padding) -> 0; run_m is finite from round 0 on
#pragma unroll
      for (int o = 16; o; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
      dsum = dsum * expf(dmax - run_m) + e;  // dmax = -inf at first: 0 * 0
      const unsigned hit = __ballot_sync(0xffffffffu, a == run_m);
      if (run_m > dmax && hit) didx = r0 + __ffs(hit) - 1;
      dmax = run_m;
    }
  }
  if (lane == 0) {
    g.gtot[(long)bh * p.NC + k] = (float)run_b;
    if (dominance) {
      g.csum[(long)bh * p.NC + k] = dsum;
      g.cidx[(long)bh * p.NC + k] = didx;
    }
  }
}

// One warp per (b, h): m_{k+1} = max(m_k + g_k, c_k) with c_k = g_k + amax at
// the chunk end.  The maps x -> max(x + G, C) compose associatively:
// (later o earlier) has G = G_l + G_e and C = max(C_e + G_l, C_l).  The same
// prefix maps give M (another starting value) and, with the index of the term
// that attains C carried along, the dominant token.  Chunks go in groups of
// 32 (one per lane); the next group's loads are issued before this group's
// scans.
__global__ void gates_state_kernel(Problem p, const float* __restrict__ m0, Gates g) {
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (bh >= p.BH) return;
  const bool dominance = g.dom != nullptr;
  float carry = m0 ? m0[bh] : 0.f;
  float* mchk = g.mchk + (long)bh * (p.NC + 1);
  if (lane == 0) mchk[0] = carry;
  const long tpad = (long)p.NC * p.L;
  // dominance carries: M (-inf without an initial state), its index (-1: the
  // initial state), and z
  float cM = m0 ? m0[bh] : -INFINITY, cz = m0 ? 1.f : 0.f;
  int cI = -1;
  int* dom = dominance ? g.dom + (long)bh * p.NC : nullptr;
  bool any = false;
  float* mdom = dominance ? g.mdom + (long)bh * p.NC : nullptr;
  if (dominance && lane == 0 && p.NC > 0) {
    dom[0] = -1;
    mdom[0] = cM;
  }
  auto load = [&](int k, float& gk, float& amx, int& ci, float& cs) {
    gk = 0.f;
    amx = -INFINITY;
    ci = 0;
    cs = 0.f;
    if (k < p.NC) {
      gk = g.gtot[(long)bh * p.NC + k];
      amx = g.amax[(long)bh * tpad + (long)k * p.L + p.L - 1];
      if (dominance) {
        ci = g.cidx[(long)bh * p.NC + k];
        cs = g.csum[(long)bh * p.NC + k];
      }
    }
  };
  float n_gk, n_amx, n_cs;
  int n_ci;
  load(lane, n_gk, n_amx, n_ci, n_cs);
  for (int k0 = 0; k0 < p.NC; k0 += 32) {
    const int k = k0 + lane;
    const float gk = n_gk, amx = n_amx, cs = n_cs;
    const int ci = n_ci;
    if (k0 + 32 < p.NC) load(k + 32, n_gk, n_amx, n_ci, n_cs);
    float G = gk, C = k < p.NC ? gk + amx : -INFINITY;  // identity map past NC
    int I = k * p.L + ci;
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
    const float m = fmaxf(carry + G, C);
    if (k < p.NC) mchk[k + 1] = m;
    carry = __shfl_sync(0xffffffffu, m, 31);
    if (!dominance) continue;

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
    any = any || __any_sync(0xffffffffu, k + 1 < p.NC && z < 2.f && Io >= 0);
    cM = __shfl_sync(0xffffffffu, Mo, 31);
    cI = __shfl_sync(0xffffffffu, Io, 31);
    cz = __shfl_sync(0xffffffffu, z, 31);
  }
  if (dominance && lane == 0) g.hdom[bh] = any ? 1 : 0;
}

}  // namespace

cudaError_t launch_gates(const Problem& p, const float* i_pre, const float* f_pre,
                         const float* m0, Gates g, cudaStream_t st) {
  if (p.NC > 0 && g.dom && p.L > 128) {
    dim3 grid(p.NC, p.BH);
    gates_chunk_kernel<true><<<grid, kGateThreads, 0, st>>>(p, i_pre, f_pre, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else if (p.NC > 0 && g.dom) {
    const long chunks = (long)p.BH * p.NC;
    const long blocks = (chunks + kChunksPerBlock - 1) / kChunksPerBlock;
    if (blocks > 0x7fffffffL) return cudaErrorInvalidValue;
    gates_chunk_warp_kernel<<<(unsigned)blocks, kGateThreads, 0, st>>>(p, i_pre, f_pre, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else if (p.NC > 0) {
    dim3 grid(p.NC, p.BH);
    gates_chunk_kernel<false><<<grid, kGateThreads, 0, st>>>(p, i_pre, f_pre, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int warps = 8;
  gates_state_kernel<<<(p.BH + warps - 1) / warps, warps * 32, 0, st>>>(p, m0, g);
  return cudaGetLastError();
}

}  // namespace mlstm
