// Backward pass of the chunkwise mLSTM on tcgen05: the gradients dq, dk, dv
// of 128-token chunks ("Tiled Flash Linear Attention: More Efficient Linear
// RNN and xLSTM Kernels", abstract: the mLSTM as an inter-chunk recurrence
// plus an intra-chunk parallel part; its backward has the same two parts).
//
// In the stabilised frame of the forward (mu_t = max(m_k, amax_t) for token t
// of chunk k, k^ = s k with s = 1/sqrt(d_qk)) the per-chunk gradients are
//
//   dP_ts = (du~_t . v_s + da~_t) e^{acol_s - mu_t} [s <= t]
//   Sg_ts = (q_t . k^_s) e^{acol_s - mu_t} [s <= t]
//   dq_t  = sum_s dP_ts k^_s + e^{m_k - mu_t} (C_k du~_t + da~_t n_k)
//   dk^_s = sum_t dP_ts q_t  + w_s (G~_{k+1} v_s + g~_{k+1})
//   dv_s  = sum_t Sg_ts du~_t + w_s G~_{k+1}^T k^_s,     w_s = e^{g_k + acol_s - m_{k+1}}
//
// (the SIMT kernels of bwd.cu state the same sums; G~, g~ come from the
// reverse state recurrence).  Every gradient is two GEMMs with 128 rows: an
// intra-chunk term (a gated 128 x 128 square times a token-major operand) and
// a state term (a token-major operand times a [d_qk, d_v] state), each in its
// own TMEM accumulator because the state term carries a per-row factor the
// intra term does not; the epilogue combines them.
//
// The reverse states G~_k = e^{g_k + m_k - m_{k+1}} G~_{k+1} + Q_k^T dUr_k
// (dUr: a bf16 copy of du~ whose rows carry e^{m_k - mu_t}) run in
// tc_bwd_rev_kernel: a CTA per 128 x 128 tile of the state walks the chunks
// from the last, the chunk updates computed ahead on the tensor cores and the
// running G~ in registers, writing every G~_k as the bf16 operand copy (and
// G~_0 in fp32: the gradient of the initial state); g~ follows from the
// per-chunk sums of e^{m_k - mu_t} da~_t q_t.
//
// Launches: one for both squares (dP and Sg, written as bf16 in the block
// layout of cb_block_row, so that the gradient kernels can read them as K- or
// MN-major operand tiles with single bulk copies), then one each for dq, dk
// and dv.  Token-major operands (Q, K, V, du~ in bf16) arrive by TMA in
// 64 x 64 boxes with the 128-byte swizzle; the states (the forward's bf16
// operand copy C_k and the reverse states G~ in the same block layout) and the
// squares by untiled bulk copies.
//
// Roles (192 threads): warp 0 producer (TMA and bulk copies through a
// 3-stage ring of 32 KB stages), warp 1 TMEM owner and MMA issuer, warps 2..5
// the epilogue (TMEM lane = chunk row), which stages its output tile in the
// ring's first stage (idle once every MMA has completed) for bulk / TMA
// stores.  About 100 KB of shared memory and 256 TMEM columns per CTA: two
// CTAs share an SM, so one's epilogue overlaps the other's loads.
#include <cuda.h>

#include "tc.h"
#include "tc_bwd.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kBT = 128;  // tokens per chunk = MMA rows
constexpr int kThreads = 192;
constexpr int kStages = 3;
constexpr uint32_t kTileBytes = 16384;               // 128 rows x 128 bytes
constexpr uint32_t kStageBytes = 2 * kTileBytes;      // A + B
constexpr uint32_t kOffBar = kStages * kStageBytes;   // full[3], empty[3], acc
constexpr uint32_t kOffSlot = kOffBar + 8 * 8;
constexpr uint32_t kOffVec = kOffSlot + 16;           // 128 floats
constexpr uint32_t kBytes = kOffVec + kBT * 4;
constexpr uint32_t kSmem = kBytes + 1024;             // + alignment slack
constexpr uint32_t kTmemCols = 256;                   // acc1 at 0, acc2 at 128

enum Job : int { kSquares = 0, kDQ = 1, kDK = 2, kDV = 3 };

struct TcBwdArgs {
  Problem p;                       // chunking of 128 tokens
  Gates g;
  const float* dA;                 // da~ [BH, T]
  const float* n_states;           // n_k [BH, NC, DK]
  const float* g_states;           // g~_k [BH, NC + 1, DK]
  const __nv_bfloat16* Cb;         // C_k, block layout, index bh NC + k
  const __nv_bfloat16* Gb;         // G~_k, block layout, index bh (NC + 1) + k
  __nv_bfloat16* sq;               // squares [BH NC][dP, Sg][2 s blocks][128 t][64]
  const __nv_bfloat16* X;          // dq: Q, dk: K (for q.dq and k.dk)
  __nv_bfloat16* out;              // dQ, dK or dV [BH, T, D]
  float* dot;                      // q.dq or k.dk [BH, T] (accumulated)
};

// Element offset of row r of s-block sb of square `which` of chunk bhk.
__device__ __forceinline__ size_t sq_row(long bhk, int which, int sb, int r) {
  return (((size_t)bhk * 2 + which) * 2 + sb) * (size_t)(kBT * 64) + (size_t)r * 64;
}

template <int kJob, int NT>
__global__ void __launch_bounds__(kThreads, 2)
tc_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_du,
              const __grid_constant__ CUtensorMap tm_out, const TcBwdArgs a) {
  static_assert(NT == 128, "output tiles of 128 columns (d_qk and d_v are multiples of 128)");
  const Problem& p = a.p;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + kOffBar, bar_empty = bar_full + 8 * kStages;
  const uint32_t bar_acc = bar_full + 16 * kStages;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffSlot);
  float* vec = reinterpret_cast<float*>(smem + kOffVec);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.y, bh = blockIdx.z;
  const int NC = p.NC, T = p.T, DK = p.DK, DV = p.DV;
  const int t0 = k * kBT;
  const int n0 = kJob == kSquares ? 0 : blockIdx.x * NT;
  const int which = kJob == kSquares ? blockIdx.x : 0;  // squares: 0 = dP, 1 = Sg
  const long bhk = (long)bh * NC + k;
  const long bhk1 = (long)bh * (NC + 1) + k + 1;  // G~_{k+1}
  const int n_vb = DV / 64;
  // slabs of 64 along the contraction: term 1, then term 2
  const int n1 = kJob == kSquares ? (which == 0 ? DV : DK) / 64 : 2;
  const int n2 = kJob == kDQ || kJob == kDK ? DV / 64 : (kJob == kDV ? DK / 64 : 0);
  const int nS = n1 + n2;
  constexpr int kN = kJob == kSquares ? kBT : NT;  // MMA N
  constexpr uint32_t kBBytes = kN * 128;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_acc, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_du);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nS && ok; ++i) {
        const int s = i % kStages, u = i / kStages;
        if (u > 0) ok = mbar_wait(bar_empty + 8 * s, (u - 1) & 1, p, 1);
        if (!ok) break;
        const uint32_t sa = sbase + (uint32_t)s * kStageBytes, sb = sa + kTileBytes;
        const uint32_t fb = bar_full + 8 * s;
        mbar_expect_tx(fb, kTileBytes + kBBytes);
        // token-major K-major tile: 128 rows of the chunk, contraction columns x0..x0+63
        auto tok_rows = [&](const CUtensorMap* m, uint32_t dst, int x0) {
          tma_load_3d(dst, m, x0, t0, bh, fb);
          tma_load_3d(dst + 8192, m, x0, t0 + 64, bh, fb);
        };
        // token-major MN-major tile: columns n0.., contraction tokens t0 + 64 i..
        auto tok_cols = [&](const CUtensorMap* m, uint32_t dst, int i1) {
#pragma unroll
          for (int b = 0; b < NT / 64; ++b)
            tma_load_3d(dst + b * 8192, m, n0 + b * 64, t0 + i1 * 64, bh, fb);
        };
        // square as an MN-major A: rows s (two 64-blocks), contraction tokens 64 i..
        auto sq_cols = [&](int w, uint32_t dst, int i1) {
          bulk_load(dst, a.sq + sq_row(bhk, w, 0, i1 * 64), 8192, fb);
          bulk_load(dst + 8192, a.sq + sq_row(bhk, w, 1, i1 * 64), 8192, fb);
        };
        if constexpr (kJob == kSquares) {
          const CUtensorMap* ma = which == 0 ? &tm_du : &tm_q;
          const CUtensorMap* mb = which == 0 ? &tm_v : &tm_k;
          tok_rows(ma, sa, i * 64);
          tok_rows(mb, sb, i * 64);
        } else if constexpr (kJob == kDQ) {
          if (i < n1) {
            bulk_load(sa, a.sq + sq_row(bhk, 0, i, 0), kTileBytes, fb);  // dP, K-major
            tok_cols(&tm_k, sb, i);
          } else {
            const int j = i - n1;
            tok_rows(&tm_du, sa, j * 64);
            bulk_load(sb, a.Cb + cb_block_row(bhk, j, n0, DK, n_vb), kBBytes, fb);
          }
        } else if constexpr (kJob == kDK) {
          if (i < n1) {
            sq_cols(0, sa, i);  // dP^T
            tok_cols(&tm_q, sb, i);
          } else {
            const int j = i - n1;
            tok_rows(&tm_v, sa, j * 64);
            bulk_load(sb, a.Gb + cb_block_row(bhk1, j, n0, DK, n_vb), kBBytes, fb);
          }
        } else {
          if (i < n1) {
            sq_cols(1, sa, i);  // Sg^T
            tok_cols(&tm_du, sb, i);
          } else {
            const int j = i - n1;
            tok_rows(&tm_k, sa, j * 64);
#pragma unroll
            for (int b = 0; b < NT / 64; ++b)
              bulk_load(sb + b * 8192, a.Gb + cb_block_row(bhk1, n0 / 64 + b, j * 64, DK, n_vb),
                        8192, fb);
          }
        }
        issued = i + 1;
      }
      // every copy issued has landed before the CTA may exit
      for (int q = (issued > kStages ? issued - kStages : 0); q < issued; ++q)
        mbar_wait(bar_full + 8 * (q % kStages), (q / kStages) & 1, p, 2);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      // operand majors per term: 1 = MN-major
      constexpr int a1 = (kJob == kDK || kJob == kDV) ? 1 : 0;
      constexpr int b1 = kJob == kSquares ? 0 : 1;
      constexpr int b2 = kJob == kDV ? 1 : 0;
      constexpr uint32_t id1 = idesc_bf16(128, kN, a1, b1);
      constexpr uint32_t id2 = idesc_bf16(128, kN, 0, b2);
      bool ok = true;
      for (int i = 0; i < nS && ok; ++i) {
        const int s = i % kStages;
        ok = mbar_wait(bar_full + 8 * s, (i / kStages) & 1, p, 3);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = sbase + (uint32_t)s * kStageBytes, sb = sa + kTileBytes;
        const bool t2 = i >= n1;
        const bool first = i == 0 || i == n1;
        const uint32_t d = tmem + (t2 ? 128u : 0u);
        const int am = t2 ? 0 : a1, bm = t2 ? b2 : b1;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = am ? sdesc_sw128(sa + kk * 2048, 8192, 1024)
                                 : sdesc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = bm ? sdesc_sw128(sb + kk * 2048, 8192, 1024)
                                 : sdesc_sw128(sb + kk * 32, 16, 1024);
          mma_bf16_ss(d, ad, bd, t2 ? id2 : id1, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(bar_empty + 8 * s);
      }
      mma_commit(bar_acc);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // chunk row = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
    const long tpad = (long)NC * kBT;
    const int t = t0 + r;
    const bool valid = t < T;
    const float m_in = a.g.mchk[(long)bh * (NC + 1) + k];
    const float m_out = a.g.mchk[(long)bh * (NC + 1) + k + 1];
    const float acol_r = a.g.acol[(long)bh * tpad + t];  // -inf on padding
    const float mu = fmaxf(m_in, a.g.amax[(long)bh * tpad + t]);
    // Output staging: the ring's first stage (32 KB), free once every MMA has
    // completed; the rows of a thread go out with bulk or TMA stores (a store
    // per thread and row would half-fill a 32-byte sector per 16 bytes).
    uint8_t* stg = smem;
    const bool issuer = warp == 2 && lane == 0;
    // per-column vector of the chunk in shared memory: the squares' column
    // weights acol_s; dq's n_k, dk's g~_{k+1} over this CTA's NT columns
    if constexpr (kJob == kSquares) {
      vec[r] = acol_r;
      named_bar_sync(1, 128);
    } else if constexpr (kJob == kDQ || kJob == kDK) {
      if (r < NT)
        vec[r] = kJob == kDQ ? a.n_states[bhk * DK + n0 + r] : a.g_states[bhk1 * DK + n0 + r];
      named_bar_sync(1, 128);
    }
    const bool ok = mbar_wait(bar_acc, 0, p, 4);
    tc_fence_after();
    if (ok) {
      if constexpr (kJob == kSquares) {
        const float da = (which == 0 && valid) ? a.dA[(long)bh * T + t] : 0.f;
#pragma unroll 1
        for (int c = 0; c < kBT / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(trow + c * 32, v);
          tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float f[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int s = c * 32 + j + e;
              const float x = __uint_as_float(v[j + e]);
              const float val = which == 0 ? x + da : p.key_scale * x;
              f[e] = (valid && s <= r) ? val * expf(vec[s] - mu) : 0.f;
            }
            w[j / 2] = pack_bf16x2(f[0], f[1]);
          }
          // into the staging copy of s-block c / 2 (the block layout of sq)
          uint8_t* blk = stg + (c >> 1) * 16384;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(blk + sw128_offset((uint32_t)r, (uint32_t)((c & 1) * 4 + u))) =
                make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      } else {
        const int D = kJob == kDV ? DV : DK;
        float rs, alpha = 0.f, s1, s2;
        if constexpr (kJob == kDQ) {
          rs = expf(m_in - mu);
          alpha = valid ? a.dA[(long)bh * T + t] : 0.f;
          s1 = p.key_scale;
          s2 = 1.f;
        } else {
          const float gk = a.g.gtot[(long)bh * NC + k];
          rs = expf(gk + acol_r - m_out);  // w_s, 0 on padding
          if constexpr (kJob == kDK) {
            alpha = 1.f;
            s1 = p.key_scale;
            s2 = p.key_scale;
          } else {
            s1 = 1.f;
            s2 = p.key_scale;
          }
        }
        float dot = 0.f;
        const long orow = ((long)bh * T + t) * D + n0;
#pragma unroll 1
        for (int c = 0; c < NT / 32; ++c) {
          // this row's q or k for the dot product, loaded ahead of the TMEM reads
          uint4 xv[4];
          if (kJob != kDV && valid) {
            const uint4* xs = reinterpret_cast<const uint4*>(a.X + orow + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) xv[u] = xs[u];
          }
          uint32_t v1[32], v2[32];
          tmem_ld32(trow + c * 32, v1);
          tmem_ld32(trow + 128 + c * 32, v2);
          tmem_wait_ld();
          float o[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float x2 = __uint_as_float(v2[j]);
            if (kJob != kDV) x2 = fmaf(alpha, vec[c * 32 + j], x2);
            // dq: s acc1 + rs (acc2 + da n);  dk: s (acc1 + w (acc2 + g~));  dv: acc1 + s w acc2
            o[j] = kJob == kDK ? s1 * fmaf(rs, x2, __uint_as_float(v1[j]))
                               : fmaf(s1, __uint_as_float(v1[j]), s2 * rs * x2);
          }
          // into the staging box of columns (c / 2) * 64.. (the TMA store's layout)
          uint8_t* box = stg + (c >> 1) * 16384;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(box + sw128_offset((uint32_t)r, (uint32_t)((c & 1) * 4 + u))) =
                make_uint4(pack_bf16x2(o[8 * u], o[8 * u + 1]),
                           pack_bf16x2(o[8 * u + 2], o[8 * u + 3]),
                           pack_bf16x2(o[8 * u + 4], o[8 * u + 5]),
                           pack_bf16x2(o[8 * u + 6], o[8 * u + 7]));
          if (valid) {
            if constexpr (kJob != kDV) {
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint32_t xw[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 f = __bfloat1622float2(
                      *reinterpret_cast<const __nv_bfloat162*>(&xw[e]));
                  dot = fmaf(f.x, o[8 * u + 2 * e], dot);
                  dot = fmaf(f.y, o[8 * u + 2 * e + 1], dot);
                }
              }
            }
          }
        }
        if (kJob != kDV && valid) atomicAdd(&a.dot[(long)bh * T + t], dot);
      }
    }
    // Every epilogue thread reaches this barrier whatever its wait returned;
    // the staged tile goes out only when the issuer's wait succeeded.
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (issuer && ok) {
      if constexpr (kJob == kSquares) {
        for (int b = 0; b < 2; ++b)
          bulk_store(a.sq + sq_row(bhk, which, b, 0), sbase + (uint32_t)b * 16384u, 16384u);
      } else {
        // the tile's rows past T are clipped by the tensor map
        for (int b = 0; b < NT / 64; ++b)
          tma_store_3d(&tm_out, sbase + (uint32_t)b * 16384u, n0 + b * 64, t0, bh);
      }
      tma_store_commit();
      tma_store_wait_all();  // the staged tile has landed
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(bar_acc, 0, p, 5);  // every MMA has completed
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Per-chunk increments of g~: u_k[d] = sum_{t in k, t < T} e^{m_k - mu_t} da~_t q_t[d].
// One block of 256 threads per (chunk, b h): a thread sums 8 consecutive d
// (16-byte loads of q) over every (256 / (DK / 8))-th token of the chunk, and
// the token groups are added up in shared memory.
__global__ void __launch_bounds__(256)
tc_bwd_gvec_kernel(Problem p, Gates g, const __nv_bfloat16* __restrict__ Q,
                   const float* __restrict__ dA, float* __restrict__ u) {
  __shared__ float red[256 * 8];
  const int k = blockIdx.x, bh = blockIdx.y, NC = p.NC, T = p.T, DK = p.DK;
  const int n_dg = DK / 8, n_tg = 256 / n_dg;
  const int dg = threadIdx.x % n_dg, tg = threadIdx.x / n_dg;
  const long tpad = (long)NC * kBT;
  const float m_in = g.mchk[(long)bh * (NC + 1) + k];
  const int t1 = min(T, (k + 1) * kBT);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int t = k * kBT + tg; t < t1; t += n_tg) {
    const float w = expf(m_in - fmaxf(m_in, g.amax[(long)bh * tpad + t])) * dA[(long)bh * T + t];
    const uint4 qv = *reinterpret_cast<const uint4*>(Q + ((long)bh * T + t) * DK + dg * 8);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw[e]));
      acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < DK; d += blockDim.x) {
    float sum = 0.f;
    for (int q = 0; q < n_tg; ++q) sum += red[(q * n_dg + d / 8) * 8 + d % 8];
    u[((long)bh * NC + k) * DK + d] = sum;
  }
}

// Reverse recurrence on tcgen05: one CTA per (b, h) and 128 x NT tile of
// the [d_qk, d_v] gradient state, walking the chunks from the last,
//
//   G~_k = e^{g_k + m_k - m_{k+1}} G~_{k+1} + U_k,   U_k = Q_k^T dUr_k,   G~_NC = 0
//
// (dUr: du~ with rows scaled by e^{m_k - mu_t}).  The chunk updates U_k do not
// depend on the recurrence, so the MMA warp computes them ahead into two
// alternating TMEM accumulators; the running G~ lives in the registers of the
// epilogue threads (eight warps, two per TMEM lane quadrant, each thread one
// state row and half of the tile's columns).  Per chunk an epilogue thread
// stores G~_{k+1} as the bf16 operand copy Gb (block layout of cb_block_row,
// index bh (NC + 1) + k + 1), then waits for U_k, folds it in and releases the
// accumulator; the MMAs of the next chunks run meanwhile.  G~_0 also goes to
// dC0 in fp32.  The CTAs of the first column tile carry g~ along (one row per
// thread of the first column half) from the increments u.
// The bf16 copy of a step goes out through shared memory: in the block
// layout the tile's rows of one 64-column block are 16 KB in a row of the
// global array, so the epilogue threads write their rows into a staging copy
// of the two blocks and one thread issues two bulk stores (stores from each
// thread straight to its own row would half-fill a 32-byte sector per 16-byte
// store, twice the bytes on the way to L2).  Two staging buffers alternate.
// Roles (320 threads): warp 0 producer, warp 1 TMEM owner and MMA issuer,
// warps 2..9 epilogue; ring of four 64-token stages (A = Q^T 16 KB, B = dUr
// 16 KB), one CTA per SM.
constexpr int kRevThreads = 320;
template <int NT>
struct RevCfg {
  static_assert(NT == 128, "one 64-column block per epilogue column half");
  static constexpr uint32_t kBBytes = NT * 128;
  static constexpr uint32_t kStageBytes = kTileBytes + kBBytes;
  static constexpr int kStages = 4;
  static constexpr uint32_t kStgBytes = 128 * NT * 2;  // bf16 tile, two 16 KB blocks
  static constexpr uint32_t kOffStg = kStages * kStageBytes;  // two staging buffers
  static constexpr uint32_t kOffBar = kOffStg + 2 * kStgBytes;  // full, empty, u_full[2], u_empty[2]
  static constexpr uint32_t kOffSlot = kOffBar + 8 * (2 * kStages + 4);
  static constexpr uint32_t kSmem = kOffSlot + 16 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static constexpr int kCols = NT / 2;   // columns per epilogue thread
  static constexpr uint32_t kTmemCols = 2 * NT;
};

template <int NT>
__global__ void __launch_bounds__(kRevThreads, 1)
tc_bwd_rev_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_dur,
                  Problem p, Gates g, const float* __restrict__ u, __nv_bfloat16* __restrict__ Gb,
                  float* __restrict__ g_states, float* __restrict__ dC0) {
  using R = RevCfg<NT>;
  constexpr int kSt = R::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + R::kOffBar, bar_empty = bar_full + 8 * kSt;
  const uint32_t bar_ufull = bar_full + 16 * kSt, bar_uempty = bar_ufull + 16;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + R::kOffSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NC = p.NC, DK = p.DK, DV = p.DV, bh = blockIdx.y;
  const int n_ct = DV / NT;
  const int m0 = (blockIdx.x / n_ct) * 128, n0 = (blockIdx.x % n_ct) * NT;
  const int nS = 2 * NC;  // two 64-token slabs per chunk, chunks from the last

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSt; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_ufull + 8 * b, 1);
      mbar_init(bar_uempty + 8 * b, kRevThreads - 64);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), R::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_dur);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nS && ok; ++i) {
        const int s = i % kSt, uu = i / kSt;
        if (uu > 0) ok = mbar_wait(bar_empty + 8 * s, (uu - 1) & 1, p, 6);
        if (!ok) break;
        const int t = (NC - 1 - i / 2) * kBT + (i & 1) * 64;
        const uint32_t sa = sbase + (uint32_t)s * R::kStageBytes, sb = sa + kTileBytes;
        const uint32_t fb = bar_full + 8 * s;
        mbar_expect_tx(fb, R::kStageBytes);
        // A = Q^T (rows d, MN-major), B = dUr (columns c, MN-major); K = tokens
        tma_load_3d(sa, &tm_q, m0, t, bh, fb);
        tma_load_3d(sa + 8192, &tm_q, m0 + 64, t, bh, fb);
#pragma unroll
        for (int b = 0; b < NT / 64; ++b) tma_load_3d(sb + b * 8192, &tm_dur, n0 + b * 64, t, bh, fb);
        issued = i + 1;
      }
      for (int q = (issued > kSt ? issued - kSt : 0); q < issued; ++q)
        mbar_wait(bar_full + 8 * (q % kSt), (q / kSt) & 1, p, 7);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, NT, 1, 1);
      bool ok = true;
      for (int kk = 0; kk < NC && ok; ++kk) {
        const int buf = kk & 1;
        // the epilogue has folded in the update that last used this accumulator
        if (kk >= 2) ok = mbar_wait(bar_uempty + 8 * buf, ((kk - 2) >> 1) & 1, p, 8);
        if (!ok) break;
        tc_fence_after();
        for (int h = 0; h < 2 && ok; ++h) {
          const int i = 2 * kk + h, s = i % kSt;
          ok = mbar_wait(bar_full + 8 * s, (i / kSt) & 1, p, 9);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = sbase + (uint32_t)s * R::kStageBytes, sb = sa + kTileBytes;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mma_bf16_ss(tmem + (uint32_t)(buf * NT), sdesc_sw128(sa + q * 2048, 8192, 1024),
                        sdesc_sw128(sb + q * 2048, 8192, 1024), idesc, (h | q) ? 1u : 0u);
          mma_commit(bar_empty + 8 * s);
        }
        mma_commit(bar_ufull + 8 * buf);
      }
    }
  } else {
    constexpr int kG = R::kCols / 32;  // 32-column groups per thread
    const int q4 = warp & 3, r = q4 * 32 + lane, d = m0 + r;
    const int ch = (warp - 2) >> 2;  // column half
    const int c0 = ch * R::kCols;    // first column of this thread within the tile
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)c0;
    const float* gt = g.gtot + (long)bh * NC;
    const float* mc = g.mchk + (long)bh * (NC + 1);
    const int n_vb = DV / 64;
    const bool g_owner = n0 == 0 && ch == 0;
    float gv = 0.f;
    float G[R::kCols];
#pragma unroll
    for (int j = 0; j < R::kCols; ++j) G[j] = 0.f;
    const bool issuer = warp == 2 && lane == 0;
    int n_st = 0;  // staged copies so far (selects the buffer)
    // The running state as bf16 at index kidx: this thread's row of its
    // column half's block into the staging buffer, then two bulk stores.
    auto store_b16 = [&](long kidx) {
      const uint32_t buf = (uint32_t)(n_st & 1) * R::kStgBytes;
      if (issuer) tma_store_wait_read_1();  // the copy from this buffer two steps ago is read
      named_bar_sync(1, kRevThreads - 64);
      uint8_t* blk = smem + R::kOffStg + buf + (uint32_t)ch * 16384u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float* x = G + 8 * j;
        *reinterpret_cast<uint4*>(blk + sw128_offset((uint32_t)r, (uint32_t)j)) =
            make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                       pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
      }
      fence_proxy_async_smem();
      named_bar_sync(1, kRevThreads - 64);
      if (issuer) {
        for (int b = 0; b < 2; ++b)
          bulk_store(Gb + cb_block_row((long)bh * (NC + 1) + kidx, n0 / 64 + b, m0, DK, n_vb),
                     sbase + R::kOffStg + buf + (uint32_t)b * 16384u, 16384u);
        tma_store_commit();
      }
      ++n_st;
    };
    bool ok = true;
    for (int kk = 0; kk < NC; ++kk) {
      const int k = NC - 1 - kk, buf = kk & 1;
      const float decay = expf(gt[k] + mc[k] - mc[k + 1]);
      const float uk = g_owner ? u[((long)bh * NC + k) * DK + d] : 0.f;
      store_b16(k + 1);  // G~_{k+1}
      if (g_owner) {
        g_states[((long)bh * (NC + 1) + k + 1) * DK + d] = gv;
        gv = fmaf(decay, gv, uk);
      }
      ok = ok && mbar_wait(bar_ufull + 8 * buf, (kk >> 1) & 1, p, 10);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kG; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + (uint32_t)(buf * NT) + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) G[c * 32 + j] = fmaf(decay, G[c * 32 + j], __uint_as_float(v[j]));
      }
      tc_fence_before();
      mbar_arrive(bar_uempty + 8 * buf);
    }
    // G~_0
    store_b16(0);
    if (g_owner) g_states[(long)bh * (NC + 1) * DK + d] = gv;
    float4* dst = reinterpret_cast<float4*>(dC0 + ((long)bh * DK + d) * DV + n0 + c0);
#pragma unroll
    for (int q = 0; q < R::kCols / 4; ++q)
      dst[q] = make_float4(G[4 * q], G[4 * q + 1], G[4 * q + 2], G[4 * q + 3]);
    if (issuer) tma_store_wait_all();  // the staged copies have landed
    (void)ok;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA has completed: the last commit of each accumulator
    if (lane == 0) {
      const int last = NC - 1;
      mbar_wait(bar_ufull + 8 * (last & 1), (last >> 1) & 1, p, 12);
      if (NC >= 2) mbar_wait(bar_ufull + 8 * ((last - 1) & 1), ((last - 1) >> 1) & 1, p, 12);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, R::kTmemCols);
  }
}

template <int NT>
cudaError_t launch_rev(const CUtensorMap& mq, const CUtensorMap& mu, const Problem& pb, Gates g,
                       const float* u, __nv_bfloat16* Gb, float* g_states, float* dC0,
                       cudaStream_t st) {
  using R = RevCfg<NT>;
  cudaError_t e = cudaFuncSetAttribute(tc_bwd_rev_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, R::kSmem);
  if (e != cudaSuccess) return e;
  tc_bwd_rev_kernel<NT><<<dim3((pb.DK / 128) * (pb.DV / NT), pb.BH), kRevThreads, R::kSmem, st>>>(
      mq, mu, pb, g, u, Gb, g_states, dC0);
  return cudaGetLastError();
}

template <int kJob, int NT>
cudaError_t launch_job(const CUtensorMap* m, const CUtensorMap& out, const TcBwdArgs& a, dim3 grid,
                       cudaStream_t st) {
  auto kern = tc_bwd_kernel<kJob, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmem, st>>>(m[0], m[1], m[2], m[3], out, a);
  return cudaGetLastError();
}

}  // namespace

bool tc_bwd_supported(const Problem& pb) {
  return pb.L == kBT && (pb.DK == 128 || pb.DK == 256) && pb.DV % 128 == 0 && pb.DV <= 1024 &&
         pb.T > 0 && tc_unfused_supported(pb);
}

size_t tc_bwd_square_elems(const Problem& pb) { return (size_t)pb.BH * pb.NC * 2 * kBT * kBT; }

cudaError_t launch_tc_bwd_states(const Problem& pb, const void* Q, const __nv_bfloat16* dUr16,
                                 Gates g, const float* dA, float* u, __nv_bfloat16* Gb,
                                 float* g_states, float* dC0, cudaStream_t st) {
  if (!tc_bwd_supported(pb)) return cudaErrorNotSupported;
  CUtensorMap mq, mu;
  if (!encode_tmap_3d(&mq, Q, 2, pb.DK, pb.T, pb.BH, 64, 64, 128) ||
      !encode_tmap_3d(&mu, dUr16, 2, pb.DV, pb.T, pb.BH, 64, 64, 128))
    return cudaErrorInvalidValue;
  tc_bwd_gvec_kernel<<<dim3(pb.NC, pb.BH), 256, 0, st>>>(pb, g, static_cast<const __nv_bfloat16*>(Q),
                                                         dA, u);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_rev<128>(mq, mu, pb, g, u, Gb, g_states, dC0, st);
}

cudaError_t launch_tc_bwd(const Problem& pb, const void* Q, const void* K, const void* V,
                          const __nv_bfloat16* dU16, Gates g, const float* dA,
                          const float* n_states, const float* g_states, const __nv_bfloat16* Cb,
                          const __nv_bfloat16* Gb, __nv_bfloat16* sq, void* dQ, void* dK,
                          void* dV, float* qdq, float* kdk, cudaStream_t st) {
  if (!tc_bwd_supported(pb)) return cudaErrorNotSupported;
  CUtensorMap m[4];
  if (!encode_tmap_3d(&m[0], Q, 2, pb.DK, pb.T, pb.BH, 64, 64, 128) ||
      !encode_tmap_3d(&m[1], K, 2, pb.DK, pb.T, pb.BH, 64, 64, 128) ||
      !encode_tmap_3d(&m[2], V, 2, pb.DV, pb.T, pb.BH, 64, 64, 128) ||
      !encode_tmap_3d(&m[3], dU16, 2, pb.DV, pb.T, pb.BH, 64, 64, 128))
    return cudaErrorInvalidValue;
  TcBwdArgs a = {};
  a.p = pb;
  a.g = g;
  a.dA = dA;
  a.n_states = n_states;
  a.g_states = g_states;
  a.Cb = Cb;
  a.Gb = Gb;
  a.sq = sq;
  // output maps: 64-column boxes of 128 rows (rows past T are not written)
  CUtensorMap oq, ok_, ov;
  if (!encode_tmap_3d(&oq, dQ, 2, pb.DK, pb.T, pb.BH, 64, 128, 128) ||
      !encode_tmap_3d(&ok_, dK, 2, pb.DK, pb.T, pb.BH, 64, 128, 128) ||
      !encode_tmap_3d(&ov, dV, 2, pb.DV, pb.T, pb.BH, 64, 128, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_job<kSquares, 128>(m, m[0], a, dim3(2, pb.NC, pb.BH), st);
  if (e != cudaSuccess) return e;
  // 128 output columns per CTA (DK and DV are multiples of 128)
  a.X = static_cast<const __nv_bfloat16*>(Q);
  a.out = static_cast<__nv_bfloat16*>(dQ);
  a.dot = qdq;
  e = launch_job<kDQ, 128>(m, oq, a, dim3(pb.DK / 128, pb.NC, pb.BH), st);
  if (e != cudaSuccess) return e;
  a.X = static_cast<const __nv_bfloat16*>(K);
  a.out = static_cast<__nv_bfloat16*>(dK);
  a.dot = kdk;
  e = launch_job<kDK, 128>(m, ok_, a, dim3(pb.DK / 128, pb.NC, pb.BH), st);
  if (e != cudaSuccess) return e;
  a.X = nullptr;
  a.out = static_cast<__nv_bfloat16*>(dV);
  a.dot = nullptr;
  return launch_job<kDV, 128>(m, ov, a, dim3(pb.DV / 128, pb.NC, pb.BH), st);
}

}  // namespace mlstm
