// G3 for chunks of at most 256 tokens: one work item per (b, h) and 128-row
// query tile, covering every value column of the head.
//
// Same per-row mathematics as tc_parallel.cu ("Tiled Flash Linear Attention:
// More Efficient Linear RNN and xLSTM Kernels", abstract: the intra-chunk part
// tiled over query and key/value blocks):
//
//   O_r   = e^{m_k - mu_r} C_k^T q_r  +  sum_{s<=r} P_rs v_s
//   P_rs  = (s q_r.k_s) e^{acol_s - mu_r}                (0 above the diagonal)
//   den_r = e^{m_k - mu_r} n_k.q_r    +  sum_{s<=r} P_rs
//   h_r   = O_r / max(|den_r|, e^{-(bcum_r + mu_r)})
//
// What differs is the work decomposition.  With at most two 128-token
// key/value tiles per query tile, the gated P tiles of an item stay on chip,
// so an item computes S and P once and then sweeps the value columns in
// 128-wide tiles d: O_d = sum_i P_i V_i[:, d] + Q~ C_k[:, d], where Q~ is the
// query tile with row r scaled by e^{m_k - mu_r} (in place, once the S MMAs
// have read Q).  The Q tile is loaded once per item, S is never recomputed per
// value tile, and the MMAs of consecutive value tiles need no hand-off from
// the row threads.  The two TMEM output accumulators alternate between value
// tiles; the epilogue of tile d (bf16 rows into a swizzled staging tile, then
// a TMA store) overlaps the MMAs of tile d + 1.
//
// P never touches shared memory: the row threads write it back as packed bf16
// over the TMEM columns of the S tile it came from, and the P.V MMAs take
// their A operand from TMEM.  The shared memory this saves deepens the TMA
// ring, which is what bounds this kernel (each item streams C_k and V through
// the ring once per value tile).
//
// Roles (320 threads): warp 0 TMA producer; warp 1 TMEM owner and MMA issuer;
// warps 2..9 two threads per query row (each owning half of the columns):
// gating of S into P, the in-place scaling of Q, row sums, epilogue.
// TMEM (512 columns): O at 0 and 128, S_0 / P_0 at 256, S_1 / P_1 at 384.
// The half of the row threads that owns S columns [64h, 64h + 64) writes its
// 64 bf16 P values (32 packed columns) to columns [64h, 64h + 32), which only
// it has read, so the halves never race.
// Chunks of 64 tokens (kPair): a 128-row query tile holds two chunks, 2j and
// 2j + 1.  S covers both, and P is masked to the causal pairs within each chunk
// (block diagonal).  The two halves of the tile need different chunk states,
// so the inter-chunk product runs over a K-stacked operand,
//   [Q~ masked to chunk 2j | Q~ masked to chunk 2j + 1] . [C_2j ; C_2j+1],
// which is one accumulation into the same O: the row threads write their
// scaled Q row into its chunk's half of a double-width Q buffer and zeros into
// the other half.
//
// MMA order per item: S_0 [, S_1], then for every value tile d:
// P_0.V_0[:, d] [, P_1.V_1[:, d]], (first tile: wait for the scaled Q),
// Q~.C_k[:, d].  S_i of the next item waits until the last P_i.V_i MMA of
// this one has completed; the Q~.C_k MMAs issued after it hide that wait.
// When the exponents of a tile allow one frame for all its rows (tile_frame:
// the entering state's m_k, as in the long-chunk kernel) Q needs no scaling,
// and each value tile issues Q.C_k[:, d] first: the inter-chunk MMAs of the
// first value tile run while the row threads still gate S.
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kQT = 128;
constexpr int kKT = 128;
constexpr int kPSlots = 2;  // key/value tiles per item (chunks of at most 256)
constexpr uint32_t kColPHalf = 64;  // P columns of the upper half within an S tile
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 256, kColS1 = 384;

template <int DK, int DVT, bool kPair>
struct WCfg {
  static_assert(DVT == 64 || DVT == 128, "value tile of 64 or 128 columns");
  static_assert(!kPair || DK <= 128, "pairs of 64-token chunks: d_qk up to 128");
  static constexpr int kChunks = kPair ? 2 : 1;  // chunks per query tile
  static constexpr int kSlabsK = DK / 64;
  static constexpr uint32_t kQLoadBytes = kQT * DK * 2;
  static constexpr uint32_t kQBytes = kChunks * kQLoadBytes;  // kPair: the stacked Q~ operand
  static constexpr uint32_t kKSlabBytes = kKT * 128;
  static constexpr uint32_t kMNSlabBytes = (DVT / 64) * 8192;
  static constexpr uint32_t kStageBytes = 16384;
  static_assert(kKSlabBytes <= kStageBytes && kMNSlabBytes <= kStageBytes, "stage size");
  static constexpr uint32_t kOutBytes = kQT * DVT * 2;  // output staging tile
  static constexpr uint32_t kMiscBytes =
      2 * kPSlots * kKT * 4 + 2 * kChunks * DK * 4 + 256 * 8 + 512;
  static constexpr uint32_t kBudget = 227 * 1024 - 1024;
  static constexpr int kStagesFit =
      (int)((kBudget - kQBytes - kOutBytes - kMiscBytes) / kStageBytes);
  static constexpr int kStages = kStagesFit > 12 ? 12 : kStagesFit;
  static_assert(kStages >= 3, "ring too shallow");
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffOut = kOffQ + kQBytes;
  static constexpr uint32_t kOffStage = kOffOut + kOutBytes;
  static constexpr uint32_t kOffAcol = kOffStage + kStages * kStageBytes;  // float[2][256]
  static constexpr uint32_t kOffN = kOffAcol + 2 * kPSlots * kKT * 4;  // float[2][kChunks][DK]
  static constexpr uint32_t kOffRed = kOffN + 2 * kChunks * DK * 4;    // float2[256]
  static constexpr uint32_t kOffBar = kOffRed + 256 * 8;
  static constexpr uint32_t kOffTmemSlot = kOffBar + 384;
  static constexpr uint32_t kBytes = kOffTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct WBars {
  uint32_t a;
  __device__ __forceinline__ uint32_t full(int i) const { return a + 8 * i; }
  __device__ __forceinline__ uint32_t empty(int i) const { return a + 128 + 8 * i; }
  __device__ __forceinline__ uint32_t q_full() const { return a + 256; }
  __device__ __forceinline__ uint32_t q_empty() const { return a + 264; }
  __device__ __forceinline__ uint32_t s_full(int i) const { return a + 272 + 8 * i; }
  // One "accumulator ready" barrier per O buffer: consecutive value tiles need
  // no hand-off from the row threads, so a single barrier could complete twice
  // before they wait on it and its parity would no longer tell the tiles apart.
  __device__ __forceinline__ uint32_t o_full(int b) const { return a + 288 + 8 * b; }
  __device__ __forceinline__ uint32_t p_full(int i) const { return a + 304 + 8 * i; }
  __device__ __forceinline__ uint32_t pv_done(int i) const { return a + 320 + 8 * i; }
  __device__ __forceinline__ uint32_t q_scaled() const { return a + 336; }
  __device__ __forceinline__ uint32_t o_empty(int b) const { return a + 360 + 8 * b; }
  __device__ __forceinline__ uint32_t mma_idle() const { return a + 376; }
};

struct WItem {
  int bh, t0, k, c0, n_kv;
};

__device__ __forceinline__ WItem decode_witem(int it, const Problem& p, int n_q) {
  WItem x;
  x.bh = it / n_q;
  x.t0 = (it % n_q) * kQT;
  x.k = x.t0 / p.L;
  x.c0 = x.k * p.L;
  x.n_kv = (x.t0 - x.c0) / kKT + 1;
  return x;
}

// Whether the item's tile works in the frame F = m_k (see the row threads),
// from the same loads and arithmetic in the MMA issuer and the row threads.
// Never with two chunks per tile (kPair) or without an entering state.
template <bool kPair>
__device__ __forceinline__ bool tile_frame(const Gates& g, const Problem& p, const WItem& x,
                                           long tpad) {
  if (kPair) return false;
  const long base = (long)x.bh * tpad;
  const float m_in = g.mchk[(long)x.bh * (p.NC + 1) + x.k];
  const float c = g.amax[base + x.t0 + kQT - 1];  // amax is a running maximum
  const float hi = -g.bcum[base + x.t0 + kQT - 1] - m_in;  // bcum falls along the chunk
  const float lo = -g.bcum[base + x.t0] - m_in;
  return m_in != -INFINITY && c - m_in <= 60.f && hi <= 80.f && lo >= -80.f;
}

// The k-th item of this CTA.  Items alternate between the first and the
// second query tile of a chunk, and the second has twice the intra-chunk work;
// a plain stride of an even grid would give each CTA only one kind (and the
// kernel the time of the slower half).  With an even grid the lowest index bit
// is therefore flipped on odd rounds: every CTA takes both kinds, and the two
// tiles of a chunk still run side by side in neighbouring CTAs (their C_k and
// V tiles are shared through L2).
__device__ __forceinline__ int item_at(int k) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return k * G + ((G & 1) ? c : (c ^ (k & 1)));
}

template <int DK, int DVT, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
tc_parallel_wide_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __nv_bfloat16* __restrict__ Cb,
                        const __grid_constant__ CUtensorMap tm_h, Problem p, Gates g,
                        const float* __restrict__ n_states,
                        float* __restrict__ n_out, float* __restrict__ m_out, int n_items,
                        const __nv_bfloat16* __restrict__ Vraw) {
  using C = WCfg<DK, DVT, kPair>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const WBars bar{sbase + C::kOffBar};
  float* acol_s = reinterpret_cast<float*>(smem + C::kOffAcol);
  float* n_s = reinterpret_cast<float*>(smem + C::kOffN);
  float2* red_s = reinterpret_cast<float2*>(smem + C::kOffRed);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_dv = p.DV / DVT;
  const int n_q = (p.T + kQT - 1) / kQT;
  const long tpad = (long)p.NC * p.L;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar.full(i), 1);
      mbar_init(bar.empty(i), 1);
    }
    mbar_init(bar.q_full(), 1);
    mbar_init(bar.q_empty(), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar.s_full(i), 1);
      mbar_init(bar.p_full(i), 256);
      mbar_init(bar.pv_done(i), 1);
      mbar_init(bar.o_full(i), 1);
      mbar_init(bar.o_empty(i), 256);
    }
    mbar_init(bar.q_scaled(), 256);
    mbar_init(bar.mma_idle(), 1);
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
    // ---------------------------- TMA producer ----------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int slab = 0;
      bool ok = true;
      auto next_stage = [&](uint32_t bytes) -> uint32_t {
        const int s = slab % C::kStages, u = slab / C::kStages;
        if (u > 0) ok = ok && mbar_wait(bar.empty(s), (u - 1) & 1, p, 1);
        mbar_expect_tx(bar.full(s), bytes);
        ++slab;
        return sbase + C::kOffStage + (uint32_t)s * C::kStageBytes;
      };
      int n = 0;
      for (int it = item_at(0); it < n_items && ok; it = item_at(n + 1), ++n) {
        const WItem x = decode_witem(it, p, n_q);
        if (n > 0) ok = mbar_wait(bar.q_empty(), (n - 1) & 1, p, 2);
        if (!ok) break;
        mbar_expect_tx(bar.q_full(), C::kQLoadBytes);
        for (int c = 0; c < C::kSlabsK; ++c)
          tma_load_3d(sbase + C::kOffQ + c * 16384, &tm_q, c * 64, x.t0, x.bh, bar.q_full());
        for (int i = 0; i < x.n_kv && ok; ++i)
          for (int c = 0; c < C::kSlabsK && ok; ++c) {
            const uint32_t dst = next_stage(C::kKSlabBytes);
            tma_load_3d(dst, &tm_k, c * 64, x.c0 + i * kKT, x.bh,
                        bar.full((slab - 1) % C::kStages));
          }
        // per value tile: the V slabs of the P.V terms and the C_k slabs of the
        // inter-chunk term, in the order the MMA issuer takes them
        const bool frame = tile_frame<kPair>(g, p, x, tpad);
        auto load_v = [&](int dv0) {
          for (int i = 0; i < x.n_kv && ok; ++i)
            for (int v = 0; v < 2 && ok; ++v) {
              const uint32_t dst = next_stage(C::kMNSlabBytes);
              for (int b = 0; b < DVT / 64; ++b)
                tma_load_3d(dst + b * 8192, &tm_v, dv0 + b * 64, x.c0 + i * kKT + v * 64, x.bh,
                            bar.full((slab - 1) % C::kStages));
            }
        };
        // C_k rows [64c, 64c + 64) (kPair: then those of chunk k + 1, or of
        // chunk k again past the last chunk, where the zero half of the
        // stacked Q~ operand meets them)
        auto load_c = [&](int dv0) {
          for (int c = 0; c < C::kChunks * C::kSlabsK && ok; ++c) {
            const int kc = x.k + c / C::kSlabsK < p.NC ? x.k + c / C::kSlabsK : p.NC - 1;
            const uint32_t dst = next_stage(C::kMNSlabBytes);
            for (int b = 0; b < DVT / 64; ++b) {
              const size_t off = cb_block_row((long)x.bh * p.NC + kc, dv0 / 64 + b,
                                              (c % C::kSlabsK) * 64, DK, p.DV / 64);
              const bool in = MLSTM_IN_BOUNDS(
                  p, off + 4096 <= (size_t)p.BH * p.NC * DK * p.DV && kc >= 0);
              bulk_load(dst + b * 8192, Cb + (in ? off : 0), 8192,
                        bar.full((slab - 1) % C::kStages));
            }
          }
        };
        for (int d = 0; d < n_dv && ok; ++d) {
          if (frame) {
            load_c(d * DVT);
            load_v(d * DVT);
          } else {
            load_v(d * DVT);
            load_c(d * DVT);
          }
        }
      }
      for (int q = (slab > C::kStages ? slab - C::kStages : 0); q < slab; ++q)
        mbar_wait(bar.full(q % C::kStages), (q / C::kStages) & 1, p, 13);
      if (n > 0) mbar_wait(bar.q_full(), (n - 1) & 1, p, 14);
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, kKT, 0, 0);
      constexpr uint32_t idO = idesc_bf16(128, DVT, 0, 1);
      bool ok = true;
      int slab = 0, dcount = 0;
      int sc0 = 0, sc1 = 0;  // times S tile 0 / 1 has been filled (no arrays: registers)
      auto take = [&]() -> uint32_t {
        const int s = slab % C::kStages, u = slab / C::kStages;
        ok = ok && mbar_wait(bar.full(s), u & 1, p, 5);
        tc_fence_after();
        ++slab;
        return (uint32_t)s;
      };
      int n = 0;
      for (int it = item_at(0); it < n_items && ok; it = item_at(n + 1), ++n) {
        const WItem x = decode_witem(it, p, n_q);
        const bool frame = tile_frame<kPair>(g, p, x, tpad);  // used after the S MMAs
        ok = mbar_wait(bar.q_full(), n & 1, p, 3);
        for (int i = 0; i < x.n_kv && ok; ++i) {  // S_i
          const int fills = i ? sc1 : sc0;
          if (fills >= 1) ok = ok && mbar_wait(bar.pv_done(i), (fills - 1) & 1, p, 4);
          tc_fence_after();
          const uint32_t dS = tmem + (i ? kColS1 : kColS0);
          for (int c = 0; c < C::kSlabsK && ok; ++c) {
            const uint32_t s = take();
            if (!ok) break;
            const uint32_t a0 = sbase + C::kOffQ + c * 16384;
            const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(dS, sdesc_sw128(a0 + kk * 32, 16, 1024),
                          sdesc_sw128(b0 + kk * 32, 16, 1024), idS, (c | kk) != 0);
            mma_commit(bar.empty(s));
          }
          mma_commit(bar.s_full(i));
          if (i) ++sc1; else ++sc0;
        }
        for (int d = 0; d < n_dv && ok; ++d, ++dcount) {
          const int ob = dcount & 1;
          const uint32_t dO = tmem + (uint32_t)ob * 128u;
          if (dcount >= 2) ok = ok && mbar_wait(bar.o_empty(ob), ((dcount >> 1) - 1) & 1, p, 6);
          tc_fence_after();
          // P_i . V_i[:, d] (A from TMEM); the first MMA into O initialises it
          auto mma_pv = [&](bool init) {
            for (int i = 0; i < x.n_kv && ok; ++i) {
              if (d == 0) ok = mbar_wait(bar.p_full(i), ((i ? sc1 : sc0) - 1) & 1, p, 8);
              tc_fence_after();
              const uint32_t aP = tmem + (i ? kColS1 : kColS0);
              for (int v = 0; v < 2 && ok; ++v) {
                const uint32_t s = take();
                if (!ok) break;
                const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ts(dO, aP + (uint32_t)v * kColPHalf + (uint32_t)kk * 8u,
                              sdesc_sw128(b0 + kk * 2048, 8192, 1024), idO,
                              !init || (i | v | kk) != 0);
                mma_commit(bar.empty(s));
              }
              if (d == n_dv - 1) mma_commit(bar.pv_done(i));
            }
          };
          // Q~ . C_k[:, d]
          auto mma_qc = [&](bool init) {
            for (int c = 0; c < C::kChunks * C::kSlabsK && ok; ++c) {
              const uint32_t s = take();
              if (!ok) break;
              const uint32_t a0 = sbase + C::kOffQ + c * 16384;
              const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(dO, sdesc_sw128(a0 + kk * 32, 16, 1024),
                            sdesc_sw128(b0 + kk * 2048, 8192, 1024), idO,
                            !init || (c | kk) != 0);
              mma_commit(bar.empty(s));
            }
          };
          if (frame) {
            // one frame for the tile: Q is used as loaded, so the inter-chunk
            // term goes first and waits for no row thread
            mma_qc(true);
            mma_pv(false);
          } else {
            mma_pv(true);
            if (!ok) break;
            if (d == 0) {
              ok = mbar_wait(bar.q_scaled(), n & 1, p, 7);  // Q rows scaled in place
              tc_fence_after();
            }
            mma_qc(false);
          }
          if (!ok) break;
          if (d == n_dv - 1) mma_commit(bar.q_empty());  // last reader of Q issued
          mma_commit(bar.o_full(ob));
        }
      }
      mma_commit(bar.mma_idle());
      mbar_wait(bar.mma_idle(), 0, p, 15);
    }
  } else {
    // ------------------- gating / softmax / epilogue ----------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int rt = threadIdx.x - 64;
    const int h = rt >> 7;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const float ks = p.key_scale;
    constexpr int kHalfO = DVT / 2;
    constexpr int kSlabsPerHalf = (C::kSlabsK + 1) / 2;
    bool ok = true;
    int dcount = 0;
    int pc0 = 0, pc1 = 0;  // times S tile 0 / 1 has been turned into P
    // kPair: rows 64..127 belong to chunk k + 1 (past the last chunk they are
    // past T, and chunk k stands in)
    const int rchunk = kPair && r >= 64 ? 1 : 0;
    auto chunk_of = [&](const WItem& x, int part) {
      return x.k + part < p.NC ? x.k + part : p.NC - 1;
    };
    auto fetch_rows = [&](const WItem& x, float& m_in, float& amax, float& bc, int& td) {
      const int t = x.t0 + r;
      m_in = g.mchk[(long)x.bh * (p.NC + 1) + chunk_of(x, rchunk)];
      amax = g.amax[(long)x.bh * tpad + t];
      bc = g.bcum[(long)x.bh * tpad + t];
      td = g.dom ? g.dom[(long)x.bh * p.NC + chunk_of(x, rchunk)] : -1;
    };
    // One frame for the tile (tile_frame): every row's terms scaled by
    // e^{mu_r - m_k}, so P_rs = s (q_r.k_s) e^{acol_s - m_k} takes one column
    // factor per key, the inter-chunk term needs no scaling of Q (factor 1)
    // and h_r = O_r / max(|den_r|, e^{-(bcum_r + m_k)}).  Otherwise each row
    // works in its own frame mu_r = max(m_k, amax_r): the column data holds
    // acol log2(e), each element takes its own exponential and Q is scaled.
    auto fetch_cols = [&](const WItem& x, int buf, bool frame, float F) {
      float* ac = acol_s + buf * kPSlots * kKT;
      float* nn = n_s + buf * C::kChunks * DK;
      for (int j = rt; j < x.n_kv * kKT; j += 256) {
        const float a = g.acol[(long)x.bh * tpad + x.c0 + j];
        ac[j] = frame ? ks * expf(a - F) : a * 1.4426950408889634f;  // -inf -> 0 / -inf
      }
      for (int j = rt; j < C::kChunks * DK; j += 256)
        nn[j] = n_states[((long)x.bh * p.NC + chunk_of(x, j / DK)) * DK + j % DK];
    };
    float nx_m_in = 0.f, nx_amax = 0.f, nx_bc = 0.f;
    int nx_td = -1;
    bool nx_frame = false;
    if (blockIdx.x < n_items) {
      const WItem x0 = decode_witem(blockIdx.x, p, n_q);
      fetch_rows(x0, nx_m_in, nx_amax, nx_bc, nx_td);
      nx_frame = tile_frame<kPair>(g, p, x0, tpad);
      fetch_cols(x0, 0, nx_frame, nx_m_in);
    }
    int n = 0;
    for (int it = item_at(0); it < n_items && ok; it = item_at(n + 1), ++n) {
      const WItem x = decode_witem(it, p, n_q);
      const int t = x.t0 + r;
      const float m_in = nx_m_in, amax = nx_amax, bc = nx_bc;
      const int td = nx_td;  // warp-uniform (kPair: rows of one chunk per warp)
      const bool frame = nx_frame;  // uniform over the CTA
      const float* ac = acol_s + (n & 1) * kPSlots * kKT;
      const float* nn = n_s + ((n & 1) * C::kChunks + rchunk) * DK;
      const float mu = fmaxf(m_in, amax);  // the row's own frame
      const float fr = frame ? m_in : mu;  // the frame this tile works in
      const float mu2 = mu * 1.4426950408889634f;
      const float f_inter = expf(m_in - fr);  // 1 with one frame
      named_bar_sync(1, 256);

      // Partial den_inter = q_r . n_k over this half's slabs; then release Q.
      ok = mbar_wait(bar.q_full(), n & 1, p, 9);
      float dn = 0.f;
      for (int c = h * kSlabsPerHalf; c < C::kSlabsK && c < (h + 1) * kSlabsPerHalf && ok; ++c) {
        const uint8_t* slab_ptr = smem + C::kOffQ + c * 16384;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(slab_ptr + sw128_offset(r, j));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(h2[e]);
            dn = fmaf(f2.x, nn[c * 64 + j * 8 + 2 * e], dn);
            dn = fmaf(f2.y, nn[c * 64 + j * 8 + 2 * e + 1], dn);
          }
        }
      }
      float den = f_inter * dn;

      // Gated P tiles, once per item, written back over their S tiles in TMEM.
      for (int i = 0; i < x.n_kv; ++i) {
        const int pc = i ? pc1 : pc0;
        ok = ok && mbar_wait(bar.s_full(i), pc & 1, p, 10);
        tc_fence_after();
        const bool diag = (i == x.n_kv - 1);
        const uint32_t scol = (i ? kColS1 : kColS0) + h * kColPHalf;
        float rs = 0.f;
        if (ok) {
          uint32_t v[64];
          tmem_ld32(trow + scol, *reinterpret_cast<uint32_t(*)[32]>(v));
          tmem_ld32(trow + scol + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          tmem_wait_ld();
          uint32_t pk[32];
          const float* acl = ac + i * kKT + h * 64;
          if (frame) {
            uint64_t rs2 = 0;  // two fp32 partial sums, +0
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const int s0 = h * 64 + j;
              const float2 cf = *reinterpret_cast<const float2*>(acl + j);
              float2 pf = f32x2_split(mul_f32x2(
                  f32x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), f32x2(cf.x, cf.y)));
              if (diag && s0 > r) pf.x = 0.f;
              if (diag && s0 + 1 > r) pf.y = 0.f;
              rs2 = add_f32x2(rs2, f32x2(pf.x, pf.y));
              pk[j >> 1] = pack_bf16x2(pf.x, pf.y);
            }
            const float2 r2 = f32x2_split(rs2);
            rs = r2.x + r2.y;
          } else {
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const int s0 = h * 64 + j;
              float pa = __uint_as_float(v[j]) * ks * ex2_approx(acl[j] - mu2);
              float pb = __uint_as_float(v[j + 1]) * ks * ex2_approx(acl[j + 1] - mu2);
              if (diag && s0 > r) pa = 0.f;
              if (diag && s0 + 1 > r) pb = 0.f;
              if (kPair && ((s0 ^ r) & 64)) pa = pb = 0.f;  // key and query in different chunks
              rs += pa + pb;
              pk[j >> 1] = pack_bf16x2(pa, pb);
            }
          }
          tmem_st32(trow + scol, pk);
          tmem_wait_st();
        }
        den += rs;
        tc_fence_before();
        mbar_arrive(bar.p_full(i));
        if (i) ++pc1; else ++pc0;
      }

      // Every S MMA of this item has completed (the waits above): scale this
      // half of the Q row by e^{m_k - mu_r} in place for the inter-chunk MMAs
      // (kPair: into the row's chunk half of the stacked operand, zeros into
      // the other half).  With one frame Q stays as loaded (its inter-chunk
      // MMAs may already be running); the arrival below still marks the item.
      if (ok && !frame) {
        for (int c = h * kSlabsPerHalf; c < C::kSlabsK && c < (h + 1) * kSlabsPerHalf; ++c) {
          uint8_t* slab_ptr = smem + C::kOffQ + c * 16384;
          uint8_t* dst_ptr = slab_ptr + rchunk * C::kSlabsK * 16384;
          uint8_t* zero_ptr = slab_ptr + (1 - rchunk) * C::kSlabsK * 16384;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 u = *reinterpret_cast<const uint4*>(slab_ptr + sw128_offset(r, j));
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f2 = __bfloat1622float2(h2[e]);
              h2[e] = __floats2bfloat162_rn(f2.x * f_inter, f2.y * f_inter);
            }
            *reinterpret_cast<uint4*>(dst_ptr + sw128_offset(r, j)) = u;
            if (kPair) *reinterpret_cast<uint4*>(zero_ptr + sw128_offset(r, j)) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar.q_scaled());

      // The next item's row values and column data (other buffer).
      const int it_next = item_at(n + 1);
      if (it_next < n_items) {
        const WItem xn = decode_witem(it_next, p, n_q);
        fetch_rows(xn, nx_m_in, nx_amax, nx_bc, nx_td);
        nx_frame = tile_frame<kPair>(g, p, xn, tpad);
        fetch_cols(xn, (n + 1) & 1, nx_frame, nx_m_in);
      }

      // Both halves' partial denominators (and inter-chunk parts) -> the row's.
      red_s[rt] = make_float2(den, dn);
      named_bar_sync(1, 256);
      const float2 other = red_s[rt ^ 128];
      den += other.x;
      // a dominated chunk's rank-one part, (n_k^T q~_r) v_{t*}, added in fp32
      const float c1 = f_inter * (dn + other.y);
      const __nv_bfloat16* vstar =
          td >= 0 ? Vraw + ((long)x.bh * p.T + td) * p.DV + h * kHalfO : nullptr;
      const float mr = bc + fr;  // the floor's exponent in the tile's frame
      // the plain sigmoid variant has no normaliser: h = e^{m_r} O
      const float floor_f = expf(-mr);
      const float denom = p.no_norm ? floor_f : fmaxf(fabsf(den), floor_f);
      const float inv = p.no_norm ? expf(mr) : 1.f / denom;
      if (t < p.T && h == 0) {  // per-token outputs in the row frame mu_r
        // (where the floor is picked, the row frame's floor itself, so that
        // a comparison with e^{-m_r} tells the two cases apart exactly)
        const float dr = !frame ? denom
                         : (p.no_norm || !(fabsf(den) > floor_f)) ? expf(-(bc + mu))
                                                                  : fabsf(den) * expf(fr - mu);
        if (n_out) n_out[(long)x.bh * p.T + t] = p.signed_den ? copysignf(dr, den) : dr;
        if (m_out) m_out[(long)x.bh * p.T + t] = bc + mu;
      }

      for (int d = 0; d < n_dv; ++d, ++dcount) {
        const uint32_t colO = (uint32_t)(dcount & 1) * 128u + h * kHalfO;
        ok = ok && mbar_wait(bar.o_full(dcount & 1), (dcount >> 1) & 1, p, 12);
        tc_fence_after();
        if (rt == 0) tma_store_wait_read_all();  // the staging tile is free again
        named_bar_sync(1, 256);
        if (ok) {
          uint32_t v0[32], v1[32];
          tmem_ld32(trow + colO, v0);
          if (kHalfO >= 64) tmem_ld32(trow + colO + 32, v1);
          tmem_wait_ld();
          if (vstar) {
            add_rank1_32(v0, c1, vstar + d * DVT);
            if (kHalfO >= 64) add_rank1_32(v1, c1, vstar + d * DVT + 32);
          }
          // this half's columns: box (h * kHalfO) / 64, 16-byte chunks from cb
          uint8_t* box = smem + C::kOffOut + ((h * kHalfO) >> 6) * 16384;
          const int cb = ((h * kHalfO) & 63) >> 3;
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2)
            pk[j >> 1] = pack_bf16x2(__uint_as_float(v0[j]) * inv, __uint_as_float(v0[j + 1]) * inv);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(box + sw128_offset(r, cb + j)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          if (kHalfO >= 64) {
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              pk[j >> 1] =
                  pack_bf16x2(__uint_as_float(v1[j]) * inv, __uint_as_float(v1[j + 1]) * inv);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(box + sw128_offset(r, cb + 4 + j)) =
                  make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar.o_empty(dcount & 1));
        fence_proxy_async_smem();
        named_bar_sync(1, 256);
        if (rt == 0 && ok) {
          for (int b = 0; b < DVT / 64; ++b)
            if (MLSTM_IN_BOUNDS(p, d * DVT + b * 64 + 64 <= p.DV && x.t0 < p.T && x.bh < p.BH))
              tma_store_3d(&tm_h, sbase + C::kOffOut + b * 16384, d * DVT + b * 64, x.t0, x.bh);
          tma_store_commit();
        }
      }
    }
    if (rt == 0) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DK, int DVT, bool kPair>
cudaError_t launch_wide_t(const Problem& p, const void* Q, const void* K, const void* V, Gates g,
                          const __nv_bfloat16* Cb, const float* n_states, void* H, float* n_out,
                          float* m_out, cudaStream_t st) {
  using C = WCfg<DK, DVT, kPair>;
  CUtensorMap tq, tk, tv, th;
  if (!encode_tmap_bf16_3d(&tq, Q, p.DK, p.T, p.BH, 64, kQT) ||
      !encode_tmap_bf16_3d(&tk, K, p.DK, p.T, p.BH, 64, kKT) ||
      !encode_tmap_bf16_3d(&tv, V, p.DV, p.T, p.BH, 64, 64) ||
      !encode_tmap_bf16_3d(&th, H, p.DV, p.T, p.BH, 64, kQT))
    return cudaErrorInvalidValue;
  auto kern = tc_parallel_wide_kernel<DK, DVT, kPair>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long items = (long)p.BH * ((p.T + kQT - 1) / kQT);
  if (items > (1L << 30)) return cudaErrorInvalidValue;
  const int grid = (int)(items < sms ? items : sms);
  kern<<<grid, kThreads, C::kSmem, st>>>(tq, tk, tv, Cb, th, p, g, n_states, n_out, m_out,
                                         (int)items, static_cast<const __nv_bfloat16*>(V));
  return cudaGetLastError();
}

}  // namespace

bool tc_parallel_wide_supported(const Problem& p) {
  const bool dk_ok = p.DK == 64 || p.DK == 128 || p.DK == 256;
  const bool dv_ok = p.DV == 64 || p.DV % 128 == 0;
  const bool l_ok = (p.L % kKT == 0 && p.L <= kPSlots * kKT) || (p.L == 64 && p.DK <= 128);
  return dk_ok && dv_ok && p.DV <= 1024 && l_ok && p.T > 0;
}

cudaError_t launch_tc_parallel_wide(const Problem& p, const void* Q, const void* K, const void* V,
                                    Gates g, const __nv_bfloat16* Cb, const float* n_states,
                                    void* H, float* n_out, float* m_out, cudaStream_t st) {
  const int dvt = p.DV >= 128 ? 128 : 64;
  const bool pair = p.L == 64;
#define MLSTM_WIDE_CASE(dk, dvt_, pair_)                                                      \
  if (p.DK == dk && dvt == dvt_ && pair == pair_)                                             \
    return launch_wide_t<dk, dvt_, pair_>(p, Q, K, V, g, Cb, n_states, H, n_out, m_out, st);
  MLSTM_WIDE_CASE(64, 64, false)
  MLSTM_WIDE_CASE(64, 128, false)
  MLSTM_WIDE_CASE(128, 64, false)
  MLSTM_WIDE_CASE(128, 128, false)
  MLSTM_WIDE_CASE(256, 64, false)
  MLSTM_WIDE_CASE(256, 128, false)
  MLSTM_WIDE_CASE(64, 64, true)
  MLSTM_WIDE_CASE(64, 128, true)
  MLSTM_WIDE_CASE(128, 64, true)
  MLSTM_WIDE_CASE(128, 128, true)
#undef MLSTM_WIDE_CASE
  return cudaErrorNotSupported;
}

}  // namespace mlstm
