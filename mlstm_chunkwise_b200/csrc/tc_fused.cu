// G4: the fused chunkwise forward pass -- chunk state carried on chip.
//
// "flash-xlstm-exp 0.1.0", "Upgrade roadmap" item 2 plans a kernel that fuses
// the recurrent (chunk state) and parallel (output) halves so that the chunk
// states never go through HBM.  This is that kernel for heads that fit one SM:
// d_qk = 128, d_v of 64 or 128, chunks of 128 tokens.  Per (b, h) the chunks
// are processed in order by one CTA; for chunk k (same quantities as the
// unfused kernels, "Tiled Flash Linear Attention", abstract):
//
//   S       = Q_k K_k^T                                   (tcgen05, TMEM)
//   P_rs    = s S_rs e^{acol_s - mu_r}  (s <= r)           (row threads, TMEM)
//   O       = P V_k + Q~ C_k,  Q~ = diag(e^{m_k - mu_r}) Q_k
//   h_r     = O_r / max(|den_r|, e^{-(bcum_r + mu_r)}),  den_r = e^{m_k - mu_r} n_k.q_r + sum_s P_rs
//   C_{k+1} = e^{g_k + m_k - m_{k+1}} C_k + (w K_k)^T V_k,  w_s = s e^{g_k + acol_s - m_{k+1}}
//   n_{k+1} = the same with V -> 1 (fp32, from the unrounded products w_s k_s)
//
// (Where the gates allow, a chunk uses one frame F for all rows instead of
// mu_r -- F = m_k, so Q~ = Q -- see the row values below.)
//
// The fp32 master state C lives in TMEM for the whole sequence of a head; the
// Q~ C_k MMA reads a bf16 copy of it that the row threads write into shared
// memory once per chunk (together with the decay of the master).  The n
// vector is carried in shared memory by the row threads.  For a chunk whose
// entering state one token t* dominates (g.dom), the copy holds C_k - n*_k
// v_{t*}^T, the denominator uses n*_k and the epilogue adds (n*_k^T q~) v_{t*}
// in fp32 (n* = n - d, d the rounding residual of t*'s weighted key; tc.h).
//
// Roles (352 threads): warp 0 TMA producer; warp 1 TMEM owner and MMA issuer;
// warp 2 stores H (a TMA store per chunk, then it releases the Q buffer the
// rows were staged in); warps 3..10 two threads per row (each owning half of
// the columns).  One
// persistent CTA per SM walks its heads; the chunk counter runs on across
// heads, so the next head's first chunk is prefetched like any other.
// MMA order per chunk j:  [ready(j)]  S(j+1)  [V(j)]  P.V(j)  Q~.C(j)  C += (wK)^T V(j)
// Row order per chunk j:  prep(j+1) (den_inter, P, Q~, wK, n)  epilogue(j)
//                         [master ready] operand copy of C_{j+1}, decay -> ready(j+1)
// TMEM (512 columns): master C [0, 128), S/P buffers [128, 256) and
// [256, 384), O [384, 512).
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kThreads = 352;
constexpr int kL = 128;   // chunk = query tile = key tile
constexpr int kDK = 128;  // key width handled by this kernel
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColC = 0, kColS0 = 128, kColS1 = 256, kColO = 384;

template <int DV>
struct FCfg {
  static_assert(DV == 64 || DV == 128, "d_v of 64 or 128");
  static constexpr uint32_t kQBytes = kL * kDK * 2;   // 2 slabs [128 rows x 64] (16 KB each)
  static constexpr uint32_t kKBytes = kL * kDK * 2;
  static constexpr uint32_t kVBytes = kL * DV * 2;    // [2 key halves][DV / 64 blocks][64 x 64]
  static constexpr uint32_t kCBytes = kDK * DV * 2;   // [2 dk slabs][DV / 64 blocks][64 x 64]
  static constexpr int kVBufs = DV <= 64 ? 2 : 1;
  static constexpr int kRG = 256 / (kDK / 8);         // row groups of the K pass (16)
  static constexpr uint32_t kOffQ = 0;                                   // 2 buffers
  static constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;                 // 2 buffers
  static constexpr uint32_t kOffV = kOffK + 2 * kKBytes;                 // kVBufs buffers
  static constexpr uint32_t kOffC = kOffV + kVBufs * kVBytes;
  static constexpr uint32_t kOffRedN = kOffC + kCBytes;                  // float[kRG][kDK]
  static constexpr uint32_t kOffN = kOffRedN + kRG * kDK * 4;            // float[kDK]
  static constexpr uint32_t kOffNPrev = kOffN + kDK * 4;                 // float[kDK]: n_k
  static constexpr uint32_t kOffDStar = kOffNPrev + kDK * 4;             // float[kDK]: d_k
  static constexpr uint32_t kOffNStar = kOffDStar + kDK * 4;             // float[kDK]: n_k - d_k
  // per chunk (2 buffers) and key column: acol, e^{acol - c}, the weight w
  static constexpr uint32_t kOffAcol = kOffNStar + kDK * 4;              // float[2][3][kL]
  static constexpr uint32_t kOffRed = kOffAcol + 2 * 3 * kL * 4;         // float2[256]
  static constexpr uint32_t kOffBar = kOffRed + 256 * 8;
  static constexpr uint32_t kOffTmemSlot = kOffBar + 256;
  static constexpr uint32_t kBytes = kOffTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct FBars {
  uint32_t a;
  __device__ __forceinline__ uint32_t q_full(int b) const { return a + 8 * b; }
  __device__ __forceinline__ uint32_t q_free(int b) const { return a + 16 + 8 * b; }
  __device__ __forceinline__ uint32_t k_full(int b) const { return a + 32 + 8 * b; }
  __device__ __forceinline__ uint32_t k_free(int b) const { return a + 48 + 8 * b; }
  __device__ __forceinline__ uint32_t v_full(int b) const { return a + 64 + 8 * b; }
  __device__ __forceinline__ uint32_t v_free(int b) const { return a + 80 + 8 * b; }
  __device__ __forceinline__ uint32_t s_full(int b) const { return a + 96 + 8 * b; }
  __device__ __forceinline__ uint32_t ready() const { return a + 112; }
  __device__ __forceinline__ uint32_t o_full() const { return a + 120; }
  __device__ __forceinline__ uint32_t upd_done() const { return a + 128; }
  __device__ __forceinline__ uint32_t mma_idle() const { return a + 136; }
  // H rows of the chunk staged in Q buffer b by all 256 row threads
  __device__ __forceinline__ uint32_t stg_full(int b) const { return a + 144 + 8 * b; }
};

// The j-th chunk of this CTA (over its heads in turn): head and chunk index.
struct FChunk {
  int bh, k;
};
__device__ __forceinline__ FChunk chunk_at(int j, int NC) {
  FChunk c;
  c.bh = (int)blockIdx.x + (j / NC) * (int)gridDim.x;
  c.k = j % NC;
  return c;
}

template <int DV>
__global__ void __launch_bounds__(kThreads, 1)
tc_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_h,
                Problem p, Gates g, const float* __restrict__ C0, const float* __restrict__ n0,
                float* __restrict__ C_T, float* __restrict__ n_T, float* __restrict__ m_T,
                const __nv_bfloat16* __restrict__ Vraw, const __nv_bfloat16* __restrict__ Kraw) {
  using F = FCfg<DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const FBars bar{sbase + F::kOffBar};
  float* redn_s = reinterpret_cast<float*>(smem + F::kOffRedN);
  float* n_s = reinterpret_cast<float*>(smem + F::kOffN);
  float* nprev_s = reinterpret_cast<float*>(smem + F::kOffNPrev);
  float* dstar_s = reinterpret_cast<float*>(smem + F::kOffDStar);
  float* nstar_s = reinterpret_cast<float*>(smem + F::kOffNStar);
  float* acol_s = reinterpret_cast<float*>(smem + F::kOffAcol);
  float2* red_s = reinterpret_cast<float2*>(smem + F::kOffRed);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + F::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NC = p.NC;
  const int my_heads = p.BH > (int)blockIdx.x
                           ? (p.BH - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                           : 0;
  const int total = my_heads * NC;  // chunks of this CTA
  const long tpad = (long)NC * p.L;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.q_full(b), 1);
      mbar_init(bar.q_free(b), 1);
      mbar_init(bar.k_full(b), 1);
      mbar_init(bar.k_free(b), 1);
      mbar_init(bar.v_full(b), 1);
      mbar_init(bar.v_free(b), 1);
      mbar_init(bar.s_full(b), 1);
    }
    mbar_init(bar.ready(), 256);
    mbar_init(bar.o_full(), 1);
    mbar_init(bar.upd_done(), 1);
    mbar_init(bar.mma_idle(), 1);
    mbar_init(bar.stg_full(0), 256);
    mbar_init(bar.stg_full(1), 256);
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
    // Order: Q(0), K(0), then per chunk j: V(j), Q(j+1), K(j+1).  Each load
    // waits for the release of its buffer by the chunk two (Q, K) or
    // kVBufs (V) before; every release completes once per chunk of its
    // buffer and the next load of that buffer is issued only after the wait.
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      bool ok = true;
      auto load_qk = [&](int j) {
        const FChunk c = chunk_at(j, NC);
        const int b = j & 1, t0 = c.k * kL;
        if (j >= 2) ok = ok && mbar_wait(bar.q_free(b), ((j >> 1) - 1) & 1, p, 1);
        if (!ok) return;
        mbar_expect_tx(bar.q_full(b), F::kQBytes);
        for (int s = 0; s < 2; ++s)
          tma_load_3d(sbase + F::kOffQ + b * F::kQBytes + s * 16384, &tm_q, s * 64, t0, c.bh,
                      bar.q_full(b));
        if (j >= 2) ok = ok && mbar_wait(bar.k_free(b), ((j >> 1) - 1) & 1, p, 2);
        if (!ok) return;
        mbar_expect_tx(bar.k_full(b), F::kKBytes);
        for (int s = 0; s < 2; ++s)
          tma_load_3d(sbase + F::kOffK + b * F::kKBytes + s * 16384, &tm_k, s * 64, t0, c.bh,
                      bar.k_full(b));
      };
      auto load_v = [&](int j) {
        const FChunk c = chunk_at(j, NC);
        const int b = j % F::kVBufs, t0 = c.k * kL;
        if (j >= F::kVBufs) ok = ok && mbar_wait(bar.v_free(b), ((j / F::kVBufs) - 1) & 1, p, 3);
        if (!ok) return;
        mbar_expect_tx(bar.v_full(b), F::kVBytes);
        for (int v = 0; v < 2; ++v)
          for (int blk = 0; blk < DV / 64; ++blk)
            tma_load_3d(sbase + F::kOffV + b * F::kVBytes + (v * (DV / 64) + blk) * 8192, &tm_v,
                        blk * 64, t0 + v * 64, c.bh, bar.v_full(b));
      };
      load_qk(0);
      for (int j = 0; j < total && ok; ++j) {
        load_v(j);
        if (j + 1 < total) load_qk(j + 1);
      }
      // Drain: the last loads of every buffer must land before the CTA exits.
      for (int j = (total > 2 ? total - 2 : 0); j < total; ++j) {
        mbar_wait(bar.q_full(j & 1), (j >> 1) & 1, p, 12);
        mbar_wait(bar.k_full(j & 1), (j >> 1) & 1, p, 12);
      }
      for (int j = (total > F::kVBufs ? total - F::kVBufs : 0); j < total; ++j)
        mbar_wait(bar.v_full(j % F::kVBufs), (j / F::kVBufs) & 1, p, 12);
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0 && total > 0) {
      constexpr uint32_t idS = idesc_bf16(128, kL, 0, 0);
      constexpr uint32_t idO = idesc_bf16(128, DV, 0, 1);
      constexpr uint32_t idU = idesc_bf16(128, DV, 1, 1);
      bool ok = true;
      // S(j) = Q K^T into S buffer j & 1.  That buffer held P(j - 2), read by
      // P.V(j - 2), which precedes Q~.C(j - 2): o_full of chunk j - 2 (waited
      // by the caller) means it has been read.
      auto issue_s = [&](int j) {
        const int b = j & 1;
        ok = ok && mbar_wait(bar.q_full(b), (j >> 1) & 1, p, 4);
        ok = ok && mbar_wait(bar.k_full(b), (j >> 1) & 1, p, 4);
        tc_fence_after();
        if (!ok) return;
        const uint32_t qa = sbase + F::kOffQ + b * F::kQBytes;
        const uint32_t ka = sbase + F::kOffK + b * F::kKBytes;
        const uint32_t dS = tmem + (b ? kColS1 : kColS0);
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(dS, sdesc_sw128(qa + s * 16384 + kk * 32, 16, 1024),
                        sdesc_sw128(ka + s * 16384 + kk * 32, 16, 1024), idS, (s | kk) != 0);
        mma_commit(bar.s_full(b));
      };
      issue_s(0);
      for (int j = 0; j < total && ok; ++j) {
        const int b = j & 1, vb = j % F::kVBufs;
        // ready(j): P(j), Q~(j), w K(j) in place, the operand copy of C_j and
        // the decayed master; it also follows the epilogue of chunk j - 1, so
        // the single O accumulator is free.  (Completes once per chunk; the
        // next completion needs this chunk's MMAs.)
        ok = ok && mbar_wait(bar.ready(), j & 1, p, 5);
        tc_fence_after();
        // S(j + 1) first: the row threads turn it into P while V(j) arrives.
        if (j + 1 < total) {
          if (j >= 1) ok = ok && mbar_wait(bar.o_full(), (j - 1) & 1, p, 7);
          issue_s(j + 1);
        }
        ok = ok && mbar_wait(bar.v_full(vb), (j / F::kVBufs) & 1, p, 6);
        tc_fence_after();
        if (!ok) break;
        const uint32_t qa = sbase + F::kOffQ + b * F::kQBytes;
        const uint32_t ka = sbase + F::kOffK + b * F::kKBytes;
        const uint32_t va = sbase + F::kOffV + vb * F::kVBytes;
        const uint32_t ca = sbase + F::kOffC;
        const uint32_t aP = tmem + (b ? kColS1 : kColS0);
        // P . V, A = P from TMEM (key half v: columns [64 v, 64 v + 32))
#pragma unroll
        for (int v = 0; v < 2; ++v)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmem + kColO, aP + v * 64 + kk * 8,
                        sdesc_sw128(va + v * (DV / 64) * 8192 + kk * 2048, 8192, 1024), idO,
                        (v | kk) != 0);
        // Q~ . C_j (operand copy in shared memory, MN-major)
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + kColO, sdesc_sw128(qa + s * 16384 + kk * 32, 16, 1024),
                        sdesc_sw128(ca + s * (DV / 64) * 8192 + kk * 2048, 8192, 1024), idO, 1);
        mma_commit(bar.o_full());
        // master += (w K)^T V: A = K^T MN-major (dk halves 16 KB apart), B = V
#pragma unroll
        for (int kk = 0; kk < kL / 16; ++kk)
          mma_bf16_ss(tmem + kColC, sdesc_sw128(ka + kk * 2048, 16384, 1024),
                      sdesc_sw128(va + (kk >> 2) * (DV / 64) * 8192 + (kk & 3) * 2048, 8192, 1024),
                      idU, 1);
        mma_commit(bar.upd_done());
        mma_commit(bar.k_free(b));
        mma_commit(bar.v_free(vb));
      }
      mma_commit(bar.mma_idle());
      mbar_wait(bar.mma_idle(), 0, p, 15);
    }
  } else if (warp == 2) {
    // ------------------------------ H stores ------------------------------
    // stg_full(b) completes once per chunk staged in buffer b; the next chunk
    // of that buffer is staged only after its Q has been loaded, which waits
    // for the q_free this thread arrives on.
    if (lane == 0 && total > 0) {
      bool ok = true;
      for (int j = 0; j < total && ok; ++j) {
        const int b = j & 1;
        const FChunk c = chunk_at(j, NC);
        ok = mbar_wait(bar.stg_full(b), (j >> 1) & 1, p, 11);
        if (!ok) break;
        for (int bx = 0; bx < DV / 64; ++bx)
          if (MLSTM_IN_BOUNDS(p, c.k < NC && c.bh < p.BH))
            tma_store_3d(&tm_h, sbase + F::kOffQ + b * F::kQBytes + bx * 16384, bx * 64,
                         c.k * kL, c.bh);
        tma_store_commit();
        tma_store_wait_read_all();  // the Q buffer may take chunk j + 2's Q
        mbar_arrive(bar.q_free(b));
      }
      tma_store_wait_all();
    }
  } else {
    // ------------------------------ row threads ---------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;   // query row / TMEM lane / dk row of the master
    const int rt = threadIdx.x - 96;
    const int h = rt >> 7;         // half of the columns
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const float ks = p.key_scale;
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int kHalfV = DV / 2;
    // K pass mapping: 16-byte chunk cc (8 dk columns) of rows rg * 8 .. + 7
    const int cc = rt % (kDK / 8);
    const int rg = rt / (kDK / 8);
    bool ok = true;

    // Per-chunk row values.  Every term of a row may be scaled by a common
    // factor, so when the exponents allow it (frame) the whole chunk works in
    // one frame F = m_k (or, with no entering state, c = the chunk's largest
    // acol): P_rs = s S_rs e^{acol_s - F} is one column factor per key, the
    // inter-chunk factor e^{m_k - F} is 1 (Q is used as loaded) or 0, and
    // h_r = O_r / max(|den_r|, e^{-(bcum_r + F)}).  frame needs c - F <= 60
    // (with F = c, the first row's amax no lower than c - 60) and the floor's
    // exponent within +-80 over the chunk.  Otherwise, when sep is set, the
    // exponent of P splits into a column factor e^{acol_s - c} (<= 1) and a
    // row factor e^{c - mu_r} below e^60 (two multiplies per element); else
    // each element takes its own exponential.  Without frame the rows use
    // their own mu_r and Q is scaled by e^{m_k - mu_r}.
    struct Rows {
      float m_in, m_out, mu, bc, gk, decay, rowf;
      float fr;       // the frame of this row: F, or mu_r
      float f_inter;  // e^{m_k - fr}
      bool sep, frame, scaleq;
      int bh, td;  // td: dominant token of the chunk's entering state, or -1
    };
    // Gate values of a chunk, loaded two chunks ahead of their use (the
    // loads stay in flight while the chunk in between is processed).
    struct Raw {
      float m_in, m_out, amax, bc, gk, acol, amax0, amax_last, bc0, bc_last;
      int bh, k, td;
    };
    auto load_raw = [&](const FChunk& c) -> Raw {
      Raw v;
      const long base = (long)c.bh * tpad + (long)c.k * kL;
      v.m_in = g.mchk[(long)c.bh * (NC + 1) + c.k];
      v.m_out = g.mchk[(long)c.bh * (NC + 1) + c.k + 1];
      v.amax = g.amax[base + r];
      v.bc = g.bcum[base + r];
      v.gk = g.gtot[(long)c.bh * NC + c.k];
      v.acol = rt < kL ? g.acol[base + rt] : 0.f;
      v.amax0 = g.amax[base];
      v.amax_last = g.amax[base + kL - 1];
      v.bc0 = g.bcum[base];
      v.bc_last = g.bcum[base + kL - 1];  // bcum falls along the chunk
      v.bh = c.bh;
      v.k = c.k;
      v.td = g.dom ? g.dom[(long)c.bh * NC + c.k] : -1;
      return v;
    };
    auto finish = [&](const Raw& w, int buf) -> Rows {
      Rows v;
      v.m_in = w.m_in;
      v.m_out = w.m_out;
      v.mu = fmaxf(w.m_in, w.amax);
      v.bc = w.bc;
      v.gk = w.gk;
      v.decay = expf(w.gk + w.m_in - w.m_out);
      v.bh = w.bh;
      v.td = w.td;
      // dominated chunk: d = the rounding residual of t*'s weighted key, per
      // d_qk column (read after the barrier that precedes prep)
      if (w.td >= 0 && rt < kDK) dstar_s[rt] = dom_residual(g, p, w.bh, w.k, w.td, rt, Kraw);
      const float cmax = w.amax_last;               // max over the chunk (amax is a running max)
      const float mu0 = fmaxf(w.m_in, w.amax0);     // the smallest mu_r of the chunk
      // one frame for the chunk (uniform: the same loads in every thread)
      const bool fresh = w.m_in == -INFINITY;
      const float F = fresh ? cmax : w.m_in;
      const float spread = fresh ? cmax - w.amax0 : cmax - w.m_in;
      v.frame = spread <= 60.f && -w.bc_last - F <= 80.f && -w.bc0 - F >= -80.f;
      v.sep = !v.frame && (cmax - mu0) <= 60.f;
      v.rowf = v.sep ? ks * expf(cmax - v.mu) : 0.f;
      v.fr = v.frame ? F : v.mu;
      v.f_inter = expf(w.m_in - v.fr);
      // Q is scaled unless its factor is 1 (with no entering state it is 0:
      // a C0 given with m0 = -inf weighs nothing)
      v.scaleq = !v.frame || fresh;
      if (rt < kL) {
        float* col = acol_s + buf * 3 * kL;
        col[rt] = w.acol;
        col[kL + rt] = v.frame ? ks * expf(w.acol - F) : expf(w.acol - cmax);  // -inf -> 0
        col[2 * kL + rt] = ks * expf(w.gk + w.acol - w.m_out);              // -inf -> 0
      }
      return v;
    };
    // master <- C0 of head bh (or zero)
    auto init_master = [&](int bh) {
      for (int c = 0; c < kHalfV; c += 32) {
        uint32_t v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          v[e] = __float_as_uint(C0 ? C0[((long)bh * kDK + r) * DV + h * kHalfV + c + e] : 0.f);
        tmem_st32(trow + kColC + h * kHalfV + c, v);
      }
      tmem_wait_st();
    };
    // C_T and m_T of head bh from the master (all its updates completed);
    // n_T is written where the n vector of the head ends (see the loop).
    auto write_final = [&](int bh) {
      for (int c = 0; c < kHalfV; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + kColC + h * kHalfV + c, v);
        tmem_wait_ld();
        if (C_T && MLSTM_IN_BOUNDS(p, bh < p.BH && h * kHalfV + c + 32 <= DV)) {
          float4* dst = reinterpret_cast<float4*>(C_T + ((long)bh * kDK + r) * DV + h * kHalfV + c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      if (rt == 0 && m_T) m_T[bh] = g.mchk[(long)bh * (NC + 1) + NC];
    };
    // Operand copy of the master (C of the chunk about to start) into shared
    // memory as bf16 (MN-major, 128-byte swizzle), then the decay of the
    // master in place.  Called once every MMA of the previous chunk has
    // completed (its Q~.C read the old copy; its update wrote the master).
    auto copy_and_decay = [&](const Rows& rv) {
      const float decay = rv.decay;
      const int sl = r >> 6, rr = r & 63;
      uint8_t* crow = smem + F::kOffC + sl * (DV / 64) * 8192 + rr * 128;
      // a dominated state leaves as C - n v_{t*}^T (n_k: kept by prep)
      const __nv_bfloat16* vstar =
          rv.td >= 0 ? Vraw + ((long)rv.bh * p.T + rv.td) * DV + h * kHalfV : nullptr;
      const float nrow = vstar ? dstar_s[r] - nprev_s[r] : 0.f;  // -(n - d)
      for (int c = 0; c < kHalfV; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + kColC + h * kHalfV + c, v);
        tmem_wait_ld();
        const int col0 = h * kHalfV + c;  // first d_v column of these 32
        uint8_t* blk = crow + (col0 >> 6) * 8192;
        const int ch0 = (col0 & 63) >> 3;
        if (vstar) {
          uint32_t x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = v[e];
          add_rank1_32(x, nrow, vstar + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<uint4*>(blk + (((ch0 + e) ^ (rr & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(x[8 * e]), __uint_as_float(x[8 * e + 1])),
                pack_bf16x2(__uint_as_float(x[8 * e + 2]), __uint_as_float(x[8 * e + 3])),
                pack_bf16x2(__uint_as_float(x[8 * e + 4]), __uint_as_float(x[8 * e + 5])),
                pack_bf16x2(__uint_as_float(x[8 * e + 6]), __uint_as_float(x[8 * e + 7])));
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<uint4*>(blk + (((ch0 + e) ^ (rr & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                pack_bf16x2(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                pack_bf16x2(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                pack_bf16x2(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * decay);
        tmem_st32(trow + kColC + h * kHalfV + c, v);
      }
      tmem_wait_st();
    };
    // Everything of chunk j that needs S(j) but not the MMAs of chunk j - 1:
    // den_inter from the unscaled Q and n_j, P into TMEM, the scaled Q~ and
    // the weighted K in place, and n_{j+1} (n_j moves to nprev_s).  Returns
    // this half's partial denominator and its inter-chunk part q_r . n_j.
    auto prep = [&](int j, const Rows& rv) -> float2 {
      const int b = j & 1;
      uint8_t* qbuf = smem + F::kOffQ + b * F::kQBytes;
      uint8_t* kbuf = smem + F::kOffK + b * F::kKBytes;
      const float* ac = acol_s + b * 3 * kL;   // acol
      const float* cf = ac + kL;                // s e^{acol - F} (frame) or e^{acol - c}
      const float* wc = ac + 2 * kL;            // s e^{g + acol - m_out}
      const float f_inter = rv.f_inter;
      const float mu2 = rv.mu * kLog2e;
      // den_inter needs Q(j) and n_j only: it overlaps the S MMA.  (q_full of
      // a buffer completes once per load; the next load of the buffer needs
      // this chunk's Q released, after this wait.)
      ok = ok && mbar_wait(bar.q_full(b), (j >> 1) & 1, p, 8);
      // den_inter over this half's 64 dk columns (slab h of Q); a dominated
      // chunk uses n* = n - d
      const float* nvec = n_s;
      if (rv.td >= 0) {
        if (rt < kDK) nstar_s[rt] = n_s[rt] - dstar_s[rt];
        named_bar_sync(1, 256);
        nvec = nstar_s;
      }
      float dn = 0.f;
      {
        const uint8_t* slab = qbuf + h * 16384;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(slab + sw128_offset(r, c));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const float4 nv = *reinterpret_cast<const float4*>(nvec + h * 64 + c * 8 + 2 * e);
            const float2 fa = __bfloat1622float2(h2[e]);
            const float2 fb = __bfloat1622float2(h2[e + 1]);
            dn = fmaf(fa.x, nv.x, dn);
            dn = fmaf(fa.y, nv.y, dn);
            dn = fmaf(fb.x, nv.z, dn);
            dn = fmaf(fb.y, nv.w, dn);
          }
        }
      }
      float den = f_inter * dn;
      ok = ok && mbar_wait(bar.s_full(b), (j >> 1) & 1, p, 8);  // S(j) done: Q, K read
      tc_fence_after();
      // P = gated S over this half's 64 keys, back into the S columns it read
      // (in two passes of 32 keys: the packed 16 columns of the first pass
      // land on columns that pass has already read).
      {
        const uint32_t scol = (b ? kColS1 : kColS0) + h * 64;
        float rs = 0.f;
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
          uint32_t v[32];
          tmem_ld32(trow + scol + hp * 32, v);
          tmem_wait_ld();
          uint32_t pk[16];
          if (rv.frame) {
            uint64_t rs2 = 0;  // two fp32 partial sums, +0
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int s0 = h * 64 + hp * 32 + e;
              const float2 c2 = *reinterpret_cast<const float2*>(cf + s0);
              float2 pf = f32x2_split(mul_f32x2(
                  f32x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), f32x2(c2.x, c2.y)));
              if (s0 > r) pf.x = 0.f;
              if (s0 + 1 > r) pf.y = 0.f;
              rs2 = add_f32x2(rs2, f32x2(pf.x, pf.y));
              pk[e >> 1] = pack_bf16x2(pf.x, pf.y);
            }
            const float2 r2 = f32x2_split(rs2);
            rs += r2.x + r2.y;
          } else {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int s0 = h * 64 + hp * 32 + e;
            float pa, pb;
            if (rv.sep) {
              pa = __uint_as_float(v[e]) * cf[s0] * rv.rowf;
              pb = __uint_as_float(v[e + 1]) * cf[s0 + 1] * rv.rowf;
            } else {
              pa = __uint_as_float(v[e]) * ks * ex2_approx(ac[s0] * kLog2e - mu2);
              pb = __uint_as_float(v[e + 1]) * ks * ex2_approx(ac[s0 + 1] * kLog2e - mu2);
            }
            if (s0 > r) pa = 0.f;
            if (s0 + 1 > r) pb = 0.f;
            rs += pa + pb;
            pk[e >> 1] = pack_bf16x2(pa, pb);
          }
          }
          tmem_st16(trow + scol + hp * 16, pk);
        }
        den += rs;
      }
      // Q~ = e^{m_k - mu_r} q_r in place (slab h); with one frame Q stays
      if (rv.scaleq) {
        uint8_t* slab = qbuf + h * 16384;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(slab + sw128_offset(r, c));
          uint4 u = *ptr;
          __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(h2[e]);
            h2[e] = __floats2bfloat162_rn(f2.x * f_inter, f2.y * f_inter);
          }
          *ptr = u;
        }
      }
      // w K in place and the n partials from the unrounded products
      float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      {
        uint8_t* slab = kbuf + (cc >> 3) * 16384;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int row = rg * 8 + i;
          const float w = wc[row];
          uint4* ptr = reinterpret_cast<uint4*>(slab + sw128_offset(row, cc & 7));
          uint4 u = *ptr;
          __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(h2[e]);
            part[2 * e] = fmaf(f2.x, w, part[2 * e]);
            part[2 * e + 1] = fmaf(f2.y, w, part[2 * e + 1]);
            h2[e] = __floats2bfloat162_rn(f2.x * w, f2.y * w);
          }
          *ptr = u;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) redn_s[rg * kDK + cc * 8 + e] = part[e];
      tmem_wait_st();
      named_bar_sync(1, 256);  // n_j reads done, partials in place
      if (rt < kDK) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < F::kRG; ++i) acc += redn_s[i * kDK + rt];
        nprev_s[rt] = n_s[rt];               // n_j, for the operand copy of C_j
        n_s[rt] = rv.decay * n_s[rt] + acc;  // n_{j+1}
      }
      fence_proxy_async_smem();  // Q~ and w K for the MMAs
      named_bar_sync(1, 256);  // n_{j+1} visible; redn_s free
      return make_float2(den, dn);
    };

    // Epilogue of chunk j: the row's denominator from both halves, then
    // O / den as bf16 through the chunk's (now free) Q buffer and TMA stores.
    auto epilogue = [&](int j, const FChunk& c, const Rows& rv, float2 den_part) {
      const int b = j & 1;
      red_s[rt] = den_part;
      named_bar_sync(1, 256);
      const float2 other = red_s[rt ^ 128];
      const float den = den_part.x + other.x;
      // the plain sigmoid variant has no normaliser: h = e^{m_r} O
      const float mr = rv.bc + rv.fr;  // the floor's exponent in the chunk's frame
      const float inv = p.no_norm ? expf(mr) : 1.f / fmaxf(fabsf(den), expf(-mr));
      ok = ok && mbar_wait(bar.o_full(), j & 1, p, 9);  // Q~.C(j) done: Q(j) free
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(trow + kColO + h * kHalfV, v0);
      if (kHalfV >= 64) tmem_ld32(trow + kColO + h * kHalfV + 32, v1);
      tmem_wait_ld();
      if (rv.td >= 0) {  // a dominated chunk's rank-one part, (n_j^T q~_r) v_{t*}
        const float c1 = rv.f_inter * (den_part.y + other.y);
        const __nv_bfloat16* vstar = Vraw + ((long)c.bh * p.T + rv.td) * DV + h * kHalfV;
        add_rank1_32(v0, c1, vstar);
        if (kHalfV >= 64) add_rank1_32(v1, c1, vstar + 32);
      }
      uint8_t* stg = smem + F::kOffQ + b * F::kQBytes;  // [DV / 64 boxes][128 rows][128 B]
      const int col0 = h * kHalfV;
      uint8_t* box = stg + (col0 >> 6) * 16384;
      const int ch0 = (col0 & 63) >> 3;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4*>(box + sw128_offset(r, ch0 + e)) = make_uint4(
            pack_bf16x2(__uint_as_float(v0[8 * e]) * inv, __uint_as_float(v0[8 * e + 1]) * inv),
            pack_bf16x2(__uint_as_float(v0[8 * e + 2]) * inv, __uint_as_float(v0[8 * e + 3]) * inv),
            pack_bf16x2(__uint_as_float(v0[8 * e + 4]) * inv, __uint_as_float(v0[8 * e + 5]) * inv),
            pack_bf16x2(__uint_as_float(v0[8 * e + 6]) * inv, __uint_as_float(v0[8 * e + 7]) * inv));
      if (kHalfV >= 64) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(box + sw128_offset(r, ch0 + 4 + e)) = make_uint4(
              pack_bf16x2(__uint_as_float(v1[8 * e]) * inv, __uint_as_float(v1[8 * e + 1]) * inv),
              pack_bf16x2(__uint_as_float(v1[8 * e + 2]) * inv,
                          __uint_as_float(v1[8 * e + 3]) * inv),
              pack_bf16x2(__uint_as_float(v1[8 * e + 4]) * inv,
                          __uint_as_float(v1[8 * e + 5]) * inv),
              pack_bf16x2(__uint_as_float(v1[8 * e + 6]) * inv,
                          __uint_as_float(v1[8 * e + 7]) * inv));
      }
      fence_proxy_async_smem();
      mbar_arrive(bar.stg_full(b));  // the store warp takes it from here
    };

    if (total > 0) {
      const FChunk c0 = chunk_at(0, NC);
      Raw pending = load_raw(c0);
      init_master(c0.bh);
      if (rt < kDK) n_s[rt] = n0 ? n0[(long)c0.bh * kDK + rt] : 0.f;
      Rows cur = finish(pending, 0);
      if (total > 1) pending = load_raw(chunk_at(1, NC));
      named_bar_sync(1, 256);  // acol, n visible
      float2 den_cur = prep(0, cur);
      copy_and_decay(cur);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar.ready());
      for (int j = 0; j < total && ok; ++j) {
        const FChunk c = chunk_at(j, NC);
        const bool last_of_head = (c.k == NC - 1);
        Rows nxt = cur;
        float2 den_nxt = make_float2(0.f, 0.f);
        FChunk cn{};
        if (j + 1 < total) {
          cn = chunk_at(j + 1, NC);
          nxt = finish(pending, (j + 1) & 1);
          if (j + 2 < total) pending = load_raw(chunk_at(j + 2, NC));
          if (last_of_head) {
            // n_T of this head before the next head's n0 replaces it
            named_bar_sync(1, 256);
            if (rt < kDK && n_T) n_T[(long)c.bh * kDK + rt] = n_s[rt];
            if (rt < kDK) n_s[rt] = n0 ? n0[(long)cn.bh * kDK + rt] : 0.f;
          }
          named_bar_sync(1, 256);  // acol of chunk j + 1 and n visible
          den_nxt = prep(j + 1, nxt);
        } else if (last_of_head) {
          named_bar_sync(1, 256);
          if (rt < kDK && n_T) n_T[(long)c.bh * kDK + rt] = n_s[rt];
        }
        epilogue(j, c, cur, den_cur);
        // Every MMA of chunk j has completed (upd_done is committed last).
        ok = ok && mbar_wait(bar.upd_done(), j & 1, p, 10);
        tc_fence_after();
        if (last_of_head) write_final(c.bh);
        if (j + 1 < total) {
          if (last_of_head) init_master(cn.bh);  // master <- C0 of the next head
          copy_and_decay(nxt);
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(bar.ready());
        }
        cur = nxt;
        den_cur = den_nxt;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DV>
cudaError_t launch_fused_t(const Problem& p, const void* Q, const void* K, const void* V,
                           const float* C0, const float* n0, Gates g, void* H, float* C_T,
                           float* n_T, float* m_T, cudaStream_t st) {
  using F = FCfg<DV>;
  CUtensorMap tq, tk, tv, th;
  if (!encode_tmap_bf16_3d(&tq, Q, p.DK, p.T, p.BH, 64, kL) ||
      !encode_tmap_bf16_3d(&tk, K, p.DK, p.T, p.BH, 64, kL) ||
      !encode_tmap_bf16_3d(&tv, V, p.DV, p.T, p.BH, 64, 64) ||
      !encode_tmap_bf16_3d(&th, H, p.DV, p.T, p.BH, 64, kL))
    return cudaErrorInvalidValue;
  auto kern = tc_fused_kernel<DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, F::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = p.BH < sms ? p.BH : sms;
  kern<<<grid, kThreads, F::kSmem, st>>>(tq, tk, tv, th, p, g, C0, n0, C_T, n_T, m_T,
                                         static_cast<const __nv_bfloat16*>(V),
                                         static_cast<const __nv_bfloat16*>(K));
  return cudaGetLastError();
}

}  // namespace

bool tc_fused_supported(const Problem& p) {
  return p.DK == kDK && (p.DV == 64 || p.DV == 128) && p.L == kL && p.T > 0;
}

cudaError_t launch_tc_fused(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* C0, const float* n0, Gates g, void* H, float* C_T,
                            float* n_T, float* m_T, cudaStream_t st) {
  if (p.DV == 64) return launch_fused_t<64>(p, Q, K, V, C0, n0, g, H, C_T, n_T, m_T, st);
  if (p.DV == 128) return launch_fused_t<128>(p, Q, K, V, C0, n0, g, H, C_T, n_T, m_T, st);
  return cudaErrorNotSupported;
}

}  // namespace mlstm
