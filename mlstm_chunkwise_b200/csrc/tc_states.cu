// G2: inter-chunk state recurrence on tcgen05 (the recurrent half of the
// chunkwise mLSTM forward pass).
//
// flash-xlstm-exp 0.1.0 ("Upgrade roadmap" item 2) describes the recurrent
// kernel that materialises the intermediate chunk states in HBM between two
// launches; this is that kernel, written for sm_100a.  Per chunk k:
//
//   C_{k+1} = e^{g_k + m_k - m_{k+1}} C_k + K_k^T diag(w) V_k,
//   w_s     = s e^{g_k + acol_s - m_{k+1}},   n likewise with V -> 1,
//
// a dense rank-L update of the [DK, DV] state.  One CTA owns the whole DK
// extent (one or two 128-row halves, each a TMEM accumulator) and DVT columns
// of DV of one (b, h), for the whole sequence; the fp32 master state lives in
// TMEM and the MMA accumulates each chunk's update straight into it.  K and V
// stream in 64-token stages through a ring deep enough to keep ~190 KB of
// loads in flight.  Before each chunk the worker threads read the master (the
// state entering the chunk), write it out (fp32 and/or bf16 operand copy) and
// scale it by the decay.  The write-out goes through a 2 KB shared-memory tile
// per warp (32 state rows x 64 bytes) and a TMA store: a warp whose lanes each
// stored their own state row would touch 32 rows per instruction, and those
// scattered stores, not the MMAs, would then set the pace of the recurrence.
//
// When there are too few (b, h, d_v tile) units to fill the GPU, each one's
// chunk sequence is split into segments that run side by side (grid z).  A
// segment after the first starts from a zero state; since the recurrence is
// linear in the state, the state entering chunk k of segment s is
//   C_k = C_k(local) + e^{G(k0, k) + m_{k0} - m_k} C_{k0},   G = sum of g_j, j in [k0, k)
// and tc_states_fixup_kernel adds that term, with the states C_{k0} entering
// each segment obtained by a short scan over the segments' end states.
//
// For d_qk = 128 and value tiles of at most 128 columns the running state
// fits the workers' registers (a row and half of the tile's columns each, 64
// values at most): there the MMAs write each chunk's update U_k into one of
// two TMEM buffers, and per chunk the workers store the state from registers,
// then fold in the update, C_{k+1} = decay C_k + U_k, and release the buffer,
// so the MMAs of the next chunk wait for no decay of a TMEM master.
//
// Dominated states (g.dom[k] = t* >= 0, bf16 operand copy only): one token
// holds most of the state entering chunk k, so C_k ~ n_k v_{t*}^T and the
// output kernels' h = C^T q / |n^T q| would divide the independent bf16
// rounding of C by a small n^T q.  The copy then holds R_k = C_k - n*_k
// v_{t*}^T (fp32 subtraction, then rounding), n_states holds n*_k, and the
// output kernels add (n*_k^T q) v_{t*} back in fp32; n*_k = n_k - d_k, d_k the
// rounding residual of t*'s weighted key (dom_residual in tc.h).  Segments
// after the first subtract their local n; the fix-up adds the carried-in part
// the same way (the split is linear in (C, n)) and then d_k.
//
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 2..9 workers: per chunk, the store and decay of the master state; per
// stage, one pass that computes its token weights, accumulates the n-vector
// partial sums (fp32, from the unrounded products w_s k_s) and weights the K
// rows in place.  The first stage of chunk k is weighted before the workers
// wait for chunk k - 1's MMAs to drain, so that work leaves the critical path;
// the n-vector needs no MMA and is carried by the workers alone.
#include <cuda.h>

#include <cstring>

#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kWorkers = 256;
constexpr int kStageTok = 64;  // tokens per ring stage

template <int DK, int DVT>
struct SCfg {
  static_assert(DK == 128 || DK == 256, "DK of 128 or 256");
  static_assert(DVT == 64 || DVT == 128 || DVT == 256, "value tile");
  static constexpr int kHalves = DK / 128;
  static constexpr uint32_t kKBytes = kStageTok * DK * 2;   // DK/64 boxes of [64 tok x 64 dk]
  static constexpr uint32_t kVBytes = kStageTok * DVT * 2;  // DVT/64 boxes of [64 tok x 64 dv]
  static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
  static constexpr int kCC = DK / 8;             // 16-byte column chunks per token row
  static constexpr int kRowsPer = kStageTok * kCC / 256;  // rows per worker per stage
  static constexpr uint32_t kRedBytes = (256 / kCC) * DK * 4;  // n partials [row group][dk]
  // Two 32 x 64-byte store tiles per worker warp; the n-partial exchange
  // reuses the same bytes (it never overlaps a state store).
  static constexpr uint32_t kStgBytes = 8 * 2 * 2048;
  static_assert(kRedBytes <= kStgBytes, "n partials must fit in the store tiles");
  static constexpr uint32_t kBudget = 227 * 1024 - 1024 - 512 - DK * 4 - kStgBytes;
  static constexpr int kStagesFit = (int)(kBudget / kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static_assert(kStages >= 2, "ring too shallow");
  static constexpr uint32_t kOffStage = 0;
  static constexpr uint32_t kOffStg = kStages * kStageBytes;  // [8 warps][2][32 rows][64 B], 64 B swizzle
  static_assert(kOffStg % 1024 == 0, "store tiles must sit on a swizzle-atom boundary");
  static constexpr uint32_t kOffBar = kOffStg + kStgBytes;
  static constexpr uint32_t kOffSlot = kOffBar + 8 * 32;
  static constexpr uint32_t kOffNs = kOffSlot + 16;  // float[DK]: n entering the chunk
  static constexpr uint32_t kBytes = kOffNs + DK * 4;
  static constexpr uint32_t kSmem = kBytes + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  // d_qk = 128 with value tiles of at most 128 columns: the running state
  // lives in the workers' registers (64 values a thread at most) and the MMAs
  // write each chunk's update into one of two TMEM buffers (see the workers).
  static constexpr bool kReg = DK == 128 && DVT <= 128;
  static constexpr uint32_t kTmemCols =
      kReg ? 2 * DVT : ((kHalves * DVT) < 32 ? 32 : kHalves * DVT);
};

struct SBars {
  uint32_t a;
  __device__ __forceinline__ uint32_t full(int i) const { return a + 8 * i; }
  __device__ __forceinline__ uint32_t empty(int i) const { return a + 64 + 8 * i; }
  __device__ __forceinline__ uint32_t kready(int i) const { return a + 128 + 8 * i; }
  // per d_qk half: the state entering the chunk is ready (workers) / the
  // half's MMAs of the chunk have completed (commit)
  __device__ __forceinline__ uint32_t master(int hf) const { return a + 192 + 8 * hf; }
  __device__ __forceinline__ uint32_t chunk(int hf) const { return a + 208 + 8 * hf; }
  __device__ __forceinline__ uint32_t done() const { return a + 224; }
};

// x[e] -= n * v[e] for 8 consecutive value columns (v: bf16, 16-byte aligned).
__device__ __forceinline__ void deflate8(float (&x)[8], float n, const __nv_bfloat16* v) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(v));
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h2[e]);
    x[2 * e] = fmaf(-n, f.x, x[2 * e]);
    x[2 * e + 1] = fmaf(-n, f.y, x[2 * e + 1]);
  }
}

template <int DK, int DVT>
__global__ void __launch_bounds__(kThreads, 1)
tc_states_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_cs, Problem p, Gates g, const float* __restrict__ C0, const float* __restrict__ n0,
                 float* __restrict__ C_states, __nv_bfloat16* __restrict__ Cb,
                 float* __restrict__ n_states, float* __restrict__ C_T, float* __restrict__ n_T,
                 float* __restrict__ m_T, float* __restrict__ seg_C, float* __restrict__ seg_n,
                 const __nv_bfloat16* __restrict__ Vraw, const __nv_bfloat16* __restrict__ Kraw) {
  using S = SCfg<DK, DVT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const SBars bar{sbase + S::kOffBar};
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + S::kOffSlot);
  float* red_s = reinterpret_cast<float*>(smem + S::kOffStg);  // aliases the store tiles
  float* n_s = reinterpret_cast<float*>(smem + S::kOffNs);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dv0 = blockIdx.x * DVT, bh = blockIdx.y;
  const int L = p.L, NC = p.NC, DV = p.DV;
  const int stages_per_chunk = L / kStageTok;
  const long tpad = (long)NC * L;
  const bool n_owner = blockIdx.x == 0;
  // this CTA's segment of chunks [k0, k1)
  const int seg = blockIdx.z, n_seg = gridDim.z;
  const int ncs = (NC + n_seg - 1) / n_seg;
  const int k0 = seg * ncs, k1 = (k0 + ncs < NC) ? k0 + ncs : NC;
  const int nk = k1 - k0;  // >= 1 (the host picks n_seg so)
  const int s0 = k0 * stages_per_chunk;  // first ring stage, counted from token 0

  if (threadIdx.x == 0) {
    for (int i = 0; i < S::kStages; ++i) {
      mbar_init(bar.full(i), 1);
      mbar_init(bar.empty(i), 1);
      mbar_init(bar.kready(i), kWorkers);
    }
    for (int hf = 0; hf < 2; ++hf) {
      mbar_init(bar.master(hf), kWorkers);
      mbar_init(bar.chunk(hf), 1);
    }
    mbar_init(bar.done(), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------- TMA producer ----------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      bool ok = true;
      const int total = nk * stages_per_chunk;
      int issued = 0;
      for (int n = 0; n < total && ok; ++n) {
        const int s = n % S::kStages, u = n / S::kStages;
        if (u > 0) ok = mbar_wait(bar.empty(s), (u - 1) & 1, p, 1);
        if (!ok) break;
        const int tok0 = (s0 + n) * kStageTok;  // chunks are whole stages: k * L + j * 64
        const uint32_t st = sbase + S::kOffStage + (uint32_t)s * S::kStageBytes;
        mbar_expect_tx(bar.full(s), S::kStageBytes);
        for (int b = 0; b < DK / 64; ++b)
          tma_load_3d(st + b * 8192, &tm_k, b * 64, tok0, bh, bar.full(s));
        for (int b = 0; b < DVT / 64; ++b)
          tma_load_3d(st + S::kKBytes + b * 8192, &tm_v, dv0 + b * 64, tok0, bh, bar.full(s));
        issued = n + 1;
      }
      for (int q = (issued > S::kStages ? issued - S::kStages : 0); q < issued; ++q)
        mbar_wait(bar.full(q % S::kStages), (q / S::kStages) & 1, p, 13);
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, DVT, 1, 1);
      bool ok = true;
      int n = 0;
      if constexpr (S::kReg) {
        // chunk k's update U_k into buffer k mod 2, once the workers have
        // folded U_{k-2} (the release of that buffer)
        for (int k = 0; k < nk && ok; ++k) {
          const int buf = k & 1;
          if (k >= 2) ok = mbar_wait(bar.master(buf), ((k - 2) >> 1) & 1, p, 2);
          if (!ok) break;
          tc_fence_after();
          for (int j = 0; j < stages_per_chunk && ok; ++j, ++n) {
            const int s = n % S::kStages;
            ok = mbar_wait(bar.kready(s), (n / S::kStages) & 1, p, 3);
            if (!ok) break;
            tc_fence_after();
            const uint32_t st = sbase + S::kOffStage + (uint32_t)s * S::kStageBytes;
#pragma unroll
            for (int kk = 0; kk < kStageTok / 16; ++kk)
              mma_bf16_ss(tmem + (uint32_t)(buf * DVT), sdesc_sw128(st + kk * 2048, 8192, 1024),
                          sdesc_sw128(st + S::kKBytes + kk * 2048, 8192, 1024), idesc,
                          (j | kk) ? 1u : 0u);
            mma_commit(bar.empty(s));
          }
          mma_commit(bar.chunk(buf));
        }
      }
      for (int k = 0; k < nk && ok && !S::kReg; ++k) {
        for (int j = 0; j < stages_per_chunk && ok; ++j, ++n) {
          const int s = n % S::kStages;
          ok = mbar_wait(bar.kready(s), (n / S::kStages) & 1, p, 3);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = sbase + S::kOffStage + (uint32_t)s * S::kStageBytes;
#pragma unroll
          for (int hf = 0; hf < S::kHalves; ++hf) {
            // master(hf) completes once per chunk; its next completion needs
            // this half's MMAs of the chunk (chunk(hf), committed below).
            if (j == 0) {
              ok = ok && mbar_wait(bar.master(hf), k & 1, p, 2);
              tc_fence_after();
            }
            // A = (w K)^T: M = the 128 dk rows of this half (two 64-dk boxes,
            // MN-major), K = tokens.  B = V: N = the value columns (MN-major).
            const uint32_t a0 = st + hf * 16384;
#pragma unroll
            for (int kk = 0; kk < kStageTok / 16; ++kk)
              mma_bf16_ss(tmem + hf * DVT, sdesc_sw128(a0 + kk * 2048, 8192, 1024),
                          sdesc_sw128(st + S::kKBytes + kk * 2048, 8192, 1024), idesc, 1);
            // the half's last MMAs of the chunk: its boundary pass may start
            if (j == stages_per_chunk - 1) mma_commit(bar.chunk(hf));
          }
          mma_commit(bar.empty(s));
        }
      }
      mma_commit(bar.done());
    }
  } else {
    // ------------------------------ workers -------------------------------
    const int wt = threadIdx.x - 64;  // 0..255
    const int q = warp & 3;
    const int r = q * 32 + lane;      // TMEM lane = state row within a half
    const int ch = wt >> 7;           // which half of the value columns
    constexpr int kColsPer = DVT / 2;  // value columns per worker in the state passes
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const float* mchk = g.mchk + (long)bh * (NC + 1);
    const float* acol = g.acol + (long)bh * tpad + (long)s0 * kStageTok;  // -inf on padding
    // this warp's two store tiles
    uint8_t* stg = smem + S::kOffStg + (warp - 2) * 4096;
    const uint32_t stg_u = sbase + S::kOffStg + (uint32_t)(warp - 2) * 4096u;
    int n_st = 0;  // state stores issued by this warp (selects the tile)
    // n-vector: worker wt owns dk column wt (DK <= 256) for the running n.
    // The first value tile's CTA carries it and writes it out; the others
    // carry it only when the (b, h) has dominated chunks (their operand copy
    // then needs n).  need_n is uniform over the CTA, so are fold_n's barriers.
    const bool need_n = n_owner || (Cb && g.hdom && g.hdom[bh] != 0);
    const bool n_mine = need_n && wt < DK;
    const bool n_write = n_owner && n_mine;
    float nval = (n_mine && n0 && seg == 0) ? n0[(long)bh * DK + wt] : 0.f;
    // Stage pass mapping: 16-byte column chunk cc (8 dk columns) of token rows
    // rg * kRowsPer .. + kRowsPer - 1.
    const int cc = wt % S::kCC;
    const int rg = wt / S::kCC;
    float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // n partials, this chunk
    bool ok = true;

    // kReg: the running state, row r and this worker's column half
    float creg[S::kReg ? kColsPer : 1];
    if constexpr (S::kReg) {
#pragma unroll
      for (int j = 0; j < kColsPer; ++j)
        creg[j] = (C0 && seg == 0) ? C0[((long)bh * DK + r) * DV + dv0 + ch * kColsPer + j] : 0.f;
    }
    // master <- C0 (or zero): row r of each half, this worker's column half
    for (int hf = 0; hf < S::kHalves && !S::kReg; ++hf) {
      const int dk = hf * 128 + r;
      for (int c = 0; c < kColsPer; c += 32) {
        const int col = ch * kColsPer + c;
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = __float_as_uint((C0 && seg == 0) ? C0[((long)bh * DK + dk) * DV + dv0 + col + j]
                                                  : 0.f);
        tmem_st32(trow + hf * DVT + col, v);
      }
    }
    tmem_wait_st();

    // Adds this chunk's n partials into the running n (all workers take part).
    // red_s spans several warps' store tiles, so every warp's stores must have
    // read them first.
    auto fold_n = [&]() {
      if (need_n) {
        if (lane == 0) tma_store_wait_read_all();
        named_bar_sync(1, kWorkers);
#pragma unroll
        for (int e = 0; e < 8; ++e) red_s[rg * DK + cc * 8 + e] = part[e];
        named_bar_sync(1, kWorkers);
        if (n_mine) {
          float acc = 0.f;
          for (int q2 = 0; q2 < 256 / S::kCC; ++q2) acc += red_s[q2 * DK + wt];
          nval += acc;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) part[e] = 0.f;
    };

    // Column weights of this worker's rows, one stage ahead.
    constexpr int kRP = S::kRowsPer;
    static_assert(kRP % 4 == 0, "rows per worker in float4 groups");
    float4 a_nxt[kRP / 4];
    auto load_acol = [&](int stage_idx) {
#pragma unroll
      for (int i = 0; i < kRP / 4; ++i)
        a_nxt[i] = *reinterpret_cast<const float4*>(acol + (long)stage_idx * kStageTok +
                                                    rg * kRP + 4 * i);
    };
    load_acol(0);

    // One pass over ring stage n: weights w = s e^{g_k + acol - m_{k+1}} of its
    // rows, the n partials from the unrounded products w k (the normaliser
    // enters h through |n^T q|, which can cancel, so it must not see the bf16
    // rounding), and the K rows weighted in place for the rank-64 update.
    auto stage_pass = [&](int n, float gk, float m_out) {
      const int s = n % S::kStages;
      float a_cur[kRP];
#pragma unroll
      for (int i = 0; i < kRP / 4; ++i) {
        a_cur[4 * i] = a_nxt[i].x;
        a_cur[4 * i + 1] = a_nxt[i].y;
        a_cur[4 * i + 2] = a_nxt[i].z;
        a_cur[4 * i + 3] = a_nxt[i].w;
      }
      if (n + 1 < nk * stages_per_chunk) load_acol(n + 1);
      ok = ok && mbar_wait(bar.full(s), (n / S::kStages) & 1, p, 5);
      uint8_t* box = smem + S::kOffStage + (uint32_t)s * S::kStageBytes + (cc >> 3) * 8192;
#pragma unroll
      for (int rr = 0; rr < kRP; ++rr) {
        const int row = rg * kRP + rr;
        const float w = p.key_scale * expf(gk + a_cur[rr] - m_out);  // -inf -> 0
        uint4* ptr = reinterpret_cast<uint4*>(box + sw128_offset(row, cc & 7));
        uint4 u = *ptr;
        __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          part[2 * e] = fmaf(f.x, w, part[2 * e]);
          part[2 * e + 1] = fmaf(f.y, w, part[2 * e + 1]);
          h2[e] = __floats2bfloat162_rn(f.x * w, f.y * w);
        }
        *ptr = u;
      }
      fence_proxy_async_smem();
      mbar_arrive(bar.kready(s));
    };

    // Packs 16 words into this warp's next store tile and stores it with TMA
    // at (x, y, z) of `map`; the tile used two stores ago must have been read.
    auto store_tile = [&](const CUtensorMap* map, const uint32_t (&w16)[16], int x, int y, int z) {
      const uint32_t t = (uint32_t)(n_st & 1) * 2048u;
      if (lane == 0) tma_store_wait_read_1();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(stg + t + sw64_offset(lane, j)) =
            make_uint4(w16[4 * j], w16[4 * j + 1], w16[4 * j + 2], w16[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (MLSTM_IN_BOUNDS(p, x >= 0 && x + 16 <= DV && y >= 0 && y + 32 <= DK &&
                                   z >= 0 && z < p.BH * NC))
          tma_store_3d(map, stg_u + t, x, y, z);
        tma_store_commit();
      }
      ++n_st;
    };

    int n = 0;
    // the chunk's gate scalars, loaded one chunk ahead (they open every
    // iteration's dependence chain)
    float nx_m_in = mchk[k0], nx_m_out = mchk[k0 + 1], nx_gk = g.gtot[(long)bh * NC + k0];
    int nx_dom = g.dom ? g.dom[(long)bh * NC + k0] : -1;
    for (int k = k0; k < k1 && ok; ++k) {
      if (k > k0) fold_n();  // chunk k - 1's partials: every worker has passed its stages
      const float m_in = nx_m_in, m_out = nx_m_out, gk = nx_gk;
      // dominated state: the operand copy leaves as C - n* v_{t*}^T, n* = n - d
      // (the first segment; later ones get d from the fix-up)
      const int tdom = Cb ? nx_dom : -1;
      if (k + 1 < k1) {
        nx_m_in = m_out;
        nx_m_out = mchk[k + 2];
        nx_gk = g.gtot[(long)bh * NC + k + 1];
        if (g.dom) nx_dom = g.dom[(long)bh * NC + k + 1];
      }
      const float decay = expf(gk + m_in - m_out);
      const __nv_bfloat16* vstar =
          tdom >= 0 ? Vraw + ((long)bh * p.T + tdom) * DV + dv0 : nullptr;
      float nout = nval;
      if (tdom >= 0 && seg == 0 && n_mine) nout -= dom_residual(g, p, bh, k, tdom, wt, Kraw);
      if (n_write && MLSTM_IN_BOUNDS(p, (long)bh * NC + k < (long)p.BH * NC))
        n_states[((long)bh * NC + k) * DK + wt] = nout;
      if (n_mine) n_s[wt] = nout;  // read by the boundary pass after the barrier below
      nval *= decay;

      // The first stage of chunk k needs nothing from the MMAs.
      stage_pass(n++, gk, m_out);
      named_bar_sync(1, kWorkers);  // the n-partial reads are done: store tiles free

      if constexpr (S::kReg) {
        // The state entering chunk k is in registers: store it (this warp's
        // tiles, as below), weight the rest of the chunk's stages, then fold in
        // the chunk's update, C_{k+1} = decay C_k + U_k, and release its buffer.
        const int dk0 = q * 32;
        if (Cb) {
          for (int c = 0; c < kColsPer; c += 64) {
            const int col = ch * kColsPer + c;
            if (lane == 0) tma_store_wait_read_all();  // the previous tile has been read
            __syncwarp();
            if (vstar) {  // dominated: C - n* v_{t*}^T
              const float nrow = n_s[dk0 + lane];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = creg[c + 8 * j + e];
                deflate8(x, nrow, vstar + col + 8 * j);
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                               pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float* x = creg + c + 8 * j;
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                               pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const size_t off = cb_block_row((long)bh * NC + k, (dv0 + col) / 64, dk0, DK, DV / 64);
              if (MLSTM_IN_BOUNDS(p, off + 2048 <= (size_t)p.BH * NC * DK * DV))
                bulk_store(Cb + off, stg_u, 4096);
              tma_store_commit();
            }
          }
        } else if (C_states) {
          for (int c = 0; c < kColsPer; c += 32) {
            const int col = ch * kColsPer + c;
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(creg[c + j]);
            store_tile(&tm_cs, *reinterpret_cast<const uint32_t(*)[16]>(v), dv0 + col, dk0,
                       bh * NC + k);
            store_tile(&tm_cs, *reinterpret_cast<const uint32_t(*)[16]>(v + 16), dv0 + col + 16,
                       dk0, bh * NC + k);
          }
        }
        for (int j = 1; j < stages_per_chunk && ok; ++j) stage_pass(n++, gk, m_out);
        const int kl = k - k0, buf = kl & 1;
        ok = ok && mbar_wait(bar.chunk(buf), (kl >> 1) & 1, p, 4);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kColsPer; c += 32) {
          uint32_t v[32];
          tmem_ld32(trow + (uint32_t)(buf * DVT + ch * kColsPer + c), v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) creg[c + j] = fmaf(decay, creg[c + j], __uint_as_float(v[j]));
        }
        tc_fence_before();
        mbar_arrive(bar.master(buf));
      } else {
      // The state entering chunk k, half by half (row halves of d_qk): store it
      // (from this warp's tiles), then decay it in place.  Half hf waits only
      // for its own MMAs of chunk k - 1 and releases itself to the MMAs of
      // chunk k, so one half's MMAs overlap the other half's pass.
      for (int hf = 0; hf < S::kHalves && ok; ++hf) {
        if (k > k0) {
          ok = ok && mbar_wait(bar.chunk(hf), (k - k0 - 1) & 1, p, 4);
          tc_fence_after();
        }
        const int dk0 = hf * 128 + q * 32;  // first state row of this warp's lanes
        if (Cb) {
          // bf16 operand copy: one 32-row x 64-column tile per warp, already in
          // the swizzled block layout, leaves with one 4 KB bulk store.
          for (int c = 0; c < kColsPer; c += 64) {
            const int col = ch * kColsPer + c;
            if (lane == 0) tma_store_wait_read_all();  // the previous tile has been read
            __syncwarp();
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t v[32];
              tmem_ld32(trow + hf * DVT + col + 32 * hh, v);
              tmem_wait_ld();
              if (vstar) {  // dominated: C - n* v_{t*}^T
                const float nrow = n_s[dk0 + lane];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  float x[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(v[8 * j + e]);
                  deflate8(x, nrow, vstar + col + 32 * hh + 8 * j);
                  *reinterpret_cast<uint4*>(stg + lane * 128 +
                                            (((4 * hh + j) ^ (lane & 7)) << 4)) =
                      make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
                }
              } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  *reinterpret_cast<uint4*>(stg + lane * 128 +
                                            (((4 * hh + j) ^ (lane & 7)) << 4)) = make_uint4(
                      pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                      pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                      pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                      pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * decay);
              tmem_st32(trow + hf * DVT + col + 32 * hh, v);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const size_t off = cb_block_row((long)bh * NC + k, (dv0 + col) / 64, dk0, DK, DV / 64);
              if (MLSTM_IN_BOUNDS(p, off + 2048 <= (size_t)p.BH * NC * DK * DV))
                bulk_store(Cb + off, stg_u, 4096);
              tma_store_commit();
            }
          }
        } else {
          // fp32 states (or none): 16-column tiles through the tensor map
          for (int c = 0; c < kColsPer; c += 32) {
            const int col = ch * kColsPer + c;
            uint32_t v[32];
            tmem_ld32(trow + hf * DVT + col, v);
            tmem_wait_ld();
            if (C_states) {
              store_tile(&tm_cs, *reinterpret_cast<const uint32_t(*)[16]>(v), dv0 + col, dk0,
                         bh * NC + k);
              store_tile(&tm_cs, *reinterpret_cast<const uint32_t(*)[16]>(v + 16), dv0 + col + 16,
                         dk0, bh * NC + k);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * decay);
            tmem_st32(trow + hf * DVT + col, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar.master(hf));
      }

      for (int j = 1; j < stages_per_chunk && ok; ++j) stage_pass(n++, gk, m_out);
      }
    }
    // final state (fold the last chunk's n partials first); kReg: the last
    // fold has already waited for the last update
    for (int hf = 0; hf < S::kHalves && ok && !S::kReg; ++hf)
      ok = mbar_wait(bar.chunk(hf), (nk - 1) & 1, p, 6);
    tc_fence_after();
    fold_n();
    // The last segment's end state is C_T (local when segmented: the fix-up
    // adds the rest); an earlier segment's goes to its slot of seg_C / seg_n.
    const bool last_seg = seg == n_seg - 1;
    if (ok && (C_T || !last_seg)) {
      for (int hf = 0; hf < S::kHalves; ++hf) {
        const int dk = hf * 128 + r;
        for (int c = 0; c < kColsPer; c += 32) {
          const int col = ch * kColsPer + c;
          uint32_t v[32];
          if constexpr (S::kReg) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(creg[c + j]);
          } else {
            tmem_ld32(trow + hf * DVT + col, v);
            tmem_wait_ld();
          }
          float* row_dst =
              last_seg ? C_T + ((long)bh * DK + dk) * DV + dv0 + col
                       : seg_C + ((((long)bh * gridDim.x + blockIdx.x) * (n_seg - 1) + seg) * DK + dk) *
                                     DVT + col;
          float4* dst = reinterpret_cast<float4*>(row_dst);
          if (!MLSTM_IN_BOUNDS(p, dv0 + col + 32 <= DV && dk < DK)) continue;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
      }
    }
    if (n_write && last_seg && n_T) n_T[(long)bh * DK + wt] = nval;
    if (n_write && !last_seg) seg_n[((long)bh * (n_seg - 1) + seg) * DK + wt] = nval;
    if (m_T && last_seg && blockIdx.x == 0 && wt == 0) m_T[bh] = mchk[NC];
    if (lane == 0) tma_store_wait_all();  // the state stores have landed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(bar.done(), 0, p, 15);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

// Segment fix-up (see the top of this file).  A thread owns 8 consecutive
// value columns of one state row in one segment s >= 1 (grid z = s - 1): it
// forms the state entering the segment from the earlier segments' end states,
// then walks the segment's chunks adding a_k times it to each stored state,
//   a_k = e^{sum of e_j, j in [k0, k)},   e_j = g_j + m_j - m_{j+1} <= 0,
// the same per-chunk decay factors the recurrence applies.  kOperand: the
// states are the bf16 operand copy (block layout of cb_block_row), else fp32
// [b h k][DK][DV].  For a dominated chunk (dom[k] = t* >= 0) the copy holds
// C - n* v_{t*}^T and n_states n*, n* = n - d: the terms added are
// a_k (C_{k0} - n_{k0} v_{t*}^T) + d v_{t*}^T and a_k n_{k0} - d.
template <bool kOperand>
__global__ void __launch_bounds__(256)
tc_states_fixup_kernel(Problem p, Gates g, int DVT, const float* __restrict__ seg_C,
                       const float* __restrict__ seg_n, float* __restrict__ C_states,
                       __nv_bfloat16* __restrict__ Cb, float* __restrict__ n_states,
                       float* __restrict__ C_T, float* __restrict__ n_T,
                       const __nv_bfloat16* __restrict__ Vraw,
                       const __nv_bfloat16* __restrict__ Kraw) {
  const int DK = p.DK, DV = p.DV, NC = p.NC;
  const int bh = blockIdx.y, seg = blockIdx.z + 1, n_seg = gridDim.z + 1;
  const int ncs = (NC + n_seg - 1) / n_seg;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;  // < DK * DV / 8 (exact grid)
  int dk, col, vb = 0, jp = 0;
  if (kOperand) {
    jp = t & 7;  // 16-byte position within the 128-byte row
    dk = (t >> 3) % DK;
    vb = (t >> 3) / DK;
    col = vb * 64 + ((jp ^ (dk & 7)) << 3);
  } else {
    dk = t / (DV / 8);
    col = (t % (DV / 8)) * 8;
  }
  const bool n_thread = col == 0;  // one thread per state row carries n
  // with dominated chunks every thread needs its row's carried-in n
  const bool dominated = kOperand && g.hdom && g.hdom[bh] != 0;
  const float* gt = g.gtot + (long)bh * NC;
  const float* mc = g.mchk + (long)bh * (NC + 1);
  auto e_of = [&](int k) { return gt[k] + mc[k] - mc[k + 1]; };

  // The state entering segment seg: C_{k0(s+1)} = E_s + A_s C_{k0(s)}, with E_s
  // segment s's end state from a zero start (segment 0 started from C0).
  const int n_dvt = DV / DVT, dvt = col / DVT, cin = col % DVT;
  float cs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float ns = 0.f;
  for (int s = 0; s < seg; ++s) {
    float A = 0.f;  // multiplies a zero state when s == 0
    if (s > 0) {
      const int a0 = s * ncs, a1 = min(a0 + ncs, NC);
      float acc = 0.f;
      for (int k = a0 + lane; k < a1; k += 32) acc += e_of(k);
#pragma unroll
      for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      A = expf(acc);
    }
    const float4* e = reinterpret_cast<const float4*>(
        seg_C + ((((long)bh * n_dvt + dvt) * (n_seg - 1) + s) * DK + dk) * DVT + cin);
    const float4 e0 = e[0], e1 = e[1];
    const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) cs[i] = fmaf(A, cs[i], ev[i]);
    if (n_thread || dominated) ns = fmaf(A, ns, seg_n[((long)bh * (n_seg - 1) + s) * DK + dk]);
  }

  const int k0 = seg * ncs, k1 = min(k0 + ncs, NC);
  float lg = 0.f;  // sum of e_j over [k0, kb)
  for (int kb = k0; kb < k1; kb += 32) {
    // coefficients of chunks kb .. kb + 31: an exclusive warp scan of e
    const int kl = kb + lane;
    const float x = kl < k1 ? e_of(kl) : 0.f;
    float inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    float exc = __shfl_up_sync(0xffffffffu, inc, 1);
    if (lane == 0) exc = 0.f;
    const float a_lane = expf(lg + exc);
    const int td_lane = (dominated && kl < k1) ? g.dom[(long)bh * NC + kl] : -1;
    const bool any_td = dominated && __any_sync(0xffffffffu, td_lane >= 0);
    lg += __shfl_sync(0xffffffffu, inc, 31);
    const int nb = min(32, k1 - kb);
    for (int c0 = 0; c0 < nb; c0 += 4) {
      // four chunks at a time: loads first, so that they overlap
      constexpr int kB = 4;
      float a[kB];
      int tds[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        a[u] = __shfl_sync(0xffffffffu, a_lane, (c0 + u) & 31);
        tds[u] = -1;
      }
      if (any_td) {
#pragma unroll
        for (int u = 0; u < kB; ++u) tds[u] = __shfl_sync(0xffffffffu, td_lane, (c0 + u) & 31);
      }
      if (kOperand) {
        uint4 v[kB];
        __nv_bfloat16* ptr[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (c0 + u < nb) {
            const size_t off = cb_block_row((long)bh * NC + kb + c0 + u, vb, dk, DK, DV / 64) + jp * 8;
            // out of bounds (debug builds): neither read nor written back
            ptr[u] = MLSTM_IN_BOUNDS(p, off + 8 <= (size_t)p.BH * NC * DK * DV) ? Cb + off : nullptr;
            if (ptr[u]) v[u] = *reinterpret_cast<const uint4*>(ptr[u]);
          }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (c0 + u < nb && ptr[u]) {
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&v[u]);
            if (any_td && tds[u] >= 0) {
              const int td = tds[u];
              float add[8], res[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                add[i] = cs[i];
                res[i] = 0.f;
              }
              const __nv_bfloat16* vs = Vraw + ((long)bh * p.T + td) * DV + col;
              deflate8(add, ns, vs);
              deflate8(res, -dom_residual(g, p, bh, kb + c0 + u, td, dk, Kraw), vs);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                h2[e] = __floats2bfloat162_rn(fmaf(a[u], add[2 * e], f.x) + res[2 * e],
                                              fmaf(a[u], add[2 * e + 1], f.y) + res[2 * e + 1]);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                h2[e] = __floats2bfloat162_rn(fmaf(a[u], cs[2 * e], f.x),
                                              fmaf(a[u], cs[2 * e + 1], f.y));
              }
            }
            *reinterpret_cast<uint4*>(ptr[u]) = v[u];
          }
        }
      } else {
        float4 v[kB][2];
        float* ptr[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (c0 + u < nb) {
            ptr[u] = C_states + (((long)bh * NC + kb + c0 + u) * DK + dk) * DV + col;
            v[u][0] = reinterpret_cast<const float4*>(ptr[u])[0];
            v[u][1] = reinterpret_cast<const float4*>(ptr[u])[1];
          }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (c0 + u < nb) {
            float* f = reinterpret_cast<float*>(&v[u][0]);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = fmaf(a[u], cs[i], f[i]);
            reinterpret_cast<float4*>(ptr[u])[0] = v[u][0];
            reinterpret_cast<float4*>(ptr[u])[1] = v[u][1];
          }
        }
      }
      if (n_thread) {
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (c0 + u < nb) {
            const int kc = kb + c0 + u;
            const int td = tds[u];
            const float d = td >= 0 ? dom_residual(g, p, bh, kc, td, dk, Kraw) : 0.f;
            n_states[((long)bh * NC + kc) * DK + dk] += a[u] * ns - d;
          }
        }
      }
    }
  }
  // the last segment's end state is the final state
  if (seg == n_seg - 1) {
    const float aT = expf(lg);
    if (C_T) {
      float4* d = reinterpret_cast<float4*>(C_T + ((long)bh * DK + dk) * DV + col);
      float4 d0 = d[0], d1 = d[1];
      d0 = make_float4(fmaf(aT, cs[0], d0.x), fmaf(aT, cs[1], d0.y), fmaf(aT, cs[2], d0.z),
                       fmaf(aT, cs[3], d0.w));
      d1 = make_float4(fmaf(aT, cs[4], d1.x), fmaf(aT, cs[5], d1.y), fmaf(aT, cs[6], d1.z),
                       fmaf(aT, cs[7], d1.w));
      d[0] = d0;
      d[1] = d1;
    }
    if (n_thread && n_T) n_T[(long)bh * DK + dk] += aT * ns;
  }
}

template <int DK, int DVT>
cudaError_t launch_states_t(const Problem& p, const void* K, const void* V, const float* C0,
                            const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                            float* n_states, float* C_T, float* n_T, float* m_T, float* seg_ws,
                            cudaStream_t st) {
  using S = SCfg<DK, DVT>;
  CUtensorMap tk, tv, tcs;
  memset(&tcs, 0, sizeof(tcs));
  // One of the two state copies per launch (they share the store tiles); the
  // operand copy is written in 64-column tiles, two per worker row at least.
  if (C_states && Cb) return cudaErrorInvalidValue;
  if (Cb && (DVT < 128 || p.DV % 64 != 0)) return cudaErrorNotSupported;
  const uint64_t n_boxes = (uint64_t)p.BH * p.NC;  // state tiles [DK][DV] per (b, h, chunk)
  if (!encode_tmap_bf16_3d(&tk, K, p.DK, p.T, p.BH, 64, kStageTok) ||
      !encode_tmap_bf16_3d(&tv, V, p.DV, p.T, p.BH, 64, kStageTok) ||
      (C_states && !encode_tmap_3d(&tcs, C_states, 4, p.DV, p.DK, n_boxes, 16, 32, 64)))
    return cudaErrorInvalidValue;
  auto kern = tc_states_kernel<DK, DVT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  const int n_seg = tc_states_segments(p);
  if (n_seg > 1 && !seg_ws) return cudaErrorInvalidValue;
  float* seg_C = seg_ws;
  float* seg_n = n_seg > 1 ? seg_ws + (size_t)p.BH * (n_seg - 1) * p.DK * p.DV : nullptr;
  dim3 grid(p.DV / DVT, p.BH, n_seg);
  // the dominance marks apply to the bf16 operand copy only
  Gates gk = g;
  if (!Cb) gk.dom = nullptr;
  const __nv_bfloat16* Vraw = static_cast<const __nv_bfloat16*>(V);
  const __nv_bfloat16* Kraw = static_cast<const __nv_bfloat16*>(K);
  kern<<<grid, kThreads, S::kSmem, st>>>(tk, tv, tcs, p, gk, C0, n0, C_states, Cb, n_states, C_T,
                                         n_T, m_T, seg_C, seg_n, Vraw, Kraw);
  e = cudaGetLastError();
  if (e != cudaSuccess || n_seg == 1) return e;
  dim3 fgrid(p.DK * p.DV / 8 / 256, p.BH, n_seg - 1);
  if (Cb)
    tc_states_fixup_kernel<true><<<fgrid, 256, 0, st>>>(p, gk, DVT, seg_C, seg_n, C_states, Cb,
                                                        n_states, C_T, n_T, Vraw, Kraw);
  else
    tc_states_fixup_kernel<false><<<fgrid, 256, 0, st>>>(p, gk, DVT, seg_C, seg_n, C_states, Cb,
                                                         n_states, C_T, n_T, Vraw, Kraw);
  return cudaGetLastError();
}

}  // namespace

bool tc_states_supported(const Problem& p) {
  const bool dv_ok = p.DV == 64 || p.DV == 128 || p.DV % 256 == 0;
  return (p.DK == 128 || p.DK == 256) && dv_ok && p.DV <= 1024 && p.L % kStageTok == 0 &&
         p.L <= 1024 && p.T > 0;
}

int tc_states_dvt(const Problem& p) { return p.DV >= 256 ? 256 : p.DV; }

int tc_states_segments(const Problem& p) {
  // Split chunk sequences only while the (b, h, d_v tile) units leave SMs of a
  // 148-SM B200 idle; at most 8 segments, each at least 2 chunks long.  A
  // function of the shape alone, so the workspace the host sizes always fits.
  constexpr int kSMs = 148, kMaxSegments = 8;
  const int units = p.BH * (p.DV / tc_states_dvt(p));
  int s = kSMs / units;
  if (s > kMaxSegments) s = kMaxSegments;
  if (s > p.NC / 2) s = p.NC / 2;
  // segment s covers chunks [s * ncs, min((s + 1) * ncs, NC)), ncs = ceil(NC / n):
  // none may be empty
  while (s > 1 && (s - 1) * ((p.NC + s - 1) / s) >= p.NC) --s;
  return s < 1 ? 1 : s;
}

size_t tc_states_segment_floats(const Problem& p) {
  const size_t extra = (size_t)tc_states_segments(p) - 1;
  return extra * p.BH * p.DK * ((size_t)p.DV + 1);
}

cudaError_t launch_tc_states_impl(const Problem& p, const void* K, const void* V, const float* C0,
                                  const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                                  float* n_states, float* C_T, float* n_T, float* m_T,
                                  float* seg_ws, cudaStream_t st) {
  const int dvt = tc_states_dvt(p);
#define MLSTM_ST_CASE(dk, dvt_)                                                                  \
  if (p.DK == dk && dvt == dvt_)                                                                 \
    return launch_states_t<dk, dvt_>(p, K, V, C0, n0, g, C_states, Cb, n_states, C_T, n_T, m_T, \
                                     seg_ws, st);
  MLSTM_ST_CASE(128, 64)
  MLSTM_ST_CASE(128, 128)
  MLSTM_ST_CASE(128, 256)
  MLSTM_ST_CASE(256, 64)
  MLSTM_ST_CASE(256, 128)
  MLSTM_ST_CASE(256, 256)
#undef MLSTM_ST_CASE
  return cudaErrorNotSupported;
}

}  // namespace mlstm
