// G3: intra-chunk TFLA kernel on tcgen05 (the parallel half of the chunkwise
// mLSTM forward pass).
//
// "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
// (abstract): the intra-chunk part is tiled a second time, over query and
// key/value blocks, so the chunk size is not tied to the tile size.  Here one
// CTA owns 128 query rows (one L_Q tile) of one chunk and DVT value columns of
// one (b, h); it walks the L_KV = 128 key/value tiles of the chunk up to the
// diagonal.  For row r (token t) of chunk k with mu_r = max(m_k, amax_r):
//
//   O_r   = e^{m_k - mu_r} C_k^T q_r  +  sum_{s<=r} P_rs v_s
//   P_rs  = (s q_r.k_s) e^{acol_s - mu_r}                (0 above the diagonal)
//   den_r = e^{m_k - mu_r} n_k.q_r    +  sum_{s<=r} P_rs
//   h_r   = O_r / max(|den_r|, e^{-(bcum_r + mu_r)})
//
// Roles (192 threads):
//   warp 0      TMA producer: Q tile once, then K / C / V slabs through a ring
//   warp 1      TMEM owner and single-thread MMA issuer
//   warps 2..5  one thread per query row (= TMEM lane): gating of S into P,
//               rescaling of the inter-chunk term, row sums, epilogue.
// TMEM (512 columns): O accumulator [128 x DVT] at column 0, two S buffers
// [128 x 128] at columns 256 and 384.  Shared memory: Q tile (DK/64 swizzled
// slabs), a ring of NSTAGE slabs, the bf16 P tile (A operand of P.V).
// MMA order: S_0, Q.C, { S_i, P_{i-1}.V_{i-1} }, P_last.V_last.
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kQT = 128;  // query rows per CTA
constexpr int kKT = 128;  // key/value rows per intra tile
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 256, kColS1 = 384;
constexpr int kMaxL = 1024;  // largest chunk this kernel handles

template <int DK, int DVT>
struct Cfg {
  static constexpr int kSlabsK = DK / 64;
  static constexpr uint32_t kQBytes = kQT * DK * 2;
  static constexpr uint32_t kKSlabBytes = kKT * 128;        // 128 rows x 64 bf16
  static constexpr uint32_t kMNSlabBytes = (DVT / 64) * 8192;  // 64 rows x DVT bf16
  static constexpr uint32_t kStageBytes = kKSlabBytes > kMNSlabBytes ? kKSlabBytes : kMNSlabBytes;
  static constexpr int kStages = kStageBytes >= 32768 ? 3 : 4;
  static constexpr uint32_t kPBytes = kQT * kKT * 2;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffStage = kOffQ + kQBytes;
  static constexpr uint32_t kOffP = kOffStage + kStages * kStageBytes;
  static constexpr uint32_t kOffAcol = kOffP + kPBytes;          // float[kMaxL]
  static constexpr uint32_t kOffN = kOffAcol + kMaxL * 4;        // float[DK]
  static constexpr uint32_t kOffBar = kOffN + DK * 4;            // barriers
  static constexpr int kNumBars = 2 * 4 + 1 + 2 + 2 + 1 + 1 + 1 + 1;
  static constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kOffTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;  // slack for 1024-byte alignment
};

struct Bars {
  uint32_t full[4], empty[4], q_full, s_full[2], s_empty[2], inter_done, p_full, p_empty, o_done;
};

template <int DK, int DVT>
__device__ __forceinline__ Bars make_bars(uint32_t base) {
  Bars b;
  uint32_t a = base + Cfg<DK, DVT>::kOffBar;
  for (int i = 0; i < 4; ++i) b.full[i] = a + 8 * i;
  for (int i = 0; i < 4; ++i) b.empty[i] = a + 32 + 8 * i;
  b.q_full = a + 64;
  b.s_full[0] = a + 72;
  b.s_full[1] = a + 80;
  b.s_empty[0] = a + 88;
  b.s_empty[1] = a + 96;
  b.inter_done = a + 104;
  b.p_full = a + 112;
  b.p_empty = a + 120;
  b.o_done = a + 128;
  return b;
}

template <int DK, int DVT>
__global__ void __launch_bounds__(kThreads, 1)
tc_parallel_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_c,
                   Problem p, Gates g, const float* __restrict__ n_states,
                   __nv_bfloat16* __restrict__ H, float* __restrict__ n_out,
                   float* __restrict__ m_out) {
  using C = Cfg<DK, DVT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const Bars bar = make_bars<DK, DVT>(sbase);
  float* acol_s = reinterpret_cast<float*>(smem + C::kOffAcol);
  float* n_s = reinterpret_cast<float*>(smem + C::kOffN);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dv0 = blockIdx.x * DVT;
  const int t0 = blockIdx.y * kQT;
  const int bh = blockIdx.z;
  const int L = p.L;
  const int k = t0 / L;
  const int c0 = k * L;                    // first token of the chunk
  const int n_kv = (t0 - c0) / kKT + 1;    // key/value tiles up to the diagonal
  const long tpad = (long)p.NC * L;
  const float m_in = g.mchk[(long)bh * (p.NC + 1) + k];

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar.full[i], 1);
      mbar_init(bar.empty[i], 1);
    }
    mbar_init(bar.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar.s_full[i], 1);
      mbar_init(bar.s_empty[i], 128);
    }
    mbar_init(bar.inter_done, 1);
    mbar_init(bar.p_full, 128);
    mbar_init(bar.p_empty, 1);
    mbar_init(bar.o_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  // Column weights of the chunk prefix [c0, t0 + 128), pre-multiplied by log2(e).
  for (int j = threadIdx.x; j < n_kv * kKT; j += kThreads)
    acol_s[j] = g.acol[(long)bh * tpad + c0 + j] * 1.4426950408889634f;
  for (int j = threadIdx.x; j < DK; j += kThreads)
    n_s[j] = n_states[((long)bh * p.NC + k) * DK + j];
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
      tma_prefetch_desc(&tm_c);
      mbar_expect_tx(bar.q_full, C::kQBytes);
      for (int c = 0; c < C::kSlabsK; ++c)
        tma_load_3d(sbase + C::kOffQ + c * 16384, &tm_q, c * 64, t0, bh, bar.q_full);
      int slab = 0;
      bool ok = true;
      auto next_stage = [&](uint32_t bytes) -> uint32_t {
        const int s = slab % C::kStages, u = slab / C::kStages;
        if (u > 0) ok = ok && mbar_wait(bar.empty[s], (u - 1) & 1, p);
        mbar_expect_tx(bar.full[s], bytes);
        ++slab;
        return (uint32_t)s;
      };
      auto load_k = [&](int i) {
        for (int c = 0; c < C::kSlabsK && ok; ++c) {
          const uint32_t s = next_stage(C::kKSlabBytes);
          tma_load_3d(sbase + C::kOffStage + s * C::kStageBytes, &tm_k, c * 64, c0 + i * kKT, bh,
                      bar.full[s]);
        }
      };
      auto load_v = [&](int i) {
        for (int v = 0; v < 2 && ok; ++v) {
          const uint32_t s = next_stage(C::kMNSlabBytes);
          for (int b = 0; b < DVT / 64; ++b)
            tma_load_3d(sbase + C::kOffStage + s * C::kStageBytes + b * 8192, &tm_v, dv0 + b * 64,
                        c0 + i * kKT + v * 64, bh, bar.full[s]);
        }
      };
      load_k(0);
      for (int c = 0; c < C::kSlabsK && ok; ++c) {
        const uint32_t s = next_stage(C::kMNSlabBytes);
        for (int b = 0; b < DVT / 64; ++b)
          tma_load_3d(sbase + C::kOffStage + s * C::kStageBytes + b * 8192, &tm_c, dv0 + b * 64,
                      c * 64, bh * p.NC + k, bar.full[s]);
      }
      for (int i = 1; i < n_kv && ok; ++i) {
        load_k(i);
        load_v(i - 1);
      }
      load_v(n_kv - 1);
      // Drain: every issued stage must have landed before the CTA may exit.
      for (int q = (slab > C::kStages ? slab - C::kStages : 0); q < slab; ++q)
        mbar_wait(bar.full[q % C::kStages], (q / C::kStages) & 1, p);
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, kKT, 0, 0);
      constexpr uint32_t idO = idesc_bf16(128, DVT, 0, 1);
      bool ok = mbar_wait(bar.q_full, 0, p);
      int slab = 0;
      auto take = [&]() -> uint32_t {
        const int s = slab % C::kStages, u = slab / C::kStages;
        ok = ok && mbar_wait(bar.full[s], u & 1, p);
        tc_fence_after();
        ++slab;
        return (uint32_t)s;
      };
      auto mma_s = [&](int i) {
        const int buf = i & 1;
        if (i >= 2) ok = ok && mbar_wait(bar.s_empty[buf], ((i >> 1) - 1) & 1, p);
        tc_fence_after();
        const uint32_t d = tmem + (buf ? kColS1 : kColS0);
        for (int c = 0; c < C::kSlabsK; ++c) {
          const uint32_t s = take();
          if (!ok) return;
          const uint32_t a0 = sbase + C::kOffQ + c * 16384;
          const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(d, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                        idS, (c | kk) != 0);
          mma_commit(bar.empty[s]);
        }
        mma_commit(bar.s_full[buf]);
      };
      auto mma_pv = [&](int i) {
        ok = ok && mbar_wait(bar.p_full, i & 1, p);
        tc_fence_after();
        for (int v = 0; v < 2; ++v) {
          const uint32_t s = take();
          if (!ok) return;
          const uint32_t a0 = sbase + C::kOffP + v * 16384;
          const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + kColO, sdesc_sw128(a0 + kk * 32, 16, 1024),
                        sdesc_sw128(b0 + kk * 2048, 8192, 1024), idO, 1);
          mma_commit(bar.empty[s]);
        }
        mma_commit(bar.p_empty);
      };
      if (ok) mma_s(0);
      for (int c = 0; c < C::kSlabsK && ok; ++c) {  // inter-chunk term Q.C_k
        const uint32_t s = take();
        if (!ok) break;
        const uint32_t a0 = sbase + C::kOffQ + c * 16384;
        const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem + kColO, sdesc_sw128(a0 + kk * 32, 16, 1024),
                      sdesc_sw128(b0 + kk * 2048, 8192, 1024), idO, (c | kk) != 0);
        mma_commit(bar.empty[s]);
      }
      if (ok) mma_commit(bar.inter_done);
      for (int i = 1; i < n_kv && ok; ++i) {
        mma_s(i);
        if (ok) mma_pv(i - 1);
      }
      if (ok) mma_pv(n_kv - 1);
      mma_commit(bar.o_done);  // also orders every MMA above before teardown
      mbar_wait(bar.o_done, 0, p);
    }
  } else {
    // ------------------- gating / softmax / epilogue ----------------------
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;         // query row in the tile = TMEM lane
    const int t = t0 + r;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const float amax = g.amax[(long)bh * tpad + t];
    const float bc = g.bcum[(long)bh * tpad + t];
    const float mu = fmaxf(m_in, amax);
    const float mu2 = mu * 1.4426950408889634f;
    const float f_inter = expf(m_in - mu);
    const float ks = p.key_scale;
    bool ok = true;

    // den_inter = q_r . n_k from the swizzled Q tile.
    ok = mbar_wait(bar.q_full, 0, p);
    float dn = 0.f;
    for (int c = 0; c < C::kSlabsK; ++c) {
      const uint8_t* slab_ptr = smem + C::kOffQ + c * 16384;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(slab_ptr + sw128_offset(r, j));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f2 = __bfloat1622float2(h2[e]);
          dn = fmaf(f2.x, n_s[c * 64 + j * 8 + 2 * e], dn);
          dn = fmaf(f2.y, n_s[c * 64 + j * 8 + 2 * e + 1], dn);
        }
      }
    }
    float den = f_inter * dn;

    // Rescale the inter-chunk term of the accumulator to the row frame mu_r.
    ok = ok && mbar_wait(bar.inter_done, 0, p);
    tc_fence_after();
    if (ok) {
      for (int c = 0; c < DVT; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + kColO + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f_inter);
        tmem_st32(trow + kColO + c, v);
      }
      tmem_wait_st();
    }

    for (int i = 0; i < n_kv; ++i) {
      const int buf = i & 1;
      ok = ok && mbar_wait(bar.s_full[buf], (i >> 1) & 1, p);
      if (i >= 1) ok = ok && mbar_wait(bar.p_empty, (i - 1) & 1, p);
      tc_fence_after();
      const bool diag = (i == n_kv - 1);
      const uint32_t scol = buf ? kColS1 : kColS0;
      float rs = 0.f;
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < kKT; c += 32) {
          uint32_t v[32];
          tmem_ld32(trow + scol + c, v);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int s0 = c + j;
            float pa = __uint_as_float(v[j]) * ks * ex2_approx(acol_s[i * kKT + s0] - mu2);
            float pb = __uint_as_float(v[j + 1]) * ks * ex2_approx(acol_s[i * kKT + s0 + 1] - mu2);
            if (diag && s0 > r) pa = 0.f;
            if (diag && s0 + 1 > r) pb = 0.f;
            rs += pa + pb;
            pk[j >> 1] = pack_bf16x2(pa, pb);
          }
          // 32 columns = 64 bytes = 4 chunks of the swizzled 128-byte row.
          uint8_t* prow = smem + C::kOffP + (c >> 6) * 16384;
          const int cb = (c & 63) >> 3;  // first 16-byte chunk within the row
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(prow + sw128_offset(r, cb + j)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      den += rs;
      tc_fence_before();
      mbar_arrive(bar.s_empty[buf]);
      fence_proxy_async_smem();
      mbar_arrive(bar.p_full);
    }

    // Epilogue: h = O / max(|den|, e^{-m_r}).
    ok = ok && mbar_wait(bar.o_done, 0, p);
    tc_fence_after();
    const float mr = bc + mu;
    const float denom = fmaxf(fabsf(den), expf(-mr));
    const float inv = 1.f / denom;
    if (ok) {
      for (int c = 0; c < DVT; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + kColO + c, v);
        tmem_wait_ld();
        if (t < p.T) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2)
            pk[j >> 1] = pack_bf16x2(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(H + ((long)bh * p.T + t) * p.DV + dv0 + c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
    }
    if (t < p.T && blockIdx.x == 0) {
      if (n_out) n_out[(long)bh * p.T + t] = denom;
      if (m_out) m_out[(long)bh * p.T + t] = mr;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DK, int DVT>
cudaError_t launch_parallel_t(const Problem& p, const void* Q, const void* K, const void* V,
                              Gates g, const __nv_bfloat16* Cb, const float* n_states, void* H,
                              float* n_out, float* m_out, cudaStream_t st) {
  using C = Cfg<DK, DVT>;
  CUtensorMap tq, tk, tv, tcm;
  if (!encode_tmap_bf16_3d(&tq, Q, p.DK, p.T, p.BH, 64, kQT) ||
      !encode_tmap_bf16_3d(&tk, K, p.DK, p.T, p.BH, 64, kKT) ||
      !encode_tmap_bf16_3d(&tv, V, p.DV, p.T, p.BH, 64, 64) ||
      !encode_tmap_bf16_3d(&tcm, Cb, p.DV, p.DK, (uint64_t)p.BH * p.NC, 64, 64))
    return cudaErrorInvalidValue;
  auto kern = tc_parallel_kernel<DK, DVT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.DV / DVT, (p.T + kQT - 1) / kQT, p.BH);
  kern<<<grid, kThreads, C::kSmem, st>>>(tq, tk, tv, tcm, p, g, n_states,
                                         static_cast<__nv_bfloat16*>(H), n_out, m_out);
  return cudaGetLastError();
}

}  // namespace

bool tc_parallel_supported(const Problem& p) {
  const bool dk_ok = p.DK == 64 || p.DK == 128 || p.DK == 256;
  const bool dv_ok = p.DV == 64 || p.DV == 128 || p.DV % 256 == 0;
  return dk_ok && dv_ok && p.DV <= 1024 && p.L % kKT == 0 && p.L <= kMaxL && p.T > 0;
}

cudaError_t launch_tc_parallel_bf16states(const Problem& p, const void* Q, const void* K,
                                          const void* V, Gates g, const __nv_bfloat16* Cb,
                                          const float* n_states, void* H, float* n_out,
                                          float* m_out, cudaStream_t st) {
  const int dvt = p.DV >= 256 ? 256 : p.DV;
#define MLSTM_PAR_CASE(dk, dvt_)                                                                \
  if (p.DK == dk && dvt == dvt_)                                                                \
    return launch_parallel_t<dk, dvt_>(p, Q, K, V, g, Cb, n_states, H, n_out, m_out, st);
  MLSTM_PAR_CASE(64, 64)
  MLSTM_PAR_CASE(64, 128)
  MLSTM_PAR_CASE(64, 256)
  MLSTM_PAR_CASE(128, 64)
  MLSTM_PAR_CASE(128, 128)
  MLSTM_PAR_CASE(128, 256)
  MLSTM_PAR_CASE(256, 64)
  MLSTM_PAR_CASE(256, 128)
  MLSTM_PAR_CASE(256, 256)
#undef MLSTM_PAR_CASE
  return cudaErrorNotSupported;
}

}  // namespace mlstm
