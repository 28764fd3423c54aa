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
// a dense rank-L update of the [DK, DV] state.  One CTA owns 128 rows of DK
// (TMEM lanes) and DVT columns of DV of one (b, h); the fp32 master state
// lives in TMEM for the whole sequence and the MMA accumulates each chunk's
// update straight into it.  Before each chunk the row threads read the master
// (the state entering the chunk), write it out (fp32 and/or bf16 operand
// copy), and scale it by the decay.
//
// Roles (192 threads): warp 0 TMA producer (one 128-token K/V tile at a time),
// warp 1 TMEM owner + MMA issuer, warps 2..5 one thread per state row: the
// decay pass, the n-vector column sums (fp32, from the unrounded products
// w_s k_s), the per-token weights (applied to the K tile in place, row by row)
// and the stores.
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kRows = 128;  // DK rows per CTA
constexpr int kKT = 128;    // tokens per tile

template <int DVT>
struct SCfg {
  static constexpr uint32_t kKBytes = kKT * kRows * 2;     // 2 boxes of [128 tokens x 64 dk]
  static constexpr uint32_t kVBytes = kKT * DVT * 2;       // DVT/64 boxes of [128 x 64 dv]
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffV = kKBytes;
  static constexpr uint32_t kOffW = kOffV + kVBytes;       // float[128] token weights
  static constexpr uint32_t kOffBar = kOffW + kKT * 4;
  static constexpr uint32_t kOffSlot = kOffBar + 8 * 8;
  static constexpr uint32_t kBytes = kOffSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;
  static constexpr uint32_t kTmemCols = DVT < 32 ? 32 : DVT;
};

template <int DVT>
__global__ void __launch_bounds__(kThreads)
tc_states_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 Problem p, Gates g, const float* __restrict__ C0, const float* __restrict__ n0,
                 float* __restrict__ C_states, __nv_bfloat16* __restrict__ Cb,
                 float* __restrict__ n_states, float* __restrict__ C_T, float* __restrict__ n_T,
                 float* __restrict__ m_T) {
  using S = SCfg<DVT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t b_full = sbase + S::kOffBar, b_kready = b_full + 8, b_empty = b_full + 16,
                 b_master = b_full + 24, b_chunk = b_full + 32, b_done = b_full + 40;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + S::kOffSlot);
  float* w_s = reinterpret_cast<float*>(smem + S::kOffW);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dv0 = blockIdx.x * DVT, dk0 = blockIdx.y * kRows, bh = blockIdx.z;
  const int L = p.L, NC = p.NC, T = p.T, DK = p.DK, DV = p.DV;
  const int tiles = L / kKT;
  const long tpad = (long)NC * L;
  const bool n_owner = blockIdx.x == 0;

  if (threadIdx.x == 0) {
    mbar_init(b_full, 1);
    mbar_init(b_kready, 128);
    mbar_init(b_empty, 1);
    mbar_init(b_master, 128);
    mbar_init(b_chunk, 1);
    mbar_init(b_done, 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      bool ok = true;
      int n = 0;
      for (int k = 0; k < NC && ok; ++k) {
        for (int i = 0; i < tiles && ok; ++i, ++n) {
          if (n > 0) ok = mbar_wait(b_empty, (n - 1) & 1, p);
          if (!ok) break;
          const int kv0 = k * L + i * kKT;
          mbar_expect_tx(b_full, S::kKBytes + S::kVBytes);
          for (int b = 0; b < 2; ++b)
            tma_load_3d(sbase + S::kOffK + b * 16384, &tm_k, dk0 + b * 64, kv0, bh, b_full);
          for (int b = 0; b < DVT / 64; ++b)
            tma_load_3d(sbase + S::kOffV + b * 16384, &tm_v, dv0 + b * 64, kv0, bh, b_full);
        }
      }
      if (n > 0) mbar_wait(b_full, (n - 1) & 1, p);  // last load landed before exit
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, DVT, 1, 1);
      bool ok = true;
      int n = 0;
      for (int k = 0; k < NC && ok; ++k) {
        ok = mbar_wait(b_master, k & 1, p);
        for (int i = 0; i < tiles && ok; ++i, ++n) {
          ok = mbar_wait(b_kready, n & 1, p);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kKT / 16; ++kk)
            mma_bf16_ss(tmem, sdesc_sw128(sbase + S::kOffK + kk * 2048, 16384, 1024),
                        sdesc_sw128(sbase + S::kOffV + kk * 2048, 16384, 1024), idesc, 1);
          mma_commit(b_empty);
        }
        if (ok) mma_commit(b_chunk);
      }
      mma_commit(b_done);  // completes once every MMA above has finished
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;  // state row within the CTA = TMEM lane
    const int dk = dk0 + r;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const float* mchk = g.mchk + (long)bh * (NC + 1);
    bool ok = true;
    float nval = (n_owner && n0) ? n0[(long)bh * DK + dk] : 0.f;

    // master <- C0 (or zero)
    for (int c = 0; c < DVT; c += 32) {
      uint32_t v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = __float_as_uint(C0 ? C0[((long)bh * DK + dk) * DV + dv0 + c + j] : 0.f);
      tmem_st32(trow + c, v);
    }
    tmem_wait_st();

    int n = 0;
    for (int k = 0; k < NC && ok; ++k) {
      if (k > 0) {
        ok = mbar_wait(b_chunk, (k - 1) & 1, p);
        tc_fence_after();
      }
      const float m_in = mchk[k], m_out = mchk[k + 1];
      const float gk = g.gtot[(long)bh * NC + k];
      const float decay = expf(gk + m_in - m_out);
      // state entering chunk k: store, then decay in place
      const long row_off = (((long)bh * NC + k) * DK + dk) * DV + dv0;
      for (int c = 0; c < DVT && ok; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + c, v);
        tmem_wait_ld();
        if (C_states) {
          float4* dst = reinterpret_cast<float4*>(C_states + row_off + c);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
        if (Cb) {
          uint4* dst = reinterpret_cast<uint4*>(Cb + row_off + c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(
                pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * decay);
        tmem_st32(trow + c, v);
      }
      tmem_wait_st();
      if (n_owner) n_states[((long)bh * NC + k) * DK + dk] = nval;
      nval *= decay;
      tc_fence_before();
      mbar_arrive(b_master);

      for (int i = 0; i < tiles && ok; ++i, ++n) {
        ok = mbar_wait(b_full, n & 1, p);
        // Token weights of this tile: thread r owns token row r.
        const long t = (long)k * L + i * kKT + r;
        const float w = (t < T) ? p.key_scale * expf(gk + g.acol[(long)bh * tpad + t] - m_out) : 0.f;
        w_s[r] = w;
        named_bar_sync(1, 128);
        if (n_owner) {
          // n update in fp32 from the unrounded products w_s k_s (thread r owns
          // dk column r).  The normaliser enters h through |n^T q|, which can
          // cancel, so it must not see the bf16 rounding of w_s k_s.
          const uint8_t* box = smem + S::kOffK + (r >> 6) * 16384;
          const int cc = r & 63;
          float acc = 0.f;
#pragma unroll 8
          for (int s = 0; s < kKT; ++s) {
            const __nv_bfloat16 x = *reinterpret_cast<const __nv_bfloat16*>(
                box + sw128_offset(s, cc >> 3) + (cc & 7) * 2);
            acc = fmaf(__bfloat162float(x), w_s[s], acc);
          }
          nval += acc;
          named_bar_sync(1, 128);  // every column read done before the rows are rescaled
        }
        // Thread r scales token row r of the K tile by its weight, in place
        // (bf16 operand of the rank-128 update).
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint8_t* box = smem + S::kOffK + b * 16384;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4* ptr = reinterpret_cast<uint4*>(box + sw128_offset(r, j));
            uint4 u = *ptr;
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float2 f = __bfloat1622float2(h2[e]);
              h2[e] = __floats2bfloat162_rn(f.x * w, f.y * w);
            }
            *ptr = u;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(b_kready);
      }
    }
    // final state
    if (ok) ok = mbar_wait(b_chunk, (NC - 1) & 1, p);
    tc_fence_after();
    if (ok && C_T) {
      for (int c = 0; c < DVT; c += 32) {
        uint32_t v[32];
        tmem_ld32(trow + c, v);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(C_T + ((long)bh * DK + dk) * DV + dv0 + c);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                               __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
      }
    }
    if (n_owner && n_T) n_T[(long)bh * DK + dk] = nval;
    if (m_T && blockIdx.x == 0 && blockIdx.y == 0 && r == 0) m_T[bh] = mchk[NC];
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(b_done, 0, p);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

template <int DVT>
cudaError_t launch_states_t(const Problem& p, const void* K, const void* V, const float* C0,
                            const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                            float* n_states, float* C_T, float* n_T, float* m_T, cudaStream_t st) {
  using S = SCfg<DVT>;
  CUtensorMap tk, tv;
  if (!encode_tmap_bf16_3d(&tk, K, p.DK, p.T, p.BH, 64, kKT) ||
      !encode_tmap_bf16_3d(&tv, V, p.DV, p.T, p.BH, 64, kKT))
    return cudaErrorInvalidValue;
  auto kern = tc_states_kernel<DVT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.DV / DVT, p.DK / kRows, p.BH);
  kern<<<grid, kThreads, S::kSmem, st>>>(tk, tv, p, g, C0, n0, C_states, Cb, n_states, C_T, n_T,
                                         m_T);
  return cudaGetLastError();
}

}  // namespace

bool tc_states_supported(const Problem& p) {
  const bool dv_ok = p.DV == 64 || p.DV == 128 || p.DV % 256 == 0;
  return (p.DK == 128 || p.DK == 256) && dv_ok && p.DV <= 1024 && p.L % kKT == 0 && p.T > 0;
}

cudaError_t launch_tc_states_impl(const Problem& p, const void* K, const void* V, const float* C0,
                                  const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                                  float* n_states, float* C_T, float* n_T, float* m_T,
                                  cudaStream_t st) {
  const int dvt = p.DV >= 256 ? 256 : p.DV;
  switch (dvt) {
    case 64: return launch_states_t<64>(p, K, V, C0, n0, g, C_states, Cb, n_states, C_T, n_T, m_T, st);
    case 128: return launch_states_t<128>(p, K, V, C0, n0, g, C_states, Cb, n_states, C_T, n_T, m_T, st);
    case 256: return launch_states_t<256>(p, K, V, C0, n0, g, C_states, Cb, n_states, C_T, n_T, m_T, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace mlstm
