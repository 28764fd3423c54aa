// Support predicates, host-side tensor maps and launch glue of the
// tensor-core kernels.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "device_address.h"
#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// One thread per 16-byte chunk (8 values) of the destination: reads 8
// consecutive fp32 values of a state row and writes them as one bf16 chunk at
// its swizzled position.
__global__ void states_to_operand_kernel(const float4* __restrict__ src, uint4* __restrict__ dst,
                                         long n_bhk, int DK, int DV,
                                         const float* __restrict__ n_states,
                                         const __nv_bfloat16* __restrict__ V,
                                         const int* __restrict__ dom, int NC, int T) {
  const int n_vb = DV / 64;
  const size_t n_chunks = (size_t)n_bhk * DK * (DV / 8);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_chunks;
       i += (size_t)gridDim.x * blockDim.x) {
    const int cj = (int)(i % (DV / 8));  // 8-column chunk of the state row
    const size_t row = i / (DV / 8);      // bhk * DK + dk
    const int dk = (int)(row % DK);
    const long bhk = (long)(row / DK);
    float4 a = src[2 * i], b = src[2 * i + 1];
    const int td = dom ? dom[bhk] : -1;
    if (td >= 0) {  // dominated: C - n v_{t*}^T
      const float n = n_states[bhk * DK + dk];
      const uint4 u = *reinterpret_cast<const uint4*>(V + ((bhk / NC) * T + td) * (long)DV + cj * 8);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
      const float2 v0 = __bfloat1622float2(h2[0]), v1 = __bfloat1622float2(h2[1]);
      const float2 v2 = __bfloat1622float2(h2[2]), v3 = __bfloat1622float2(h2[3]);
      a = make_float4(fmaf(-n, v0.x, a.x), fmaf(-n, v0.y, a.y), fmaf(-n, v1.x, a.z),
                      fmaf(-n, v1.y, a.w));
      b = make_float4(fmaf(-n, v2.x, b.x), fmaf(-n, v2.y, b.y), fmaf(-n, v3.x, b.z),
                      fmaf(-n, v3.y, b.w));
    }
    const int vb = cj >> 3, j = cj & 7;
    uint4 v = make_uint4(tc::pack_bf16x2(a.x, a.y), tc::pack_bf16x2(a.z, a.w),
                         tc::pack_bf16x2(b.x, b.y), tc::pack_bf16x2(b.z, b.w));
    dst[cb_block_row(bhk, vb, dk, DK, n_vb) / 8 + (j ^ (dk & 7))] = v;
  }
}

}  // namespace

bool current_context_id(unsigned long long* id) {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    (void)cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  if (!g_ctx_current || !g_ctx_id || g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return g_ctx_id(ctx, id) == CUDA_SUCCESS;
}

bool encode_tmap_3d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t d0, uint64_t d1,
                    uint64_t d2, uint32_t b0, uint32_t b1, int swizzle_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc || (elem_bytes != 2 && elem_bytes != 4)) return false;
  if (b0 * (uint32_t)elem_bytes != (uint32_t)swizzle_bytes) return false;
  CUtensorMapSwizzle sw;
  switch (swizzle_bytes) {
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    default: return false;
  }
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      enc(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
          3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint32_t b0, uint32_t b1) {
  return encode_tmap_3d(map, base, 2, d0, d1, d2, b0, b1, 128);
}

bool tc_unfused_supported(const Problem& p) {
  // The chunk-state kernel writes the operand copy in 64-column blocks, one
  // warp per 32 x 64 tile, which needs at least 128 value columns per CTA.
  return tc_states_supported(p) && (tc_parallel_supported(p) || tc_parallel_wide_supported(p)) &&
         p.DV % 128 == 0;
}

cudaError_t launch_tc_states(const Problem& p, const void* K, const void* V, const float* C0,
                             const float* n0, Gates g, float* C_states, __nv_bfloat16* Cb,
                             float* n_states, float* C_T, float* n_T, float* m_T, float* seg_ws,
                             cudaStream_t st) {
  return launch_tc_states_impl(p, K, V, C0, n0, g, C_states, Cb, n_states, C_T, n_T, m_T, seg_ws,
                               st);
}

cudaError_t launch_tc_parallel(const Problem& p, const void* Q, const void* K, const void* V,
                               Gates g, const __nv_bfloat16* Cb, const float* n_states, void* H,
                               float* n_out, float* m_out, cudaStream_t st) {
  // Chunks of at most 256 tokens: one item per query tile covering every value
  // column (S computed once).  Longer chunks: one item per query tile and
  // value tile.
  if (tc_parallel_wide_supported(p))
    return launch_tc_parallel_wide(p, Q, K, V, g, Cb, n_states, H, n_out, m_out, st);
  return launch_tc_parallel_bf16states(p, Q, K, V, g, Cb, n_states, H, n_out, m_out, st);
}

cudaError_t launch_states_to_operand(const float* src, __nv_bfloat16* dst, long n_bhk, int DK,
                                     int DV, cudaStream_t st, const float* n_states,
                                     const void* V, const int* dom, const Problem& p) {
  if (dom && (!n_states || !V || p.NC < 1)) return cudaErrorInvalidValue;
  if (DV % 64 != 0) return cudaErrorNotSupported;
  const size_t n_chunks = (size_t)n_bhk * DK * (DV / 8);
  if (n_chunks == 0) return cudaSuccess;
  const size_t want = (n_chunks + 255) / 256;
  const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
  states_to_operand_kernel<<<blocks, 256, 0, st>>>(
      reinterpret_cast<const float4*>(src), reinterpret_cast<uint4*>(dst), n_bhk, DK, DV,
      n_states, static_cast<const __nv_bfloat16*>(V), dom, p.NC, p.T);
  return cudaGetLastError();
}

}  // namespace mlstm
