// Single-token step of the mLSTM: the inference step kernel that "xLSTM: the
// NX-AI repository behind the extended LSTM architecture" names as a kernel
// choice of its own next to the chunkwise one (section "Exponential gating,
// matrix memory, and why the kernels decide everything").  It is the forward
// recurrence for one token: for every (b, h),
//
//   lf = logsigmoid(f~),  li = i~ | logsigmoid(i~)
//   m' = max(lf + m, li),  fa = e^{lf + m - m'},  ia = e^{li - m'}
//   C' = fa C + ia (s k) v^T            C: [d_qk][d_v]
//   n' = fa n + ia (s k)
//   h  = C'^T q / max(|n'.q|, e^{-m'})
//
// The step reads and writes the fp32 state once: it is bound by HBM (2 x
// 4 d_qk d_v bytes per head against 4 d_qk d_v FLOPs).  step_state_kernel
// owns a (b, h, column tile) of C: each lane owns kVec consecutive columns
// (16-byte accesses when d_v is a multiple of 4, so a warp moves 512
// contiguous bytes of a state row per instruction), eight warps split the
// rows with eight rows in flight per thread, and h of the tile comes out of
// the same pass (a shared-memory reduction over the warps).
// The denominator only needs n'.q = fa (n.q) + ia (s k.q), which every block
// forms from the old n.  The blocks of one (b, h) are launched as one thread-
// block cluster (at most 8 column tiles): once every block of the cluster has
// read the old n and m, a cluster barrier lets block 0 write n' and m' in
// place.  Where the tiles of a head do not fit one cluster, step_norm_kernel
// writes them in a second launch instead (stream order puts it after every
// read of the old values).
#include "common.cuh"

namespace mlstm {
namespace {

constexpr int kStepWarps = 8;   // warps per block, splitting the state rows
constexpr int kStepUnroll = 8;  // state rows in flight per thread

struct StepGate {
  float m_new, fa, ia;
};

__device__ __forceinline__ StepGate step_gate(float i_pre, float f_pre, float m_old, bool sig) {
  const float lf = logsigmoidf(f_pre);
  const float li = sig ? logsigmoidf(i_pre) : i_pre;
  StepGate g;
  g.m_new = fmaxf(lf + m_old, li);
  g.fa = expf(lf + m_old - g.m_new);
  g.ia = expf(li - g.m_new);
  return g;
}

template <int kVec>
struct VecF;
template <> struct VecF<1> {
  using type = float;
  __device__ static void load(const float* p, float (&x)[1]) { x[0] = *p; }
  __device__ static void store(float* p, const float (&x)[1]) { *p = x[0]; }
};
template <> struct VecF<4> {
  using type = float4;
  __device__ static void load(const float* p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  __device__ static void store(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

template <typename T, int kVec>
__global__ void __launch_bounds__(kStepWarps * 32)
step_state_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ i_pre, const float* __restrict__ f_pre,
                  float* __restrict__ C, float* __restrict__ n, float* __restrict__ m,
                  T* __restrict__ h, int DK, int DV, int sig, float key_scale, int cluster_nm) {
  // sig: 0 exponential input gate, 1 sigmoid, 2 the sigmoid variant without
  // normaliser (same state update as 1)
  constexpr int kCols = 32 * kVec;       // value columns per block
  extern __shared__ float sh[];
  float* sk = sh;                        // s k   [DK]
  float* sq = sh + DK;                   // q     [DK]
  float* red = sh + 2 * DK;              // [kStepWarps][kCols] partial C'^T q
  float* dots = red + kStepWarps * kCols;  // [kStepWarps][2] partial n.q, (s k).q
  const int bh = blockIdx.y;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const StepGate gt = step_gate(i_pre[bh], f_pre[bh], m[bh], sig != 0);

  float nq = 0.f, kq = 0.f;
  for (int i = threadIdx.x; i < DK; i += blockDim.x) {
    const float kk = key_scale * to_float(k[(long)bh * DK + i]);
    const float qq = to_float(q[(long)bh * DK + i]);
    sk[i] = kk;
    sq[i] = qq;
    nq = fmaf(n[(long)bh * DK + i], qq, nq);
    kq = fmaf(kk, qq, kq);
  }
  nq = warp_sum(nq);
  kq = warp_sum(kq);
  if (tx == 0) {
    dots[2 * ty] = nq;
    dots[2 * ty + 1] = kq;
  }
  __syncthreads();
  if (cluster_nm) {
    // every block of this head's cluster has read the old n and m
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
    if (blockIdx.x == 0) {
      for (int i = threadIdx.x; i < DK; i += blockDim.x)
        n[(long)bh * DK + i] = fmaf(gt.fa, n[(long)bh * DK + i], gt.ia * sk[i]);
      if (threadIdx.x == 0) m[bh] = gt.m_new;
    }
  }

  // columns col .. col + kVec - 1 (kVec == 4 needs DV % 4 == 0, so all or none are valid)
  const int col = blockIdx.x * kCols + tx * kVec;
  const bool valid = col < DV;
  float vv[kVec], acc[kVec];
#pragma unroll
  for (int e = 0; e < kVec; ++e) {
    vv[e] = valid ? gt.ia * to_float(v[(long)bh * DV + col + e]) : 0.f;
    acc[e] = 0.f;
  }
  if (valid) {
    float* cp = C + (long)bh * DK * DV + col;
    int dk = ty;
    // kStepUnroll rows per batch: all loads issued before the first store
    for (; dk + (kStepUnroll - 1) * kStepWarps < DK; dk += kStepUnroll * kStepWarps) {
      float c[kStepUnroll][kVec];
#pragma unroll
      for (int u = 0; u < kStepUnroll; ++u) VecF<kVec>::load(cp + (long)(dk + u * kStepWarps) * DV, c[u]);
#pragma unroll
      for (int u = 0; u < kStepUnroll; ++u) {
        const int r = dk + u * kStepWarps;
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          c[u][e] = fmaf(gt.fa, c[u][e], sk[r] * vv[e]);
          acc[e] = fmaf(c[u][e], sq[r], acc[e]);
        }
        VecF<kVec>::store(cp + (long)r * DV, c[u]);
      }
    }
    for (; dk < DK; dk += kStepWarps) {
      float c[kVec];
      VecF<kVec>::load(cp + (long)dk * DV, c);
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        c[e] = fmaf(gt.fa, c[e], sk[dk] * vv[e]);
        acc[e] = fmaf(c[e], sq[dk], acc[e]);
      }
      VecF<kVec>::store(cp + (long)dk * DV, c);
    }
  }
#pragma unroll
  for (int e = 0; e < kVec; ++e) red[ty * kCols + tx * kVec + e] = acc[e];
  __syncthreads();
  // h of the tile: thread j < kCols sums column j over the warps
  float nq_all = 0.f, kq_all = 0.f;
#pragma unroll
  for (int w = 0; w < kStepWarps; ++w) {
    nq_all += dots[2 * w];
    kq_all += dots[2 * w + 1];
  }
  const float den = gt.fa * nq_all + gt.ia * kq_all;  // n'.q
  // sig == 2: the plain sigmoid variant, h = e^{m'} C'^T q (no normaliser)
  const float scale = sig == 2 ? expf(gt.m_new) : 1.f / fmaxf(fabsf(den), expf(-gt.m_new));
  for (int j = threadIdx.x; j < kCols; j += blockDim.x) {
    const int cj = blockIdx.x * kCols + j;
    if (cj >= DV) break;
    float num = 0.f;
#pragma unroll
    for (int w = 0; w < kStepWarps; ++w) num += red[w * kCols + j];
    h[(long)bh * DV + cj] = from_float<T>(num * scale);
  }
}

// n' and m' in place, one block per (b, h).
__global__ void __launch_bounds__(256)
step_norm_kernel(const void* __restrict__ k, int k_bf16, const float* __restrict__ i_pre,
                 const float* __restrict__ f_pre, float* __restrict__ n, float* __restrict__ m,
                 int DK, int sig, float key_scale) {
  const int bh = blockIdx.x;
  const StepGate gt = step_gate(i_pre[bh], f_pre[bh], m[bh], sig != 0);
  __syncthreads();  // every thread has read the old m before thread 0 writes m'
  for (int i = threadIdx.x; i < DK; i += blockDim.x) {
    const float kk =
        k_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(k)[(long)bh * DK + i])
               : static_cast<const float*>(k)[(long)bh * DK + i];
    n[(long)bh * DK + i] = fmaf(gt.fa, n[(long)bh * DK + i], gt.ia * key_scale * kk);
  }
  if (threadIdx.x == 0) m[bh] = gt.m_new;
}

}  // namespace

size_t step_smem_bytes(int DK, int cols) {
  return (2 * (size_t)DK + kStepWarps * (size_t)cols + 2 * kStepWarps) * sizeof(float);
}

constexpr int kMaxCluster = 8;  // portable cluster size

// Launches the state kernel; with one cluster per head (the tiles of a head
// fit one cluster) it also writes n' and m' and returns true.
template <typename T, int kVec>
cudaError_t launch_state(const Problem& p, const void* q, const void* k, const void* v,
                         const float* i_pre, const float* f_pre, float* C, float* n, float* m,
                         void* h, cudaStream_t st, bool* nm_done) {
  constexpr int kCols = 32 * kVec;
  const int gx = (p.DV + kCols - 1) / kCols;
  const int cluster = gx <= kMaxCluster ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, p.BH);
  cfg.blockDim = dim3(kStepWarps * 32);
  cfg.dynamicSmemBytes = step_smem_bytes(p.DK, kCols);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster ? gx : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  *nm_done = cluster != 0;
  return cudaLaunchKernelEx(&cfg, step_state_kernel<T, kVec>, static_cast<const T*>(q),
                            static_cast<const T*>(k), static_cast<const T*>(v), i_pre, f_pre, C, n,
                            m, static_cast<T*>(h), p.DK, p.DV, p.gate_sigmoid + p.no_norm,
                            p.key_scale, cluster);
}

int step_launches(const Problem& p) {
  const int cols = p.DV % 4 == 0 ? 128 : 32;
  return (p.DV + cols - 1) / cols <= kMaxCluster ? 1 : 2;
}

cudaError_t launch_step(const Problem& p, mlstm_dtype dt, const void* q, const void* k,
                        const void* v, const float* i_pre, const float* f_pre, float* C,
                        float* n, float* m, void* h, cudaStream_t st) {
  if (step_smem_bytes(p.DK, 128) > 48 * 1024) return cudaErrorNotSupported;
  // 16-byte state accesses when every row starts on a 16-byte boundary
  const bool vec = p.DV % 4 == 0;
  bool nm_done = false;
  cudaError_t e;
  if (dt == MLSTM_DT_BF16)
    e = vec ? launch_state<__nv_bfloat16, 4>(p, q, k, v, i_pre, f_pre, C, n, m, h, st, &nm_done)
            : launch_state<__nv_bfloat16, 1>(p, q, k, v, i_pre, f_pre, C, n, m, h, st, &nm_done);
  else
    e = vec ? launch_state<float, 4>(p, q, k, v, i_pre, f_pre, C, n, m, h, st, &nm_done)
            : launch_state<float, 1>(p, q, k, v, i_pre, f_pre, C, n, m, h, st, &nm_done);
  if (e != cudaSuccess || nm_done) return e;
  step_norm_kernel<<<p.BH, 256, 0, st>>>(k, dt == MLSTM_DT_BF16, i_pre, f_pre, n, m, p.DK,
                                         p.gate_sigmoid, p.key_scale);
  return cudaGetLastError();
}

}  // namespace mlstm
