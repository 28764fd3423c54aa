// C ABI of the mLSTM forward library: argument checks, workspace layout and
// dispatch to the kernels.  Every check happens before the first launch, so an
// error return means nothing was enqueued.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "device_address.h"
#include "tc.h"
#include "tc_bwd.h"

namespace mlstm {
namespace {

__device__ uint32_t g_error_word = 0;

constexpr unsigned long long kDefaultPolls = 1ull << 26;
uint32_t g_last_error_word = 0;
unsigned long long g_max_polls = kDefaultPolls;

constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Address of g_error_word in the current context (nullptr if it cannot be
// looked up).
DeviceAddressCache g_err_cache;
uint32_t* error_word_ptr() {
  return static_cast<uint32_t*>(cached_device_address(
      g_err_cache, [](void** p) { return cudaGetSymbolAddress(p, g_error_word); }));
}

mlstm_status check_sizes(int B, int NH, int T, int DK, int DV, int L) {
  if (B < 1 || NH < 1 || T < 0 || DK < 1 || DV < 1) return MLSTM_ERR_INVALID_ARG;
  if (L < 64 || L % 64 != 0) return MLSTM_ERR_INVALID_ARG;
  if (L > 4096 || DK > 1024 || DV > 1024) return MLSTM_ERR_UNSUPPORTED;
  if ((long long)B * NH > 65535) return MLSTM_ERR_UNSUPPORTED;
  if (T > (1 << 22)) return MLSTM_ERR_UNSUPPORTED;
  return MLSTM_OK;
}

Problem make_problem(int B, int NH, int T, int DK, int DV, int L, mlstm_gate_mode gm) {
  Problem p{};
  p.B = B;
  p.NH = NH;
  p.T = T;
  p.DK = DK;
  p.DV = DV;
  p.L = L;
  p.NC = (T + L - 1) / L;
  p.BH = B * NH;
  p.gate_sigmoid = gm == MLSTM_GATE_SIGMOID || gm == MLSTM_GATE_SIGMOID_PLAIN;
  p.no_norm = gm == MLSTM_GATE_SIGMOID_PLAIN;
  p.key_scale = (float)(1.0 / sqrt((double)DK));
  p.signed_den = 0;
  p.err = nullptr;
  p.max_polls = g_max_polls;
  return p;
}

struct Layout {
  size_t gates_bytes;   // bcum, acol, amax, gtot, mchk
  size_t states_bytes;  // chunk states kept between two kernels
  size_t total;
};

// What a call needs the workspace for.
enum class Mode { kFull, kStates, kParallel };

size_t cb_bytes(const Problem& p) {
  return round_up((size_t)p.BH * p.NC * (size_t)p.DK * p.DV * sizeof(__nv_bfloat16));
}

size_t seg_bytes(const Problem& p) { return round_up(tc_states_segment_floats(p) * sizeof(float)); }

// Workspace layout: the gate arrays, then
//   kFull/SIMT:     C_states fp32 [BH, NC, DK, DV], n_states fp32 [BH, NC, DK]
//   kFull/TC:       C_states bf16 (operand copy), n_states fp32, segment end states
//   kStates/TC:     segment end states
//   kParallel/TC:   C_states bf16 (converted from the caller's fp32 states)
//   everything else: nothing more.
Layout layout_for(const Problem& p, mlstm_algo a, Mode mode) {
  Layout l{};
  const size_t BH = (size_t)p.BH, tpad = (size_t)p.NC * p.L;
  l.gates_bytes = 3 * round_up(BH * tpad * sizeof(float)) + round_up(BH * p.NC * sizeof(float)) +
                  round_up(BH * (p.NC + 1) * sizeof(float)) + 4 * round_up(BH * p.NC * 4) +
                  round_up(BH * 4);
  const size_t n_bytes = round_up(BH * p.NC * (size_t)p.DK * sizeof(float));
  if (mode == Mode::kFull && a == MLSTM_ALGO_SIMT)
    l.states_bytes = round_up(BH * p.NC * (size_t)p.DK * p.DV * sizeof(float)) + n_bytes;
  else if (mode == Mode::kFull && a == MLSTM_ALGO_TC)
    l.states_bytes = cb_bytes(p) + n_bytes + seg_bytes(p);
  else if (mode == Mode::kStates && a == MLSTM_ALGO_TC)
    l.states_bytes = seg_bytes(p);
  else if (mode == Mode::kParallel && a == MLSTM_ALGO_TC)
    l.states_bytes = cb_bytes(p);
  l.total = l.gates_bytes + l.states_bytes;
  return l;
}

// Carves the gate arrays out of `ws`; returns the first byte after them.
// `dominance`: the gate kernels also mark the chunks whose entering state one
// token dominates (used by the tensor-core paths that hand states on in bf16).
char* carve_gates(const Problem& p, char* ws, Gates* g, float* mchk_override,
                  bool dominance = false) {
  const size_t BH = (size_t)p.BH, tpad = (size_t)p.NC * p.L;
  g->bcum = reinterpret_cast<float*>(ws);
  ws += round_up(BH * tpad * sizeof(float));
  g->acol = reinterpret_cast<float*>(ws);
  ws += round_up(BH * tpad * sizeof(float));
  g->amax = reinterpret_cast<float*>(ws);
  ws += round_up(BH * tpad * sizeof(float));
  g->gtot = reinterpret_cast<float*>(ws);
  ws += round_up(BH * p.NC * sizeof(float));
  g->mchk = mchk_override ? mchk_override : reinterpret_cast<float*>(ws);
  ws += round_up(BH * (p.NC + 1) * sizeof(float));
  g->csum = dominance ? reinterpret_cast<float*>(ws) : nullptr;
  ws += round_up(BH * p.NC * 4);
  g->cidx = dominance ? reinterpret_cast<int*>(ws) : nullptr;
  ws += round_up(BH * p.NC * 4);
  g->dom = dominance ? reinterpret_cast<int*>(ws) : nullptr;
  ws += round_up(BH * p.NC * 4);
  g->mdom = dominance ? reinterpret_cast<float*>(ws) : nullptr;
  ws += round_up(BH * p.NC * 4);
  g->hdom = dominance ? reinterpret_cast<int*>(ws) : nullptr;
  ws += round_up(BH * 4);
  return ws;
}

bool valid_enums(mlstm_dtype dt, mlstm_gate_mode gm, mlstm_algo algo) {
  return (dt == MLSTM_DT_F32 || dt == MLSTM_DT_BF16) &&
         (gm == MLSTM_GATE_EXP || gm == MLSTM_GATE_SIGMOID || gm == MLSTM_GATE_SIGMOID_PLAIN) &&
         (algo == MLSTM_ALGO_AUTO || algo == MLSTM_ALGO_SIMT || algo == MLSTM_ALGO_TC ||
          algo == MLSTM_ALGO_TC_FUSED);
}

// Resolves AUTO and checks that the chosen algorithm supports the problem.
mlstm_status resolve_algo(const Problem& p, mlstm_dtype dt, mlstm_algo req, bool allow_fused,
                          mlstm_algo* out) {
  if (req == MLSTM_ALGO_AUTO) {
    // The fused kernel walks each head's chunks in order on one SM: a chunk
    // there costs about 5 us of one SM against about 9-11 us of SM time on the
    // unfused path, so it wins once its waves of 148 heads are at least half
    // full.  Below 74 heads the unfused state kernel also splits each head's
    // sequence into segments and wins (measured at d = 128, chunks of 128:
    // fused faster at 96, 128, 160, 192, 256 and 1024 heads, slower at 64).
    // The threshold is a constant of the shape (half of a 148-SM B200) so
    // that the workspace size computed on the host always matches the
    // algorithm a call picks.
    constexpr int kFusedMinHeads = 148 / 2;
    if (dt == MLSTM_DT_BF16 && p.T > 0 && allow_fused && tc_fused_supported(p) &&
        p.BH >= kFusedMinHeads) {
      *out = MLSTM_ALGO_TC_FUSED;
    } else if (dt == MLSTM_DT_BF16 && p.T > 0 && tc_unfused_supported(p)) {
      *out = MLSTM_ALGO_TC;
    } else {
      *out = MLSTM_ALGO_SIMT;
    }
    return MLSTM_OK;
  }
  if (req == MLSTM_ALGO_SIMT) {
    *out = req;
    return MLSTM_OK;
  }
  if (dt != MLSTM_DT_BF16 || p.T == 0) return MLSTM_ERR_UNSUPPORTED;
  if (req == MLSTM_ALGO_TC) {
    if (!tc_unfused_supported(p)) return MLSTM_ERR_UNSUPPORTED;
  } else {
    if (!allow_fused || !tc_fused_supported(p)) return MLSTM_ERR_UNSUPPORTED;
  }
  *out = req;
  return MLSTM_OK;
}

inline mlstm_status from_cuda(cudaError_t e) {
  return e == cudaSuccess ? MLSTM_OK : MLSTM_ERR_CUDA;
}

// --- launch accounting and the optional per-kernel event timing -----------
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_profile_on{0};
struct Pending {
  int id;
  int launches;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
std::vector<Pending> g_pending;

// Runs one launcher `fn` (which enqueues `n_launch` kernels on `st`), counting
// the launches and, when profiling is on, bracketing them with events.
template <typename Fn>
cudaError_t launch_family(int id, int n_launch, cudaStream_t st, Fn&& fn) {
  Pending pd{id, n_launch, nullptr, nullptr};
  const bool prof = g_profile_on.load(std::memory_order_relaxed) != 0;
  if (prof) {
    if (cudaEventCreate(&pd.start) != cudaSuccess) return cudaGetLastError();
    if (cudaEventCreate(&pd.stop) != cudaSuccess) return cudaGetLastError();
    cudaEventRecord(pd.start, st);
  }
  cudaError_t e = fn();
  if (e == cudaSuccess) g_launches.fetch_add((uint64_t)n_launch, std::memory_order_relaxed);
  if (prof) {
    cudaEventRecord(pd.stop, st);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_pending.push_back(pd);
  }
  return e;
}

int gate_launches(const Problem& p) { return p.NC > 0 ? 2 : 1; }

}  // namespace
}  // namespace mlstm

using namespace mlstm;

extern "C" {

int mlstm_abi_version(void) { return 100; }

uint32_t mlstm_last_device_error_word(void) { return g_last_error_word; }

uint64_t mlstm_kernel_launches(void) { return g_launches.load(); }

void mlstm_profile_enable(int on) { g_profile_on.store(on ? 1 : 0); }

mlstm_status mlstm_profile_read(double* ms, uint64_t* launches, int n) {
  if (n < 0 || n > MLSTM_KERNEL_COUNT || (n > 0 && (!ms || !launches)))
    return MLSTM_ERR_INVALID_ARG;
  std::vector<Pending> pend;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    pend.swap(g_pending);
  }
  for (int i = 0; i < n; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  mlstm_status st = MLSTM_OK;
  for (Pending& pd : pend) {
    float t = 0.f;
    if (cudaEventSynchronize(pd.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, pd.start, pd.stop) != cudaSuccess)
      st = MLSTM_ERR_CUDA;
    else if (pd.id < n) {
      ms[pd.id] += t;
      launches[pd.id] += (uint64_t)pd.launches;
    }
    cudaEventDestroy(pd.start);
    cudaEventDestroy(pd.stop);
  }
  return st;
}

const char* mlstm_kernel_name(int id) {
  switch (id) {
    case MLSTM_KERNEL_GATES: return "gates";
    case MLSTM_KERNEL_SIMT_STATES: return "simt_states";
    case MLSTM_KERNEL_SIMT_PARALLEL: return "simt_parallel";
    case MLSTM_KERNEL_TC_STATES: return "tc_states";
    case MLSTM_KERNEL_TC_PARALLEL: return "tc_parallel";
    case MLSTM_KERNEL_TC_FUSED: return "tc_fused";
    case MLSTM_KERNEL_STEP: return "step";
    case MLSTM_KERNEL_BW: return "bw";
    case MLSTM_KERNEL_FW_TRAIN: return "fw_train";
  }
  return "unknown";
}

const char* mlstm_status_string(mlstm_status s) {
  switch (s) {
    case MLSTM_OK: return "ok";
    case MLSTM_ERR_INVALID_ARG: return "invalid argument";
    case MLSTM_ERR_UNSUPPORTED: return "unsupported by the selected algorithm";
    case MLSTM_ERR_CUDA: return "CUDA error";
    case MLSTM_ERR_TIMEOUT: return "device-side bounded wait timed out";
    case MLSTM_ERR_DEVICE: return "device-side check failed";
    case MLSTM_ERR_SCRATCH_TOO_SMALL:
      return "problem needs more scratch than the library's static array holds";
  }
  return "unknown status";
}

void mlstm_set_watchdog(uint64_t max_polls) {
  g_max_polls = max_polls ? (unsigned long long)max_polls : kDefaultPolls;
}

mlstm_status mlstm_watchdog_selftest(mlstm_stream_t stream) {
  uint32_t* w = error_word_ptr();
  if (!w) return MLSTM_ERR_CUDA;
  return from_cuda(
      launch_watchdog_selftest(w, g_max_polls, reinterpret_cast<cudaStream_t>(stream)));
}

mlstm_status mlstm_fw_workspace_size(int B, int NH, int T, int DK, int DV, int chunk_size,
                                     mlstm_dtype dtype, mlstm_algo algo, size_t* bytes) {
  if (!bytes || !valid_enums(dtype, MLSTM_GATE_EXP, algo)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  Problem p = make_problem(B, NH, T, DK, DV, chunk_size, MLSTM_GATE_EXP);
  mlstm_algo a;
  s = resolve_algo(p, dtype, algo, true, &a);
  if (s != MLSTM_OK) return s;
  *bytes = layout_for(p, a, Mode::kFull).total;
  return MLSTM_OK;
}

mlstm_status mlstm_fw_substep_workspace_size(int B, int NH, int T, int DK, int DV, int chunk_size,
                                             mlstm_dtype dtype, mlstm_algo algo, size_t* bytes) {
  if (!bytes || !valid_enums(dtype, MLSTM_GATE_EXP, algo)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  Problem p = make_problem(B, NH, T, DK, DV, chunk_size, MLSTM_GATE_EXP);
  mlstm_algo a;
  s = resolve_algo(p, dtype, algo, false, &a);
  if (s != MLSTM_OK) return s;
  const size_t st = layout_for(p, a, Mode::kStates).total;
  const size_t pa = layout_for(p, a, Mode::kParallel).total;
  *bytes = st > pa ? st : pa;
  return MLSTM_OK;
}

mlstm_status mlstm_fw(const void* Q, const void* K, const void* V, const float* i_pre,
                      const float* f_pre, const float* C0, const float* n0, const float* m0,
                      void* H, float* C_T, float* n_T, float* m_T, int B, int NH, int T, int DK,
                      int DV, int chunk_size, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                      mlstm_algo algo, void* workspace, size_t workspace_bytes,
                      mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, algo)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  if (T > 0 && (!Q || !K || !V || !i_pre || !f_pre || !H)) return MLSTM_ERR_INVALID_ARG;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return MLSTM_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, i_pre, f_pre, C0, n0, m0, H, C_T, n_T, m_T, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MLSTM_ERR_INVALID_ARG;
  Problem p = make_problem(B, NH, T, DK, DV, chunk_size, gate_mode);
  mlstm_algo a;
  s = resolve_algo(p, dtype, algo, true, &a);
  if (s != MLSTM_OK) return s;
  const Layout lay = layout_for(p, a, Mode::kFull);
  if (workspace_bytes < lay.total || (lay.total > 0 && !workspace)) return MLSTM_ERR_INVALID_ARG;
  p.err = error_word_ptr();
  if (!p.err) return MLSTM_ERR_CUDA;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Gates g;
  char* rest = carve_gates(p, static_cast<char*>(workspace), &g, nullptr, a != MLSTM_ALGO_SIMT);
  s = from_cuda(launch_family(MLSTM_KERNEL_GATES, gate_launches(p), st,
                              [&] { return launch_gates(p, i_pre, f_pre, m0, g, st); }));
  if (s != MLSTM_OK) return s;
  if (a == MLSTM_ALGO_TC_FUSED)
    return from_cuda(launch_family(MLSTM_KERNEL_TC_FUSED, 1, st, [&] {
      return launch_tc_fused(p, Q, K, V, C0, n0, g, H, C_T, n_T, m_T, st);
    }));

  if (a == MLSTM_ALGO_TC) {
    __nv_bfloat16* Cb = reinterpret_cast<__nv_bfloat16*>(rest);
    float* n_states = reinterpret_cast<float*>(rest + cb_bytes(p));
    float* seg_ws = reinterpret_cast<float*>(
        rest + cb_bytes(p) + round_up((size_t)p.BH * p.NC * (size_t)DK * sizeof(float)));
    s = from_cuda(launch_family(MLSTM_KERNEL_TC_STATES, tc_states_launches(p), st, [&] {
      return launch_tc_states(p, K, V, C0, n0, g, nullptr, Cb, n_states, C_T, n_T, m_T, seg_ws,
                              st);
    }));
    if (s != MLSTM_OK) return s;
    return from_cuda(launch_family(MLSTM_KERNEL_TC_PARALLEL, 1, st, [&] {
      return launch_tc_parallel(p, Q, K, V, g, Cb, n_states, H, nullptr, nullptr, st);
    }));
  }
  float* C_states = reinterpret_cast<float*>(rest);
  float* n_states =
      reinterpret_cast<float*>(rest + round_up((size_t)p.BH * p.NC * (size_t)DK * DV * 4));
  s = from_cuda(launch_family(MLSTM_KERNEL_SIMT_STATES, 1, st, [&] {
    return launch_simt_states(p, dtype, K, V, C0, n0, g, C_states, n_states, C_T, n_T, m_T, st);
  }));
  if (s != MLSTM_OK) return s;
  if (T == 0) return MLSTM_OK;
  return from_cuda(launch_family(MLSTM_KERNEL_SIMT_PARALLEL, 1, st, [&] {
    return launch_simt_parallel(p, dtype, Q, K, V, g, C_states, n_states, H, nullptr, nullptr,
                                st);
  }));
}

mlstm_status mlstm_fw_chunk_states(const void* K, const void* V, const float* i_pre,
                                   const float* f_pre, const float* C0, const float* n0,
                                   const float* m0, float* C_states, float* n_states,
                                   float* m_states, float* C_T, float* n_T, float* m_T, int B,
                                   int NH, int T, int DK, int DV, int chunk_size,
                                   mlstm_dtype dtype, mlstm_gate_mode gate_mode, mlstm_algo algo,
                                   void* workspace, size_t workspace_bytes,
                                   mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, algo)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  if (T > 0 && (!K || !V || !i_pre || !f_pre || !C_states || !n_states))
    return MLSTM_ERR_INVALID_ARG;
  if (!m_states) return MLSTM_ERR_INVALID_ARG;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return MLSTM_ERR_INVALID_ARG;
  const void* ptrs[] = {K,  V,        i_pre,    f_pre,    C0,  n0,  m0,       C_states,
                        n_states, m_states, C_T, n_T, m_T, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MLSTM_ERR_INVALID_ARG;
  Problem p = make_problem(B, NH, T, DK, DV, chunk_size, gate_mode);
  mlstm_algo a;
  s = resolve_algo(p, dtype, algo, false, &a);
  if (s != MLSTM_OK) return s;
  const Layout lay = layout_for(p, a, Mode::kStates);
  if (workspace_bytes < lay.total || (lay.total > 0 && !workspace)) return MLSTM_ERR_INVALID_ARG;
  p.err = error_word_ptr();
  if (!p.err) return MLSTM_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Gates g;
  float* seg_ws = reinterpret_cast<float*>(carve_gates(p, static_cast<char*>(workspace), &g, m_states));
  s = from_cuda(launch_family(MLSTM_KERNEL_GATES, gate_launches(p), st,
                              [&] { return launch_gates(p, i_pre, f_pre, m0, g, st); }));
  if (s != MLSTM_OK) return s;
  if (a == MLSTM_ALGO_TC)
    return from_cuda(launch_family(MLSTM_KERNEL_TC_STATES, tc_states_launches(p), st, [&] {
      return launch_tc_states(p, K, V, C0, n0, g, C_states, nullptr, n_states, C_T, n_T, m_T,
                              seg_ws, st);
    }));
  return from_cuda(launch_family(MLSTM_KERNEL_SIMT_STATES, 1, st, [&] {
    return launch_simt_states(p, dtype, K, V, C0, n0, g, C_states, n_states, C_T, n_T, m_T, st);
  }));
}

mlstm_status mlstm_fw_parallel(const void* Q, const void* K, const void* V, const float* i_pre,
                               const float* f_pre, const float* m0, const float* C_states,
                               const float* n_states, void* H, float* n_out, float* m_out, int B,
                               int NH, int T, int DK, int DV, int chunk_size, mlstm_dtype dtype,
                               mlstm_gate_mode gate_mode, mlstm_algo algo, void* workspace,
                               size_t workspace_bytes, mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, algo)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  if (T > 0 && (!Q || !K || !V || !i_pre || !f_pre || !C_states || !n_states || !H))
    return MLSTM_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, i_pre, f_pre, m0, C_states, n_states, H, n_out, m_out,
                        workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MLSTM_ERR_INVALID_ARG;
  Problem p = make_problem(B, NH, T, DK, DV, chunk_size, gate_mode);
  mlstm_algo a;
  s = resolve_algo(p, dtype, algo, false, &a);
  if (s != MLSTM_OK) return s;
  const Layout lay = layout_for(p, a, Mode::kParallel);
  if (workspace_bytes < lay.total || (lay.total > 0 && !workspace)) return MLSTM_ERR_INVALID_ARG;
  if (T == 0) return MLSTM_OK;
  p.err = error_word_ptr();
  if (!p.err) return MLSTM_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Gates g;
  char* rest = carve_gates(p, static_cast<char*>(workspace), &g, nullptr, a == MLSTM_ALGO_TC);
  s = from_cuda(launch_family(MLSTM_KERNEL_GATES, gate_launches(p), st,
                              [&] { return launch_gates(p, i_pre, f_pre, m0, g, st); }));
  if (s != MLSTM_OK) return s;
  if (a == MLSTM_ALGO_TC) {
    __nv_bfloat16* Cb = reinterpret_cast<__nv_bfloat16*>(rest);
    s = from_cuda(launch_family(MLSTM_KERNEL_TC_PARALLEL, 1, st, [&] {
      cudaError_t e = launch_states_to_operand(C_states, Cb, (long)p.BH * p.NC, DK, DV, st,
                                               n_states, V, g.dom, p);
      if (e != cudaSuccess) return e;
      return launch_tc_parallel(p, Q, K, V, g, Cb, n_states, H, n_out, m_out, st);
    }));
    return s;
  }
  return from_cuda(launch_family(MLSTM_KERNEL_SIMT_PARALLEL, 1, st, [&] {
    return launch_simt_parallel(p, dtype, Q, K, V, g, C_states, n_states, H, n_out, m_out, st);
  }));
}

mlstm_status mlstm_bw_workspace_size(int B, int NH, int T, int DK, int DV, int chunk_size,
                                     mlstm_dtype dtype, size_t* bytes) {
  if (!bytes || !valid_enums(dtype, MLSTM_GATE_EXP, MLSTM_ALGO_AUTO)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  *bytes = bwd_workspace_bytes(make_problem(B, NH, T, DK, DV, chunk_size, MLSTM_GATE_EXP), dtype);
  return MLSTM_OK;
}

mlstm_status mlstm_bw(const void* Q, const void* K, const void* V, const float* i_pre,
                      const float* f_pre, const float* C0, const float* n0, const float* m0,
                      const void* dH, void* dQ, void* dK, void* dV, float* di_pre, float* df_pre,
                      float* dC0, float* dn0, float* dm0, int B, int NH, int T, int DK, int DV,
                      int chunk_size, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                      void* workspace, size_t workspace_bytes, mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, MLSTM_ALGO_AUTO)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, chunk_size);
  if (s != MLSTM_OK) return s;
  if (gate_mode == MLSTM_GATE_SIGMOID_PLAIN) return MLSTM_ERR_UNSUPPORTED;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return MLSTM_ERR_INVALID_ARG;
  if (T > 0 && (!Q || !K || !V || !i_pre || !f_pre || !dH || !dQ || !dK || !dV || !di_pre ||
                !df_pre))
    return MLSTM_ERR_INVALID_ARG;
  const void* ptrs[] = {Q,  K,      V,      i_pre, f_pre, C0,  n0,  m0, dH,
                        dQ, dK,     dV,     di_pre, df_pre, dC0, dn0, dm0, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MLSTM_ERR_INVALID_ARG;
  Problem p = make_problem(B, NH, T, DK, DV, chunk_size, gate_mode);
  const size_t need = bwd_workspace_bytes(p, dtype);
  if (workspace_bytes < need || !workspace) return MLSTM_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // no output token: the initial state gets no gradient
    if (dC0 && cudaMemsetAsync(dC0, 0, sizeof(float) * p.BH * DK * DV, st) != cudaSuccess)
      return MLSTM_ERR_CUDA;
    if (dn0 && cudaMemsetAsync(dn0, 0, sizeof(float) * p.BH * DK, st) != cudaSuccess)
      return MLSTM_ERR_CUDA;
    if (dm0 && cudaMemsetAsync(dm0, 0, sizeof(float) * p.BH, st) != cudaSuccess)
      return MLSTM_ERR_CUDA;
    return MLSTM_OK;
  }
  p.err = error_word_ptr();
  if (!p.err) return MLSTM_ERR_CUDA;
  return from_cuda(launch_family(MLSTM_KERNEL_BW, bwd_launches(p, dtype), st, [&] {
    return launch_backward(p, dtype, Q, K, V, i_pre, f_pre, C0, n0, m0, dH, dQ, dK, dV, di_pre,
                           df_pre, dC0, dn0, dm0, workspace, st);
  }));
}

mlstm_status mlstm_train_sizes(int B, int NH, int T, int DK, int DV, mlstm_dtype dtype,
                               size_t* saved_bytes, size_t* fw_workspace_bytes,
                               size_t* bw_workspace_bytes) {
  if (!saved_bytes || !fw_workspace_bytes || !bw_workspace_bytes ||
      !valid_enums(dtype, MLSTM_GATE_EXP, MLSTM_ALGO_AUTO))
    return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, 128);
  if (s != MLSTM_OK) return s;
  const Problem p = make_problem(B, NH, T, DK, DV, 128, MLSTM_GATE_EXP);
  if (!train_supported(p, dtype)) return MLSTM_ERR_UNSUPPORTED;
  *saved_bytes = train_saved_bytes(p);
  *fw_workspace_bytes = fw_train_workspace_bytes(p);
  *bw_workspace_bytes = bw_saved_workspace_bytes(p);
  return MLSTM_OK;
}

mlstm_status mlstm_fw_train(const void* Q, const void* K, const void* V, const float* i_pre,
                            const float* f_pre, const float* C0, const float* n0, const float* m0,
                            void* H, float* C_T, float* n_T, float* m_T, void* saved,
                            size_t saved_bytes, int B, int NH, int T, int DK, int DV,
                            mlstm_dtype dtype, mlstm_gate_mode gate_mode, void* workspace,
                            size_t workspace_bytes, mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, MLSTM_ALGO_AUTO)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, 128);
  if (s != MLSTM_OK) return s;
  Problem p = make_problem(B, NH, T, DK, DV, 128, gate_mode);
  if (!train_supported(p, dtype) || p.no_norm) return MLSTM_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !i_pre || !f_pre || !H || !saved || !workspace)
    return MLSTM_ERR_INVALID_ARG;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return MLSTM_ERR_INVALID_ARG;
  if (!((C_T && n_T && m_T) || (!C_T && !n_T && !m_T))) return MLSTM_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, i_pre, f_pre, C0, n0, m0, H, C_T, n_T, m_T, saved, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MLSTM_ERR_INVALID_ARG;
  if (saved_bytes < train_saved_bytes(p) || workspace_bytes < fw_train_workspace_bytes(p))
    return MLSTM_ERR_INVALID_ARG;
  p.err = error_word_ptr();
  if (!p.err) return MLSTM_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return from_cuda(launch_family(MLSTM_KERNEL_FW_TRAIN, fw_train_launches(p), st, [&] {
    return launch_fw_train(p, Q, K, V, i_pre, f_pre, C0, n0, m0, H, C_T, n_T, m_T, saved,
                           workspace, st);
  }));
}

mlstm_status mlstm_bw_saved(const void* Q, const void* K, const void* V, const float* i_pre,
                            const float* f_pre, const float* C0, const float* n0, const float* m0,
                            const void* H, const void* saved, size_t saved_bytes, const void* dH,
                            void* dQ, void* dK, void* dV, float* di_pre, float* df_pre,
                            float* dC0, float* dn0, float* dm0, int B, int NH, int T, int DK,
                            int DV, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                            void* workspace, size_t workspace_bytes, mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, MLSTM_ALGO_AUTO)) return MLSTM_ERR_INVALID_ARG;
  mlstm_status s = check_sizes(B, NH, T, DK, DV, 128);
  if (s != MLSTM_OK) return s;
  Problem p = make_problem(B, NH, T, DK, DV, 128, gate_mode);
  if (!train_supported(p, dtype) || p.no_norm) return MLSTM_ERR_UNSUPPORTED;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return MLSTM_ERR_INVALID_ARG;
  if (!Q || !K || !V || !i_pre || !f_pre || !H || !saved || !dH || !dQ || !dK || !dV ||
      !di_pre || !df_pre || !workspace)
    return MLSTM_ERR_INVALID_ARG;
  const void* ptrs[] = {Q,  K,  V,      i_pre,  f_pre, C0,  n0,  m0,  H,        saved,
                        dH, dQ, dK,     dV,     di_pre, df_pre, dC0, dn0, dm0, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MLSTM_ERR_INVALID_ARG;
  if (saved_bytes < train_saved_bytes(p) || workspace_bytes < bw_saved_workspace_bytes(p))
    return MLSTM_ERR_INVALID_ARG;
  p.err = error_word_ptr();
  if (!p.err) return MLSTM_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return from_cuda(launch_family(MLSTM_KERNEL_BW, bw_saved_launches(p), st, [&] {
    return launch_bw_saved(p, Q, K, V, i_pre, f_pre, C0, n0, m0, H, saved, dH, dQ, dK, dV,
                           di_pre, df_pre, dC0, dn0, dm0, workspace, st);
  }));
}

mlstm_status mlstm_step(const void* q, const void* k, const void* v, const float* i_pre,
                        const float* f_pre, float* C, float* n, float* m, void* h, int B, int NH,
                        int DK, int DV, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                        mlstm_stream_t stream) {
  if (!valid_enums(dtype, gate_mode, MLSTM_ALGO_AUTO)) return MLSTM_ERR_INVALID_ARG;
  if (B < 1 || NH < 1 || DK < 1 || DV < 1) return MLSTM_ERR_INVALID_ARG;
  if (DK > 1024 || DV > 1024 || (long long)B * NH > 65535) return MLSTM_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, i_pre, f_pre, C, n, m, h};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return MLSTM_ERR_INVALID_ARG;
  Problem p = make_problem(B, NH, 1, DK, DV, 64, gate_mode);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return from_cuda(launch_family(MLSTM_KERNEL_STEP, step_launches(p), st, [&] {
    return launch_step(p, dtype, q, k, v, i_pre, f_pre, C, n, m, h, st);
  }));
}

mlstm_status mlstm_last_device_error(mlstm_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLSTM_ERR_CUDA;
  uint32_t* w = error_word_ptr();
  if (!w) return MLSTM_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MLSTM_ERR_CUDA;
  g_last_error_word = v;
  if (v != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return MLSTM_ERR_CUDA;
  }
  if (v & kErrWatchdog) return MLSTM_ERR_TIMEOUT;
  if (v) return MLSTM_ERR_DEVICE;
  return MLSTM_OK;
}

}  // extern "C"
