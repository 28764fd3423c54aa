/*
 * mlstm_fw.h -- C ABI of the B200 (sm_100a) chunkwise mLSTM forward library.
 *
 * The operation.  For every (batch b, head h) the mLSTM ("xLSTM: the NX-AI
 * repository behind the extended LSTM architecture", section "Exponential
 * gating, matrix memory, and why the kernels decide everything": exponential
 * gating with normalisation and stabilisation, a matrix memory) runs, for
 * t = 1..T,
 *
 *   lf_t = logsigmoid(f~_t),   li_t = i~_t (EXP) or logsigmoid(i~_t) (SIGMOID)
 *   m_t  = max(lf_t + m_{t-1}, li_t)
 *   C_t  = e^{lf_t + m_{t-1} - m_t} C_{t-1} + e^{li_t - m_t} (s k_t) v_t^T
 *   n_t  = e^{lf_t + m_{t-1} - m_t} n_{t-1} + e^{li_t - m_t} (s k_t)
 *   h_t  = C_t^T q_t / max(|n_t^T q_t|, e^{-m_t}),     s = 1/sqrt(DK)
 *
 * and returns H and the final state (C_T, n_T, m_T).  It is computed
 * chunkwise, as in "Tiled Flash Linear Attention: More Efficient Linear RNN
 * and xLSTM Kernels" (abstract): an inter-chunk state recurrence plus an
 * intra-chunk parallel part that is tiled a second time over query and
 * key/value blocks, so the chunk size is not limited by the tile size.  The
 * sigmoid input gate is that page's mLSTM variant with a sigmoid input gate.
 * The split into a recurrent (chunk-state) call and a parallel (output) call
 * mirrors flash-xlstm-exp 0.1.0 ("Usage": the parallel kernel takes matQ,
 * matK, matV, vecI, vecF and matC_states, vecN_states, scaMinter_states and
 * returns matH_out, vecN_out, vecM_out).
 *
 * Layouts (all row-major, contiguous, 16-byte aligned device pointers):
 *   Q, K    [B, NH, T, DK]   dtype      V, H [B, NH, T, DV]   dtype
 *   i_pre, f_pre [B, NH, T]  fp32       (gate pre-activations)
 *   C0, C_T [B, NH, DK, DV]  fp32       (C stored as sum of (s k) v^T, i.e. [DK, DV])
 *   n0, n_T [B, NH, DK]      fp32       m0, m_T [B, NH] fp32
 * Initial states: C0, n0, m0 are all NULL (zero state, m0 = 0) or all given.
 * Final states: each of C_T, n_T, m_T may be NULL independently.
 *
 * Ownership: the caller owns every buffer, including the workspace; the
 * library allocates no device memory and keeps no state other than a 32-bit
 * device error word.  All calls are asynchronous on `stream`; the outputs are
 * valid once the stream has reached that point.
 *
 * Errors: shape/pointer problems return MLSTM_ERR_INVALID_ARG and launch
 * nothing; shapes outside what a chosen algorithm supports return
 * MLSTM_ERR_UNSUPPORTED and launch nothing; a failed launch returns
 * MLSTM_ERR_CUDA.  Kernels never trap: a bounded wait that runs out sets the
 * device error word, which mlstm_last_device_error() reports as
 * MLSTM_ERR_TIMEOUT.  Inputs must be finite; NaN/inf inputs give unspecified
 * (but memory-safe) results.
 */
#ifndef MLSTM_FW_H_
#define MLSTM_FW_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* mlstm_stream_t;

typedef enum {
  MLSTM_OK = 0,
  MLSTM_ERR_INVALID_ARG = 1,  /* bad pointer, shape or enum value          */
  MLSTM_ERR_UNSUPPORTED = 2,  /* valid, but not supported by that algorithm */
  MLSTM_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed       */
  MLSTM_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out         */
  MLSTM_ERR_DEVICE = 5,       /* another device-side check failed           */
  MLSTM_ERR_SCRATCH_TOO_SMALL = 6 /* needs more than the static scratch array */
} mlstm_status;

typedef enum { MLSTM_DT_F32 = 0, MLSTM_DT_BF16 = 1 } mlstm_dtype;

/* Gate activations.
 *   EXP             log i = i~ (exponential input gate)
 *   SIGMOID         log i = logsigmoid(i~)
 *   SIGMOID_PLAIN   the sigmoid-input-gate variant with reduced computation
 *                   ("Tiled Flash Linear Attention: More Efficient Linear RNN
 *                   and xLSTM Kernels", abstract).  Read as: with both gates
 *                   sigmoids every gate value lies in (0, 1), so the output
 *                   needs no normaliser and no stabiliser,
 *                     h_t = C_t^T q_t  with the unstabilised
 *                     C_t = sig(f~_t) C_{t-1} + sig(i~_t) (s k_t) v_t^T.
 *                   The kernels still carry the stabiliser internally (a
 *                   choice of frame that h does not depend on); what the
 *                   variant removes is the normaliser's reductions and the
 *                   division.  The returned final state is the SIGMOID mode's
 *                   (C_T, n_T in the frame m_T: the unstabilised state is
 *                   e^{m_T} C_T).  Forward, chunk-state, parallel and step
 *                   calls only: the backward and training calls return
 *                   MLSTM_ERR_UNSUPPORTED. */
typedef enum {
  MLSTM_GATE_EXP = 0,
  MLSTM_GATE_SIGMOID = 1,
  MLSTM_GATE_SIGMOID_PLAIN = 2
} mlstm_gate_mode;

/* Which kernels compute the path.
 *   AUTO      TC_FUSED where it is supported and there are at least 74
 *             (b, h) pairs (half the SMs of a 148-SM B200), else TC where it is
 *             supported, else SIMT.  A fixed rule, so workspace sizes computed
 *             for AUTO always match the algorithm the call picks.
 *   SIMT      fp32 CUDA-core kernels (the only choice for fp32 inputs).
 *   TC        bf16 tensor-core kernels, unfused: the state entering every
 *             chunk goes to the workspace (as a bf16 operand copy plus fp32
 *             n) between the state and the output kernels.  Needs d_qk of
 *             128 or 256, d_v of 128 or a multiple of 256 (up to 1024), and a
 *             chunk size that is a multiple of 128 up to 1024, or 64 with
 *             d_qk = 128 (two chunks per 128-row query tile).  With few
 *             (b, h) pairs the state kernel splits each sequence into
 *             segments and adds a fix-up launch; the workspace then also
 *             holds the segments' end states.
 *   TC_FUSED  bf16 tensor-core kernel that carries the chunk state on chip
 *             ("Upgrade roadmap" item 2 of the flash-xlstm-exp page): d_qk =
 *             128, d_v of 64 or 128, chunk size 128. */
typedef enum {
  MLSTM_ALGO_AUTO = 0,
  MLSTM_ALGO_SIMT = 1,
  MLSTM_ALGO_TC = 2,
  MLSTM_ALGO_TC_FUSED = 3
} mlstm_algo;

/* Bytes of workspace mlstm_fw() needs for these arguments (written to
 * *bytes).  Sizes: B, NH >= 1; T >= 0; DK, DV in [1, 1024]; chunk_size a
 * multiple of 64 in [64, 4096].  Returns MLSTM_ERR_INVALID_ARG or
 * MLSTM_ERR_UNSUPPORTED like mlstm_fw() would. */
mlstm_status mlstm_fw_workspace_size(int B, int NH, int T, int DK, int DV, int chunk_size,
                                     mlstm_dtype dtype, mlstm_algo algo, size_t* bytes);

/* The whole forward pass: H and, where non-NULL, the final (C_T, n_T, m_T).
 * T need not be a multiple of chunk_size (the last chunk is ragged); T = 0
 * copies the initial state to the final state.  `workspace` must hold at
 * least mlstm_fw_workspace_size() bytes (it may be NULL when that is 0). */
mlstm_status mlstm_fw(const void* Q, const void* K, const void* V, const float* i_pre,
                      const float* f_pre, const float* C0, const float* n0, const float* m0,
                      void* H, float* C_T, float* n_T, float* m_T, int B, int NH, int T, int DK,
                      int DV, int chunk_size, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                      mlstm_algo algo, void* workspace, size_t workspace_bytes,
                      mlstm_stream_t stream);

/* Bytes of workspace either of the two calls below needs for these
 * arguments (the gate arrays, plus a bf16 copy of the chunk states for the
 * tensor-core parallel call). */
mlstm_status mlstm_fw_substep_workspace_size(int B, int NH, int T, int DK, int DV, int chunk_size,
                                             mlstm_dtype dtype, mlstm_algo algo, size_t* bytes);

/* Recurrent half of the chunkwise pass: the state entering every chunk,
 *   C_states [B, NH, NC, DK, DV], n_states [B, NH, NC, DK], m_states
 *   [B, NH, NC + 1] (m_states[..., k] is the stabiliser entering chunk k;
 *   index NC is the final m), NC = ceil(T / chunk_size),
 * plus the optional final state.  Algorithm SIMT or TC (AUTO picks). */
mlstm_status mlstm_fw_chunk_states(const void* K, const void* V, const float* i_pre,
                                   const float* f_pre, const float* C0, const float* n0,
                                   const float* m0, float* C_states, float* n_states,
                                   float* m_states, float* C_T, float* n_T, float* m_T, int B,
                                   int NH, int T, int DK, int DV, int chunk_size,
                                   mlstm_dtype dtype, mlstm_gate_mode gate_mode, mlstm_algo algo,
                                   void* workspace, size_t workspace_bytes,
                                   mlstm_stream_t stream);

/* Parallel half: H from Q, K, V, the gates and the chunk states produced by
 * mlstm_fw_chunk_states (same m0 and gates).  Optional per-token outputs:
 *   n_out [B, NH, T] = max(|n_t^T q_t|, e^{-m_t}) (the denominator; e^{-m_t}
 *   for MLSTM_GATE_SIGMOID_PLAIN), and
 *   m_out [B, NH, T] = m_t.  Algorithm SIMT or TC (AUTO picks). */
mlstm_status mlstm_fw_parallel(const void* Q, const void* K, const void* V, const float* i_pre,
                               const float* f_pre, const float* m0, const float* C_states,
                               const float* n_states, void* H, float* n_out, float* m_out, int B,
                               int NH, int T, int DK, int DV, int chunk_size, mlstm_dtype dtype,
                               mlstm_gate_mode gate_mode, mlstm_algo algo, void* workspace,
                               size_t workspace_bytes, mlstm_stream_t stream);

/* Workspace bytes of mlstm_bw() for these sizes and input type (sizes as
 * mlstm_fw). */
mlstm_status mlstm_bw_workspace_size(int B, int NH, int T, int DK, int DV, int chunk_size,
                                     mlstm_dtype dtype, size_t* bytes);

/* Backward pass: the gradients of a loss L(H) of the forward's output, given
 * dH = dL/dH, with respect to every input of mlstm_fw.  It recomputes the
 * forward (gates, chunk states, outputs) and then runs the chunkwise
 * gradient: a reverse recurrence over the chunks for the gradient of the
 * state entering each chunk, dQ / dK / dV from the intra-chunk tiles plus the
 * inter-chunk terms, and the gate gradients from the identities
 * dL/d log i_s = k_s . dk_s and dL/d log f_l = sum_{t >= l} (q_t . dq_t -
 * k_t . dk_t) ("Tiled Flash Linear Attention: More Efficient Linear RNN and
 * xLSTM Kernels": the chunkwise split applied to the gradient).
 * Two paths.  bf16 inputs with DK of 128 or 256, a DV the tensor-core forward
 * takes (128, or a multiple of 256 up to 1024) and T >= 128: the whole
 * backward runs on tensor cores in 128-token chunks whatever chunk_size says
 * (the gradients do not depend on the chunking, up to rounding); the
 * recomputed forward, the reverse state recurrence and the gradient GEMMs
 * use bf16 operands with fp32 accumulation.  Everything else: fp32 CUDA-core
 * gradient kernels on chunk_size (the forward recomputed on the tensor cores
 * for bf16 shapes the TC algorithm supports).  The derivation and its
 * stabilisation are in the header of the implementation files (bwd.cu,
 * tc_bwd.cu).
 *   Q, K, V, dH in `dtype` as in mlstm_fw; dQ, dK, dV out, same shapes and
 *   dtype; di_pre, df_pre [B, NH, T] fp32 out; C0/n0/m0 all given or all
 *   null; dC0 [B, NH, DK, DV], dn0 [B, NH, DK], dm0 [B, NH] fp32 out
 *   (nullable; zero-state calls get the gradient a zero initial state would
 *   have).  The loss is on H only (no gradient arrives through C_T/n_T/m_T).
 * Errors as mlstm_fw; the workspace must hold mlstm_bw_workspace_size bytes.
 * 10 to 14 launches, asynchronous on `stream`. */
mlstm_status mlstm_bw(const void* Q, const void* K, const void* V, const float* i_pre,
                      const float* f_pre, const float* C0, const float* n0, const float* m0,
                      const void* dH, void* dQ, void* dK, void* dV, float* di_pre, float* df_pre,
                      float* dC0, float* dn0, float* dm0, int B, int NH, int T, int DK, int DV,
                      int chunk_size, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                      void* workspace, size_t workspace_bytes, mlstm_stream_t stream);

/* Training pair ("Tiled Flash Linear Attention: More Efficient Linear RNN and
 * xLSTM Kernels": the forward's per-token normaliser and stabiliser outputs
 * serve the backward).  mlstm_fw_train is the forward pass of mlstm_fw (same
 * arguments and outputs, no chunk size) that also keeps, in a caller buffer
 * `saved`, what the backward needs: the bf16 chunk states and fp32 n states
 * entering every 128-token chunk and, per token, the signed denominator
 * copysign(max(|n.q|, e^{-m}), n.q) and the stabiliser m.  mlstm_bw_saved is
 * mlstm_bw (same gradients) that takes `saved` and the forward's H instead of
 * recomputing the forward.  Both run in 128-token chunks on the tensor cores
 * and exist only for the shapes of the tensor-core backward: bf16 inputs,
 * DK of 128 or 256, DV of 128 or a multiple of 256 up to 1024, T >= 128
 * (else MLSTM_ERR_UNSUPPORTED, from mlstm_train_sizes first).
 * mlstm_train_sizes: bytes of `saved` and of each call's workspace.
 * Buffers 16-byte aligned; C0/n0/m0 and C_T/n_T/m_T each all given or all
 * null; `saved` must not change between the two calls.  mlstm_fw_train: 4 or
 * 5 launches; mlstm_bw_saved: 10; asynchronous on `stream`.  Errors as
 * mlstm_fw. */
mlstm_status mlstm_train_sizes(int B, int NH, int T, int DK, int DV, mlstm_dtype dtype,
                               size_t* saved_bytes, size_t* fw_workspace_bytes,
                               size_t* bw_workspace_bytes);
mlstm_status mlstm_fw_train(const void* Q, const void* K, const void* V, const float* i_pre,
                            const float* f_pre, const float* C0, const float* n0, const float* m0,
                            void* H, float* C_T, float* n_T, float* m_T, void* saved,
                            size_t saved_bytes, int B, int NH, int T, int DK, int DV,
                            mlstm_dtype dtype, mlstm_gate_mode gate_mode, void* workspace,
                            size_t workspace_bytes, mlstm_stream_t stream);
mlstm_status mlstm_bw_saved(const void* Q, const void* K, const void* V, const float* i_pre,
                            const float* f_pre, const float* C0, const float* n0, const float* m0,
                            const void* H, const void* saved, size_t saved_bytes, const void* dH,
                            void* dQ, void* dK, void* dV, float* di_pre, float* df_pre,
                            float* dC0, float* dn0, float* dm0, int B, int NH, int T, int DK,
                            int DV, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                            void* workspace, size_t workspace_bytes, mlstm_stream_t stream);

/* Single-token step (decode), the recurrence of mlstm_fw for T = 1: advances
 * the state of every (b, h) by one token in place and writes that token's
 * output ("xLSTM: the NX-AI repository behind the extended LSTM
 * architecture", section "Exponential gating, matrix memory, and why the
 * kernels decide everything": the step kernel is a separate choice from the
 * chunkwise one).
 *   q, k [B, NH, DK] and v, h [B, NH, DV] in `dtype` (device, contiguous);
 *   i_pre, f_pre [B, NH] fp32;
 *   C [B, NH, DK, DV], n [B, NH, DK], m [B, NH] fp32: the state before the
 *   token on entry, after it on return (a zero state is C = n = 0, m = 0).
 *   m' = max(logsigmoid(f~) + m, li), C' = fa C + ia (s k) v^T,
 *   n' = fa n + ia s k, h = C'^T q / max(|n'^T q|, e^{-m'}), s = 1/sqrt(DK)
 *   (MLSTM_GATE_SIGMOID_PLAIN: h = e^{m'} C'^T q).
 * Sizes: B, NH >= 1, DK, DV in [1, 1024].  No workspace; asynchronous on
 * `stream`: one launch (a thread-block cluster per head), or two when d_v is
 * not a multiple of 4 and above 256 (a head then spans more column tiles
 * than one cluster holds).  All pointers 16-byte aligned and non-null, else
 * MLSTM_ERR_INVALID_ARG before any launch. */
mlstm_status mlstm_step(const void* q, const void* k, const void* v, const float* i_pre,
                        const float* f_pre, float* C, float* n, float* m, void* h, int B, int NH,
                        int DK, int DV, mlstm_dtype dtype, mlstm_gate_mode gate_mode,
                        mlstm_stream_t stream);

/* Synchronises `stream`, then returns and clears the device error word:
 * MLSTM_OK, MLSTM_ERR_TIMEOUT (a bounded wait ran out) or MLSTM_ERR_DEVICE;
 * MLSTM_ERR_CUDA if the synchronisation itself failed. */
mlstm_status mlstm_last_device_error(mlstm_stream_t stream);

/* The raw device error word read by the last mlstm_last_device_error() call:
 * bit 0 a bounded wait ran out, bit 1 a bounds check failed, bit 2 a TMEM
 * allocation check failed; bits 8..15 identify the first wait that ran out
 * (a kernel-specific site number, for diagnosis). */
uint32_t mlstm_last_device_error_word(void);

/* Spin limit of every bounded device-side wait (default 2^26 polls, about a
 * second or more).  Affects launches made after the call.  0 restores the
 * default.  Not thread-safe with concurrent launches. */
void mlstm_set_watchdog(uint64_t max_polls);

/* Failure-detection self-test.  Enqueues on `stream` one tiny kernel whose
 * only waiting thread waits on an mbarrier that nothing ever completes,
 * through the same bounded wait that every kernel of the library uses.  After
 * the watchdog limit (mlstm_set_watchdog) the wait gives up, sets bit 0 of the
 * device error word and the site 0xF7 in bits 8..15, and the kernel returns
 * normally: the next mlstm_last_device_error() on the stream reports
 * MLSTM_ERR_TIMEOUT and the CUDA context stays usable.  Nothing traps or
 * faults.  Returns MLSTM_OK once enqueued, MLSTM_ERR_CUDA if the launch
 * fails.  The pages have no counterpart: it exists to exercise the watchdog
 * that backs every wait of the forward pass. */
mlstm_status mlstm_watchdog_selftest(mlstm_stream_t stream);

/* Kernel families, as reported by the profiling calls below. */
typedef enum {
  MLSTM_KERNEL_GATES = 0,         /* gate preprocessing (2 launches per call)  */
  MLSTM_KERNEL_SIMT_STATES = 1,   /* fp32 chunk-state recurrence               */
  MLSTM_KERNEL_SIMT_PARALLEL = 2, /* fp32 intra-chunk + inter-chunk output     */
  MLSTM_KERNEL_TC_STATES = 3,     /* tensor-core chunk-state recurrence        */
  MLSTM_KERNEL_TC_PARALLEL = 4,   /* tensor-core intra-chunk TFLA kernel       */
  MLSTM_KERNEL_TC_FUSED = 5,      /* tensor-core fused kernel                  */
  MLSTM_KERNEL_STEP = 6,          /* single-token step (1 or 2 launches)       */
  MLSTM_KERNEL_BW = 7,            /* backward pass (10 to 14 launches per call) */
  MLSTM_KERNEL_FW_TRAIN = 8,      /* training forward (4 or 5 launches)        */
  MLSTM_KERNEL_COUNT = 9
} mlstm_kernel_id;

/* Total number of kernels this library has enqueued since it was loaded. */
uint64_t mlstm_kernel_launches(void);

/* Measurement hook, off by default.  While on, every kernel family launch is
 * bracketed by a pair of CUDA events on the launch stream. */
void mlstm_profile_enable(int on);

/* Waits for the recorded events, then writes, per kernel family id
 * (0 <= id < n, n <= MLSTM_KERNEL_COUNT), the summed device time in ms and the
 * number of launches since the previous read, and clears the record.
 * Returns MLSTM_ERR_CUDA if an event query fails. */
mlstm_status mlstm_profile_read(double* ms, uint64_t* launches, int n);

/* Static name of a kernel family id (never NULL). */
const char* mlstm_kernel_name(int id);

/* The forward pass for callers that cannot allocate device memory.  The
 * pages have no counterpart: this is a deployment variant of mlstm_fw().
 *
 * Some callers hold their inputs and outputs but have no way to allocate a
 * workspace -- a plugin hook in a host framework that hands over tensors but
 * no allocator, or a latency-critical loop that forbids cudaMalloc after
 * start-up because it can synchronise the device.  This call takes the same
 * arguments as mlstm_fw() minus the workspace and uses a scratch array that is
 * part of the library's device image instead; it never allocates.
 *
 * Limits: the array holds mlstm_fw_static_scratch_capacity() bytes (16 MiB),
 * which every GPU that loads the library keeps until the process exits.  A
 * problem whose mlstm_fw_workspace_size() is larger returns
 * MLSTM_ERR_SCRATCH_TOO_SMALL and launches nothing.  All calls share the one
 * array, so calls that overlap on the GPU (other streams or host threads)
 * race and must be serialised by the caller.  The first call in a CUDA context
 * looks up the array's address with that context current and caches it for
 * that context; make it before any stream capture.  After a cudaDeviceReset
 * (which ends the context) the next call looks the address up again.  Other
 * errors are those of mlstm_fw(). */
mlstm_status mlstm_fw_static_scratch(const void* Q, const void* K, const void* V,
                                     const float* i_pre, const float* f_pre, const float* C0,
                                     const float* n0, const float* m0, void* H, float* C_T,
                                     float* n_T, float* m_T, int B, int NH, int T, int DK, int DV,
                                     int chunk_size, mlstm_dtype dtype,
                                     mlstm_gate_mode gate_mode, mlstm_algo algo,
                                     mlstm_stream_t stream);

/* Bytes of the static scratch array used by mlstm_fw_static_scratch(). */
size_t mlstm_fw_static_scratch_capacity(void);

/* Static text for a status code (never NULL). */
const char* mlstm_status_string(mlstm_status status);

/* Library ABI version: 100 * major + minor. */
int mlstm_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLSTM_FW_H_ */
