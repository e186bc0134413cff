/*
 * mlstm.h -- C ABI of the B200 mLSTM / retention recurrence library (libmlstm.so).
 *
 * The recurrence (DeepChrInteract-v2 "mLSTM Model", "Core idea"; gates stabilised
 * in log space as stated there):
 *
 *     m_t = max(log f_t + m_{t-1}, log i_t)        log f_t = logsigmoid(ftilde_t),
 *                                                  log i_t = itilde_t
 *     C_t = f'_t C_{t-1} + i'_t v_t k_t^T          f'_t = exp(log f_t + m_{t-1} - m_t)
 *     n_t = f'_t n_{t-1} + i'_t k_t                i'_t = exp(itilde_t - m_t)
 *     h_t = o_t * (C_t q_t) / max(|n_t . q_t|, exp(-m_t))
 *
 * C and n are kept in stabilised units (the raw state times exp(-m_t)); the floor
 * exp(-m_t) is the floor 1 of the raw form, so h does not depend on the stabiliser.
 *
 * Retention flag (Edifice.Attention.RetNet, "Key Innovation", recurrent form, and
 * "Multi-Scale Retention"): i = 1, f = gamma_h = 1 - 2^(-5-h) for head h (0-based),
 * no normaliser, no stabiliser, no output gate:  C_t = gamma_h C_{t-1} + v_t k_t^T,
 * h_t = C_t q_t.
 *
 * Block-diagonal memory (Edifice.Recurrent.XLSTMv2, "Key Improvements" #1):
 * num_blocks = nb splits each head's q, k (DHQK) and v, o, h (DHV) into nb
 * contiguous slices; block j owns C_j [DHV/nb x DHQK/nb] and n_j [DHQK/nb] and
 * shares the head's gates and m.
 *
 * Two evaluation orders of the same recurrence (RetNet "Triple Paradigm"):
 *   mlstm_fwd_chunkwise  chunkwise-parallel prefill over a whole sequence,
 *   mlstm_step           one recurrent decode step, state updated in place.
 *
 * Conventions for every entry point
 *   - Every data pointer is DEVICE memory owned by the caller.  The library never
 *     allocates, frees or keeps a pointer past the call.  Scratch memory of the
 *     prefill is a caller-supplied workspace sized by
 *     mlstm_fwd_chunkwise_workspace_size().  (One exception, for callers that cannot
 *     allocate: mlstm_fwd_chunkwise_noalloc uses a scratch buffer built into the
 *     library instead; see there.)
 *   - All tensors are dense, row-major (last index fastest), 16-byte aligned.
 *   - q, k, v, o, h use the dtype of the params (fp32 or bf16); gates are always
 *     fp32; the state (C, n, m) is always fp32.
 *   - Work is enqueued on `stream`; the call returns without synchronising.
 *   - Arguments are validated on the host before anything is enqueued; on any
 *     error nothing is enqueued and no output is touched.  Errors raised by the
 *     CUDA runtime at launch are returned as MLSTM_ERR_CUDA.
 *   - Device-side waits are bounded.  The tensor-core prefill kernels wait on
 *     mbarriers for their own copies and tensor-core results; each wait gives up
 *     after params->wait_limit_cycles SM cycles (0 = about 4e9, ~2 s).  A wait that
 *     runs out is reported after the work, by mlstm_fwd_chunkwise_status
 *     (MLSTM_ERR_TIMEOUT), never by a hang: the kernel stops issuing work, waits for
 *     the copies it has in flight, frees its tensor memory and returns.
 *   - Calls that share no output buffer may run concurrently on different
 *     streams.  The library holds no global mutable state, except the built-in
 *     scratch buffer of mlstm_fwd_chunkwise_noalloc: calls of that entry point
 *     whose GPU work overlaps race on it, so they must not overlap.
 */
#ifndef MLSTM_H_
#define MLSTM_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying types as cudaStream_t / cudaEvent_t of the CUDA runtime. */
typedef struct CUstream_st* mlstm_stream_t;
typedef struct CUevent_st* mlstm_event_t;

typedef enum {
  MLSTM_OK = 0,
  MLSTM_ERR_NULL = 1,       /* a required pointer is NULL                          */
  MLSTM_ERR_SHAPE = 2,      /* a size is negative, inconsistent or unsupported     */
  MLSTM_ERR_DTYPE = 3,      /* dtype is not MLSTM_F32 or MLSTM_BF16                */
  MLSTM_ERR_ALIGN = 4,      /* a pointer is not 16-byte aligned                    */
  MLSTM_ERR_WORKSPACE = 5,  /* workspace NULL or smaller than the size query       */
  MLSTM_ERR_CUDA = 6,       /* the CUDA runtime reported an error at launch        */
  MLSTM_ERR_ALIAS = 7,      /* an output overlaps an input it must not overlap     */
  MLSTM_ERR_TIMEOUT = 8,    /* a bounded device-side wait ran out (reported by the
                               status calls after the work has finished)           */
  MLSTM_ERR_BOUNDS = 9      /* bounds-checked build only: an access failed its check
                               and was skipped (status calls; see
                               mlstm_fwd_chunkwise_bounds_record)                  */
} mlstm_status_t;

typedef enum { MLSTM_F32 = 0, MLSTM_BF16 = 1 } mlstm_dtype_t;

/* Sizes of one chunkwise prefill.  B, NH >= 0; S >= 0; DHQK, DHV >= 1 and
 * divisible by num_blocks (>= 1); chunk >= 1 (the intra-chunk tile length; the
 * result does not depend on it beyond rounding; S need not be a multiple of it).
 * retention: 0 = mLSTM, 1 = retention.
 * wait_limit_cycles: bound of each device-side wait of the tensor-core kernels in SM
 * cycles; 0 (or negative) = the default, about 4e9 (~2 s).  Only tests and watchdogs
 * set it: a limit shorter than a copy takes makes the call fail with MLSTM_ERR_TIMEOUT
 * (see mlstm_fwd_chunkwise_status).  Ignored by the other entry points. */
typedef struct {
  int B, NH, S, DHQK, DHV;
  int chunk;
  int num_blocks;
  mlstm_dtype_t dtype;
  int retention;
  long long wait_limit_cycles;
} mlstm_fwd_params_t;

/* Sizes of one decode step (one token per sequence). */
typedef struct {
  int B, NH, DHQK, DHV;
  int num_blocks;
  mlstm_dtype_t dtype;
  int retention;
} mlstm_step_params_t;

/* How a prefill will be executed (for tests, benchmarks and logs). */
typedef struct {
  int tensor_core;      /* 1: tcgen05/TMEM kernels; 0: SIMT fp32 kernels            */
  int segments;         /* sequence segments run in parallel per head (>= 1)        */
  int dv_tile;          /* value rows of the state owned by one CTA                 */
  int ctas_main;        /* CTAs of the dominant (intra-chunk + state walk) kernel   */
  int kernels;          /* kernel launches one call enqueues                         */
  size_t workspace_bytes;
  int seg0_chunks;      /* chunks of the first segment (tensor-core path; it walks while the
                           others are summarised, so it may be longer)                */
  int seg_chunks;       /* chunks of each later segment (the last may be shorter)    */
  int summary_units;    /* segment summaries computed before the walk (0: one segment) */
} mlstm_fwd_plan_t;

/* Workspace bytes mlstm_fwd_chunkwise needs for these sizes (0 if none); returns
 * 0 as well for invalid sizes, which mlstm_fwd_chunkwise then rejects. */
size_t mlstm_fwd_chunkwise_workspace_size(const mlstm_fwd_params_t* p);

/* Fills *plan for these sizes.  MLSTM_ERR_NULL / MLSTM_ERR_SHAPE / MLSTM_ERR_DTYPE
 * as for mlstm_fwd_chunkwise. */
mlstm_status_t mlstm_fwd_chunkwise_plan(const mlstm_fwd_params_t* p, mlstm_fwd_plan_t* plan);

/*
 * Chunkwise-parallel prefill of a whole sequence (RetNet "Triple Paradigm",
 * chunkwise mode: O(S) work, state carried between chunks).
 *
 *   q, k    [B,NH,S,DHQK]  dtype          required (if S > 0)
 *   v       [B,NH,S,DHV]   dtype          required (if S > 0)
 *   igate   [B,NH,S]       fp32           input-gate pre-activation itilde; required
 *                                          unless retention (then ignored, may be NULL)
 *   fgate   [B,NH,S]       fp32           forget-gate pre-activation ftilde; same rule
 *   ogate   [B,NH,S,DHV]   dtype          already-activated output gate o_t; NULL = 1;
 *                                          ignored in retention mode
 *   C0      [B,NH,nb,DHV/nb,DHQK/nb] fp32 initial state (value row, key column),
 *   n0      [B,NH,nb,DHQK/nb]        fp32 stabilised units; NULL = zeros.  n0 and m0
 *   m0      [B,NH]                   fp32 are ignored in retention mode.
 *   h       [B,NH,S,DHV]   dtype          output; required (if S > 0)
 *   C_out, n_out, m_out               fp32 final state in the sequential recurrence's
 *                                          representation (same m_S); NULL = not written.
 *                                          May alias C0 / n0 / m0 exactly (in place);
 *                                          any other overlap with an input is an error.
 *   workspace, workspace_bytes        device scratch of at least
 *                                          mlstm_fwd_chunkwise_workspace_size(p) bytes,
 *                                          16-byte aligned; contents need not be
 *                                          initialised and are garbage afterwards.
 *                                          Two calls in flight must not share it.
 *   stream                            CUDA stream (NULL = legacy default stream)
 */
mlstm_status_t mlstm_fwd_chunkwise(const mlstm_fwd_params_t* p,
                                   const void* q, const void* k, const void* v,
                                   const float* igate, const float* fgate, const void* ogate,
                                   const float* C0, const float* n0, const float* m0,
                                   void* h, float* C_out, float* n_out, float* m_out,
                                   void* workspace, size_t workspace_bytes,
                                   mlstm_stream_t stream);

/* mlstm_fwd_chunkwise, plus: if main_begin / main_end are non-NULL, they are recorded
 * on `stream` immediately before and after the dominant kernel (intra-chunk
 * contraction + state walk), so its duration can be timed with cudaEventElapsedTime. */
mlstm_status_t mlstm_fwd_chunkwise_timed(const mlstm_fwd_params_t* p,
                                         const void* q, const void* k, const void* v,
                                         const float* igate, const float* fgate, const void* ogate,
                                         const float* C0, const float* n0, const float* m0,
                                         void* h, float* C_out, float* n_out, float* m_out,
                                         void* workspace, size_t workspace_bytes,
                                         mlstm_stream_t stream,
                                         mlstm_event_t main_begin, mlstm_event_t main_end);

/*
 * mlstm_fwd_chunkwise without a caller workspace (the pages have no counterpart; this
 * is a deployment convenience).  For callers that cannot call cudaMalloc -- for example
 * code running inside a host framework that owns all device memory and forbids outside
 * allocations, or a loop where an allocation's implicit device synchronisation is not
 * acceptable.  The scratch memory comes from one fixed buffer compiled into the library
 * (mlstm_noalloc_scratch_bytes() bytes, 32 MiB), which every GPU that loads the library
 * holds until the process exits.  Arguments are those of mlstm_fwd_chunkwise minus the
 * workspace.  Returns MLSTM_ERR_WORKSPACE if the sizes need more scratch than the buffer
 * holds (see mlstm_fwd_chunkwise_workspace_size).  The first call on a device looks up
 * the buffer's device address (cudaGetSymbolAddress) and caches it; make that first
 * call before any stream capture.  Nothing is allocated or freed.  All calls share the
 * buffer: calls whose GPU work overlaps (other streams, other host threads) race.  The
 * buffer used is the one of the CURRENT device, so every pointer must be memory of the
 * current device.  Bounded-wait failures are read with mlstm_fwd_chunkwise_noalloc_status.
 */
mlstm_status_t mlstm_fwd_chunkwise_noalloc(const mlstm_fwd_params_t* p,
                                           const void* q, const void* k, const void* v,
                                           const float* igate, const float* fgate, const void* ogate,
                                           const float* C0, const float* n0, const float* m0,
                                           void* h, float* C_out, float* n_out, float* m_out,
                                           mlstm_stream_t stream);

/* Size in bytes of the built-in scratch buffer used by mlstm_fwd_chunkwise_noalloc. */
size_t mlstm_noalloc_scratch_bytes(void);

/*
 * Outcome of the bounded device-side waits of the last prefill enqueued on `stream` with
 * `workspace` (mlstm_fwd_chunkwise, _timed, _reversed or _msr, called with the same params):
 * synchronises `stream`, then reads the error word the tensor-core kernels keep in the first
 * bytes of the workspace (each prefill call clears it first).
 *   MLSTM_OK           no wait ran out (always, for sizes that run the SIMT kernels, which
 *                      have no such waits)
 *   MLSTM_ERR_TIMEOUT  a wait ran out (params->wait_limit_cycles); that call's outputs and
 *                      final state are unspecified, the workspace can be used again
 *   MLSTM_ERR_BOUNDS   (bounds-checked build only) an access failed its check and was
 *                      skipped; outputs unspecified; mlstm_fwd_chunkwise_bounds_record says
 *                      which
 *   MLSTM_ERR_CUDA     the synchronisation or the read failed (for example an earlier
 *                      asynchronous error on the stream)
 *   MLSTM_ERR_NULL / _SHAPE / _DTYPE as for mlstm_fwd_chunkwise (workspace NULL: _NULL when
 *                      the sizes have a workspace)
 * mlstm_fwd_chunkwise_noalloc_status does the same for mlstm_fwd_chunkwise_noalloc, reading
 * the built-in scratch buffer of the current device.
 */
mlstm_status_t mlstm_fwd_chunkwise_status(const mlstm_fwd_params_t* p, const void* workspace,
                                          mlstm_stream_t stream);
mlstm_status_t mlstm_fwd_chunkwise_noalloc_status(const mlstm_fwd_params_t* p, mlstm_stream_t stream);

/*
 * Bounds-checked debug build.  libmlstm_checked.so is the same library compiled with every
 * plain global access of the tensor-core prefill kernels (gate preparation, segment
 * summaries, walk) checked against its buffer's extent, every TMA copy's coordinates checked
 * against the copy rules (innermost coordinate on a 16-byte boundary, stores from
 * non-negative coordinates, the box overlapping its tensor) and every offset into the h
 * staging tile checked against the tile, before the access is made.  A failing check skips
 * the access and records the first failure in the workspace; nothing traps.  The status calls
 * above then return MLSTM_ERR_BOUNDS.  The checks cost time: the build is for tests.
 *
 * mlstm_bounds_checked: 1 in libmlstm_checked.so, 0 in libmlstm.so.
 * mlstm_fwd_chunkwise_bounds_record: synchronises `stream` and copies the first failure of
 * the last prefill with `workspace` (arguments as for mlstm_fwd_chunkwise_status) to *site (0:
 * none; the site numbers name the kernel step and buffer, see the library's bounds.cuh),
 * *index (the offending index or coordinate) and *extent (its limit).  Any of the three
 * pointers may be NULL.  In libmlstm.so it reports no failure.  MLSTM_ERR_CUDA if the read
 * fails; argument errors as for mlstm_fwd_chunkwise_status.
 */
int mlstm_bounds_checked(void);
mlstm_status_t mlstm_fwd_chunkwise_bounds_record(const mlstm_fwd_params_t* p, const void* workspace,
                                                 mlstm_stream_t stream, int* site, long long* index,
                                                 long long* extent);

/*
 * The same prefill over the reversed sequence: token S-1 is read first and token 0 last;
 * h[t] is written at the token's own position t, and the final state is the state after
 * token 0.  This is the backward direction of a bidirectional encoder (DeepChrInteract-v2
 * "mLSTM Model": a bidirectional wrapper so that the encoder sees context from both sides);
 * a caller combines it with mlstm_fwd_chunkwise as it likes.  Arguments as for
 * mlstm_fwd_chunkwise; workspace: mlstm_fwd_chunkwise_reversed_workspace_size bytes.  On the
 * tensor-core path (bf16, chunk 64) the kernels read the chunks and their rows backwards in
 * place (the chunks stay aligned to multiples of 64 rows from the start of the sequence, so a
 * ragged chunk is the first one taken) and the workspace is the forward's; elsewhere it also
 * holds reversed copies of the inputs and of h and must not overlap any argument.
 */
size_t mlstm_fwd_chunkwise_reversed_workspace_size(const mlstm_fwd_params_t* p);
mlstm_status_t mlstm_fwd_chunkwise_reversed(const mlstm_fwd_params_t* p,
                                            const void* q, const void* k, const void* v,
                                            const float* igate, const float* fgate, const void* ogate,
                                            const float* C0, const float* n0, const float* m0,
                                            void* h, float* C_out, float* n_out, float* m_out,
                                            void* workspace, size_t workspace_bytes,
                                            mlstm_stream_t stream);

/*
 * The prefill with the normaliser of Edifice.Recurrent.XLSTMv2 ("Key Improvements" #2): a
 * scalar n_t = f_t n_{t-1} + i_t and a learnable bias,  h_t = o_t (C_t q_t) / max(|n_t + bias|, 1)
 * (gates and stabiliser as above; in stabilised units the denominator is
 * max(|n'_t + bias e^{-m_t}|, e^{-m_t})).  n depends on the gates only, so it is one value per
 * (batch, head), shared by the head's blocks.  Arguments as for mlstm_fwd_chunkwise, except:
 *   bias    [NH]   fp32   required (if S > 0)
 *   n0, n_out [B,NH] fp32 stabilised scalar normaliser (NULL = zero / not written)
 * retention is rejected (MLSTM_ERR_SHAPE: retention has no normaliser).  Runs on the
 * tensor-core kernels for the sizes mlstm_fwd_chunkwise runs there (bf16, chunk 64, block
 * widths 64/128/256; status calls as for mlstm_fwd_chunkwise), else on the SIMT fp32 kernels;
 * workspace: mlstm_fwd_chunkwise_scalar_normaliser_workspace_size.
 */
size_t mlstm_fwd_chunkwise_scalar_normaliser_workspace_size(const mlstm_fwd_params_t* p);
mlstm_status_t mlstm_fwd_chunkwise_scalar_normaliser(const mlstm_fwd_params_t* p,
                                                     const void* q, const void* k, const void* v,
                                                     const float* igate, const float* fgate, const void* ogate,
                                                     const float* bias,
                                                     const float* C0, const float* n0, const float* m0,
                                                     void* h, float* C_out, float* n_out, float* m_out,
                                                     void* workspace, size_t workspace_bytes,
                                                     mlstm_stream_t stream);

/*
 * Backward of the recurrence: gradients of a loss with respect to the inputs of
 * mlstm_fwd_chunkwise, given its gradient dh with respect to h (and optionally dC, dn
 * with respect to the final state).  Reverse-mode differentiation of the sequential
 * steps (RetNet "Triple Paradigm": the parallel / chunkwise form is the training mode;
 * this computes its gradients).  h does not depend on the stabiliser m, so the steps
 * are differentiated with m held fixed, which is exact; the final state (C'_S, n'_S) is
 * differentiated in stabilised units with m_S fixed (dC = exp(m_S) dL/dC_S for a loss on
 * the raw state C_S = exp(m_S) C'_S), and the initial state enters as exp(m0) C0, so
 * dm0 = <dC0, C0> + dn0 . n0.
 *
 *   p                       sizes as for the forward (chunk is ignored).  Supported: block
 *                           key and value widths DHQK/nb, DHV/nb <= 256 with
 *                           (DHV/nb) x (DHQK/nb + 1) fp32 of state in one CTA's shared memory
 *                           (about 48 K values), else MLSTM_ERR_SHAPE.
 *   q, k, v, igate, fgate,  the forward's inputs, same layouts and rules (ogate, C0, n0,
 *   ogate, C0, n0, m0       m0 may be NULL)
 *   dh      [B,NH,S,DHV]   dtype   gradient of h; required (if S > 0)
 *   dC      [B,NH,nb,DHV/nb,DHQK/nb] fp32  gradient of C_out (stabilised units); NULL = 0
 *   dn      [B,NH,nb,DHQK/nb]        fp32  gradient of n_out; NULL = 0; ignored in retention
 *   dq, dk  [B,NH,S,DHQK]  fp32    required (if S > 0)
 *   dv      [B,NH,S,DHV]   fp32    required (if S > 0)
 *   digate, dfgate [B,NH,S] fp32   gradients of the gate pre-activations; NULL = not
 *                                  written; not written in retention mode
 *   dogate  [B,NH,S,DHV]   fp32    gradient of the output gate; written only if ogate
 *                                  is given (and not in retention mode)
 *   dC0 [B,NH,nb,DHV/nb,DHQK/nb], dn0 [B,NH,nb,DHQK/nb], dm0 [B,NH]  fp32  gradients of the
 *                                  initial state; NULL = not written; dn0 and dm0 not in
 *                                  retention mode
 *   workspace, workspace_bytes     at least mlstm_bwd_workspace_size(p) bytes, 16-byte
 *                                  aligned; contents need not be initialised; required
 *                                  whenever that size is nonzero (B*NH > 0, also for S = 0)
 * Outputs must not overlap the inputs, each other or the workspace (MLSTM_ERR_ALIAS).
 * Other conventions as for the forward.
 */
size_t mlstm_bwd_workspace_size(const mlstm_fwd_params_t* p);
mlstm_status_t mlstm_bwd(const mlstm_fwd_params_t* p,
                         const void* q, const void* k, const void* v,
                         const float* igate, const float* fgate, const void* ogate,
                         const float* C0, const float* n0, const float* m0,
                         const void* dh, const float* dC, const float* dn,
                         float* dq, float* dk, float* dv, float* digate, float* dfgate, float* dogate,
                         float* dC0, float* dn0, float* dm0,
                         void* workspace, size_t workspace_bytes, mlstm_stream_t stream);

/*
 * The steps either side of retention in a multi-scale retention block
 * (Edifice.Attention.RetNet, "Key Innovation": Y = (Q Theta) D (K Theta)^T V; "Multi-Scale
 * Retention (MSR)": GroupNorm over heads, Y = SiLU(X W_G) * GroupNorm(Retention(X))).  The
 * projections X W_G and W_O are matrix products outside the library.
 *
 * mlstm_theta_rotate: q_out = q Theta, k_out = k Theta.  Entries (2j, 2j+1) of each head
 * vector are one complex number, multiplied by e^{i p theta_j} at sequence position
 * p = pos0[b] + t, theta_j = theta_base^{-2j/DHQK}; the same rotation on q and k makes the
 * scores depend on positions only through their difference.
 *   p            B, NH, S, DHQK, dtype used (the rest ignored but validated as for the
 *                forward).  DHQK a multiple of 8 (bf16) or 4 (fp32), at most 2048 / 1024.
 *   q, k         [B,NH,S,DHQK]  dtype   required (if the tensor is not empty)
 *   pos0         [B]  int64, device, 8-byte aligned: position of token 0 of each sequence
 *                (a decode step passes the sequence's current length); NULL = 0
 *   theta_base   > 0 (10000 is the common choice)
 *   q_out, k_out [B,NH,S,DHQK]  dtype   may equal q / k exactly (in place); no other overlap
 *
 * mlstm_group_norm_gate: each (batch, head, token) row of DHV values is one group,
 * y = (h - mean) / sqrt(var + eps) * weight + bias (biased variance), then y *= silu(g).
 *   p            B, NH, S, DHV, dtype used.  DHV = 8 x 2^k (bf16) or 4 x 2^k (fp32), k <= 8.
 *   h, y         [B,NH,S,DHV]  dtype   y may equal h exactly (in place)
 *   g            [B,NH,S,DHV]  dtype   gate pre-activation X W_G; NULL = no gate
 *   weight, bias [NH*DHV] fp32 per channel; NULL = 1 / 0
 *   eps          >= 0
 *
 * mlstm_fwd_chunkwise_msr: the block in one call: rotate q and k (into the workspace), run
 * mlstm_fwd_chunkwise on them (retention or mLSTM per p->retention; no ogate), GroupNorm
 * and gate h into y (the kernel of mlstm_group_norm_gate, in place on y).  Other
 * arguments as for mlstm_fwd_chunkwise and the two calls
 * above; workspace: mlstm_fwd_chunkwise_msr_workspace_size (rotated q and k plus the
 * forward's).  g, weight, bias, pos0, q and k must not overlap y, the state outputs or the
 * workspace (MLSTM_ERR_ALIAS).
 */
mlstm_status_t mlstm_theta_rotate(const mlstm_fwd_params_t* p, const void* q, const void* k,
                                  const long long* pos0, float theta_base, void* q_out, void* k_out,
                                  mlstm_stream_t stream);
mlstm_status_t mlstm_group_norm_gate(const mlstm_fwd_params_t* p, const void* h, const void* g,
                                     const float* weight, const float* bias, float eps, void* y,
                                     mlstm_stream_t stream);
size_t mlstm_fwd_chunkwise_msr_workspace_size(const mlstm_fwd_params_t* p);
mlstm_status_t mlstm_fwd_chunkwise_msr(const mlstm_fwd_params_t* p,
                                       const void* q, const void* k, const void* v,
                                       const float* igate, const float* fgate,
                                       const long long* pos0, float theta_base,
                                       const void* g, const float* gn_weight, const float* gn_bias, float eps,
                                       const float* C0, const float* n0, const float* m0,
                                       void* y, float* C_out, float* n_out, float* m_out,
                                       void* workspace, size_t workspace_bytes, mlstm_stream_t stream);

/*
 * Gated DeltaNet-2 (burn-gdn2 config.rs): the delta rule with a per-key-channel decay and two
 * channel-wise gates, an erase gate b (how much of each key channel to erase) and a write
 * gate w (how much of each value channel to write); b = w = beta 1 is KDA, and a scalar decay
 * on top is Gated DeltaNet.  Per (batch, head), state S [K, V] fp32, for each token t:
 *     S' = Diag(exp(g_t)) S;   r = S'^T k_t;   S = S' - (b_t o k_t) r^T + k_t (w_t o v_t)^T;
 *     o_t = S^T q_t
 * (the page names the gates and modes but prints no update; this is the KDA step with its
 * erase and write strengths split by channel).  Projections, the short convolution, key
 * normalisation and the output norm are outside the library.
 *
 *   p->mode   MLSTM_GDN2_RECURRENT: token by token, the state on chip for the whole sequence
 *             (Gdn2Mode::FusedRecurrent; with T = 1 and S_out == S0 it is the decode step);
 *             K in {32, 64, 128, 256}.
 *             MLSTM_GDN2_CHUNK: chunks of p->chunk tokens (a multiple of 4, at most 64), dense
 *             products and one triangular solve per chunk (Gdn2Mode::Chunk); needs g <= 0.
 *             bf16 with chunk 64, K = 128 and V = 64 or 128 runs on the tensor cores (the
 *             per-chunk matrices for all chunks at once, then one pass per head with the
 *             state in tensor memory; bf16 operands, fp32 accumulation and state); other sizes
 *             on fp32 SIMT kernels.  Unsupported sizes: MLSTM_ERR_SHAPE.
 *   q, k      [B,H,T,K]  dtype       required (if T > 0); k usually unit-norm (caller's choice)
 *   v         [B,H,T,V]  dtype       required
 *   g         [B,H,T,K]  fp32        log decay (log alpha), <= 0 for a decay
 *   b         [B,H,T,K]  fp32        erase gate (in [0,1], or [0,2] with negative eigenvalues)
 *   w         [B,H,T,V]  fp32        write gate in [0,1]
 *   S0        [B,H,K,V]  fp32        initial state; NULL = zeros
 *   o         [B,H,T,V]  dtype       output, required (if T > 0)
 *   S_out     [B,H,K,V]  fp32        final state; NULL = not written; may equal S0 exactly
 *   workspace, workspace_bytes  chunk mode: at least mlstm_gdn2_workspace_size(p) bytes, 16-byte
 *             aligned (one prepared slot of per-chunk matrices per batch, head and chunk);
 *             recurrent mode: none needed (size 0), may be NULL
 * Outputs and the workspace must not overlap the inputs or each other (MLSTM_ERR_ALIAS).
 */
typedef enum { MLSTM_GDN2_RECURRENT = 0, MLSTM_GDN2_CHUNK = 1 } mlstm_gdn2_mode_t;
typedef struct {
  int B, H, T, K, V;
  mlstm_dtype_t dtype;
  int mode;  /* mlstm_gdn2_mode_t */
  int chunk; /* chunk mode only */
  /* Bound of every device-side wait of the tensor-core chunk kernels, in SM cycles; 0 = the
   * default (about two seconds).  A limit shorter than a copy takes makes the call fail with
   * MLSTM_ERR_TIMEOUT (see mlstm_gdn2_status).  Ignored by the other paths. */
  long long wait_limit_cycles;
} mlstm_gdn2_params_t;
size_t mlstm_gdn2_workspace_size(const mlstm_gdn2_params_t* p);
mlstm_status_t mlstm_gdn2_fwd(const mlstm_gdn2_params_t* p, const void* q, const void* k, const void* v,
                              const float* g, const float* b, const float* w, const float* S0, void* o,
                              float* S_out, void* workspace, size_t workspace_bytes, mlstm_stream_t stream);
/* Outcome of the bounded device-side waits of the last mlstm_gdn2_fwd enqueued on `stream` with
 * `workspace` and these params: synchronises `stream`; MLSTM_OK, or MLSTM_ERR_TIMEOUT when a
 * wait of the tensor-core chunk kernels ran out (that call's o and S_out are unspecified; the
 * workspace can be used again); MLSTM_OK always for the other paths, which have no such waits.
 * MLSTM_ERR_CUDA if the synchronisation or the read fails; argument errors as mlstm_gdn2_fwd
 * (workspace NULL: MLSTM_ERR_NULL when the tensor-core path would run).  In the bounds-checked
 * build (see mlstm_bounds_checked) a failed check gives MLSTM_ERR_BOUNDS, with the first failure
 * at bytes 16..39 of the workspace as {int site; int count; long long index; long long extent}. */
mlstm_status_t mlstm_gdn2_status(const mlstm_gdn2_params_t* p, const void* workspace, mlstm_stream_t stream);

/*
 * One recurrent decode step for every sequence of the batch, state updated in
 * place (RetNet recurrent_retention_step: O(1) per token; burn-gdn2 Gdn2Mode
 * FusedRecurrent: state [B,H,K,V] carried across tokens and updated in place).
 *
 *   q, k    [B,NH,DHQK]  dtype      required
 *   v       [B,NH,DHV]   dtype      required
 *   igate, fgate [B,NH]  fp32       pre-activations; required unless retention
 *   ogate   [B,NH,DHV]   dtype      activated output gate; NULL = 1; ignored in retention
 *   C       [B,NH,nb,DHV/nb,DHQK/nb] fp32  in/out, required
 *   n       [B,NH,nb,DHQK/nb]        fp32  in/out, required unless retention
 *   m       [B,NH]                   fp32  in/out, required unless retention
 *   h       [B,NH,DHV]   dtype      output, required; must not overlap the state
 *   stream
 * Supported block key widths DHQK/nb: 4, 8, 16, 32, 64, 128, 256, 512 (else
 * MLSTM_ERR_SHAPE).
 */
mlstm_status_t mlstm_step(const mlstm_step_params_t* p,
                          const void* q, const void* k, const void* v,
                          const float* igate, const float* fgate, const void* ogate,
                          float* C, float* n, float* m, void* h,
                          mlstm_stream_t stream);

/* Static, never-NULL description of a status code. */
const char* mlstm_status_string(mlstm_status_t s);

/* ABI version: (major << 16) | minor.  2.3: mlstm_bwd needs its workspace whenever
 * mlstm_bwd_workspace_size is nonzero, an empty sequence included. */
int mlstm_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLSTM_H_ */
