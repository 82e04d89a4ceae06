/*
 * xlstm_mlstm.h -- C ABI of the B200 (sm_100a) mLSTM cell library.
 *
 * The operation is the mLSTM cell of "xLSTM: Extended Long Short-Term Memory":
 * a matrix memory C (section 2.3) updated by the gated covariance rule (eq. (18)
 * with the forget gate as decay rate and the input gate as learning rate), a
 * normaliser state n whose dot product with the query is floored at 1.0
 * (section 2.3), exponential input gating with the stabiliser state m
 * (section 2.2, applied to mLSTM as section 2.3 says), and the output gate
 * scaling the retrieved vector.  Per batch b and head h, with d = DH:
 *
 *   log i_t = itilde_t;  log f_t = log sigmoid(ftilde_t)  or  ftilde_t;
 *   o_t = sigmoid(otilde_t) (per element);   khat_t = k_t / sqrt(d)
 *   m_t  = max(log f_t + m_{t-1}, log i_t)
 *   C'_t = exp(log f_t + m_{t-1} - m_t) C'_{t-1} + exp(log i_t - m_t) v_t khat_t^T
 *   n'_t = exp(log f_t + m_{t-1} - m_t) n'_{t-1} + exp(log i_t - m_t) khat_t
 *   h_t  = o_t * (C'_t q_t) / max(|n'_t^T q_t|, exp(-m_t))
 *
 * The state (C', n', m) is kept in stabilised units (C' = C exp(-m)); the
 * floor exp(-m_t) is the section 2.3 bound of 1.0 expressed in those units.
 * C' is [value row, key column].  Heads are independent (section 2.3: no
 * memory mixing between heads).
 *
 * Conventions for every entry point
 *  - Pointers are DEVICE pointers owned by the caller; the library keeps none
 *    of them after the call returns and allocates no device memory.
 *  - Tensors are dense, row-major (C order) with the shapes given, and every
 *    pointer is 16-byte aligned (else XLSTM_ERR_ALIGN).
 *  - Work is enqueued on the CUDA stream `cuda_stream` (a cudaStream_t; NULL =
 *    the legacy default stream) on the current device, asynchronously; no call
 *    synchronises.  The returned status covers argument validation and kernel
 *    launch only.  Errors found on the device (a bounded wait that ran out) are
 *    latched in a device status word read by xlstm_device_status().
 *  - No entry point exits, aborts, traps or throws.
 */
#ifndef XLSTM_MLSTM_H
#define XLSTM_MLSTM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    XLSTM_OK = 0,
    XLSTM_ERR_NULL = 1,        /* a required pointer is NULL                       */
    XLSTM_ERR_SHAPE = 2,       /* a size is negative, DH unsupported, or too large */
    XLSTM_ERR_DTYPE = 3,       /* dtype or gate kind out of range                  */
    XLSTM_ERR_CHUNK = 4,       /* chunk size not supported for this dtype          */
    XLSTM_ERR_ALIGN = 5,       /* a pointer is not 16-byte aligned                 */
    XLSTM_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed      */
    XLSTM_ERR_TIMEOUT = 7,     /* a bounded device-side wait ran out               */
    XLSTM_ERR_WORKSPACE = 8,   /* workspace NULL or smaller than required          */
    XLSTM_ERR_UNSUPPORTED = 9  /* option combination not supported                 */
} xlstm_status;

typedef enum { XLSTM_F32 = 0, XLSTM_BF16 = 1 } xlstm_dtype;          /* dtype of q, k, v, h */
typedef enum { XLSTM_FGATE_SIGMOID = 0, XLSTM_FGATE_EXP = 1 } xlstm_fgate;
/* Activation of the mLSTM block's external output gate (xlstm_mlstm_headnorm_gate). */
typedef enum { XLSTM_OGATE_SILU = 0, XLSTM_OGATE_SIGMOID = 1 } xlstm_ogate;

/* Kernel family for the forward.  AUTO picks the tensor-core (tcgen05) kernels
 * for bf16 inputs where they apply (chunk 64 or 128 with DH 64, 128, 256 or
 * 512; chunk 256 with DH 64, 128 or 256), and the fp32 SIMT kernels for every
 * other case.  SIMT forces the fp32-arithmetic kernels for any supported
 * arguments (a second, independent path the tests compare against).  TENSOR
 * forces the tensor-core kernels; for arguments they do not take the call
 * returns XLSTM_ERR_UNSUPPORTED and launches nothing.  Two tensor-core output
 * kernels exist: one keeps the state in tensor memory and retrieves with tf32
 * operands (TENSOR_TMEM: DH 128 or 256, chunk 64; about 11 significant bits
 * in the retrieval), the other keeps the state in fp32 registers and
 * retrieves with two bf16 parts (TENSOR_RS: every tensor-core case above; 15
 * to 16 bits).  TENSOR_RS splits the key columns of the state over two CTAs
 * at DH 512, and at DH 256 with chunk 256, and a combining kernel adds the two
 * partial numerators and denominators.  TENSOR takes TENSOR_TMEM where it
 * applies (it is the faster at DH 128 / 256, chunk 64) and TENSOR_RS
 * elsewhere. */
typedef enum {
    XLSTM_PATH_AUTO = 0, XLSTM_PATH_SIMT = 1, XLSTM_PATH_TENSOR = 2, XLSTM_PATH_TENSOR_TMEM = 3,
    XLSTM_PATH_TENSOR_RS = 4
} xlstm_path;

typedef struct {
    int path;       /* xlstm_path                                                       */
    int segments;   /* sequence segments per head for the two-level scan; 0 = automatic */
} xlstm_fwd_options;

/* ABI version of this header (bumped on any signature change). */
#define XLSTM_ABI_VERSION 1
int xlstm_abi_version(void);

/* Human-readable name of a status; never NULL. */
const char *xlstm_status_string(xlstm_status status);

/*
 * Bytes of device workspace xlstm_mlstm_fwd needs for these arguments (written
 * to *bytes; may be 0).  The workspace holds per-chunk gate prefix sums and,
 * when a head's sequence is split into segments that run in parallel, one
 * summary state per segment (the two-level chunk-state scan).  Same validation
 * as xlstm_mlstm_fwd.  Launches nothing; it reads the current device's SM
 * count (the segment plan fills one wave of SMs), and without a usable device
 * plans for 148 SMs.  Ask with the device current that the forward will run on.
 */
xlstm_status xlstm_mlstm_fwd_workspace_size(int B, int NH, int S, int DH, int chunk,
                                            xlstm_dtype dt, size_t *bytes);
xlstm_status xlstm_mlstm_fwd_workspace_size_ex(int B, int NH, int S, int DH, int chunk,
                                               xlstm_dtype dt, const xlstm_fwd_options *opts,
                                               size_t *bytes);

/*
 * Chunkwise-parallel forward (prefill) over S tokens.
 *
 *   q, k, v      [B, NH, S, DH]  dtype dt (float or bfloat16)
 *   i_pre, f_pre [B, NH, S]      float   (input / forget gate pre-activations)
 *   o_pre        [B, NH, S, DH]  float   (output gate pre-activation, per element)
 *   h            [B, NH, S, DH]  dtype dt, output
 *   C0 [B, NH, DH, DH], n0 [B, NH, DH], m0 [B, NH]  float, initial state in
 *                stabilised units; each may be NULL, meaning zeros.
 *   C_out, n_out, m_out  same shapes, final state; each may be NULL (not written).
 *                They must not overlap C0, n0, m0 or any input (the same
 *              pointer passed twice is rejected with XLSTM_ERR_UNSUPPORTED).
 *   chunk        tokens per chunk of the chunkwise form: 64, 128 or 256 for
 *                bf16; 1..1024 for f32.  S need not be a multiple of chunk.
 *   DH           multiple of 16 in [16, 512].
 *   fg           forget gate activation (sigmoid or exponential).
 *   workspace    device buffer of at least xlstm_mlstm_fwd_workspace_size()
 *                bytes (may be NULL when that size is 0); contents on entry
 *                are ignored, on exit unspecified.
 * S == 0 is allowed: h is untouched and the final state equals the initial one.
 * B == 0 or NH == 0 is a no-op.
 */
xlstm_status xlstm_mlstm_fwd(const void *q, const void *k, const void *v,
                             const float *i_pre, const float *f_pre, const float *o_pre,
                             void *h,
                             const float *C0, const float *n0, const float *m0,
                             float *C_out, float *n_out, float *m_out,
                             int B, int NH, int S, int DH, int chunk,
                             xlstm_dtype dt, xlstm_fgate fg,
                             void *workspace, size_t workspace_bytes, void *cuda_stream);

/*
 * Which kernel family xlstm_mlstm_fwd_ex would run for these arguments
 * (written to *path: XLSTM_PATH_SIMT or XLSTM_PATH_TENSOR after resolving
 * XLSTM_PATH_AUTO; a forced family is returned as given when it applies); same validation and error codes as the forward for DH,
 * chunk, dt and the options.  The paper has no counterpart: this lets a caller
 * (and the tests) know whether the fp32 CUDA-core kernels or the tcgen05
 * tensor-core kernels will compute the result.  Pure host function.
 */
xlstm_status xlstm_mlstm_fwd_path(int DH, int chunk, xlstm_dtype dt, const xlstm_fwd_options *opts,
                                  int *path);

/* As xlstm_mlstm_fwd, with explicit options (NULL = defaults). */
xlstm_status xlstm_mlstm_fwd_ex(const void *q, const void *k, const void *v,
                                const float *i_pre, const float *f_pre, const float *o_pre,
                                void *h,
                                const float *C0, const float *n0, const float *m0,
                                float *C_out, float *n_out, float *m_out,
                                int B, int NH, int S, int DH, int chunk,
                                xlstm_dtype dt, xlstm_fgate fg,
                                void *workspace, size_t workspace_bytes,
                                const xlstm_fwd_options *opts, void *cuda_stream);

/*
 * xlstm_mlstm_fwd without a workspace argument.  (The paper has no
 * counterpart: this is a calling convention of this library.)
 *
 * For callers that cannot allocate device memory: code that reaches this
 * library only through the C ABI and owns no device allocator (a plugin inside
 * a runtime that owns all device memory), or a serving loop that must not call
 * cudaMalloc, which can synchronise the device, fail under memory pressure or
 * stall for an unbounded time.  Inputs and outputs are passed exactly as for
 * xlstm_mlstm_fwd; the scratch comes from one device array inside the library
 * of XLSTM_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library
 * holds until the process exits.
 *  - Calls whose xlstm_mlstm_fwd_workspace_size() exceeds that size return
 *    XLSTM_ERR_WORKSPACE and launch nothing.  Nothing is allocated, ever.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress)
 *    on the current device; the first call on a device also loads the
 *    library's device code there, so make that first call before any stream
 *    capture.  Nothing is cached between calls, so the entry point stays valid
 *    after a cudaDeviceReset.
 *  - All calls share the one array: two calls whose kernels overlap on the GPU
 *    (different streams, or different host threads) race on it and give wrong
 *    results.  Serialise them, e.g. by issuing them on one stream.  The array
 *    keeps the last call's contents; the forward overwrites whatever it reads,
 *    so no clearing is needed.
 */
#define XLSTM_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
xlstm_status xlstm_mlstm_fwd_noalloc(const void *q, const void *k, const void *v,
                                     const float *i_pre, const float *f_pre, const float *o_pre,
                                     void *h,
                                     const float *C0, const float *n0, const float *m0,
                                     float *C_out, float *n_out, float *m_out,
                                     int B, int NH, int S, int DH, int chunk,
                                     xlstm_dtype dt, xlstm_fgate fg, void *cuda_stream);

/*
 * One recurrent decode token for every (b, h), updating the resident state in
 * place (section 2.5 of the paper: constant memory in the sequence length).
 *
 *   q, k, v      [B, NH, DH]      dtype dt
 *   i_pre, f_pre [B, NH]          float
 *   o_pre        [B, NH, DH]      float
 *   h            [B, NH, DH]      dtype dt, output
 *   C [B, NH, DH, DH], n [B, NH, DH], m [B, NH]  float, stabilised state,
 *                read and overwritten with the state after this token.  This
 *                is exactly the state xlstm_mlstm_fwd returns.
 * DH: multiple of 16 in [16, 512].  B == 0 or NH == 0 is a no-op.
 * If a bounded wait inside the step runs out (xlstm_device_status() then
 * reports XLSTM_ERR_TIMEOUT), h and the state are undefined: synchronise and
 * restore the state before the next step.
 */
xlstm_status xlstm_mlstm_step(const void *q, const void *k, const void *v,
                              const float *i_pre, const float *f_pre, const float *o_pre,
                              void *h, float *C, float *n, float *m,
                              int B, int NH, int DH, xlstm_dtype dt, xlstm_fgate fg,
                              void *cuda_stream);

/*
 * Sequence parallelism: a sequence cut into consecutive slices, one per GPU
 * (or per call), each slice's forward started from the state the slices before
 * it leave.  Unrolling the recurrence of section 2.3 over a slice j that
 * starts from the zero state summarises it as (C'_j, n'_j) under the slice's
 * own stabiliser mloc_j = max_s(log i_s + F_j - F_{j,s}), plus F_j, the slice's
 * total log forget (F_{j,s}: its prefix up to token s).  Slices then join
 * exactly as tokens do:
 *   M = max(F_j + M_prev, mloc_j),
 *   (C', n') = e^{F_j + M_prev - M} (C', n')_prev + e^{mloc_j - M} (C'_j, n'_j).
 * The state a rank starts from is therefore the fold of the summaries of the
 * slices before it (an all-gather of summaries, then a local fold: no
 * sequential hand-off between GPUs), and its forward (xlstm_mlstm_fwd with that
 * state as C0/n0/m0) reproduces the single-sequence result.
 *
 * A summary is one "packed" float buffer of xlstm_mlstm_seg_state_floats()
 * floats: C' [B, NH, DH, DH], then n' [B, NH, DH], then mloc [B, NH], then
 * F [B, NH], then zero to three floats of padding (the size is a multiple of 4
 * floats, so packed summaries laid end to end stay 16-byte aligned).  An empty
 * slice (S == 0) is summarised as zero state, mloc = -inf, F = 0, which the
 * fold treats as the identity.
 */
xlstm_status xlstm_mlstm_seg_state_floats(int B, int NH, int DH, size_t *floats);

/*
 * Summary of one slice (see above): k, v [B, NH, S, DH] dtype dt, i_pre, f_pre
 * [B, NH, S] float, packed: output of xlstm_mlstm_seg_state_floats() floats.
 * Runs the forward's gate pass and segment summaries (tensor-core kernels for
 * bf16 where the forward has them, fp32 SIMT kernels otherwise) and a fold of
 * the segments; no h is formed and q, o are not read.  chunk, dtype and shape
 * rules and error codes as xlstm_mlstm_fwd; workspace of at least
 * xlstm_mlstm_seg_state_workspace_size() bytes (overwritten).  B or NH == 0 is
 * a no-op.
 */
xlstm_status xlstm_mlstm_seg_state_workspace_size(int B, int NH, int S, int DH, int chunk,
                                                  xlstm_dtype dt, size_t *bytes);
xlstm_status xlstm_mlstm_seg_state(const void *k, const void *v, const float *i_pre, const float *f_pre,
                                   float *packed, int B, int NH, int S, int DH, int chunk,
                                   xlstm_dtype dt, xlstm_fgate fg, void *workspace,
                                   size_t workspace_bytes, void *cuda_stream);

/*
 * Folds `count` packed summaries (laid end to end at `parts`, each
 * xlstm_mlstm_seg_state_floats() floats; count == 0 allowed, parts may then be
 * NULL) into the state that the token-by-token recurrence reaches after those
 * slices when it starts from (C0, n0, m0) ([B, NH, DH, DH], [B, NH, DH],
 * [B, NH] float; each NULL = zeros, m0 NULL = 0, the forward's convention).
 * Writes C_out [B, NH, DH, DH], n_out [B, NH, DH], m_out [B, NH] (all
 * required); they must not be C0, n0 or m0 (XLSTM_ERR_UNSUPPORTED) nor overlap
 * parts.  DH: multiple of 16 in [16, 512].
 */
xlstm_status xlstm_mlstm_state_combine(const float *parts, int count, const float *C0, const float *n0,
                                       const float *m0, float *C_out, float *n_out, float *m_out,
                                       int B, int NH, int DH, void *cuda_stream);

/*
 * Backward of the cell (gradients for training): for the forward with a zero
 * initial state and the loss L = sum(dh * h) + sum(dC * C'_T) + sum(dn * n'_T),
 * writes dL/dq, dL/dk, dL/dv, dL/d(itilde), dL/d(ftilde), dL/d(otilde).  The
 * stabiliser is held fixed, which "xLSTM: Extended Long Short-Term Memory"
 * section 2.2 (appendix A.2) shows leaves the derivatives unchanged; the
 * returned state's own stabiliser m_T is differentiated where the final-state
 * cotangents need it.  The chunk-start and reverse states are materialised in
 * the workspace.  bf16 inputs with DH 64, 128 or 256 run on the tensor cores
 * (tcgen05, fp32 accumulation; every fp32 operand enters as a bf16 high + low
 * pair, about 16 significant bits); other arguments run fp32 arithmetic on
 * CUDA cores.
 *
 *   q, k, v, dh     [B, NH, S, DH]  dtype dt (dh: cotangent of h)
 *   i_pre, f_pre    [B, NH, S]      float
 *   o_pre           [B, NH, S, DH]  float
 *   dC [B, NH, DH, DH], dn [B, NH, DH]  float, cotangents of the final
 *                   stabilised state; each may be NULL (zero)
 *   dq, dk, dv      [B, NH, S, DH]  dtype dt, outputs
 *   di, df          [B, NH, S]      float, outputs
 *   d_o             [B, NH, S, DH]  float, output
 *   chunk           1..64 tokens per chunk (XLSTM_ERR_CHUNK otherwise)
 *   workspace       at least xlstm_mlstm_bwd_workspace_size() bytes
 * Outputs must not be any input or each other (the same pointer twice is
 * rejected with XLSTM_ERR_UNSUPPORTED).  DH: multiple of 16 in [16, 512].
 * B, NH or S == 0 is a no-op.
 */
xlstm_status xlstm_mlstm_bwd_workspace_size(int B, int NH, int S, int DH, int chunk,
                                            xlstm_dtype dt, size_t *bytes);
xlstm_status xlstm_mlstm_bwd(const void *q, const void *k, const void *v,
                             const float *i_pre, const float *f_pre, const float *o_pre,
                             const void *dh, const float *dC, const float *dn,
                             void *dq, void *dk, void *dv, float *di, float *df, float *d_o,
                             int B, int NH, int S, int DH, int chunk,
                             xlstm_dtype dt, xlstm_fgate fg,
                             void *workspace, size_t workspace_bytes, void *cuda_stream);

/*
 * sLSTM forward ("xLSTM: Extended Long Short-Term Memory" section 2.2): scalar
 * memory cells with exponential input gating, a sigmoid or exponential forget
 * gate, a normaliser state, the stabiliser m_t, and memory mixing through
 * recurrent connections from h_{t-1} to the cell input z and the gates i, f, o
 * within each head.  Per batch b, head hd, unit j:
 *
 *   zt = zx + R_z h_{t-1}, it = ix + R_i h_{t-1}, ft = fx + R_f h_{t-1},
 *   ot = ox + R_o h_{t-1};  z = tanh(zt), log i = it,
 *   log f = log sigmoid(ft) | ft, o = sigmoid(ot)
 *   m_t = max(log f + m_{t-1}, log i)
 *   c_t = exp(log f + m_{t-1} - m_t) c_{t-1} + exp(log i - m_t) z
 *   n_t = exp(log f + m_{t-1} - m_t) n_{t-1} + exp(log i - m_t),  h_t = o c_t / n_t
 *
 *   zx, ix, fx, ox  [B, NH, S, DH] float, input pre-activations (projection and
 *                   bias already applied)
 *   R               [NH, 4, DH, DH] float, recurrent blocks in the order z, i, f,
 *                   o; R[hd][g][j][l] multiplies h_{t-1}[l] into unit j's gate g
 *   h               [B, NH, S, DH] float, output
 *   c0, n0, m0, h0  [B, NH, DH] float, initial state (c, n stabilised); each
 *                   may be NULL (zeros)
 *   c_out, n_out, m_out, h_out  [B, NH, DH] float, final state; each nullable
 * Outputs must not be any input or each other (XLSTM_ERR_UNSUPPORTED).
 * DH in [1, 512].  S == 0 copies the initial state to the state outputs.
 * fp32 throughout.  DH 64, 128, 256 (and 512 where the device can place a
 * 16-CTA cluster): a cluster of DH/32 CTAs per (batch, head) keeps the
 * recurrent blocks on chip for the whole sequence and exchanges h_t through
 * distributed shared memory, one cluster barrier per step; other DH: one CTA
 * per (batch, head) reading R from L2 at every step.
 */
xlstm_status xlstm_slstm_fwd(const float *zx, const float *ix, const float *fx, const float *ox,
                             const float *R, float *h,
                             const float *c0, const float *n0, const float *m0, const float *h0,
                             float *c_out, float *n_out, float *m_out, float *h_out,
                             int B, int NH, int S, int DH, xlstm_fgate fg, void *cuda_stream);

/*
 * The mLSTM block's epilogue after the cell ("xLSTM: Extended Long Short-Term
 * Memory" section 2.4, Figure 10): the cell output is normalised by a GroupNorm
 * whose groups are the heads (a LayerNorm over each head's DH channels, per
 * token; GroupNorm as defined by Wu & He: biased variance, eps inside the square
 * root, per-channel scale and shift), the learnable skip input is added, and the
 * sum is gated component-wise by the block's external output gate.  One pass;
 * the output is in the block's layout, ready for the down-projection:
 *
 *   y[b, t, c] = ((h[b, hd, t, j] - mean) / sqrt(var + eps) * gamma[c] + beta[c]
 *                 + skip_w[c] * x_skip[b, t, c]) * act(z[b, t, c]),
 *   c = hd * DH + j,  mean / var over j of h[b, hd, t, :],
 *   act(z) = z * sigmoid(z) (XLSTM_OGATE_SILU) or sigmoid(z) (XLSTM_OGATE_SIGMOID).
 *
 *   h            [B, NH, S, DH]  dtype dt, the cell output (as xlstm_mlstm_fwd
 *                writes it; run the cell with o_pre = +inf for the block's form,
 *                where the output gate is outside the cell)
 *   gamma, beta  [NH * DH]       float, GroupNorm scale and shift per channel
 *   skip_w       [NH * DH]       float, learnable skip weight per channel
 *   x_skip       [B, S, NH * DH] dtype dt, skip input (the cell input after the
 *                block's causal convolution); skip_w and x_skip are both NULL
 *                (no skip term) or both given
 *   z            [B, S, NH * DH] dtype dt, external output-gate pre-activation
 *   y            [B, S, NH * DH] dtype dt, output; must not be any input buffer
 *                (the same pointer passed twice is rejected with
 *                XLSTM_ERR_UNSUPPORTED)
 *   eps          > 0 and finite (else XLSTM_ERR_UNSUPPORTED)
 * DH: multiple of 16 in [16, 512].  B, NH or S == 0 is a no-op.  Statistics
 * and arithmetic are fp32; y is rounded once to dt.
 */
xlstm_status xlstm_mlstm_headnorm_gate(const void *h, const float *gamma, const float *beta,
                                       const float *skip_w, const void *x_skip, const void *z,
                                       void *y, int B, int NH, int S, int DH, float eps,
                                       xlstm_dtype dt, xlstm_ogate og, void *cuda_stream);

/*
 * Synchronises `cuda_stream`, then reads and clears the device status word of
 * the current device.  Returns XLSTM_OK, XLSTM_ERR_TIMEOUT if a kernel gave up
 * a bounded wait since the last call, or XLSTM_ERR_CUDA.
 *
 * The status word is one per device and per process, shared by every stream
 * and host thread, and this call clears it: a timeout latched by a kernel on
 * another stream is reported (and consumed) by whichever caller reads the
 * word first, and only work on `cuda_stream` is waited for.  Callers that use
 * several streams should read it after synchronising all of them.  After a
 * timeout the outputs of the call whose kernel gave up (h, the state) are
 * undefined; synchronise and re-run that call before relying on them.
 */
xlstm_status xlstm_device_status(void *cuda_stream);

/*
 * Per-kernel timing (tracing).  Between xlstm_profile_begin() and
 * xlstm_profile_end(), every kernel this library launches, from any thread, is
 * bracketed by a pair of CUDA events recorded on the stream it is launched
 * on.  xlstm_profile_end() waits for those events and writes, per kernel
 * name, the launch count and the summed device time, for at most `max`
 * kernels into `out`; *count receives the number of distinct kernels.  The
 * events cost one stream operation each and do not serialise streams.
 */
typedef struct {
    char name[48];       /* kernel name, NUL-terminated */
    int launches;
    double total_ms;     /* sum of event-to-event times of its launches */
} xlstm_kernel_time;

xlstm_status xlstm_profile_begin(void);
xlstm_status xlstm_profile_end(xlstm_kernel_time *out, int max, int *count);

/*
 * Self-test of the failure path (the paper has no counterpart).  Enqueues on
 * `cuda_stream` one single-CTA kernel that waits, with the same bounded wait the
 * forward and decode kernels use, on a shared-memory barrier that nothing
 * completes; after about `limit_us` microseconds (1..1000000) the wait gives up
 * and latches the device status word, and the kernel returns normally.  A
 * following xlstm_device_status() then reports XLSTM_ERR_TIMEOUT (and clears
 * the word).  No fault, trap or hang is involved; the context stays usable.
 * Returns XLSTM_ERR_SHAPE for a limit out of range, XLSTM_ERR_CUDA if the
 * launch fails.
 */
xlstm_status xlstm_selftest_wait_timeout(int limit_us, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* XLSTM_MLSTM_H */
