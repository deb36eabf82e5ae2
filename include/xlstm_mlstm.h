/*
 * xlstm_mlstm.h -- C ABI of the B200 (sm_100a) mLSTM forward library.
 *
 * The operation (xLSTM page, obsidian-dorae222.pages.dev, section "mLSTM
 * (matrix LSTM)", eq. 1-3, with the stabilizer of its "sLSTM" section):
 *
 *   m_t  = max(f~_t + m_{t-1}, i~_t)                       (log-space stabilizer)
 *   f'_t = exp(f~_t + m_{t-1} - m_t),  i'_t = exp(i~_t - m_t)
 *   C~_t = f'_t C~_{t-1} + i'_t v_t k_t^T                   (eq. 1, stabilized)
 *   n~_t = f'_t n~_{t-1} + i'_t k_t                         (eq. 2, stabilized)
 *   h~_t = C~_t q_t / max(|n~_t^T q_t|, exp(-m_t))          (eq. 3 without o_t)
 *
 * with q_t multiplied by desc->qk_scale first.  (C~, n~, m) is the stabilized
 * state: the unstabilized state of eq. 1-2 is (e^m C~, e^m n~), and the readout
 * above equals eq. 3's C q / max(|n^T q|, 1) exactly.  The output gate o_t of
 * eq. 3 and the input projections of the page's listing are not part of this
 * library: q, k, v, i~, f~ arrive already projected.
 *
 * Layouts (row-major, contiguous, device memory):
 *   q, k    [B][H][T][d_qk]  qkv_dtype (bf16 or fp32)
 *   v       [B][H][T][d_v]   qkv_dtype
 *   i_pre   [B][H][T]        fp32   input-gate pre-activation i~
 *   f_pre   [B][H][T]        fp32   forget-gate pre-activation f~ (log forget gate)
 *   h_out   [B][H][T][d_v]   fp32   pre-gate output h~
 *   C       [B][H][d_v][d_qk] fp32  row = value index, so C q is a row dot
 *   n       [B][H][d_qk]     fp32
 *   m       [B][H]           fp32
 * The step call uses the same tensors with the T axis removed.
 *
 * Ownership and execution: every pointer is caller-owned device memory.  The
 * library allocates nothing; scratch memory is the caller's workspace, sized
 * by xlstm_mlstm_workspace_size().  Calls enqueue work on `stream` and return
 * without synchronising; results are ready when the stream is.
 *
 * Errors: argument problems are reported synchronously, before anything is
 * enqueued.  XLSTM_ERR_CUDA reports a launch failure (the CUDA error is left
 * for cudaGetLastError).  Faults detected on the device (a bounded wait that
 * gave up) are recorded in the workspace status block and read back with
 * xlstm_mlstm_workspace_status().
 */
#ifndef XLSTM_MLSTM_H
#define XLSTM_MLSTM_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define XLSTM_API __attribute__((visibility("default")))
#else
#define XLSTM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    XLSTM_OK = 0,
    XLSTM_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, overlap   */
    XLSTM_ERR_UNSUPPORTED = 2,  /* valid request this build has no kernel for   */
    XLSTM_ERR_CUDA = 3,         /* a CUDA launch or enqueue failed              */
    XLSTM_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up           */
    XLSTM_ERR_WORKSPACE = 5     /* workspace missing or smaller than required   */
} xlstm_status_t;

typedef enum {
    XLSTM_F32 = 0,
    XLSTM_BF16 = 1
} xlstm_dtype_t;

typedef struct {
    int32_t B, H;        /* batch, heads: >= 1                                   */
    int32_t T;           /* sequence length: >= 0 (ignored by the step call)     */
    int32_t d_qk, d_v;   /* head dims: multiples of 16 in [16, 512]              */
    int32_t qkv_dtype;   /* xlstm_dtype_t of q, k, v                             */
    float qk_scale;      /* multiplies q before use (1 = the page literally)     */
    int32_t chunk;       /* chunk length L for the chunkwise call; 0 = 64        */
} xlstm_mlstm_desc_t;

/*
 * Chunkwise-parallel forward over a whole sequence.
 *
 * Splits T into chunks of L tokens (the last one ragged).  Inside a chunk the
 * unrolled recurrence is evaluated in parallel form:
 *   F_t = sum_{r<=t} f~_r (cumulative log forget gate, reset every chunk),
 *   m_t = F_t + max(m_0, max_{s<=t}(i~_s - F_s))   -- exactly the stabilizer,
 *   h~_t = [e^{F_t+m_0-m_t} C~_0 q_t + sum_{s<=t} e^{F_t-F_s+i~_s-m_t}(q_t.k_s) v_s]
 *          / max(|same with n~_0 and 1 in place of C~_0 and v_s|, e^{-m_t})
 * and the state is carried from chunk to chunk in fp32.  bf16 inputs run on
 * tcgen05 tensor cores (fp32 accumulation); fp32 inputs on fp32 CUDA cores.
 *
 *   C_in, n_in, m_in : initial state; all three NULL means zero state (m = 0),
 *                      otherwise all three must be given.
 *   h_out            : required when T > 0.
 *   C_out, n_out, m_out : final state; each may be NULL (then not written).
 *                      The canonical stabilizer m_T of the recurrence is
 *                      written, with C~ and n~ in that gauge.
 *   workspace        : device scratch of >= xlstm_mlstm_workspace_size(desc)
 *                      bytes, 256-byte aligned; its first 16 bytes are the
 *                      status block.  With >= xlstm_mlstm_workspace_size_parallel
 *                      (desc) bytes a long sequence with few heads runs as
 *                      parallel segments.  Calls sharing a workspace must not
 *                      overlap on the device.
 * Chunk lengths: 0 (= 64) and 64 for both input types; 16, 32 and 128 for
 * fp32 inputs (CUDA-core kernel); 128 for bf16 inputs with d_qk = 64 or 128
 * and d_v a multiple of 64 (the shapes the tensor-core kernel takes).  Every
 * other length (256 among them), 16 or 32 with bf16 inputs, and bf16 128 at
 * d_qk = 256 return XLSTM_ERR_UNSUPPORTED: the tensor-core kernel that runs bf16 inputs holds
 * the state, its readout copy and one chunk's S and H accumulators in tensor
 * memory (512 columns), which at d_qk = 256 fits a chunk of 64 tokens only, and
 * at L = 256 no d_qk.  The chunk length is an evaluation order, not part of the
 * method: results differ only by rounding.
 * Outputs must not overlap inputs.  T = 0 copies the state through.
 */
XLSTM_API xlstm_status_t xlstm_mlstm_fwd_chunkwise(
    const xlstm_mlstm_desc_t *desc,
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    const float *C_in, const float *n_in, const float *m_in,
    float *h_out, float *C_out, float *n_out, float *m_out,
    void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Output stage of xlstm_mlstm_fwd_chunkwise_out (xLSTM page, "mLSTM (matrix
 * LSTM)" eq. 3, h_t = o_t * h~_t, with o_t = sigmoid(o~_t) as in the o_t line of
 * the page's forward_recurrent listing, the projection removed).
 *   o_pre   : [B][H][T][d_v] output-gate pre-activations o~ (device), or NULL
 *             for no gate (h = h~).  An input: must not overlap any output.
 *   o_dtype : XLSTM_F32 or XLSTM_BF16, the element type of o_pre.
 *   h_dtype : XLSTM_F32 or XLSTM_BF16, the element type of h_out (bf16: rounded
 *             to nearest even from the fp32 result).
 */
typedef struct {
    const void *o_pre;
    xlstm_dtype_t o_dtype;
    xlstm_dtype_t h_dtype;
} xlstm_mlstm_output_t;

/*
 * xlstm_mlstm_fwd_chunkwise with the output stage:
 * h_out[b][h][t][:] = sigmoid(o_pre[b][h][t][:]) * h~_t (elementwise), stored as
 * out->h_dtype.  out == NULL is xlstm_mlstm_fwd_chunkwise exactly.  Same
 * arguments, rules, workspace and status block otherwise; h_out holds
 * B*H*T*d_v elements of h_dtype.  Invalid dtypes or a misaligned o_pre give
 * XLSTM_ERR_INVALID_ARG.  The state outputs are the recurrence's, untouched by
 * the gate.  On the tensor-core path the chunkwise kernel stores h~ in h_dtype
 * and a streaming kernel applies the gate in place (with a bf16 h, h~ is rounded
 * to bf16 before the gate and the gated value again); on the fp32 CUDA-core path
 * the gate is applied in the epilogue.  When the tensor-core grid ends in a
 * partial wave, the call splits it in two launches on `stream`. It gates the
 * first launch's h~ on a second stream of the library's own (one per device,
 * made on the first such call and kept) while the second launch runs. The
 * caller's stream waits for that gate before its last kernel, so all of the
 * call's work is ordered on `stream` as usual, CUDA-graph capture included
 * (the second stream joins the capture through events).  Make the first such
 * call on a device outside a capture: it creates that stream and its events.
 */
XLSTM_API xlstm_status_t xlstm_mlstm_fwd_chunkwise_out(
    const xlstm_mlstm_desc_t *desc, const xlstm_mlstm_output_t *out,
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    const float *C_in, const float *n_in, const float *m_in,
    void *h_out, float *C_out, float *n_out, float *m_out,
    void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Recurrent forward over a whole sequence: the recurrence above evaluated one
 * token at a time with the state held on chip (O(1) state memory per head,
 * O(T) time).  Same arguments and rules as xlstm_mlstm_fwd_chunkwise;
 * desc->chunk is ignored; the workspace may be NULL (it needs none).
 */
XLSTM_API xlstm_status_t xlstm_mlstm_fwd_recurrent(
    const xlstm_mlstm_desc_t *desc,
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    const float *C_in, const float *n_in, const float *m_in,
    float *h_out, float *C_out, float *n_out, float *m_out,
    void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * One decode step (the page's forward_recurrent without projections and o_t):
 *   q, k [B][H][d_qk], v [B][H][d_v], i_pre, f_pre [B][H];
 *   C, n, m : state in (required);  h_out [B][H][d_v];
 *   C_new, n_new, m_new : state out (required).  Each may equal its input
 *   exactly (in-place update); any other overlap is rejected.
 * desc->T and desc->chunk are ignored.  Memory-bound: C is read and written
 * once with 128-bit coalesced accesses.
 */
XLSTM_API xlstm_status_t xlstm_mlstm_step(
    const xlstm_mlstm_desc_t *desc,
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    const float *C, const float *n, const float *m,
    float *h_out, float *C_new, float *n_new, float *m_new,
    cudaStream_t stream);

/*
 * xlstm_mlstm_fwd_chunkwise without a caller workspace, for callers that cannot
 * allocate device memory: a plug-in inside a host framework that owns every
 * device allocation and offers no allocator, or code on a latency-critical path
 * where cudaMalloc (which may synchronise the device and may fail) is not
 * allowed.  (The xLSTM pages have no counterpart to this call; it is a library
 * convenience.)
 *
 * Same arguments, rules and results as xlstm_mlstm_fwd_chunkwise, minus the
 * workspace.  The scratch is a fixed 4096-byte array in the library's own
 * device memory, held on every GPU that loads the library until the process
 * exits; a desc whose xlstm_mlstm_workspace_size exceeds 4096 bytes is refused
 * with XLSTM_ERR_WORKSPACE.  The call allocates nothing and frees nothing.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before capturing any stream.
 *   - All calls share the one array: calls that overlap on the device (other
 *     streams, other host threads) race on it.  Each call clears the part that
 *     must start at zero (the status block) on its stream before its kernel.
 *   - The device status block lives at the start of that array; read it after
 *     the call's stream with xlstm_mlstm_noalloc_status.
 *   - The array holds only the status block, never segment summaries, so this
 *     call always runs a sequence in one piece: a long sequence with few heads
 *     (e.g. 8 heads of 65536 tokens) takes about ten times as long as through
 *     xlstm_mlstm_fwd_chunkwise given xlstm_mlstm_workspace_size_parallel bytes.
 *   - The device address is cached per device for the life of the process: do
 *     not use this call across cudaDeviceReset on a device.
 */
XLSTM_API xlstm_status_t xlstm_mlstm_fwd_chunkwise_noalloc(
    const xlstm_mlstm_desc_t *desc,
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    const float *C_in, const float *n_in, const float *m_in,
    float *h_out, float *C_out, float *n_out, float *m_out,
    cudaStream_t stream);

/*
 * The device status block of the last xlstm_mlstm_fwd_chunkwise_noalloc call on
 * the current device (the allocation-free counterpart of
 * xlstm_mlstm_workspace_status; the pages have no counterpart either): copies
 * the block to the host on `stream` and waits for that stream, so call it after
 * the call you want to check, on its stream.  Returns the block's code (XLSTM_OK
 * or XLSTM_ERR_TIMEOUT) and, if where != NULL, the code of the wait that gave
 * up; XLSTM_ERR_CUDA if the copy fails.  Allocates nothing.
 */
XLSTM_API xlstm_status_t xlstm_mlstm_noalloc_status(int32_t *where, cudaStream_t stream);

/*
 * Backward pass (training; xLSTM page, "mLSTM (matrix LSTM)" eq. 1-3 with the
 * "sLSTM" stabilizer): the vector-Jacobian product of xlstm_mlstm_fwd_chunkwise.
 * What is differentiated is the readout with the true states,
 * h_t = C_t q_t / max(|n_t^T q_t|, 1), f_t = e^{f~_t}, i_t = e^{i~_t}; the stabilizer
 * only stores those states and is a constant of the derivative (h~ does not
 * depend on it).
 *   Inputs: desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in as given to the forward
 *     call (state all NULL: zero state, m = 0); dh [B][H][T][d_v] the upstream
 *     gradient of h~ (fp32; h~ itself is recomputed); dC_out [B][H][d_v][d_qk]
 *     and dn_out [B][H][d_qk] that of the final stored state, for a consumer of the
 *     true state such as the next call of the recurrence (both NULL: zero).
 *   Outputs (fp32, whatever the input type): dq, dk [B][H][T][d_qk], dv
 *     [B][H][T][d_v], di_pre, df_pre [B][H][T]; dC_in, dn_in, dm_in: gradients of
 *     the initial state (each may be NULL; with no initial state they are the
 *     gradients at the zero state).
 *   workspace: >= xlstm_mlstm_bwd_workspace_size(desc) bytes, 256-byte aligned
 *     (the stored state at every chunk entry and the adjoint at every chunk
 *     exit: about 2 (T / 64) B H d_v d_qk floats).  Chunk: 0 or 64.
 * Runs on fp32 CUDA cores: the states at chunk entries (sequential in t, with
 * h~ recomputed in fp32 for dh . h~), the adjoints at chunk exits (sequential
 * backwards in t), then every chunk's gradients at once.  Outputs must not
 * overlap inputs.
 */
XLSTM_API size_t xlstm_mlstm_bwd_workspace_size(const xlstm_mlstm_desc_t *desc);
XLSTM_API xlstm_status_t xlstm_mlstm_bwd_chunkwise(
    const xlstm_mlstm_desc_t *desc,
    const void *q, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    const float *C_in, const float *n_in, const float *m_in,
    const float *dh, const float *dC_out, const float *dn_out,
    float *dq, float *dk, float *dv, float *di_pre, float *df_pre,
    float *dC_in, float *dn_in, float *dm_in,
    void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Sequences cut along T (e.g. across GPUs).  Over a stretch of tokens the
 * recurrence (xLSTM page, "mLSTM (matrix LSTM)" eq. 1-2 with the stabilizer of
 * the "sLSTM" section) maps the entering state to the leaving one affinely:
 * the true state is scaled by e^F (F = the stretch's summed f~) and the
 * stretch's own contribution is added.  A stretch is therefore summarised by F
 * and by the state it leaves from a zero state whose stabilizer starts at -inf:
 *   C_seg = sum_t e^{u_t - u*} v_t k_t^T,  n_seg = sum_t e^{u_t - u*} k_t,
 *   m_seg = F + u*,  with F_t = sum_{r<=t} f~_r, u_t = i~_t - F_t, u* = max_t u_t.
 *
 * xlstm_mlstm_segment_summary: the summary of each (b, h) sequence of desc.
 *   k [B][H][T][d_qk], v [B][H][T][d_v] (desc->qkv_dtype), i_pre, f_pre [B][H][T];
 *   C_seg [B][H][d_v][d_qk], n_seg [B][H][d_qk] (fp32), F_m [B][H][2] (float64:
 *   F, m_seg).  Runs on the tcgen05 summary kernel: bf16 inputs, d_qk in
 *   {64, 128, 256}, d_v a multiple of 64, T a multiple of 64 and at most 65536,
 *   chunk 0 or 64; other descs return XLSTM_ERR_UNSUPPORTED.  Workspace and
 *   status block as for xlstm_mlstm_fwd_chunkwise (>= 256 bytes).
 */
XLSTM_API xlstm_status_t xlstm_mlstm_segment_summary(
    const xlstm_mlstm_desc_t *desc, const void *k, const void *v,
    const float *i_pre, const float *f_pre,
    float *C_seg, float *n_seg, double *F_m,
    void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * xlstm_mlstm_combine_states: the state after nsum summarised stretches in order,
 * chained onto (C_in, n_in, m_in) (all NULL: zero state, m = 0):
 *   m' = max(F + m, m_seg),  C' = e^{F+m-m'} C + e^{m_seg-m'} C_seg  (n likewise),
 * every coefficient <= 1, the gauge chain in float64 with each m' rounded to the
 * fp32 it is stored as.  The result carries the recurrence's canonical m, so it
 * is the entry state of the next stretch for xlstm_mlstm_fwd_chunkwise.
 *   C_seg [nsum][B][H][d_v][d_qk], n_seg [nsum][B][H][d_qk], F_m [nsum][B][H][2];
 *   C_out, n_out, m_out: required, must not overlap the inputs.
 * desc gives B, H, d_qk, d_v; its T, dtype and chunk are ignored.  nsum = 0
 * copies the entry state (or writes the zero state).
 */
XLSTM_API xlstm_status_t xlstm_mlstm_combine_states(
    const xlstm_mlstm_desc_t *desc, int32_t nsum,
    const float *C_in, const float *n_in, const float *m_in,
    const float *C_seg, const float *n_seg, const double *F_m,
    float *C_out, float *n_out, float *m_out, cudaStream_t stream);

/* Workspace bytes xlstm_mlstm_fwd_chunkwise needs for desc (>= 256), or 0 for
 * a NULL desc. */
XLSTM_API size_t xlstm_mlstm_workspace_size(const xlstm_mlstm_desc_t *desc);

/*
 * Workspace bytes with which xlstm_mlstm_fwd_chunkwise may run a long sequence
 * as parallel segments (>= xlstm_mlstm_workspace_size(desc); equal to it when
 * desc gains nothing from segments), or 0 for a NULL desc.
 *
 * The recurrence over a stretch of tokens is an affine map of the state (xLSTM
 * page, "mLSTM (matrix LSTM)" eq. 1-3, with the stabilizer of the "sLSTM"
 * section), so when B*H leaves most of the GPU idle (the tensor-core kernel's
 * shapes only: bf16, chunk 64) the sequence is cut into segments of whole
 * chunks: each segment but the last is first summarised from a zero state, the
 * summaries are chained into every segment's entry state, and then all
 * segments run at once.  The extra memory is about
 * (segments - 1) * B * H * (d_v * d_qk + d_qk + 4) * 4 bytes; the extra traffic
 * is one more read of k, v and the gates.  Results agree with the sequential
 * evaluation to within rounding (the final state keeps the canonical m).
 * With a smaller workspace (>= xlstm_mlstm_workspace_size) the call runs the
 * sequence in one piece, as before.
 */
XLSTM_API size_t xlstm_mlstm_workspace_size_parallel(const xlstm_mlstm_desc_t *desc);

/*
 * Reads the workspace status block written by the device: waits for `stream`,
 * returns XLSTM_OK or the recorded device error (e.g. XLSTM_ERR_TIMEOUT), and
 * stores the code of the wait that gave up in *where (may be NULL).
 * Each chunkwise call clears the block before its kernels run.
 */
XLSTM_API xlstm_status_t xlstm_mlstm_workspace_status(const void *workspace, int32_t *where,
                                            cudaStream_t stream);

/* Human-readable name of a status code (static storage). */
XLSTM_API const char *xlstm_status_string(xlstm_status_t status);

/* Library version string (static storage). */
XLSTM_API const char *xlstm_mlstm_version(void);

/*
 * Which kernel xlstm_mlstm_fwd_chunkwise runs for desc: "tcgen05" (bf16
 * inputs, chunk 64, d_qk in {64, 128, 256}, d_v a multiple of 64), "simt"
 * (fp32 CUDA-core kernel: fp32 inputs and every other supported shape),
 * "copy" (T = 0) or "none" (invalid or unsupported desc).  Static storage.
 */
XLSTM_API const char *xlstm_mlstm_chunkwise_kernel(const xlstm_mlstm_desc_t *desc);

/*
 * Testing hook for the device-side bounded waits.  When enable != 0, the next
 * tcgen05 chunkwise launch withholds one internal hand-off, so that the waits
 * depending on it run out after their 1 s limit: the kernel then records
 * XLSTM_ERR_TIMEOUT in the workspace status block, drains its in-flight copies
 * and tensor-core work, frees its tensor memory and returns (its outputs are
 * not valid).  The flag is consumed by that one launch.  No other effect.
 */
XLSTM_API void xlstm_mlstm_test_timeout_next(int32_t enable);

#ifdef __cplusplus
}
#endif
#endif /* XLSTM_MLSTM_H */
