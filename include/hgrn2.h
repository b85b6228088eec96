/*
 * hgrn2.h -- C ABI of the B200 (sm_100a) HGRN2 recurrence library (libhgrn2.so).
 *
 * The operation ("HGRN2: Gated Linear RNNs with State Expansion", Qin et al.
 * 2024, arXiv 2404.07904; section numbers refer to the paper as summarised on
 * the paperlayer.ai page):
 *
 *   per batch b and head h (heads are independent, §3.2 "multihead"), with a
 *   d_k x d_v fp32 state S (row j = key dimension):
 *
 *     f_t = exp(log_f_t)                        forget gate, one per key dim (§5)
 *     k_t = 1 - f_t = -expm1(log_f_t)           input gate tied to forget gate (§2.1)
 *     S_t = Diag(f_t) S_{t-1} + k_t i_t^T       outer-product state expansion (§3.2)
 *     o_t = S_t^T q_t                           matrix-vector output, UPDATED state (§3.2)
 *
 *   Read as gated linear attention (§3.2: same recurrence as GLA up to the
 *   parameterisation) with key k = 1 - f, value v = i and query q, it is
 *   computed chunkwise on tensor cores.  There is no 1/sqrt(d) scale, no
 *   normalisation and no output gate inside the library.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layouts (row-major, innermost last, no padding):
 *      token tensors q, log_f, dlog_f, dq : [B][T][H][d_k]
 *                    i, o, dO, di         : [B][T][H][d_v]
 *      states        h0, hT, dhT, dh0, S  : [B][H][d_k][d_v]   always float32
 *      decode tensors q, log_f            : [B][H][d_k];  i, o : [B][H][d_v]
 *  - dtype (hgrn2_dtype) is the element type of all token tensors (inputs and
 *    outputs alike).  States are always float32.
 *  - All data pointers are DEVICE pointers owned by the caller, aligned to 16
 *    bytes.  The library allocates no memory, never synchronises inside
 *    hgrn2_fwd / hgrn2_bwd / hgrn2_step, and keeps no pointer after a call.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default
 *    stream).  Argument checks run on the host before anything is launched: a
 *    call that returns an error has launched nothing.  A launch failure reported
 *    by the CUDA runtime returns HGRN2_ERR_CUDA.  Everything a call puts on the
 *    stream (kernel launches, some as programmatic dependents of the launch
 *    before them, and cudaMemsetAsync of workspace or outputs) is stream-ordered,
 *    so a call can be captured into a CUDA graph (hgrn2_bwd_noalloc: see there).
 *  - No exception or abort crosses this ABI.
 *  - Supported sizes: B, H >= 1; T >= 0 (T = 0 writes hT = h0 and nothing else);
 *    1 <= d_k, d_v <= 256; chunk in {16, 32, 64, 128}.  The bf16 tensor-core
 *    path is used when dtype = BF16 and d_k = d_v = 128 or 64; every other
 *    shape up to 128 runs the exact CUDA-core path.  Unsupported shapes return
 *    HGRN2_ERR_UNSUPPORTED.
 *  - A head wider than 128 (d_k or d_v in 129..256) runs as blocks: key dims
 *    0..127 and 128..d_k-1, value dims likewise.  Diag(f) acts on each key dim and
 *    the update on each value column alone (§3.2, §5), so every block pair (a, c)
 *    is a head of its own: its state block S[a, c] evolves alone and o[c] is the
 *    sum over a of the blocks' outputs; the gradients add the same way.  Each
 *    block takes the route of its own sizes, on contiguous copies of its columns
 *    in the workspace; partial outputs are added in fp32 and rounded once.
 *    Packed sequences and the decode step take d_k, d_v <= 128.
 *  - `chunk` is the length of the chunks of the chunkwise algorithm (§3.2);
 *    results do not depend on it beyond rounding.  The CUDA-core path caps it at
 *    what fits in shared memory for the given d_k, d_v.
 *  - log_f must be finite and <= 0 (f in (0, 1]); other values are outside the
 *    method's range and their results are unspecified (no fault).
 *  - Ragged T (not a multiple of the chunk) is handled; the tail is computed
 *    exactly like any other token.
 */
#ifndef HGRN2_H
#define HGRN2_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HGRN2_OK = 0,
    HGRN2_ERR_INVALID_ARG = 1,   /* null required pointer, negative size, bad alignment, short workspace */
    HGRN2_ERR_UNSUPPORTED = 2,   /* valid but unsupported shape / chunk / dtype combination */
    HGRN2_ERR_CUDA = 3,          /* the CUDA runtime reported an error at launch */
    HGRN2_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (see hgrn2_get_device_status) */
    HGRN2_ERR_DEVICE = 5         /* a device-side consistency check failed (see hgrn2_get_device_status) */
} hgrn2_status;

typedef enum {
    HGRN2_FP32 = 0,
    HGRN2_BF16 = 1
} hgrn2_dtype;

/* Bytes of device workspace that hgrn2_fwd (want_bwd = 0), hgrn2_bwd (want_bwd = 1)
 * or hgrn2_bwd_saved (want_bwd = 2; never more than for 1) needs for these sizes.
 * May be 0.  For bf16 heads of 64, the hgrn2_bwd size includes room for the chunk
 * states and an o scratch: that backward runs the tensor-core forward into them,
 * then the saved-state backward.  Returns (size_t)-1 for invalid or unsupported
 * arguments.  Host-only, no CUDA call. */
size_t hgrn2_workspace_size(int B, int T, int H, int dk, int dv, int chunk,
                            hgrn2_dtype dtype, int want_bwd);

/* Forward over a whole sequence (§3.2 recurrence above, chunkwise).
 *   q, log_f : [B,T,H,dk]   i : [B,T,H,dv]          (dtype)
 *   h0       : [B,H,dk,dv] float32 initial state, or NULL for zeros
 *   o        : [B,T,H,dv] output (dtype)
 *   hT       : [B,H,dk,dv] float32 final state S_{T-1}, or NULL to skip
 *   workspace: device scratch of at least hgrn2_workspace_size(..., 0) bytes
 *              (may be NULL when that size is 0); contents need no initialisation
 *              and are undefined afterwards.
 * Inputs must not alias outputs. */
hgrn2_status hgrn2_fwd(const void *q, const void *log_f, const void *i, const float *h0,
                       void *o, float *hT,
                       int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                       void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Backward of L(o, hT) through the forward above, given dO = dL/do and an
 * optional dhT = dL/dhT (NULL = 0).  Writes dq, dlog_f, di (dtype, same layouts
 * as q, log_f, i) and, when dh0 != NULL, dh0 = dL/dh0 (float32).  h0 must be the
 * forward's initial state (NULL = zeros).  The gradient of log_f includes both
 * paths through which it acts: the decay Diag(f) and the tied input gate
 * k = 1 - f (§2.1).  workspace: at least hgrn2_workspace_size(..., 1) bytes.
 * dq must not alias any input: the backward reads dq back after writing it. */
hgrn2_status hgrn2_bwd(const void *q, const void *log_f, const void *i, const float *h0,
                       const void *dO, const float *dhT,
                       void *dq, void *dlog_f, void *di, float *dh0,
                       int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                       void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Training pair: a forward that keeps the chunk states, and a backward that reads
 * them instead of recomputing them.  Chunkwise training (§3.2: the GLA-style
 * chunkwise algorithm) needs the state entering every chunk in both passes;
 * storing it in the forward halves the backward's sweeps over the sequence.
 *
 * hgrn2_saved_size: bytes of the saved-state buffer for these sizes.  0 when the
 * configuration has no saved-state path (the exact CUDA-core route, or T = 0):
 * hgrn2_fwd_train and hgrn2_bwd_saved then behave exactly as hgrn2_fwd and
 * hgrn2_bwd and ignore `saved` (which may be NULL).  (size_t)-1 for invalid or
 * unsupported arguments.  Host-only, no CUDA call.
 *
 * The buffer (device memory, caller-owned, 16-byte aligned, no initialisation
 * needed) is opaque.  For the bf16 tensor-core route it holds, per (b,h), the
 * bf16-rounded state entering each 128-token chunk (the same operand the forward
 * multiplies with; ceil(T/128) x 128 x 128 x 2 bytes), the float32 final state,
 * and which (b,h) took the exact route.  For a head wider than 128 it holds one
 * such region per block pair whose sizes take the tensor-core route.
 *
 * hgrn2_fwd_train: hgrn2_fwd (same arguments and results) that also fills
 *   `saved` (saved_bytes >= hgrn2_saved_size, else HGRN2_ERR_INVALID_ARG).
 * hgrn2_bwd_saved: hgrn2_bwd (same arguments and results, same workspace size)
 *   for a forward made by hgrn2_fwd_train with the same q, log_f, i, h0 and
 *   sizes, whose `saved` buffer is passed unchanged.  A buffer from other inputs
 *   gives wrong gradients (it is not checked).  dq is only written, never read
 *   back, on this path.  The bf16 route runs one kernel launch. */
size_t hgrn2_saved_size(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype);

hgrn2_status hgrn2_fwd_train(const void *q, const void *log_f, const void *i, const float *h0,
                             void *o, float *hT, void *saved, size_t saved_bytes,
                             int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                             void *workspace, size_t ws_bytes, cudaStream_t stream);

hgrn2_status hgrn2_bwd_saved(const void *q, const void *log_f, const void *i, const float *h0,
                             const void *saved, size_t saved_bytes,
                             const void *dO, const float *dhT,
                             void *dq, void *dlog_f, void *di, float *dh0,
                             int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                             void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Packed variable-length sequences.  The paper trains on concatenated documents
 * (§4 language modelling); packing several sequences into one token tensor without
 * padding is how that is fed to a per-sequence recurrence.  The recurrence restarts
 * at every sequence boundary.
 *   token tensors q, log_f, dq, dlog_f: [total_T][H][dk];  i, o, dO, di: [total_T][H][dv]
 *   cu_seqlens: DEVICE int32 [nseq + 1], 16-byte aligned; sequence s is tokens
 *     cu_seqlens[s] .. cu_seqlens[s+1]-1 (0 = cu[0] <= cu[1] <= ... <= cu[nseq] = total_T;
 *     not checked on the host: values are clamped to [0, total_T] on the device, so a
 *     malformed array gives wrong results, never an out-of-range access).  Sequences may
 *     be empty and may start at any token.
 *   states h0, hT, dhT, dh0: [nseq][H][dk][dv] float32, one per sequence and head.
 * hgrn2_workspace_size_varlen: workspace bytes of both calls (never 0).
 * hgrn2_saved_size_varlen: bytes of the optional saved-state buffer (0 where there is
 *   no saved-state path: the exact route, or total_T = 0); (size_t)-1 for bad sizes.
 * hgrn2_fwd_varlen: forward of every sequence; `saved` (may be NULL) receives what
 *   hgrn2_bwd_varlen reads, as for hgrn2_fwd_train.
 * hgrn2_bwd_varlen: backward of every sequence.  With the `saved` buffer of the
 *   matching hgrn2_fwd_varlen call it is one reverse-sweep launch on tensor cores;
 *   without it (NULL) the exact CUDA-core route computes it. */
size_t hgrn2_workspace_size_varlen(int nseq, int total_T, int H, int dk, int dv, int chunk,
                                   hgrn2_dtype dtype);
size_t hgrn2_saved_size_varlen(int nseq, int total_T, int H, int dk, int dv, hgrn2_dtype dtype);

hgrn2_status hgrn2_fwd_varlen(const void *q, const void *log_f, const void *i, const float *h0,
                              void *o, float *hT, const int *cu_seqlens, int nseq, int total_T,
                              int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                              void *saved, size_t saved_bytes, void *workspace, size_t ws_bytes,
                              cudaStream_t stream);

hgrn2_status hgrn2_bwd_varlen(const void *q, const void *log_f, const void *i, const float *h0,
                              const void *saved, size_t saved_bytes,
                              const void *dO, const float *dhT,
                              void *dq, void *dlog_f, void *di, float *dh0,
                              const int *cu_seqlens, int nseq, int total_T, int H, int dk, int dv,
                              int chunk, hgrn2_dtype dtype, void *workspace, size_t ws_bytes,
                              cudaStream_t stream);

/* Allocation-free variant of hgrn2_bwd.  The paper has no counterpart: this
 * entry point exists for callers that cannot give the library a device
 * buffer -- for example a plain C host program that links only this library
 * and owns no device allocator, or a service whose memory policy forbids new
 * device allocations once it is running (cudaMalloc and cudaFree synchronise
 * the device and can stall unrelated work).  Arguments and results are those
 * of hgrn2_bwd without the workspace.  Its scratch is a fixed array of
 * HGRN2_NOALLOC_SCRATCH_BYTES bytes inside the library, which every GPU that
 * loads the library keeps until the process exits; sizes whose backward needs
 * more scratch than that (for d_k = 128 and bf16: B*H > 2032) return
 * HGRN2_ERR_UNSUPPORTED and launch nothing.  The first call on a device looks
 * up the array's device address on that device (make that first call before
 * any stream capture on it); the lookup is repeated when the device's current
 * context has changed since, e.g. after cudaDeviceReset.  All calls share the one array and it keeps the
 * last call's contents; nothing in it needs to start at zero, because each call
 * writes what it reads.  Calls that may overlap on the GPU (on different
 * streams, or from different host threads) race on the array: serialise them.
 * This entry point calls no device allocation routine. */
#define HGRN2_NOALLOC_SCRATCH_BYTES (1u << 20)
hgrn2_status hgrn2_bwd_noalloc(const void *q, const void *log_f, const void *i, const float *h0,
                               const void *dO, const float *dhT,
                               void *dq, void *dlog_f, void *di, float *dh0,
                               int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                               cudaStream_t stream);

/* One recurrent decode step for B sequences with one new token each (§1: linear-
 * time recurrent inference without a KV cache; the §3.2 recurrence for one t):
 *   S <- Diag(f) S + k i^T  (in place, float32),  then  o = S^T q.
 *   q, log_f : [B,H,dk]   i, o : [B,H,dv]   (dtype)     S : [B,H,dk,dv] float32
 * S must not alias q, log_f, i or o.  dv must be a multiple of 4. */
hgrn2_status hgrn2_step(const void *q, const void *log_f, const void *i, float *S, void *o,
                        int B, int H, int dk, int dv, hgrn2_dtype dtype, cudaStream_t stream);

/* hgrn2_step with the lower-bounded forget gate formed in the kernel from raw gate
 * logits (§2.2: each layer keeps its forget gate above a lower bound lb):
 *   f = lb + (1 - lb) sigmoid(g),   k = 1 - f = (1 - lb) sigmoid(-g)
 *   g : [B,H,dk] (dtype), the gate pre-activations of this token; 0 <= lb < 1 (else
 *   HGRN2_ERR_INVALID_ARG).  Everything else as hgrn2_step.  It saves the separate
 *   elementwise pass that would write log f for hgrn2_step. */
hgrn2_status hgrn2_step_lb(const void *q, const void *g, const void *i, float lb, float *S, void *o,
                           int B, int H, int dk, int dv, hgrn2_dtype dtype, cudaStream_t stream);

/* Backward of one hgrn2_step, for a loss L(o, S_new) of the step's output and updated
 * state (truncated backpropagation through recurrent decode steps):
 *   S       : [B,H,dk,dv] float32, the state BEFORE the step (what hgrn2_step read)
 *   dO      : [B,H,dv] (dtype), dL/do
 *   dS      : [B,H,dk,dv] float32, dL/dS_new, or NULL (zero)
 *   dS_prev : out [B,H,dk,dv] float32, dL/dS, or NULL; may be dS itself (in place), else
 *             must not overlap it (HGRN2_ERR_INVALID_ARG)
 *   dq, dlog_f : out [B,H,dk] (dtype);  di : out [B,H,dv] (dtype)
 * With G = dS + q dO^T:  dq = S_new dO,  dlog f = f . rowsum(G . (S - 1 i^T)),
 * di = G^T k,  dS_prev = Diag(f) G  (the §3.2 recurrence for one token, differentiated
 * with k = 1 - f tied to f as in §2.1).  It reads S and dS and writes dS_prev once.
 * Same size limits as hgrn2_step. */
hgrn2_status hgrn2_step_bwd(const void *q, const void *log_f, const void *i, const float *S,
                            const void *dO, const float *dS, float *dS_prev,
                            void *dq, void *dlog_f, void *di,
                            int B, int H, int dk, int dv, hgrn2_dtype dtype, cudaStream_t stream);

/* Backward of one hgrn2_step_lb: as hgrn2_step_bwd, with the gate logits g and lb of that
 * step in place of log f, and dg = dL/dg = dL/dlog f . (1 - lb) sigmoid(g) sigmoid(-g) / f
 * written in place of dlog f.  0 <= lb < 1, else HGRN2_ERR_INVALID_ARG. */
hgrn2_status hgrn2_step_lb_bwd(const void *q, const void *g, const void *i, float lb, const float *S,
                               const void *dO, const float *dS, float *dS_prev,
                               void *dq, void *dg, void *di,
                               int B, int H, int dk, int dv, hgrn2_dtype dtype, cudaStream_t stream);

/* Scalar-decay variant: one decay per head and token and a key of its own, the per-head
 * decay of models such as Mamba2 and RetNet that §5 contrasts with HGRN2's per-dimension
 * decay (where the masked form ((Q K^T) . D) V holds exactly):
 *   S_t = g_t S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t,   g_t = exp(log_g_t)  (log_g <= 0)
 *   q, k : [B,T,H,dk]   v, o : [B,T,H,dv]   log_g : [B,T,H]   (all dtype)
 *   h0, hT : [B,H,dk,dv] float32 (NULL allowed, as for hgrn2_fwd)
 * Forward and backward run on tensor cores for bf16 with dk = dv = 128 or 64 (128-token
 * chunks, bf16 operands, fp32 accumulation and state; a (batch, head) with a chunk whose
 * summed log decay is below -59.8 is recomputed on CUDA cores, by the forward inside its own
 * launch); everything else runs chunkwise on CUDA cores in fp32 arithmetic, exact for any
 * decay strength.
 * 1 <= dk, dv <= 128; any T >= 0; pointers 16-byte aligned.
 * hgrn2_scalar_bwd: gradients dq, dk_out (of k), dv_out (of v), dlog_g (same shapes and dtype
 * as the inputs) and dh0 (NULL: not computed) of L(o, hT) given dO and dhT (NULL: zero).
 * workspace: device scratch of at least hgrn2_scalar_workspace_size(..., 1) bytes.  On the
 * tensor-core route (bf16, dk = dv = 128 or 64) this backward runs the forward again with its
 * chunk states saved into that workspace, then a reverse sweep over them; pairs whose summed log
 * decay over a 128-token chunk is below -59.8 are recomputed on CUDA cores.
 * hgrn2_scalar_workspace_size: bytes of workspace for the forward (want_bwd = 0: none),
 * hgrn2_scalar_bwd (1) or hgrn2_scalar_bwd_saved (2); (size_t)-1 for bad sizes. */
size_t hgrn2_scalar_workspace_size(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype, int want_bwd);
hgrn2_status hgrn2_scalar_fwd(const void *q, const void *k, const void *v, const void *log_g,
                              const float *h0, void *o, float *hT,
                              int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                              cudaStream_t stream);
hgrn2_status hgrn2_scalar_bwd(const void *q, const void *k, const void *v, const void *log_g,
                              const float *h0, const void *dO, const float *dhT,
                              void *dq, void *dk_out, void *dv_out, void *dlog_g, float *dh0,
                              int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                              void *workspace, size_t ws_bytes, cudaStream_t stream);

/* The scalar-decay training pair: hgrn2_scalar_fwd_train is hgrn2_scalar_fwd that also keeps
 * what hgrn2_scalar_bwd_saved reads (the bf16 state entering every 128-token chunk, the fp32 final
 * state and the range flags) in `saved`, a device buffer of hgrn2_scalar_saved_size(...) bytes
 * (0 where there is no saved-state path: fp32, other head sizes or T = 0; then `saved` may be
 * NULL and the backward takes the exact route).  hgrn2_scalar_bwd_saved is hgrn2_scalar_bwd
 * reading that buffer instead of running the forward again; its workspace is
 * hgrn2_scalar_workspace_size(..., 2) bytes.  A buffer shorter than the saved size returns
 * HGRN2_ERR_INVALID_ARG before any launch. */
size_t hgrn2_scalar_saved_size(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype);
hgrn2_status hgrn2_scalar_fwd_train(const void *q, const void *k, const void *v, const void *log_g,
                                    const float *h0, void *o, float *hT, void *saved, size_t saved_bytes,
                                    int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                                    cudaStream_t stream);
hgrn2_status hgrn2_scalar_bwd_saved(const void *q, const void *k, const void *v, const void *log_g,
                                    const float *h0, const void *saved, size_t saved_bytes,
                                    const void *dO, const float *dhT,
                                    void *dq, void *dk_out, void *dv_out, void *dlog_g, float *dh0,
                                    int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                                    void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ---- One sequence across several GPUs (sequence parallelism) ----------------------
 * Over a contiguous slice of tokens the recurrence (§3.2) is affine in the state that
 * enters the slice, S_out = Diag(g) S_in + U, and its backward is affine in the gradient
 * that leaves it, dL/dS_in = Diag(g) dL/dS_out + W, with
 *   g = prod_t f_t,   U = sum_t (k_t * prod_{r>t} f_r) i_t^T,   W = sum_t (q_t * prod_{r<=t} f_r) dO_t^T.
 * Each GPU computes the maps of its own slice, the maps are exchanged (the caller's
 * all-gather), hgrn2_affine_scan gives each slice its boundary state, and each GPU then runs
 * hgrn2_fwd / hgrn2_bwd on its slice from those boundary states (h0 = the state entering the
 * slice, dhT = the gradient leaving it).  The chunkwise algorithm's state passing, with slices
 * in place of chunks; the pages name linear-attention sequence parallelism (LASP) for running
 * it across devices.
 *
 * hgrn2_state_map: the forward map of a slice.
 *   log_f : [B,T,H,dk] (dtype)   i : [B,T,H,dv] (dtype)
 *   g : out [B,H,dk] float32     U : out [B,H,dk,dv] float32
 * hgrn2_state_map_bwd: the backward map of a slice (g is the same as the forward's).
 *   q, log_f : [B,T,H,dk]   dO : [B,T,H,dv]   g : out [B,H,dk]   W : out [B,H,dk,dv]
 * Both: dk <= 128, dv <= 256; T >= 0 (T = 0 gives g = 1, U = W = 0).  Exact for any decay
 * strength (every product of gates is <= 1).  bf16 with dk = dv = 128 computes the forward map
 * on the tensor cores; every other case steps the recurrence token by token on CUDA cores in
 * fp32.  Asynchronous on `stream`; the library allocates nothing. */
hgrn2_status hgrn2_state_map(const void *log_f, const void *i, int B, int T, int H, int dk, int dv,
                             hgrn2_dtype dtype, float *g, float *U, cudaStream_t stream);
hgrn2_status hgrn2_state_map_bwd(const void *q, const void *log_f, const void *dO, int B, int T, int H,
                                 int dk, int dv, hgrn2_dtype dtype, float *g, float *W, cudaStream_t stream);

/* Scan of R slice maps in fp32: S = init (zeros if NULL), then for `count` maps
 * r = first, first + step, ... (step = +1 or -1, every r in [0, R)):
 *   S <- Diag(g_r) S + M_r
 *   g : [R][B,H,dk] float32   M : [R][B,H,dk,dv] float32   init, S : [B,H,dk,dv] float32
 * Forward: r = 0 .. rank-1 from h0 gives the state entering slice `rank`; all R maps give
 * hT.  Backward (M = W): r = R-1 down to rank+1 from dhT gives dL/dS leaving slice `rank`.
 * S may be init (in place); it must not overlap g or M.  count = 0 copies init (or zeros). */
hgrn2_status hgrn2_affine_scan(const float *g, const float *M, int R, int first, int count, int step,
                               const float *init, float *S, int B, int H, int dk, int dv,
                               cudaStream_t stream);

/* Check of the failure reporting: launches one block that waits, through the bounded
 * wait every kernel of the library uses, on a barrier that nothing arrives at.  The
 * wait gives up after `polls` polls (1 .. 2^24; each poll lasts at most the hardware's
 * short try-wait window), records HGRN2_ERR_TIMEOUT in the device status word and the
 * block exits normally: no fault, the context stays usable.  hgrn2_get_device_status
 * then returns HGRN2_ERR_TIMEOUT (and clears it). */
hgrn2_status hgrn2_selftest_wait_timeout(unsigned int polls, cudaStream_t stream);

/* Synchronises `stream`, then returns and clears the library's device-side
 * status word of the current device: HGRN2_OK, HGRN2_ERR_TIMEOUT (a bounded
 * wait gave up) or HGRN2_ERR_DEVICE (a consistency check failed).  Returns
 * HGRN2_ERR_CUDA if the synchronisation itself fails. */
hgrn2_status hgrn2_get_device_status(cudaStream_t stream);

/* Diagnostic counters, accumulated since the last reset:
 *   out[0] = (batch, head) passes that took the exact CUDA-core route because a
 *            chunk's cumulative log-decay spanned more than the tensor-core
 *            factorisation allows (device counter of the current device);
 *   out[1] = tensor-core chunk passes completed (device counter);
 *   out[2] = kernel launches issued by this library in this process (host count).
 * Synchronises `stream`.  n = number of entries of `out` (<= 3 are written).
 * reset != 0 zeroes the counters after reading them. */
hgrn2_status hgrn2_get_counters(long long *out, int n, int reset, cudaStream_t stream);

/* Static English description of a status code (never NULL). */
const char *hgrn2_status_string(hgrn2_status s);

/* Library version, e.g. "hgrn2-b200 0.1". */
const char *hgrn2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HGRN2_H */
