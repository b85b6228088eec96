// kernels.h -- internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace hgrn2 {

struct SimtFwdArgs {
    const void *q, *lf, *x;
    const float *h0;
    void *o;
    float *hT;
    int B, T, H, dk, dv, C;
    const int *only;   // if non-null: only (b,h) with only[b*H+h] != 0 are computed
    const int *cu;     // if non-null: packed sequences, B = their number, T = total tokens
    const int *perm;   // with cu: launch order of the sequences (longest first), or null
};

struct TcFwdArgs {
    const void *q, *lf, *x;
    const float *h0;
    void *o;
    float *hT;
    int *flags;        // [B*H] out: 1 where the (b,h) needs the exact route
    float *seg_ws;     // segment aggregates, tc_fwd_workspace(B, T, H) bytes (may be null if 0)
    int B, T, H;
    int simt_C;        // chunk of the exact route
    void *st16;        // out, or null: bf16 state entering every chunk, tc_saved_slots() tiles
    float *hTs;        // out (with st16): final state [B*H][128][128]
    const int *cu;     // if non-null: packed sequences, B = their number, T = total tokens
    const int *perm;   // with cu: launch order of the sequences (longest first), or null
    int D;             // head size d_k = d_v: 128 or 64
    const void *lgs;   // scalar-decay variant: log g [B][T][H] (lf is then the key k); else null
    // Heads of width nK * 128 = nV * 128 read in place (nK = nV = 2: 256): H counts block pairs,
    // H / (nK nV) the caller's heads; q, lf, x, o are the caller's [B][T][H / (nK nV)][256] tensors.
    // o must be zero on entry: every block pair adds its share into it.  opart: scratch
    // [nK][B][T][H / (nK nV)][256] for the shares of pairs flagged for the exact route.
    int nK = 1, nV = 1;
    void *opart = nullptr;
};

struct SimtBwdArgs {
    const void *q, *lf, *x, *dO;
    const float *h0, *dhT;
    void *dq, *dlf, *dx;
    float *dh0;
    float *rs;   // [B*H*dk] workspace: rowsum(dhT * hT)
    int B, T, H, dk, dv, C;
    const int *only;   // if non-null: only (b,h) with only[b*H+h] != 0 are computed
    const int *cu;     // if non-null: packed sequences, B = their number, T = total tokens
    const int *perm;   // with cu: launch order of the sequences (longest first), or null
};

struct TcBwdArgs {
    const void *q, *lf, *x, *dO;
    const float *h0, *dhT;
    void *dq, *dlf, *dx;
    float *dh0;
    float *rs;         // [B*H*128] workspace
    int *flags;        // [B*H] recompute: workspace, out; saved states: in, from the forward
    int B, T, H;
    int simt_C;        // chunk of the exact route
    const void *st16;  // saved bf16 chunk-entry states (tc_saved_slots() tiles), or null (recompute)
    const float *hTs;  // saved final state [B*H][128][128] (with st16)
    const int *cu;     // if non-null: packed sequences, B = their number, T = total tokens (needs st16)
    const int *perm;   // with cu: launch order of the sequences (longest first), or null
    int D;             // head size d_k = d_v: 128 or 64 (64: saved-state mode only)
    const void *lgs;   // scalar-decay variant (saved mode): log g [B][T][H]; lf is then k, dlf dk
    void *dlg;         // scalar-decay variant: d log g [B][T][H]
    // Heads read in place (saved mode, nK = nV = 2), as for TcFwdArgs: q, lf, x, dO, dq, dlf, dx are
    // the caller's 256-wide tensors; dq, dlf, dx must be zero on entry (every block pair adds its
    // share).  Scratch for the shares of flagged pairs: dq, dlf as the value blocks' partials
    // [nV][B][T][Hw][256] (dq_part, dlf_part), dx as the key blocks' [nK][B][T][Hw][256] (dx_part).
    int nK = 1, nV = 1;
    void *dq_part = nullptr, *dlf_part = nullptr, *dx_part = nullptr;
    // saved states, dense d = 128, few (b,h): sequence segments' workspace, tc_bwd_workspace(B, T, H)
    // bytes (null: one CTA per (b,h))
    float *seg_ws = nullptr;
};

struct StepBwdArgs {
    const void *q, *lf, *x;   // lf: log f, or the gate logits g with gate_lb
    const float *S;           // state before the step
    const void *dO;
    const float *dS;          // dL/dS_new or null
    float *dS_prev;           // out or null; may equal dS
    void *dq, *dlf, *dx;      // dlf: d log f, or dL/dg with gate_lb
    int B, H, dk, dv;
    bool gate_lb;
    float lb;
};
cudaError_t launch_step_bwd(const StepBwdArgs &a, bool bf16, cudaStream_t st);

// Scalar-decay variant (one decay per head and token, explicit key): exact route on CUDA cores.
struct ScalarArgs {
    const void *q, *k, *v, *lg;     // lg: log g [B][T][H]
    const float *h0;
    void *o;                        // forward outputs
    float *hT;
    const void *dO;                 // backward inputs / outputs
    const float *dhT;
    void *dq, *dk_out, *dv_out, *dlg;
    float *dh0;
    float *rs;                      // backward workspace: <dhT, hT> per (b,h)
    float *qdq;                     // backward workspace: q_t . dq_t per token [B][T][H], fp32
    int B, T, H, dk, dv;
    const int *only;                // backward: if non-null, only (b,h) with only[b*H+h] != 0
};
cudaError_t launch_scalar_fwd(const ScalarArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_scalar_bwd(const ScalarArgs &a, bool bf16, cudaStream_t st);

// Longest-first launch order of packed sequences: perm[r] = the sequence that CTA row r runs,
// ordered by decreasing number of 128-token chunks (one CTA; any nseq).
cudaError_t launch_lpt_order(const int *cu, int nseq, int T, int *perm, cudaStream_t st);
// Heads wider than 128 (wide.cu): state blocks between [nmat][dk][dv] and rw x cw matrices
// `bstride` floats apart; dst[r][off + c] = p0[r][c] + p1[r][c] (p1 may be null) in fp32, dst rows
// `pitch` elements apart, p0 / p1 rows `spitch` apart.
cudaError_t launch_state_block(float *full, float *blk, size_t bstride, size_t nmat, int dk, int dv, int ro, int rw,
                               int co, int cw, bool to_full, cudaStream_t st);
cudaError_t launch_sum_blocks(void *dst, int pitch, int off, const void *p0, const void *p1, int spitch, size_t rows,
                              int w, bool bf16, cudaStream_t st);

// State maps of a token slice (seqpar.cu): forward (g, U) from log f and v = i, or backward
// (g, W) from log f, q and v = dO; [B][H][dk] and [B][H][dk][dv] fp32.  CUDA cores, any shape
// with dk <= 128.
struct StateMapArgs {
    const void *lf, *q, *v;
    float *g, *M;
    int B, T, H, dk, dv;
    bool backward;
};
cudaError_t launch_state_map(const StateMapArgs &a, bool bf16, cudaStream_t st);
// The forward map of bf16 d = 128 slices on the tensor cores (the segment aggregate of tc_fwd.cu
// over the whole slice).
cudaError_t launch_tc_state_map(const void *lf, const void *x, int B, int T, int H, float *g, float *U,
                                cudaStream_t st);
// S = init (or 0); S <- Diag(g_r) S + M_r for r = first, first + step, ... (count maps).
cudaError_t launch_affine_scan(const float *g, const float *M, const float *init, float *S, size_t nbh, int dk, int dv,
                               int first, int count, int step, cudaStream_t st);

size_t simt_fwd_smem(int C, int dk, int dv);
size_t simt_bwd_dq_smem(int C, int dk, int dv);
size_t simt_bwd_rev_smem(int C, int dk, int dv);
cudaError_t launch_simt_fwd(const SimtFwdArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_simt_bwd(const SimtBwdArgs &a, bool bf16, cudaStream_t st);

size_t tc_fwd_smem();
int tc_saved_slots(int B, int T, int H, bool packed);
void tc_fwd_segments(int B, int T, int H, int *nseg, int *tps);
size_t tc_fwd_workspace(int B, int T, int H);
// Kernel launches of one segmented forward call with nseg segments per pair (1 without segments).
int tc_fwd_launches(int nseg);
// Sequence segments of the saved-state backward (dense, d = 128, bf16): workspace bytes (0: one
// CTA per (b,h)) and kernel launches of one call.
size_t tc_bwd_workspace(int B, int T, int H);
int tc_bwd_launches(int B, int T, int H);
size_t tc_bwd_smem();
cudaError_t launch_tc_bwd(const TcBwdArgs &a, cudaStream_t st);
cudaError_t launch_tc_fwd(const TcFwdArgs &a, cudaStream_t st);

// gate_lb: `lf` holds raw gate logits g and f = lb + (1 - lb) sigmoid(g); else `lf` is log f.
cudaError_t launch_step(const void *q, const void *lf, const void *x, float *S, void *o, int B, int H,
                        int dk, int dv, bool bf16, bool gate_lb, float lb, cudaStream_t st);

}  // namespace hgrn2
