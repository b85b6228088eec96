// api.cu -- the extern "C" boundary of libhgrn2.so (declared in include/hgrn2.h).
//
// Host-side argument validation, workspace planning and dispatch between the
// bf16 tensor-core kernels and the exact CUDA-core kernels.  Nothing here
// allocates device memory or synchronises, except the two status/counter
// queries, which synchronise the given stream by contract.
#include <stdint.h>

#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

#include <initializer_list>

using namespace hgrn2;

namespace {

constexpr size_t kMaxSmem = 227 * 1024;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool chunk_ok(int chunk) { return chunk == 16 || chunk == 32 || chunk == 64 || chunk == 128; }

// Largest chunk <= requested whose exact-route shared memory fits.
int simt_chunk(int chunk, int dk, int dv, bool bwd) {
    for (int C = chunk; C >= 16; C >>= 1) {
        size_t s = bwd ? (simt_bwd_dq_smem(C, dk, dv) > simt_bwd_rev_smem(C, dk, dv)
                              ? simt_bwd_dq_smem(C, dk, dv)
                              : simt_bwd_rev_smem(C, dk, dv))
                       : simt_fwd_smem(C, dk, dv);
        if (s <= kMaxSmem) return C;
    }
    return 0;
}

hgrn2_status check_common(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt) {
    if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return HGRN2_ERR_INVALID_ARG;
    if (dt != HGRN2_FP32 && dt != HGRN2_BF16) return HGRN2_ERR_INVALID_ARG;
    if (!chunk_ok(chunk)) return HGRN2_ERR_UNSUPPORTED;
    if (dk > 256 || dv > 256) return HGRN2_ERR_UNSUPPORTED;   // wider than 128: blocks of <= 128
    // index arithmetic is 64-bit; keep grid dimensions and per-tensor element counts sane
    if ((long long)B * H > (1ll << 30)) return HGRN2_ERR_UNSUPPORTED;
    return HGRN2_OK;
}

// The bf16 tensor-core route takes d_k = d_v = 128; everything else runs the exact route.
// The tensor-core route: bf16 with d_k = d_v = 128, or 64 (run as 128-wide tiles whose second
// half is held at zero).
bool use_tc(int dk, int dv, hgrn2_dtype dt) { return dt == HGRN2_BF16 && dk == dv && (dk == 128 || dk == 64); }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Heads wider than 128 run as blocks of the 128-wide path (wide.cu): the key dims in blocks a
// (w[0][a] dims from off[0][a]) and the value dims in blocks c (w[1][c] from off[1][c]).
bool is_wide(int dk, int dv) { return dk > 128 || dv > 128; }
struct WideSplit {
    int n[2], off[2][2], w[2][2];
};
WideSplit wide_split(int dk, int dv) {
    WideSplit s{};
    const int d[2] = {dk, dv};
    for (int x = 0; x < 2; ++x) {
        s.w[x][0] = d[x] < 128 ? d[x] : 128;
        s.w[x][1] = d[x] - s.w[x][0];
        s.off[x][0] = 0;
        s.off[x][1] = s.w[x][0];
        s.n[x] = s.w[x][1] > 0 ? 2 : 1;
    }
    return s;
}
// Scratch of a wide-head call, carved from the workspace (sizes only when base is null).
struct WideWs {
    char *q[2], *f[2], *x[2], *dO[2];          // token blocks; null: the caller's tensor serves
    char *part[2][2], *pq[2][2], *pf[2][2];    // per block pair: o (or di) and dq, d log f partials
    float *h0[2][2], *hT[2][2], *dhT[2][2], *dh0[2][2];
    char *sub;                                 // the block calls' own workspace
    size_t sub_bytes, total;
};
WideWs wide_ws(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt, int want_bwd, bool tc64, char *base);
size_t wide_saved(int B, int T, int H, int dk, int dv, hgrn2_dtype dt, size_t off[2][2]);
// Blocks of equal size (each of d_k, d_v is 256 or at most 128): the nb block pairs of a head run
// as nb heads of one call of the 128-wide path, block pair (a, c) of head h as head
// h * nb + a * n[1] + c, so that the whole problem is one launch over H * nb heads.
bool wide_uniform(int dk, int dv) { return (dk == 256 || dk <= 128) && (dv == 256 || dv <= 128); }
struct WideStack {
    char *q, *f, *x, *dO;         // [B*T*H][nb][block width]
    char *part, *pq, *pf;         // o (or di), dq, d log f of the H * nb heads
    float *h0, *hT, *dhT, *dh0;   // [B*H*nb][kw][vw]
    char *sub;
    size_t sub_bytes, total;
};
WideStack wide_stack_ws(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt, int want_bwd, bool tc64,
                        char *base);

// Saved-state buffer of the tensor-core route (written by hgrn2_fwd_train, read by
// hgrn2_bwd_saved): bf16 state entering every 128-token chunk, fp32 final state, and the
// forward's exact-route flags.
struct SavedLayout {
    size_t hTs, flags, perm, total;   // byte offsets (the bf16 states start at 0)
};
SavedLayout saved_layout(int B, int T, int H, bool packed = false) {
    const size_t BH = (size_t)B * H, slots = (size_t)tc_saved_slots(B, T, H, packed);
    SavedLayout l;
    l.hTs = align256(slots * 128 * 128 * 2);
    l.flags = l.hTs + align256(BH * 128 * 128 * sizeof(float));
    l.perm = l.flags + align256(BH * sizeof(int));
    l.total = l.perm + (packed ? align256((size_t)B * sizeof(int)) : 0);   // packed: launch order
    return l;
}

// Workspace of hgrn2_fwd / hgrn2_bwd.  The backward of 64-wide heads without saved states
// (tc64) runs the tensor-core forward into a saved-state buffer and an o scratch inside the
// workspace, then the saved-state backward; the no-alloc backward passes tc64 = false and
// takes the exact route instead.
size_t ws_bytes_base(int B, int H, int dk, int dv, hgrn2_dtype dt, int want_bwd) {
    size_t bytes = 0;
    if (want_bwd) bytes += align256(sizeof(float) * (size_t)B * H * dk);   // rowsum(dhT * hT)
    if (use_tc(dk, dv, dt)) bytes += align256(sizeof(int) * (size_t)B * H);  // exact-route flags
    return bytes;
}
// The backward without saved states for few (b,h) (sequence segments): it runs the training
// forward into its workspace and then the saved-state backward, which both run in segments,
// instead of one CTA per (b,h) walking every chunk twice.
bool segmented_recompute(int B, int T, int H, int dk, int dv, hgrn2_dtype dt) {
    return dt == HGRN2_BF16 && dk == 128 && dv == 128 && T > 0 && tc_bwd_workspace(B, T, H) > 0;
}
struct RecomputeLayout {
    size_t saved, o, fws, total;   // offsets of the saved buffer, the o scratch, the forward's workspace
};
size_t ws_bytes_needed(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt, int want_bwd, bool tc64);
// [the saved-state backward's workspace][saved buffer][o scratch][the forward's workspace]
RecomputeLayout recompute_layout(int B, int T, int H, int dv, hgrn2_dtype dt) {
    RecomputeLayout l;
    l.saved = ws_bytes_needed(B, T, H, 128, dv, 64, dt, 2, false);
    l.o = l.saved + align256(saved_layout(B, T, H).total);
    l.fws = l.o + align256((size_t)B * T * H * dv * 2);
    l.total = l.fws + ws_bytes_needed(B, T, H, 128, dv, 64, dt, 0, true);
    return l;
}
size_t ws_bytes_needed(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt, int want_bwd,
                       bool tc64 = true) {
    if (is_wide(dk, dv))
        return wide_uniform(dk, dv) ? wide_stack_ws(B, T, H, dk, dv, chunk, dt, want_bwd, tc64, nullptr).total
                                    : wide_ws(B, T, H, dk, dv, chunk, dt, want_bwd, tc64, nullptr).total;
    size_t bytes = ws_bytes_base(B, H, dk, dv, dt, want_bwd);
    if (!want_bwd && use_tc(dk, dv, dt) && dk == 128 && T > 0) bytes += align256(tc_fwd_workspace(B, T, H));
    if (want_bwd == 2 && use_tc(dk, dv, dt) && dk == 128 && T > 0) bytes += align256(tc_bwd_workspace(B, T, H));
    if (want_bwd == 1 && tc64 && segmented_recompute(B, T, H, dk, dv, dt)) bytes = recompute_layout(B, T, H, dv, dt).total;
    if (want_bwd && tc64 && use_tc(dk, dv, dt) && dk == 64 && T > 0)   // saved states + o scratch
        bytes += saved_layout(B, T, H).total + align256((size_t)B * T * H * dv * 2);
    return bytes;
}

size_t saved_bytes_needed(int B, int T, int H, int dk, int dv, hgrn2_dtype dt) {
    if (is_wide(dk, dv)) {
        if (!wide_uniform(dk, dv)) return wide_saved(B, T, H, dk, dv, dt, nullptr);
        const WideSplit s = wide_split(dk, dv);
        return saved_bytes_needed(B, T, H * s.n[0] * s.n[1], s.w[0][0], s.w[1][0], dt);
    }
    return (use_tc(dk, dv, dt) && T > 0) ? saved_layout(B, T, H).total : 0;
}

WideStack wide_stack_ws(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt, int want_bwd, bool tc64,
                        char *base) {
    const WideSplit s = wide_split(dk, dv);
    const int nb = s.n[0] * s.n[1], kw = s.w[0][0], vw = s.w[1][0];
    const size_t es = dt == HGRN2_BF16 ? 2 : 4, rows = (size_t)B * T * H * nb;
    const size_t sb = (size_t)B * H * nb * kw * vw * sizeof(float);
    WideStack w{};
    size_t p = 0;
    auto take = [&](size_t n) -> char * {
        char *r = base ? base + p : nullptr;
        p += align256(n);
        return r;
    };
    w.q = take(rows * kw * es);
    w.f = take(rows * kw * es);
    w.x = take(rows * vw * es);
    w.part = take(rows * vw * es);
    w.h0 = (float *)take(sb);
    if (want_bwd) {
        w.dO = take(rows * vw * es);
        w.pq = take(rows * kw * es);
        w.pf = take(rows * kw * es);
        w.dhT = (float *)take(sb);
        w.dh0 = (float *)take(sb);
    } else {
        w.hT = (float *)take(sb);
    }
    w.sub_bytes = ws_bytes_needed(B, T, H * nb, kw, vw, chunk, dt, want_bwd, tc64);
    w.sub = take(w.sub_bytes);
    w.total = p;
    return w;
}

// Block (a, c) regions of a wide head's saved buffer, each as saved_bytes_needed for the block.
size_t wide_saved(int B, int T, int H, int dk, int dv, hgrn2_dtype dt, size_t off[2][2]) {
    const WideSplit s = wide_split(dk, dv);
    size_t p = 0;
    for (int a = 0; a < s.n[0]; ++a)
        for (int c = 0; c < s.n[1]; ++c) {
            if (off) off[a][c] = p;
            p += align256(saved_bytes_needed(B, T, H, s.w[0][a], s.w[1][c], dt));
        }
    return p;
}

WideWs wide_ws(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dt, int want_bwd, bool tc64, char *base) {
    const WideSplit s = wide_split(dk, dv);
    const size_t es = dt == HGRN2_BF16 ? 2 : 4, rows = (size_t)B * T * H, BH = (size_t)B * H;
    WideWs w{};
    size_t p = 0;
    auto take = [&](size_t n) -> char * {
        char *r = base ? base + p : nullptr;
        p += align256(n);
        return r;
    };
    if (s.n[0] > 1)
        for (int a = 0; a < 2; ++a) {
            w.q[a] = take(rows * s.w[0][a] * es);
            w.f[a] = take(rows * s.w[0][a] * es);
        }
    if (s.n[1] > 1)
        for (int c = 0; c < 2; ++c) {
            w.x[c] = take(rows * s.w[1][c] * es);
            if (want_bwd) w.dO[c] = take(rows * s.w[1][c] * es);
        }
    size_t sub = 0;
    for (int a = 0; a < s.n[0]; ++a)
        for (int c = 0; c < s.n[1]; ++c) {
            const int kw = s.w[0][a], vw = s.w[1][c];
            const size_t sb = BH * kw * vw * sizeof(float);
            w.part[a][c] = take(rows * vw * es);
            w.h0[a][c] = (float *)take(sb);
            if (want_bwd) {
                w.pq[a][c] = take(rows * kw * es);
                w.pf[a][c] = take(rows * kw * es);
                w.dhT[a][c] = (float *)take(sb);
                w.dh0[a][c] = (float *)take(sb);
            } else {
                w.hT[a][c] = (float *)take(sb);
            }
            const size_t need = ws_bytes_needed(B, T, H, kw, vw, chunk, dt, want_bwd, tc64);
            if (need > sub) sub = need;
        }
    w.sub_bytes = sub;
    w.sub = take(sub);
    w.total = p;
    return w;
}

// Workspace of the packed-sequence calls: rowsum(dhT * hT) [nseq*H*dk], flags [nseq*H] and the
// launch order [nseq].
size_t ws_flags_varlen(int nseq, int H, int dk) { return align256(sizeof(float) * (size_t)nseq * H * dk); }
size_t ws_perm_varlen(int nseq, int H, int dk) {
    return ws_flags_varlen(nseq, H, dk) + align256(sizeof(int) * (size_t)nseq * H);
}
size_t ws_bytes_varlen(int nseq, int H, int dk) {
    return ws_perm_varlen(nseq, H, dk) + align256(sizeof(int) * (size_t)nseq);
}

hgrn2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? HGRN2_OK : HGRN2_ERR_CUDA; }

std::atomic<long long> g_launches{0};   // kernel launches issued (host side)

}  // namespace

extern "C" {

size_t hgrn2_workspace_size(int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                            int want_bwd) {
    if (check_common(B, T, H, dk, dv, chunk, dtype) != HGRN2_OK) return (size_t)-1;
    if (want_bwd < 0 || want_bwd > 2) return (size_t)-1;
    return ws_bytes_needed(B, T, H, dk, dv, chunk, dtype, want_bwd, want_bwd != 2);
}

}  // extern "C"

namespace {

hgrn2_status wide_fwd(const void *q, const void *log_f, const void *i, const float *h0, void *o, float *hT,
                      void *saved, int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                      void *workspace, cudaStream_t stream);
hgrn2_status wide_bwd(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                      const void *dO, const float *dhT, void *dq, void *dlog_f, void *di, float *dh0, int B,
                      int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype, void *workspace,
                      cudaStream_t stream, bool tc64);
hgrn2_status stack_fwd(const void *q, const void *log_f, const void *i, const float *h0, void *o, float *hT,
                       void *saved, int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                       void *workspace, cudaStream_t stream);
hgrn2_status stack_bwd(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                       const void *dO, const float *dhT, void *dq, void *dlog_f, void *di, float *dh0, int B,
                       int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype, void *workspace,
                       cudaStream_t stream, bool tc64);

// Forward; `saved` (null, or saved_bytes_needed bytes) receives what hgrn2_bwd_saved reads.
hgrn2_status fwd_impl(const void *q, const void *log_f, const void *i, const float *h0, void *o, float *hT,
                      void *saved, int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                      void *workspace, size_t ws_bytes, cudaStream_t stream, const int *cu = nullptr) {
    hgrn2_status s = check_common(B, T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    if (T > 0 && (!q || !log_f || !i || !o)) return HGRN2_ERR_INVALID_ARG;
    const void *ptrs[] = {q, log_f, i, h0, o, hT, workspace, saved};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return HGRN2_ERR_INVALID_ARG;
    if (cu && is_wide(dk, dv)) return HGRN2_ERR_UNSUPPORTED;   // packed sequences: d_k, d_v <= 128
    size_t need = cu ? ws_bytes_varlen(B, H, dk) : ws_bytes_needed(B, T, H, dk, dv, chunk, dtype, 0);
    if (ws_bytes < need || (need && !workspace)) return HGRN2_ERR_INVALID_ARG;
    if (is_wide(dk, dv))
        return (wide_uniform(dk, dv) ? stack_fwd : wide_fwd)(q, log_f, i, h0, o, hT, saved, B, T, H, dk, dv, chunk,
                                                             dtype, workspace, stream);
    const bool bf16 = dtype == HGRN2_BF16;
    if (T == 0) {
        if (!hT) return HGRN2_OK;
        size_t n = sizeof(float) * (size_t)B * H * dk * dv;
        cudaError_t e = h0 ? cudaMemcpyAsync(hT, h0, n, cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(hT, 0, n, stream);
        return from_cuda(e);
    }
    int C = simt_chunk(chunk, dk, dv, false);
    if (!C) return HGRN2_ERR_UNSUPPORTED;
    const SavedLayout sl = saved_layout(B, T, H, cu != nullptr);
    int *perm = nullptr;
    if (cu) {   // longest sequences first; kept in the saved buffer for the backward
        perm = saved ? (int *)((char *)saved + sl.perm) : (int *)((char *)workspace + ws_perm_varlen(B, H, dk));
        if (launch_lpt_order(cu, B, T, perm, stream) != cudaSuccess) return HGRN2_ERR_CUDA;
        g_launches += 1;
    }
    if (use_tc(dk, dv, dtype)) {
        // tensor-core pass; (b,h) pairs whose chunk decay span is too wide are flagged
        // and recomputed right after by the exact route (same stream, in order)
        int *flags = saved ? (int *)((char *)saved + sl.flags)
                           : (int *)((char *)workspace + (cu ? ws_flags_varlen(B, H, dk) : 0));
        float *seg_ws = cu ? nullptr : (float *)((char *)workspace + align256(sizeof(int) * (size_t)B * H));
        int nseg = 1, tps = 1;
        if (!cu && dk == 128) tc_fwd_segments(B, T, H, &nseg, &tps);   // as the launcher decides
        TcFwdArgs t{q, log_f, i, h0, o, hT, flags, seg_ws, B, T, H, C, saved,
                    saved ? (float *)((char *)saved + sl.hTs) : nullptr, cu, perm, dk};
        cudaError_t e = launch_tc_fwd(t, stream);
        if (e != cudaSuccess) return HGRN2_ERR_CUDA;
        // the exact route, if needed, runs inside the tensor-core kernel: in the pair's CTA, or with
        // segments in the pair's last segment to finish (segments, the scan beyond a few segments,
        // the carried-state fix-up)
        g_launches += tc_fwd_launches(nseg);
        return HGRN2_OK;
    }
    SimtFwdArgs a{q, log_f, i, h0, o, hT, B, T, H, dk, dv, C, nullptr, cu, perm};
    g_launches += 1;
    return from_cuda(launch_simt_fwd(a, bf16, stream));
}

// Backward; with `saved` (from fwd_impl on the same inputs) the states are read, not recomputed.
hgrn2_status bwd_impl(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                      const void *dO, const float *dhT, void *dq, void *dlog_f, void *di, float *dh0, int B,
                      int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype, void *workspace,
                      size_t ws_bytes, cudaStream_t stream, const int *cu = nullptr, bool tc64 = true) {
    hgrn2_status s = check_common(B, T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    if (T > 0 && (!q || !log_f || !i || !dO || !dq || !dlog_f || !di)) return HGRN2_ERR_INVALID_ARG;
    const void *ptrs[] = {q, log_f, i, h0, dO, dhT, dq, dlog_f, di, dh0, workspace, saved};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return HGRN2_ERR_INVALID_ARG;
    if (cu && is_wide(dk, dv)) return HGRN2_ERR_UNSUPPORTED;
    size_t need = cu ? ws_bytes_varlen(B, H, dk)
                     : ws_bytes_needed(B, T, H, dk, dv, chunk, dtype, saved ? 2 : 1, tc64 && !saved);
    if (ws_bytes < need || (need && !workspace)) return HGRN2_ERR_INVALID_ARG;
    if (is_wide(dk, dv))
        return (wide_uniform(dk, dv) ? stack_bwd : wide_bwd)(q, log_f, i, h0, saved, dO, dhT, dq, dlog_f, di, dh0, B,
                                                             T, H, dk, dv, chunk, dtype, workspace, stream,
                                                             tc64 && !saved);
    const bool bf16 = dtype == HGRN2_BF16;
    if (T > 0 && !saved && !cu && tc64 && use_tc(dk, dv, dtype) && dk == 64) {
        // 64-wide heads: the tensor-core forward keeps the chunk states in the workspace (its o
        // goes to scratch there too), then the saved-state backward reads them
        const size_t base = ws_bytes_base(B, H, dk, dv, dtype, 1);
        char *sv = (char *)workspace + base;
        void *o2 = sv + saved_layout(B, T, H).total;
        hgrn2_status st = fwd_impl(q, log_f, i, h0, o2, nullptr, sv, B, T, H, dk, dv, chunk, dtype, workspace, base,
                                   stream);
        if (st != HGRN2_OK) return st;
        return bwd_impl(q, log_f, i, h0, sv, dO, dhT, dq, dlog_f, di, dh0, B, T, H, dk, dv, chunk, dtype, workspace,
                        base, stream);
    }
    if (!saved && !cu && tc64 && segmented_recompute(B, T, H, dk, dv, dtype)) {
        // few (b,h): the training forward (segments) into the workspace, then the saved-state
        // backward (segments)
        const RecomputeLayout l = recompute_layout(B, T, H, dv, dtype);
        char *sv = (char *)workspace + l.saved;
        hgrn2_status st = fwd_impl(q, log_f, i, h0, sv + (l.o - l.saved), nullptr, sv, B, T, H, dk, dv, chunk, dtype,
                                   (char *)workspace + l.fws, l.total - l.fws, stream);
        if (st != HGRN2_OK) return st;
        return bwd_impl(q, log_f, i, h0, sv, dO, dhT, dq, dlog_f, di, dh0, B, T, H, dk, dv, chunk, dtype, workspace,
                        l.saved, stream);
    }
    if (T == 0) {
        if (!dh0) return HGRN2_OK;
        size_t n = sizeof(float) * (size_t)B * H * dk * dv;
        cudaError_t e = dhT ? cudaMemcpyAsync(dh0, dhT, n, cudaMemcpyDeviceToDevice, stream)
                            : cudaMemsetAsync(dh0, 0, n, stream);
        return from_cuda(e);
    }
    int C = simt_chunk(chunk, dk, dv, true);
    if (!C) return HGRN2_ERR_UNSUPPORTED;
    float *rs = (float *)workspace;
    const SavedLayout sl = saved_layout(B, T, H, cu != nullptr);
    const int *perm = nullptr;
    if (cu && saved) {   // the order the forward chose
        perm = (const int *)((const char *)saved + sl.perm);
    } else if (cu) {
        int *p = (int *)((char *)workspace + ws_perm_varlen(B, H, dk));
        if (launch_lpt_order(cu, B, T, p, stream) != cudaSuccess) return HGRN2_ERR_CUDA;
        g_launches += 1;
        perm = p;
    }
    // without saved states only d = 128 has a tensor-core backward (recompute); the rest take the
    // exact route
    if (use_tc(dk, dv, dtype) && (saved || (!cu && dk == 128))) {
        if (saved) {   // reverse sweep from the saved states (exact route inside); few (b,h): segments
            TcBwdArgs t{q, log_f, i, dO, h0, dhT, dq, dlog_f, di, dh0, rs,
                        (int *)((char *)saved + sl.flags), B, T, H, C, saved,
                        (const float *)((const char *)saved + sl.hTs), cu, perm, dk};
            const bool segs = !cu && dk == 128 && tc_bwd_workspace(B, T, H) > 0;
            if (segs) t.seg_ws = (float *)((char *)workspace + ws_bytes_base(B, H, dk, dv, dtype, 1));
            g_launches += segs ? tc_bwd_launches(B, T, H) : 1;
            return from_cuda(launch_tc_bwd(t, stream));
        }
        int *flags = (int *)((char *)workspace + align256(sizeof(float) * (size_t)B * H * dk));
        TcBwdArgs t{q, log_f, i, dO, h0, dhT, dq, dlog_f, di, dh0, rs, flags, B, T, H, C, nullptr, nullptr, nullptr,
                    nullptr, 128};
        g_launches += 2;   // the exact route, if needed, runs inside the forward-sweep kernel
        return from_cuda(launch_tc_bwd(t, stream));
    }
    SimtBwdArgs a{q, log_f, i, dO, h0, dhT, dq, dlog_f, di, dh0, rs, B, T, H, dk, dv, C, nullptr, cu, perm};
    g_launches += 2;
    return from_cuda(launch_simt_bwd(a, bf16, stream));
}

// Columns off .. off+w-1 of every row of a [rows][d] token tensor into contiguous [rows][w].
cudaError_t copy_cols(void *dst, const void *src, size_t rows, int d, int off, int w, size_t es, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    return cudaMemcpy2DAsync(dst, w * es, (const char *)src + off * es, d * es, w * es, rows, cudaMemcpyDeviceToDevice,
                             st);
}

// Columns off .. off+w-1 of every row of a [rows][d] token tensor into rows `dpitch` elements apart.
cudaError_t copy_cols_to(void *dst, size_t dpitch, const void *src, size_t rows, int d, int off, int w, size_t es,
                         cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    return cudaMemcpy2DAsync(dst, dpitch * es, (const char *)src + off * es, d * es, w * es, rows,
                             cudaMemcpyDeviceToDevice, st);
}

// Equal blocks: the columns of block pair j = a * n[1] + c go to head slot j of the H * nb heads
// (token rows nb blocks wide, state matrices nb per (b, h)); one forward call runs them all, and
// o[c] = sum over a of slot a * n[1] + c, added in fp32.
// bf16 heads of 256 x 256 run on the tensor cores reading the caller's 256-wide rows in place (two
// 128-wide half-heads each, key blocks for q and log f, value blocks for i and dO): no column
// copies; the blocks' partial outputs land in summable layouts.  The backward does so from saved
// states only.
bool wide_inplace(int T, int dk, int dv, hgrn2_dtype dt) { return dt == HGRN2_BF16 && dk == 256 && dv == 256 && T > 0; }

hgrn2_status stack_fwd(const void *q, const void *log_f, const void *i, const float *h0, void *o, float *hT,
                       void *saved, int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                       void *workspace, cudaStream_t stream) {
    const WideSplit s = wide_split(dk, dv);
    const int nK = s.n[0], nV = s.n[1], nb = nK * nV, kw = s.w[0][0], vw = s.w[1][0];
    const WideStack w = wide_stack_ws(B, T, H, dk, dv, chunk, dtype, 0, true, (char *)workspace);
    const bool bf16 = dtype == HGRN2_BF16;
    const size_t es = bf16 ? 2 : 4, rows = (size_t)B * T * H, BH = (size_t)B * H, sm = (size_t)kw * vw;
    if (wide_inplace(T, dk, dv, dtype)) {
        for (int a = 0; a < nK && h0; ++a)
            for (int c = 0; c < nV; ++c)
                if (launch_state_block(const_cast<float *>(h0), w.h0 + (a * nV + c) * sm, nb * sm, BH, dk, dv,
                                       s.off[0][a], kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                    return HGRN2_ERR_CUDA;
        const int C = simt_chunk(chunk, kw, vw, false);
        if (!C) return HGRN2_ERR_UNSUPPORTED;
        const SavedLayout sl = saved_layout(B, T, H * nb);
        int *flags = saved ? (int *)((char *)saved + sl.flags) : (int *)w.sub;
        // every block pair adds its share of o into o: zeroed first
        if (cudaMemsetAsync(o, 0, rows * dv * es, stream) != cudaSuccess) return HGRN2_ERR_CUDA;
        TcFwdArgs t{q, log_f, i, h0 ? w.h0 : nullptr, o, hT ? w.hT : nullptr, flags, nullptr, B, T, H * nb, C,
                    saved, saved ? (float *)((char *)saved + sl.hTs) : nullptr, nullptr, nullptr, 128};
        t.nK = nK;
        t.nV = nV;
        t.opart = w.part;
        if (launch_tc_fwd(t, stream) != cudaSuccess) return HGRN2_ERR_CUDA;
        for (int a = 0; a < nK && hT; ++a)
            for (int c = 0; c < nV; ++c)
                if (launch_state_block(hT, w.hT + (a * nV + c) * sm, nb * sm, BH, dk, dv, s.off[0][a], kw,
                                       s.off[1][c], vw, true, stream) != cudaSuccess)
                    return HGRN2_ERR_CUDA;
        g_launches += (h0 ? nb : 0) + 1 + (hT ? nb : 0);
        return HGRN2_OK;
    }
    for (int a = 0; a < nK; ++a)
        for (int c = 0; c < nV; ++c) {
            const int j = a * nV + c;
            if (copy_cols_to(w.q + j * kw * es, (size_t)nb * kw, q, rows, dk, s.off[0][a], kw, es, stream) ||
                copy_cols_to(w.f + j * kw * es, (size_t)nb * kw, log_f, rows, dk, s.off[0][a], kw, es, stream) ||
                copy_cols_to(w.x + j * vw * es, (size_t)nb * vw, i, rows, dv, s.off[1][c], vw, es, stream))
                return HGRN2_ERR_CUDA;
            if (h0 && launch_state_block(const_cast<float *>(h0), w.h0 + j * sm, nb * sm, BH, dk, dv, s.off[0][a], kw,
                                         s.off[1][c], vw, false, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
        }
    const hgrn2_status st = fwd_impl(w.q, w.f, w.x, h0 ? w.h0 : nullptr, w.part, hT ? w.hT : nullptr, saved, B, T,
                                     H * nb, kw, vw, chunk, dtype, w.sub, w.sub_bytes, stream);
    if (st != HGRN2_OK) return st;
    for (int a = 0; a < nK && hT; ++a)
        for (int c = 0; c < nV; ++c)
            if (launch_state_block(hT, w.hT + (a * nV + c) * sm, nb * sm, BH, dk, dv, s.off[0][a], kw, s.off[1][c], vw,
                                   true, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
    for (int c = 0; c < nV; ++c)
        if (launch_sum_blocks(o, dv, s.off[1][c], w.part + c * vw * es, nK > 1 ? w.part + (nV + c) * vw * es : nullptr,
                              nb * vw, rows, vw, bf16, stream) != cudaSuccess)
            return HGRN2_ERR_CUDA;
    g_launches += (h0 ? nb : 0) + (hT ? nb : 0) + (rows ? nV : 0);
    return HGRN2_OK;
}

// Backward of equal blocks: one backward call over the H * nb heads; dq[a], d log f[a] = sums of
// slots a * n[1] + c over c, di[c] = sum of slots a * n[1] + c over a, dh0 blocks as they are.
hgrn2_status stack_bwd(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                       const void *dO, const float *dhT, void *dq, void *dlog_f, void *di, float *dh0, int B,
                       int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype, void *workspace,
                       cudaStream_t stream, bool tc64) {
    const WideSplit s = wide_split(dk, dv);
    const int nK = s.n[0], nV = s.n[1], nb = nK * nV, kw = s.w[0][0], vw = s.w[1][0];
    const WideStack w = wide_stack_ws(B, T, H, dk, dv, chunk, dtype, saved ? 2 : 1, tc64, (char *)workspace);
    const bool bf16 = dtype == HGRN2_BF16;
    const size_t es = bf16 ? 2 : 4, rows = (size_t)B * T * H, BH = (size_t)B * H, sm = (size_t)kw * vw;
    if (saved && wide_inplace(T, dk, dv, dtype)) {
        for (int a = 0; a < nK; ++a)
            for (int c = 0; c < nV; ++c) {
                const int j = a * nV + c;
                if (h0 && launch_state_block(const_cast<float *>(h0), w.h0 + j * sm, nb * sm, BH, dk, dv, s.off[0][a],
                                             kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                    return HGRN2_ERR_CUDA;
                if (dhT && launch_state_block(const_cast<float *>(dhT), w.dhT + j * sm, nb * sm, BH, dk, dv,
                                              s.off[0][a], kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                    return HGRN2_ERR_CUDA;
            }
        const int C = simt_chunk(chunk, kw, vw, true);
        if (!C) return HGRN2_ERR_UNSUPPORTED;
        const SavedLayout sl = saved_layout(B, T, H * nb);
        // every block pair adds its shares of dq, d log f and di into them: zeroed first
        if (cudaMemsetAsync(dq, 0, rows * dk * es, stream) != cudaSuccess ||
            cudaMemsetAsync(dlog_f, 0, rows * dk * es, stream) != cudaSuccess ||
            cudaMemsetAsync(di, 0, rows * dv * es, stream) != cudaSuccess)
            return HGRN2_ERR_CUDA;
        TcBwdArgs t{q, log_f, i, dO, h0 ? w.h0 : nullptr, dhT ? w.dhT : nullptr, dq, dlog_f, di,
                    dh0 ? w.dh0 : nullptr, (float *)w.sub, (int *)((char *)saved + sl.flags), B, T, H * nb, C, saved,
                    (const float *)((const char *)saved + sl.hTs), nullptr, nullptr, 128};
        t.nK = nK;
        t.nV = nV;
        t.dq_part = w.pq;
        t.dlf_part = w.pf;
        t.dx_part = w.part;
        if (launch_tc_bwd(t, stream) != cudaSuccess) return HGRN2_ERR_CUDA;
        for (int a = 0; a < nK && dh0; ++a)
            for (int c = 0; c < nV; ++c)
                if (launch_state_block(dh0, w.dh0 + (a * nV + c) * sm, nb * sm, BH, dk, dv, s.off[0][a], kw,
                                       s.off[1][c], vw, true, stream) != cudaSuccess)
                    return HGRN2_ERR_CUDA;
        g_launches += (h0 ? nb : 0) + (dhT ? nb : 0) + 1 + (dh0 ? nb : 0);
        return HGRN2_OK;
    }
    for (int a = 0; a < nK; ++a)
        for (int c = 0; c < nV; ++c) {
            const int j = a * nV + c;
            if (copy_cols_to(w.q + j * kw * es, (size_t)nb * kw, q, rows, dk, s.off[0][a], kw, es, stream) ||
                copy_cols_to(w.f + j * kw * es, (size_t)nb * kw, log_f, rows, dk, s.off[0][a], kw, es, stream) ||
                copy_cols_to(w.x + j * vw * es, (size_t)nb * vw, i, rows, dv, s.off[1][c], vw, es, stream) ||
                copy_cols_to(w.dO + j * vw * es, (size_t)nb * vw, dO, rows, dv, s.off[1][c], vw, es, stream))
                return HGRN2_ERR_CUDA;
            if (h0 && launch_state_block(const_cast<float *>(h0), w.h0 + j * sm, nb * sm, BH, dk, dv, s.off[0][a], kw,
                                         s.off[1][c], vw, false, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
            if (dhT && launch_state_block(const_cast<float *>(dhT), w.dhT + j * sm, nb * sm, BH, dk, dv, s.off[0][a],
                                          kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
        }
    const hgrn2_status st = bwd_impl(w.q, w.f, w.x, h0 ? w.h0 : nullptr, saved, w.dO, dhT ? w.dhT : nullptr, w.pq,
                                     w.pf, w.part, dh0 ? w.dh0 : nullptr, B, T, H * nb, kw, vw, chunk, dtype, w.sub,
                                     w.sub_bytes, stream, nullptr, tc64);
    if (st != HGRN2_OK) return st;
    for (int a = 0; a < nK && dh0; ++a)
        for (int c = 0; c < nV; ++c)
            if (launch_state_block(dh0, w.dh0 + (a * nV + c) * sm, nb * sm, BH, dk, dv, s.off[0][a], kw, s.off[1][c],
                                   vw, true, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
    for (int a = 0; a < nK; ++a) {
        const size_t j0 = (size_t)a * nV;
        if (launch_sum_blocks(dq, dk, s.off[0][a], w.pq + j0 * kw * es, nV > 1 ? w.pq + (j0 + 1) * kw * es : nullptr,
                              nb * kw, rows, kw, bf16, stream) != cudaSuccess ||
            launch_sum_blocks(dlog_f, dk, s.off[0][a], w.pf + j0 * kw * es,
                              nV > 1 ? w.pf + (j0 + 1) * kw * es : nullptr, nb * kw, rows, kw, bf16, stream) !=
                cudaSuccess)
            return HGRN2_ERR_CUDA;
    }
    for (int c = 0; c < nV; ++c)
        if (launch_sum_blocks(di, dv, s.off[1][c], w.part + c * vw * es, nK > 1 ? w.part + (nV + c) * vw * es : nullptr,
                              nb * vw, rows, vw, bf16, stream) != cudaSuccess)
            return HGRN2_ERR_CUDA;
    g_launches += (h0 ? nb : 0) + (dhT ? nb : 0) + (dh0 ? nb : 0) + (rows ? 2 * nK + nV : 0);
    return HGRN2_OK;
}

// Heads wider than 128: every block pair (a, c) runs the forward of a head of d_k = w[0][a],
// d_v = w[1][c] on contiguous copies of its columns, with its state block as h0 / hT and its own
// region of the saved buffer; o[c] = sum over a of the blocks' outputs, added in fp32.
hgrn2_status wide_fwd(const void *q, const void *log_f, const void *i, const float *h0, void *o, float *hT,
                      void *saved, int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                      void *workspace, cudaStream_t stream) {
    const WideSplit s = wide_split(dk, dv);
    const WideWs w = wide_ws(B, T, H, dk, dv, chunk, dtype, 0, true, (char *)workspace);
    size_t soff[2][2];
    wide_saved(B, T, H, dk, dv, dtype, soff);
    const bool bf16 = dtype == HGRN2_BF16;
    const size_t es = bf16 ? 2 : 4, rows = (size_t)B * T * H, BH = (size_t)B * H;
    cudaError_t e = cudaSuccess;
    for (int a = 0; a < 2 && s.n[0] > 1 && e == cudaSuccess; ++a) {
        e = copy_cols(w.q[a], q, rows, dk, s.off[0][a], s.w[0][a], es, stream);
        if (e == cudaSuccess) e = copy_cols(w.f[a], log_f, rows, dk, s.off[0][a], s.w[0][a], es, stream);
    }
    for (int c = 0; c < 2 && s.n[1] > 1 && e == cudaSuccess; ++c)
        e = copy_cols(w.x[c], i, rows, dv, s.off[1][c], s.w[1][c], es, stream);
    if (e != cudaSuccess) return HGRN2_ERR_CUDA;
    for (int a = 0; a < s.n[0]; ++a)
        for (int c = 0; c < s.n[1]; ++c) {
            const int kw = s.w[0][a], vw = s.w[1][c];
            if (h0 && launch_state_block(const_cast<float *>(h0), w.h0[a][c], (size_t)kw * vw, BH, dk, dv,
                                         s.off[0][a], kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
            void *sv = saved && saved_bytes_needed(B, T, H, kw, vw, dtype) ? (char *)saved + soff[a][c] : nullptr;
            const hgrn2_status st = fwd_impl(s.n[0] > 1 ? w.q[a] : q, s.n[0] > 1 ? w.f[a] : log_f,
                                             s.n[1] > 1 ? w.x[c] : i, h0 ? w.h0[a][c] : nullptr, w.part[a][c],
                                             hT ? w.hT[a][c] : nullptr, sv, B, T, H, kw, vw, chunk, dtype, w.sub,
                                             w.sub_bytes, stream);
            if (st != HGRN2_OK) return st;
            if (hT && launch_state_block(hT, w.hT[a][c], (size_t)kw * vw, BH, dk, dv, s.off[0][a], kw, s.off[1][c],
                                         vw, true, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
            g_launches += (h0 ? 1 : 0) + (hT ? 1 : 0);
        }
    for (int c = 0; c < s.n[1]; ++c) {
        if (launch_sum_blocks(o, dv, s.off[1][c], w.part[0][c], s.n[0] > 1 ? w.part[1][c] : nullptr, s.w[1][c], rows,
                              s.w[1][c], bf16, stream) != cudaSuccess)
            return HGRN2_ERR_CUDA;
        g_launches += rows ? 1 : 0;
    }
    return HGRN2_OK;
}

// Backward of a wide head: every block pair runs the backward of its own head (from its saved
// region, if any); dq[a], d log f[a] = sums over c, di[c] = sum over a, dh0 block (a,c) as is.
hgrn2_status wide_bwd(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                      const void *dO, const float *dhT, void *dq, void *dlog_f, void *di, float *dh0, int B,
                      int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype, void *workspace,
                      cudaStream_t stream, bool tc64) {
    const WideSplit s = wide_split(dk, dv);
    const WideWs w = wide_ws(B, T, H, dk, dv, chunk, dtype, saved ? 2 : 1, tc64, (char *)workspace);
    size_t soff[2][2];
    wide_saved(B, T, H, dk, dv, dtype, soff);
    const bool bf16 = dtype == HGRN2_BF16;
    const size_t es = bf16 ? 2 : 4, rows = (size_t)B * T * H, BH = (size_t)B * H;
    cudaError_t e = cudaSuccess;
    for (int a = 0; a < 2 && s.n[0] > 1 && e == cudaSuccess; ++a) {
        e = copy_cols(w.q[a], q, rows, dk, s.off[0][a], s.w[0][a], es, stream);
        if (e == cudaSuccess) e = copy_cols(w.f[a], log_f, rows, dk, s.off[0][a], s.w[0][a], es, stream);
    }
    for (int c = 0; c < 2 && s.n[1] > 1 && e == cudaSuccess; ++c) {
        e = copy_cols(w.x[c], i, rows, dv, s.off[1][c], s.w[1][c], es, stream);
        if (e == cudaSuccess) e = copy_cols(w.dO[c], dO, rows, dv, s.off[1][c], s.w[1][c], es, stream);
    }
    if (e != cudaSuccess) return HGRN2_ERR_CUDA;
    for (int a = 0; a < s.n[0]; ++a)
        for (int c = 0; c < s.n[1]; ++c) {
            const int kw = s.w[0][a], vw = s.w[1][c];
            if (h0 && launch_state_block(const_cast<float *>(h0), w.h0[a][c], (size_t)kw * vw, BH, dk, dv,
                                         s.off[0][a], kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
            if (dhT && launch_state_block(const_cast<float *>(dhT), w.dhT[a][c], (size_t)kw * vw, BH, dk, dv,
                                          s.off[0][a], kw, s.off[1][c], vw, false, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
            const size_t need = saved_bytes_needed(B, T, H, kw, vw, dtype);
            const void *sv = saved && need ? (const char *)saved + soff[a][c] : nullptr;
            const hgrn2_status st = bwd_impl(s.n[0] > 1 ? w.q[a] : q, s.n[0] > 1 ? w.f[a] : log_f,
                                             s.n[1] > 1 ? w.x[c] : i, h0 ? w.h0[a][c] : nullptr, sv,
                                             s.n[1] > 1 ? w.dO[c] : dO, dhT ? w.dhT[a][c] : nullptr, w.pq[a][c],
                                             w.pf[a][c], w.part[a][c], dh0 ? w.dh0[a][c] : nullptr, B, T, H, kw, vw,
                                             chunk, dtype, w.sub, w.sub_bytes, stream, nullptr, tc64);
            if (st != HGRN2_OK) return st;
            if (dh0 && launch_state_block(dh0, w.dh0[a][c], (size_t)kw * vw, BH, dk, dv, s.off[0][a], kw,
                                          s.off[1][c], vw, true, stream) != cudaSuccess)
                return HGRN2_ERR_CUDA;
            g_launches += (h0 ? 1 : 0) + (dhT ? 1 : 0) + (dh0 ? 1 : 0);
        }
    for (int a = 0; a < s.n[0]; ++a) {
        const bool two = s.n[1] > 1;
        if (launch_sum_blocks(dq, dk, s.off[0][a], w.pq[a][0], two ? w.pq[a][1] : nullptr, s.w[0][a], rows,
                              s.w[0][a], bf16, stream) != cudaSuccess ||
            launch_sum_blocks(dlog_f, dk, s.off[0][a], w.pf[a][0], two ? w.pf[a][1] : nullptr, s.w[0][a], rows,
                              s.w[0][a], bf16, stream) != cudaSuccess)
            return HGRN2_ERR_CUDA;
        g_launches += rows ? 2 : 0;
    }
    for (int c = 0; c < s.n[1]; ++c) {
        if (launch_sum_blocks(di, dv, s.off[1][c], w.part[0][c], s.n[0] > 1 ? w.part[1][c] : nullptr, s.w[1][c], rows,
                              s.w[1][c], bf16, stream) != cudaSuccess)
            return HGRN2_ERR_CUDA;
        g_launches += rows ? 1 : 0;
    }
    return HGRN2_OK;
}

hgrn2_status step_impl(const void *q, const void *lf, const void *i, float *S, void *o, int B, int H, int dk, int dv,
                       hgrn2_dtype dtype, bool gate_lb, float lb, cudaStream_t stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return HGRN2_ERR_INVALID_ARG;
    if (dtype != HGRN2_FP32 && dtype != HGRN2_BF16) return HGRN2_ERR_INVALID_ARG;
    if (dk > 128 || dv > 128 || (dv & 3)) return HGRN2_ERR_UNSUPPORTED;
    if ((long long)B * H > (1ll << 30)) return HGRN2_ERR_UNSUPPORTED;
    if (!q || !lf || !i || !S || !o) return HGRN2_ERR_INVALID_ARG;
    const void *ptrs[] = {q, lf, i, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return HGRN2_ERR_INVALID_ARG;
    g_launches += 1;
    return from_cuda(launch_step(q, lf, i, S, o, B, H, dk, dv, dtype == HGRN2_BF16, gate_lb, lb, stream));
}

hgrn2_status step_bwd_impl(const void *q, const void *lf, const void *i, const float *S, const void *dO,
                           const float *dS, float *dS_prev, void *dq, void *dlf, void *di, int B, int H, int dk,
                           int dv, hgrn2_dtype dtype, bool gate_lb, float lb, cudaStream_t stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return HGRN2_ERR_INVALID_ARG;
    if (dtype != HGRN2_FP32 && dtype != HGRN2_BF16) return HGRN2_ERR_INVALID_ARG;
    if (dk > 128 || dv > 128 || (dv & 3)) return HGRN2_ERR_UNSUPPORTED;
    if ((long long)B * H > (1ll << 29)) return HGRN2_ERR_UNSUPPORTED;   // two blocks per (b,h)
    if (!q || !lf || !i || !S || !dO || !dq || !dlf || !di) return HGRN2_ERR_INVALID_ARG;
    const void *ptrs[] = {q, lf, i, S, dO, dS, dS_prev, dq, dlf, di};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return HGRN2_ERR_INVALID_ARG;
    // dS_prev is dS itself or does not overlap it
    if (dS && dS_prev && dS != dS_prev) {
        const size_t n = sizeof(float) * (size_t)B * H * dk * dv;
        const char *a = (const char *)dS, *b = (const char *)dS_prev;
        if (a < b + n && b < a + n) return HGRN2_ERR_INVALID_ARG;
    }
    StepBwdArgs a{q, lf, i, S, dO, dS, dS_prev, dq, dlf, di, B, H, dk, dv, gate_lb, lb};
    g_launches += 1;
    return from_cuda(launch_step_bwd(a, dtype == HGRN2_BF16, stream));
}

}  // namespace

extern "C" {

hgrn2_status hgrn2_fwd(const void *q, const void *log_f, const void *i, const float *h0, void *o,
                       float *hT, int B, int T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype,
                       void *workspace, size_t ws_bytes, cudaStream_t stream) {
    return fwd_impl(q, log_f, i, h0, o, hT, nullptr, B, T, H, dk, dv, chunk, dtype, workspace, ws_bytes, stream);
}

hgrn2_status hgrn2_bwd(const void *q, const void *log_f, const void *i, const float *h0, const void *dO,
                       const float *dhT, void *dq, void *dlog_f, void *di, float *dh0, int B, int T,
                       int H, int dk, int dv, int chunk, hgrn2_dtype dtype, void *workspace,
                       size_t ws_bytes, cudaStream_t stream) {
    return bwd_impl(q, log_f, i, h0, nullptr, dO, dhT, dq, dlog_f, di, dh0, B, T, H, dk, dv, chunk, dtype,
                    workspace, ws_bytes, stream);
}

size_t hgrn2_saved_size(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype) {
    if (check_common(B, T, H, dk, dv, 64, dtype) != HGRN2_OK) return (size_t)-1;
    return saved_bytes_needed(B, T, H, dk, dv, dtype);
}

hgrn2_status hgrn2_fwd_train(const void *q, const void *log_f, const void *i, const float *h0, void *o,
                             float *hT, void *saved, size_t saved_bytes, int B, int T, int H, int dk, int dv,
                             int chunk, hgrn2_dtype dtype, void *workspace, size_t ws_bytes,
                             cudaStream_t stream) {
    hgrn2_status s = check_common(B, T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    const size_t need = saved_bytes_needed(B, T, H, dk, dv, dtype);
    if (need && (!saved || saved_bytes < need)) return HGRN2_ERR_INVALID_ARG;
    return fwd_impl(q, log_f, i, h0, o, hT, need ? saved : nullptr, B, T, H, dk, dv, chunk, dtype, workspace,
                    ws_bytes, stream);
}

hgrn2_status hgrn2_bwd_saved(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                             size_t saved_bytes, const void *dO, const float *dhT, void *dq, void *dlog_f,
                             void *di, float *dh0, int B, int T, int H, int dk, int dv, int chunk,
                             hgrn2_dtype dtype, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    hgrn2_status s = check_common(B, T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    const size_t need = saved_bytes_needed(B, T, H, dk, dv, dtype);
    if (need && (!saved || saved_bytes < need)) return HGRN2_ERR_INVALID_ARG;
    return bwd_impl(q, log_f, i, h0, need ? saved : nullptr, dO, dhT, dq, dlog_f, di, dh0, B, T, H, dk, dv,
                    chunk, dtype, workspace, ws_bytes, stream);
}

size_t hgrn2_saved_size_varlen(int nseq, int total_T, int H, int dk, int dv, hgrn2_dtype dtype) {
    if (check_common(nseq, total_T, H, dk, dv, 64, dtype) != HGRN2_OK || is_wide(dk, dv)) return (size_t)-1;
    return (use_tc(dk, dv, dtype) && total_T > 0) ? saved_layout(nseq, total_T, H, true).total : 0;
}

size_t hgrn2_workspace_size_varlen(int nseq, int total_T, int H, int dk, int dv, int chunk, hgrn2_dtype dtype) {
    if (check_common(nseq, total_T, H, dk, dv, chunk, dtype) != HGRN2_OK || is_wide(dk, dv)) return (size_t)-1;
    return ws_bytes_varlen(nseq, H, dk);
}

hgrn2_status hgrn2_fwd_varlen(const void *q, const void *log_f, const void *i, const float *h0, void *o, float *hT,
                              const int *cu_seqlens, int nseq, int total_T, int H, int dk, int dv, int chunk,
                              hgrn2_dtype dtype, void *saved, size_t saved_bytes, void *workspace, size_t ws_bytes,
                              cudaStream_t stream) {
    hgrn2_status s = check_common(nseq, total_T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    if (!cu_seqlens || !aligned16(cu_seqlens)) return HGRN2_ERR_INVALID_ARG;
    const size_t need = hgrn2_saved_size_varlen(nseq, total_T, H, dk, dv, dtype);
    if (saved && saved_bytes < need) return HGRN2_ERR_INVALID_ARG;
    return fwd_impl(q, log_f, i, h0, o, hT, need ? saved : nullptr, nseq, total_T, H, dk, dv, chunk, dtype,
                    workspace, ws_bytes, stream, cu_seqlens);
}

hgrn2_status hgrn2_bwd_varlen(const void *q, const void *log_f, const void *i, const float *h0, const void *saved,
                              size_t saved_bytes, const void *dO, const float *dhT, void *dq, void *dlog_f,
                              void *di, float *dh0, const int *cu_seqlens, int nseq, int total_T, int H, int dk,
                              int dv, int chunk, hgrn2_dtype dtype, void *workspace, size_t ws_bytes,
                              cudaStream_t stream) {
    hgrn2_status s = check_common(nseq, total_T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    if (!cu_seqlens || !aligned16(cu_seqlens)) return HGRN2_ERR_INVALID_ARG;
    const size_t need = hgrn2_saved_size_varlen(nseq, total_T, H, dk, dv, dtype);
    if (saved && saved_bytes < need) return HGRN2_ERR_INVALID_ARG;
    return bwd_impl(q, log_f, i, h0, need ? saved : nullptr, dO, dhT, dq, dlog_f, di, dh0, nseq, total_T, H, dk, dv,
                    chunk, dtype, workspace, ws_bytes, stream, cu_seqlens);
}

hgrn2_status hgrn2_step(const void *q, const void *log_f, const void *i, float *S, void *o, int B, int H,
                        int dk, int dv, hgrn2_dtype dtype, cudaStream_t stream) {
    return step_impl(q, log_f, i, S, o, B, H, dk, dv, dtype, false, 0.0f, stream);
}

hgrn2_status hgrn2_step_lb(const void *q, const void *g, const void *i, float lb, float *S, void *o, int B, int H,
                           int dk, int dv, hgrn2_dtype dtype, cudaStream_t stream) {
    if (!(lb >= 0.0f && lb < 1.0f)) return HGRN2_ERR_INVALID_ARG;   // also rejects NaN
    return step_impl(q, g, i, S, o, B, H, dk, dv, dtype, true, lb, stream);
}

hgrn2_status hgrn2_step_bwd(const void *q, const void *log_f, const void *i, const float *S, const void *dO,
                            const float *dS, float *dS_prev, void *dq, void *dlog_f, void *di, int B, int H, int dk,
                            int dv, hgrn2_dtype dtype, cudaStream_t stream) {
    return step_bwd_impl(q, log_f, i, S, dO, dS, dS_prev, dq, dlog_f, di, B, H, dk, dv, dtype, false, 0.0f, stream);
}

hgrn2_status hgrn2_step_lb_bwd(const void *q, const void *g, const void *i, float lb, const float *S, const void *dO,
                               const float *dS, float *dS_prev, void *dq, void *dg, void *di, int B, int H, int dk,
                               int dv, hgrn2_dtype dtype, cudaStream_t stream) {
    if (!(lb >= 0.0f && lb < 1.0f)) return HGRN2_ERR_INVALID_ARG;
    return step_bwd_impl(q, g, i, S, dO, dS, dS_prev, dq, dg, di, B, H, dk, dv, dtype, true, lb, stream);
}

// ------------------------------------------------------------------ sequence parallelism
namespace {
hgrn2_status state_map_impl(const void *q, const void *log_f, const void *v, int B, int T, int H, int dk, int dv,
                            hgrn2_dtype dtype, float *g, float *M, bool backward, cudaStream_t stream) {
    if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return HGRN2_ERR_INVALID_ARG;
    if (dtype != HGRN2_FP32 && dtype != HGRN2_BF16) return HGRN2_ERR_INVALID_ARG;
    if (dk > 128 || dv > 256 || (long long)B * H > (1ll << 30)) return HGRN2_ERR_UNSUPPORTED;
    if (!g || !M || (T > 0 && (!log_f || !v || (backward && !q)))) return HGRN2_ERR_INVALID_ARG;
    const void *ptrs[] = {q, log_f, v, g, M};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return HGRN2_ERR_INVALID_ARG;
    if (!backward && T > 0 && dtype == HGRN2_BF16 && dk == 128 && dv == 128) {
        g_launches += 1;
        return from_cuda(launch_tc_state_map(log_f, v, B, T, H, g, M, stream));
    }
    StateMapArgs a{log_f, q, v, g, M, B, T, H, dk, dv, backward};
    g_launches += 1;
    return from_cuda(launch_state_map(a, dtype == HGRN2_BF16, stream));
}
}  // namespace

extern "C" {

hgrn2_status hgrn2_state_map(const void *log_f, const void *i, int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                             float *g, float *U, cudaStream_t stream) {
    return state_map_impl(nullptr, log_f, i, B, T, H, dk, dv, dtype, g, U, false, stream);
}

hgrn2_status hgrn2_state_map_bwd(const void *q, const void *log_f, const void *dO, int B, int T, int H, int dk,
                                 int dv, hgrn2_dtype dtype, float *g, float *W, cudaStream_t stream) {
    return state_map_impl(q, log_f, dO, B, T, H, dk, dv, dtype, g, W, true, stream);
}

hgrn2_status hgrn2_affine_scan(const float *g, const float *M, int R, int first, int count, int step,
                               const float *init, float *S, int B, int H, int dk, int dv, cudaStream_t stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1 || R < 0 || count < 0 || (step != 1 && step != -1))
        return HGRN2_ERR_INVALID_ARG;
    if (dk > 256 || dv > 256 || (long long)B * H > (1ll << 30)) return HGRN2_ERR_UNSUPPORTED;
    if (count > 0) {
        const long long last = (long long)first + (long long)(count - 1) * step;
        if (first < 0 || first >= R || last < 0 || last >= R || !g || !M) return HGRN2_ERR_INVALID_ARG;
    }
    if (!S) return HGRN2_ERR_INVALID_ARG;
    const size_t nbh = (size_t)B * H, ns = nbh * dk * dv * sizeof(float);
    const float *ptrs[] = {g, M, init, S};
    for (const float *p : ptrs)
        if (p && !aligned16(p)) return HGRN2_ERR_INVALID_ARG;
    if (count > 0) {   // S must not overlap the maps (init may be S itself)
        auto overlap = [](const void *a, size_t na, const void *b, size_t nb) {
            return (const char *)a < (const char *)b + nb && (const char *)b < (const char *)a + na;
        };
        if (overlap(S, ns, g, (size_t)R * nbh * dk * sizeof(float)) || overlap(S, ns, M, (size_t)R * ns))
            return HGRN2_ERR_INVALID_ARG;
    }
    g_launches += 1;
    return from_cuda(launch_affine_scan(g, M, init, S, nbh, dk, dv, first, count, step, stream));
}

}  // extern "C"

// ------------------------------------------------------------------ scalar-decay variant
namespace {
hgrn2_status check_scalar(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype) {
    if (B < 1 || H < 1 || T < 0 || dk < 1 || dv < 1) return HGRN2_ERR_INVALID_ARG;
    if (dtype != HGRN2_FP32 && dtype != HGRN2_BF16) return HGRN2_ERR_INVALID_ARG;
    if (dk > 128 || dv > 128) return HGRN2_ERR_UNSUPPORTED;
    if ((long long)B * H > (1ll << 30) || (long long)B * T * H > (1ll << 40)) return HGRN2_ERR_UNSUPPORTED;
    return HGRN2_OK;
}
// Workspace of hgrn2_scalar_bwd: <dhT, hT> per (b,h) and q . dq per token (exact route); on the
// tensor-core route also the chunk states its forward saves and an o scratch.
size_t scalar_ws_bytes(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype, int want) {
    if (want == 0) return 0;   // the forward needs none
    size_t n = align256(sizeof(float) * (size_t)B * H) + align256(sizeof(float) * (size_t)B * T * H);   // rs, q.dq
    if (want == 1 && use_tc(dk, dv, dtype) && T > 0)   // no saved states: room for them and an o scratch
        n += saved_layout(B, T, H).total + align256((size_t)B * T * H * dv * 2);
    return n;
}

bool all_aligned(std::initializer_list<const void *> ptrs) {
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return false;
    return true;
}
}  // namespace

}  // extern "C"

namespace {

// Scalar-decay forward; `saved` (null, or scalar_saved_bytes) receives the chunk states and the
// range flags that the reverse sweep reads (tensor-core route only).
hgrn2_status scalar_fwd_impl(const void *q, const void *k, const void *v, const void *log_g, const float *h0,
                             void *o, float *hT, void *saved, int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                             cudaStream_t stream) {
    hgrn2_status s = check_scalar(B, T, H, dk, dv, dtype);
    if (s != HGRN2_OK) return s;
    if (T > 0 && (!q || !k || !v || !log_g || !o)) return HGRN2_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, log_g, h0, o, hT, saved})) return HGRN2_ERR_INVALID_ARG;
    if (T == 0) {
        if (!hT) return HGRN2_OK;
        const size_t n = sizeof(float) * (size_t)B * H * dk * dv;
        return from_cuda(h0 ? cudaMemcpyAsync(hT, h0, n, cudaMemcpyDeviceToDevice, stream)
                            : cudaMemsetAsync(hT, 0, n, stream));
    }
    g_launches += 1;
    if (use_tc(dk, dv, dtype)) {   // tensor cores: the kScalar instance of the forward kernel
        const SavedLayout sl = saved_layout(B, T, H);
        int *flags = saved ? (int *)((char *)saved + sl.flags) : nullptr;
        float *hTs = saved ? (float *)((char *)saved + sl.hTs) : nullptr;
        TcFwdArgs t{q, k, v, h0, o, hT, flags, nullptr, B, T, H, 32, saved, hTs, nullptr, nullptr, dk, log_g};
        return from_cuda(launch_tc_fwd(t, stream));
    }
    ScalarArgs a{q, k, v, log_g, h0, o, hT, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                 nullptr, nullptr, B, T, H, dk, dv, nullptr};
    return from_cuda(launch_scalar_fwd(a, dtype == HGRN2_BF16, stream));
}

size_t scalar_saved_bytes(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype) {
    return (use_tc(dk, dv, dtype) && T > 0) ? saved_layout(B, T, H).total : 0;
}

// Scalar-decay backward.  With `saved` (from scalar_fwd_impl on the same inputs) the reverse sweep
// reads its chunk states; without it, on the tensor-core route, the forward runs again into the
// workspace first.
hgrn2_status scalar_bwd_impl(const void *q, const void *k, const void *v, const void *log_g, const float *h0,
                             const void *saved, const void *dO, const float *dhT, void *dq, void *dk_out,
                             void *dv_out, void *dlog_g, float *dh0, int B, int T, int H, int dk, int dv,
                             hgrn2_dtype dtype, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    hgrn2_status s = check_scalar(B, T, H, dk, dv, dtype);
    if (s != HGRN2_OK) return s;
    if (T > 0 && (!q || !k || !v || !log_g || !dO || !dq || !dk_out || !dv_out || !dlog_g))
        return HGRN2_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, log_g, h0, dO, dhT, dq, dk_out, dv_out, dlog_g, dh0, workspace, saved}))
        return HGRN2_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < scalar_ws_bytes(B, T, H, dk, dv, dtype, saved ? 2 : 1)) return HGRN2_ERR_INVALID_ARG;
    if (T == 0) {
        if (!dh0) return HGRN2_OK;
        const size_t n = sizeof(float) * (size_t)B * H * dk * dv;
        return from_cuda(dhT ? cudaMemcpyAsync(dh0, dhT, n, cudaMemcpyDeviceToDevice, stream)
                             : cudaMemsetAsync(dh0, 0, n, stream));
    }
    float *rs = (float *)workspace;
    float *qdq = (float *)((char *)workspace + align256(sizeof(float) * (size_t)B * H));
    const size_t base = align256(sizeof(float) * (size_t)B * H) + align256(sizeof(float) * (size_t)B * T * H);
    if (use_tc(dk, dv, dtype)) {
        // the reverse sweep over the saved chunk states; pairs whose chunk decay leaves the factorised
        // form's range were flagged by the forward and are recomputed on the exact route
        const SavedLayout sl = saved_layout(B, T, H);
        char *sv = (char *)saved;
        if (!sv) {   // no saved states: the forward again, into the workspace (o to scratch)
            sv = (char *)workspace + base;
            s = scalar_fwd_impl(q, k, v, log_g, h0, sv + sl.total, nullptr, sv, B, T, H, dk, dv, dtype, stream);
            if (s != HGRN2_OK) return s;
        }
        int *flags = (int *)(sv + sl.flags);
        float *hTs = (float *)(sv + sl.hTs);
        TcBwdArgs r{q, k, v, dO, h0, dhT, dq, dk_out, dv_out, dh0, rs, flags, B, T, H, 32, sv, hTs, nullptr, nullptr,
                    dk, log_g, dlog_g};
        if (launch_tc_bwd(r, stream) != cudaSuccess) return HGRN2_ERR_CUDA;
        ScalarArgs a{q, k, v, log_g, h0, nullptr, nullptr, dO, dhT, dq, dk_out, dv_out, dlog_g, dh0, rs, qdq, B, T, H,
                     dk, dv, flags};
        g_launches += 3;
        return from_cuda(launch_scalar_bwd(a, dtype == HGRN2_BF16, stream));
    }
    ScalarArgs a{q, k, v, log_g, h0, nullptr, nullptr, dO, dhT, dq, dk_out, dv_out, dlog_g, dh0, rs, qdq, B, T, H, dk,
                 dv, nullptr};
    g_launches += 2;
    return from_cuda(launch_scalar_bwd(a, dtype == HGRN2_BF16, stream));
}

}  // namespace

extern "C" {

size_t hgrn2_scalar_workspace_size(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype, int want_bwd) {
    if (check_scalar(B, T, H, dk, dv, dtype) != HGRN2_OK || want_bwd < 0 || want_bwd > 2) return (size_t)-1;
    return scalar_ws_bytes(B, T, H, dk, dv, dtype, want_bwd);
}

size_t hgrn2_scalar_saved_size(int B, int T, int H, int dk, int dv, hgrn2_dtype dtype) {
    if (check_scalar(B, T, H, dk, dv, dtype) != HGRN2_OK) return (size_t)-1;
    return scalar_saved_bytes(B, T, H, dk, dv, dtype);
}

hgrn2_status hgrn2_scalar_fwd(const void *q, const void *k, const void *v, const void *log_g, const float *h0,
                              void *o, float *hT, int B, int T, int H, int dk, int dv, hgrn2_dtype dtype,
                              cudaStream_t stream) {
    return scalar_fwd_impl(q, k, v, log_g, h0, o, hT, nullptr, B, T, H, dk, dv, dtype, stream);
}

hgrn2_status hgrn2_scalar_fwd_train(const void *q, const void *k, const void *v, const void *log_g, const float *h0,
                                    void *o, float *hT, void *saved, size_t saved_bytes, int B, int T, int H, int dk,
                                    int dv, hgrn2_dtype dtype, cudaStream_t stream) {
    if (check_scalar(B, T, H, dk, dv, dtype) != HGRN2_OK) return check_scalar(B, T, H, dk, dv, dtype);
    const size_t need = scalar_saved_bytes(B, T, H, dk, dv, dtype);
    if (need && (!saved || saved_bytes < need)) return HGRN2_ERR_INVALID_ARG;
    return scalar_fwd_impl(q, k, v, log_g, h0, o, hT, need ? saved : nullptr, B, T, H, dk, dv, dtype, stream);
}

hgrn2_status hgrn2_scalar_bwd(const void *q, const void *k, const void *v, const void *log_g, const float *h0,
                              const void *dO, const float *dhT, void *dq, void *dk_out, void *dv_out, void *dlog_g,
                              float *dh0, int B, int T, int H, int dk, int dv, hgrn2_dtype dtype, void *workspace,
                              size_t ws_bytes, cudaStream_t stream) {
    return scalar_bwd_impl(q, k, v, log_g, h0, nullptr, dO, dhT, dq, dk_out, dv_out, dlog_g, dh0, B, T, H, dk, dv,
                           dtype, workspace, ws_bytes, stream);
}

hgrn2_status hgrn2_scalar_bwd_saved(const void *q, const void *k, const void *v, const void *log_g, const float *h0,
                                    const void *saved, size_t saved_bytes, const void *dO, const float *dhT, void *dq,
                                    void *dk_out, void *dv_out, void *dlog_g, float *dh0, int B, int T, int H, int dk,
                                    int dv, hgrn2_dtype dtype, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (check_scalar(B, T, H, dk, dv, dtype) != HGRN2_OK) return check_scalar(B, T, H, dk, dv, dtype);
    const size_t need = scalar_saved_bytes(B, T, H, dk, dv, dtype);
    if (need && (!saved || saved_bytes < need)) return HGRN2_ERR_INVALID_ARG;
    return scalar_bwd_impl(q, k, v, log_g, h0, need ? saved : nullptr, dO, dhT, dq, dk_out, dv_out, dlog_g, dh0, B, T,
                           H, dk, dv, dtype, workspace, ws_bytes, stream);
}

hgrn2_status hgrn2_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return HGRN2_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return HGRN2_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return HGRN2_ERR_CUDA;
    return (hgrn2_status)v;
}

hgrn2_status hgrn2_get_counters(long long *out, int n, int reset, cudaStream_t stream) {
    if (!out || n < 0) return HGRN2_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return HGRN2_ERR_CUDA;
    unsigned long long c[2] = {0, 0};
    if (cudaMemcpyFromSymbol(c, g_counters, sizeof(c)) != cudaSuccess) return HGRN2_ERR_CUDA;
    for (int k = 0; k < n && k < 2; ++k) out[k] = (long long)c[k];
    if (n > 2) out[2] = g_launches.load();
    if (reset) {
        unsigned long long z[2] = {0, 0};
        if (cudaMemcpyToSymbol(g_counters, z, sizeof(z)) != cudaSuccess) return HGRN2_ERR_CUDA;
        g_launches = 0;
    }
    return HGRN2_OK;
}

const char *hgrn2_status_string(hgrn2_status s) {
    switch (s) {
        case HGRN2_OK: return "ok";
        case HGRN2_ERR_INVALID_ARG: return "invalid argument";
        case HGRN2_ERR_UNSUPPORTED: return "unsupported shape, chunk or dtype";
        case HGRN2_ERR_CUDA: return "CUDA runtime error";
        case HGRN2_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case HGRN2_ERR_DEVICE: return "a device-side consistency check failed";
    }
    return "unknown status";
}

const char *hgrn2_version(void) { return "hgrn2-b200 0.1"; }

}  // extern "C"

// ------------------------------------------------------------------ allocation-free backward
// Scratch of hgrn2_bwd_noalloc: a fixed-size array in the library's own device
// memory, present on every GPU the library is loaded on for the life of the
// process.  Host code only ever sees a stand-in for this symbol; the device
// address is looked up with cudaGetSymbolAddress, once per device and context:
// the cache is keyed on the current driver context, so a context made anew on
// the same device (after cudaDeviceReset, say), whose copy of the array may sit
// elsewhere, gets a fresh lookup instead of a stale address.
namespace {
constexpr size_t kNoAllocScratchBytes = HGRN2_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
struct NoAllocEntry {
    CUcontext ctx;
    void *ptr;
};
NoAllocEntry g_noalloc[kMaxDevices] = {};

// The calling thread's current driver context (null if none is current yet).
CUcontext current_context() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    }
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Device address of the scratch array in the current device's current context.
hgrn2_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return HGRN2_ERR_CUDA;
    if (dev >= kMaxDevices) return HGRN2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    CUcontext ctx = current_context();
    if (!ctx || g_noalloc[dev].ctx != ctx || !g_noalloc[dev].ptr) {
        void *p = nullptr;   // the lookup also makes the device's primary context current if none is
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HGRN2_ERR_CUDA;
        g_noalloc[dev].ctx = current_context();
        g_noalloc[dev].ptr = p;
    }
    *out = g_noalloc[dev].ptr;
    return HGRN2_OK;
}
}  // namespace

extern "C" hgrn2_status hgrn2_bwd_noalloc(const void *q, const void *log_f, const void *i, const float *h0,
                                          const void *dO, const float *dhT, void *dq, void *dlog_f, void *di,
                                          float *dh0, int B, int T, int H, int dk, int dv, int chunk,
                                          hgrn2_dtype dtype, cudaStream_t stream) {
    hgrn2_status s = check_common(B, T, H, dk, dv, chunk, dtype);
    if (s != HGRN2_OK) return s;
    // 64-wide heads take the exact route here: their tensor-core recompute needs a workspace
    // the size of the chunk states
    const size_t need = ws_bytes_needed(B, T, H, dk, dv, chunk, dtype, 1, false);
    if (need > kNoAllocScratchBytes) return HGRN2_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != HGRN2_OK) return s;
    return bwd_impl(q, log_f, i, h0, nullptr, dO, dhT, dq, dlog_f, di, dh0, B, T, H, dk, dv, chunk, dtype, scratch,
                    kNoAllocScratchBytes, stream, nullptr, false);
}
