// simt.cu -- exact chunkwise HGRN2 on CUDA cores (fp32 arithmetic, no TF32).
//
// This is the library's exact route: it serves every float32 call, every shape
// the tensor-core kernels do not take, and (batch, head) pairs whose per-chunk
// cumulative log-decay is too wide for the tensor-core factorisation.
//
// Chunkwise form of the recurrence ("HGRN2: Gated Linear RNNs with State
// Expansion", §3.2: the recurrence is gated linear attention with key
// k = 1 - f, value v = i, query q, so chunkwise algorithms apply; §5: one decay
// per key dimension).  Inside a chunk starting with state S_in, with
// b_t = sum_{r<=t} log f_r (cumulative from the chunk start, per key dim j) and
// B = b at the chunk's last token:
//
//   o_t   = (q_t * e^{b_t})^T S_in + sum_{s<=t} A_ts v_s,
//   A_ts  = sum_j q_t[j] k_s[j] e^{b_t[j] - b_s[j]}              (exact exps)
//   S_out = Diag(e^B) S_in + sum_s (k_s * e^{B - b_s}) v_s^T
//
// Every exponent formed is <= 0 when log f <= 0, so nothing overflows however
// strong the decay.  One thread block walks the chunks of one (batch, head).
//
// The bodies are device functions kept out of line (__noinline__): the tensor-core
// kernels call them only for flagged pairs, and inlined there they made those kernels'
// code large enough that instruction fetch cost the reverse sweep 10% of its time.
#include "common.cuh"
#include "kernels.h"

namespace hgrn2 {

constexpr int kSimtThreads = 256;

static __device__ __forceinline__ size_t tok(int b, int t, int h, int T, int H, int D) {
    return (((size_t)b * T + t) * H + h) * (size_t)D;
}

// ------------------------------------------------------------------ smem sizes
size_t simt_fwd_smem(int C, int dk, int dv) {
    size_t ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    return sizeof(float) * (3 * C * ldk + C * ldv + C * ldc + (size_t)dk * ldv);
}
size_t simt_bwd_dq_smem(int C, int dk, int dv) {
    size_t ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    return sizeof(float) * (2 * C * ldk + 2 * C * ldv + C * ldc + (size_t)dk * ldv);
}
size_t simt_bwd_rev_smem(int C, int dk, int dv) {
    size_t ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    return sizeof(float) * (6 * C * ldk + 2 * C * ldv + 2 * C * ldc + (size_t)dk * ldv + dk);
}

// Loads rows [c0, c0+C) of one (b,h) of a token tensor into smem (row stride ld),
// zero-filling rows past the end of the sequence.
template <typename T>
static __device__ __forceinline__ void load_tile(float *dst, int ld, const T *src, int b, int h,
                                                 int c0, int C, int n, int T_, int H, int D) {
    for (int idx = threadIdx.x; idx < C * D; idx += blockDim.x) {
        int t = idx / D, j = idx - t * D;
        dst[t * ld + j] = (t < n) ? to_f<T>(src[tok(b, c0 + t, h, T_, H, D) + j]) : 0.0f;
    }
}

// A 16-bit token tensor carries fp32 values of dq between the exact backward's two sweeps: the
// forward sweep writes each value's low half into the d log f row and its high half into the di
// row of its token (rows the reverse sweep overwrites only after reading them back), so that the
// reverse sweep's d log f sums q dq over the sequence from fp32 dq, not from the rounded output.
// Needs d_v >= d_k; tok() indexes both tensors as usual.
static __device__ __forceinline__ void stash_f32(void *lo, void *hi, size_t ilo, size_t ihi, float v) {
    const uint32_t u = __float_as_uint(v);
    reinterpret_cast<uint16_t *>(lo)[ilo] = (uint16_t)(u & 0xffffu);
    reinterpret_cast<uint16_t *>(hi)[ihi] = (uint16_t)(u >> 16);
}
static __device__ __forceinline__ void load_stash(float *dst, int ld, const void *lo, const void *hi, int b, int h,
                                                  int c0, int C, int n, int T_, int H, int dk, int dv) {
    for (int idx = threadIdx.x; idx < C * dk; idx += blockDim.x) {
        int t = idx / dk, j = idx - t * dk;
        float v = 0.0f;
        if (t < n) {
            const uint32_t l = reinterpret_cast<const uint16_t *>(lo)[tok(b, c0 + t, h, T_, H, dk) + j];
            const uint32_t u = reinterpret_cast<const uint16_t *>(hi)[tok(b, c0 + t, h, T_, H, dv) + j];
            v = __uint_as_float(l | (u << 16));
        }
        dst[t * ld + j] = v;
    }
}

// log f -> (inclusive cumsum b in place, k = 1 - f in K).  One thread per key dim.
static __device__ __forceinline__ void cumsum_gates(float *Bs, float *Ks, int ld, int C, int dk) {
    for (int j = threadIdx.x; j < dk; j += blockDim.x) {
        float acc = 0.0f;
        for (int t = 0; t < C; ++t) {
            float a = Bs[t * ld + j];
            if (Ks) Ks[t * ld + j] = one_minus_exp(a);
            acc += a;
            Bs[t * ld + j] = acc;
        }
    }
}

// ------------------------------------------------------------------ forward
template <typename T>
__device__ __noinline__ void
simt_fwd_body(const T *__restrict__ q, const T *__restrict__ lf, const T *__restrict__ x,
                const float *__restrict__ h0, T *__restrict__ o, float *__restrict__ hT,
                int T_, int H, int dk, int dv, int C, float *sm, int b, int h, int sidx) {
    const int ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    float *Qs = sm;              // [C][ldk]  q, then q * e^{b}
    float *Bs = Qs + C * ldk;    // [C][ldk]  log f, then cumulative b
    float *Ks = Bs + C * ldk;    // [C][ldk]  k, then k * e^{B - b}
    float *Vs = Ks + C * ldk;    // [C][ldv]
    float *As = Vs + C * ldv;    // [C][ldc]
    float *Ss = As + C * ldc;    // [dk][ldv] running state (fp32)
    const int tid = threadIdx.x;
    const size_t sbase = (size_t)sidx * dk * dv;

    for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
        int j = idx / dv, v = idx - j * dv;
        Ss[j * ldv + v] = h0 ? h0[sbase + idx] : 0.0f;
    }
    for (int c0 = 0; c0 < T_; c0 += C) {
        const int n = min(C, T_ - c0);
        __syncthreads();
        load_tile(Qs, ldk, q, b, h, c0, C, n, T_, H, dk);
        load_tile(Bs, ldk, lf, b, h, c0, C, n, T_, H, dk);
        load_tile(Vs, ldv, x, b, h, c0, C, n, T_, H, dv);
        __syncthreads();
        cumsum_gates(Bs, Ks, ldk, C, dk);
        __syncthreads();
        // intra-chunk scores, exact per-dimension decay
        for (int p = tid; p < C * C; p += blockDim.x) {
            int t = p / C, s = p - t * C;
            float acc = 0.0f;
            if (s <= t) {
                const float *qt = Qs + t * ldk, *ks = Ks + s * ldk, *bt = Bs + t * ldk, *bs = Bs + s * ldk;
                for (int j = 0; j < dk; ++j) acc = fmaf(qt[j] * ks[j], expf(bt[j] - bs[j]), acc);
            }
            As[t * ldc + s] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < C * dk; idx += blockDim.x) {
            int t = idx / dk, j = idx - t * dk;
            float bt = Bs[t * ldk + j];
            Qs[t * ldk + j] *= expf(bt);
            Ks[t * ldk + j] *= expf(Bs[(C - 1) * ldk + j] - bt);
        }
        __syncthreads();
        for (int idx = tid; idx < C * dv; idx += blockDim.x) {
            int t = idx / dv, v = idx - t * dv;
            float acc = 0.0f;
            const float *qt = Qs + t * ldk;
            for (int j = 0; j < dk; ++j) acc = fmaf(qt[j], Ss[j * ldv + v], acc);
            const float *at = As + t * ldc;
            for (int s = 0; s <= t; ++s) acc = fmaf(at[s], Vs[s * ldv + v], acc);
            if (t < n) o[tok(b, c0 + t, h, T_, H, dv) + v] = from_f<T>(acc);
        }
        __syncthreads();
        for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
            int j = idx / dv, v = idx - j * dv;
            float acc = expf(Bs[(C - 1) * ldk + j]) * Ss[j * ldv + v];
            for (int s = 0; s < C; ++s) acc = fmaf(Ks[s * ldk + j], Vs[s * ldv + v], acc);
            Ss[j * ldv + v] = acc;
        }
    }
    __syncthreads();
    if (hT)
        for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
            int j = idx / dv, v = idx - j * dv;
            hT[sbase + idx] = Ss[j * ldv + v];
        }
}

// ------------------------------------------------------------------ backward, forward sweep (dq)
// dq_t = S_t dO_t.  Chunkwise: dq_t = e^{b_t} * (S_in dO_t) + sum_{s<=t} dA_ts k_s e^{b_t - b_s},
// dA_ts = dO_t . v_s.  Also writes rs[j] = sum_v dhT[j,v] hT[j,v] when dhT != NULL (used by the
// reverse sweep's d log f carry).
template <typename T>
__device__ __noinline__ void
simt_bwd_dq_body(const T *__restrict__ lf, const T *__restrict__ x, const float *__restrict__ h0,
                   const T *__restrict__ dO, const float *__restrict__ dhT, T *__restrict__ dq,
                   float *__restrict__ rs, int T_, int H, int dk, int dv, int C, float *sm, int b, int h, int sidx,
                   T *stash_lo = nullptr, T *stash_hi = nullptr) {
    const int ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    float *Bs = sm;              // [C][ldk]
    float *Ks = Bs + C * ldk;    // [C][ldk]
    float *Vs = Ks + C * ldk;    // [C][ldv]
    float *Gs = Vs + C * ldv;    // [C][ldv] dO
    float *As = Gs + C * ldv;    // [C][ldc] dA
    float *Ss = As + C * ldc;    // [dk][ldv]
    const int tid = threadIdx.x;
    const size_t sbase = (size_t)sidx * dk * dv;

    for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
        int j = idx / dv, v = idx - j * dv;
        Ss[j * ldv + v] = h0 ? h0[sbase + idx] : 0.0f;
    }
    for (int c0 = 0; c0 < T_; c0 += C) {
        const int n = min(C, T_ - c0);
        __syncthreads();
        load_tile(Bs, ldk, lf, b, h, c0, C, n, T_, H, dk);
        load_tile(Vs, ldv, x, b, h, c0, C, n, T_, H, dv);
        load_tile(Gs, ldv, dO, b, h, c0, C, n, T_, H, dv);
        __syncthreads();
        cumsum_gates(Bs, Ks, ldk, C, dk);
        for (int p = tid; p < C * C; p += blockDim.x) {
            int t = p / C, s = p - t * C;
            float acc = 0.0f;
            if (s <= t)
                for (int v = 0; v < dv; ++v) acc = fmaf(Gs[t * ldv + v], Vs[s * ldv + v], acc);
            As[t * ldc + s] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < C * dk; idx += blockDim.x) {
            int t = idx / dk, j = idx - t * dk;
            float inter = 0.0f;
            for (int v = 0; v < dv; ++v) inter = fmaf(Ss[j * ldv + v], Gs[t * ldv + v], inter);
            const float bt = Bs[t * ldk + j];
            float acc = expf(bt) * inter;
            for (int s = 0; s <= t; ++s)
                acc = fmaf(As[t * ldc + s] * Ks[s * ldk + j], expf(bt - Bs[s * ldk + j]), acc);
            if (t < n) {
                dq[tok(b, c0 + t, h, T_, H, dk) + j] = from_f<T>(acc);
                if (sizeof(T) == 2 && stash_lo)
                    stash_f32(stash_lo, stash_hi, tok(b, c0 + t, h, T_, H, dk) + j, tok(b, c0 + t, h, T_, H, dv) + j, acc);
            }
        }
        __syncthreads();
        for (int idx = tid; idx < C * dk; idx += blockDim.x) {
            int t = idx / dk, j = idx - t * dk;
            Ks[t * ldk + j] *= expf(Bs[(C - 1) * ldk + j] - Bs[t * ldk + j]);
        }
        __syncthreads();
        for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
            int j = idx / dv, v = idx - j * dv;
            float acc = expf(Bs[(C - 1) * ldk + j]) * Ss[j * ldv + v];
            for (int s = 0; s < C; ++s) acc = fmaf(Ks[s * ldk + j], Vs[s * ldv + v], acc);
            Ss[j * ldv + v] = acc;
        }
    }
    __syncthreads();
    if (dhT && rs)
        for (int j = tid; j < dk; j += blockDim.x) {
            float acc = 0.0f;
            for (int v = 0; v < dv; ++v) acc = fmaf(dhT[sbase + (size_t)j * dv + v], Ss[j * ldv + v], acc);
            rs[(size_t)sidx * dk + j] = acc;
        }
}

// ------------------------------------------------------------------ backward, reverse sweep
// With dS = dL/dS_out of the chunk (dhT for the last one):
//   di_s  = sum_{t>=s} A_ts dO_t + (k_s * e^{B - b_s})^T-row . dS
//   dk_s  = sum_{t>=s} dA_ts q_t e^{b_t - b_s} + e^{B - b_s} * (dS v_s)
//   dlog f_t = sum_{t'>=t} (q*dq - k*dk)_{t'} + rowsum(dhT*hT) - f_t * dk_t
//   dS_in = Diag(e^B) dS + sum_t (q_t e^{b_t}) dO_t^T
// The reverse cumulative sum runs across chunks through `carry`.
template <typename T>
__device__ __noinline__ void
simt_bwd_rev_body(const T *__restrict__ q, const T *__restrict__ lf, const T *__restrict__ x,
                    const T *__restrict__ dO, const float *__restrict__ dhT, const T *__restrict__ dq,
                    const float *__restrict__ rs, T *__restrict__ dlf, T *__restrict__ dx,
                    float *__restrict__ dh0, int T_, int H, int dk, int dv, int C, float *sm, int b, int h, int sidx,
                    bool dq_stashed = false) {
    const int ldk = dk + 1, ldv = dv + 1, ldc = C + 1;
    float *Qs = sm;               // [C][ldk] q, later q e^{b}
    float *Bs = Qs + C * ldk;     // [C][ldk] b
    float *Ks = Bs + C * ldk;     // [C][ldk] k
    float *Es = Ks + C * ldk;     // [C][ldk] e^{B - b}
    float *Ds = Es + C * ldk;     // [C][ldk] dq (read back)
    float *DKs = Ds + C * ldk;    // [C][ldk] dk
    float *Vs = DKs + C * ldk;    // [C][ldv]
    float *Gs = Vs + C * ldv;     // [C][ldv] dO
    float *As = Gs + C * ldv;     // [C][ldc]
    float *dAs = As + C * ldc;    // [C][ldc]
    float *dS = dAs + C * ldc;    // [dk][ldv]
    float *carry = dS + dk * ldv; // [dk]
    const int tid = threadIdx.x;
    const size_t sbase = (size_t)sidx * dk * dv;

    for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
        int j = idx / dv, v = idx - j * dv;
        dS[j * ldv + v] = dhT ? dhT[sbase + idx] : 0.0f;
    }
    for (int j = tid; j < dk; j += blockDim.x) carry[j] = (dhT && rs) ? rs[(size_t)sidx * dk + j] : 0.0f;

    const int nchunks = (T_ + C - 1) / C;
    for (int c = nchunks - 1; c >= 0; --c) {
        const int c0 = c * C, n = min(C, T_ - c0);
        __syncthreads();
        load_tile(Qs, ldk, q, b, h, c0, C, n, T_, H, dk);
        load_tile(Bs, ldk, lf, b, h, c0, C, n, T_, H, dk);
        if (dq_stashed) load_stash(Ds, ldk, dlf, dx, b, h, c0, C, n, T_, H, dk, dv);   // fp32 dq
        else load_tile(Ds, ldk, dq, b, h, c0, C, n, T_, H, dk);
        load_tile(Vs, ldv, x, b, h, c0, C, n, T_, H, dv);
        load_tile(Gs, ldv, dO, b, h, c0, C, n, T_, H, dv);
        __syncthreads();
        cumsum_gates(Bs, Ks, ldk, C, dk);
        __syncthreads();
        for (int idx = tid; idx < C * dk; idx += blockDim.x) {
            int t = idx / dk, j = idx - t * dk;
            Es[idx / dk * ldk + j] = expf(Bs[(C - 1) * ldk + j] - Bs[t * ldk + j]);
        }
        for (int p = tid; p < C * C; p += blockDim.x) {
            int t = p / C, s = p - t * C;
            float a = 0.0f, da = 0.0f;
            if (s <= t) {
                const float *qt = Qs + t * ldk, *ks = Ks + s * ldk, *bt = Bs + t * ldk, *bs = Bs + s * ldk;
                for (int j = 0; j < dk; ++j) a = fmaf(qt[j] * ks[j], expf(bt[j] - bs[j]), a);
                for (int v = 0; v < dv; ++v) da = fmaf(Gs[t * ldv + v], Vs[s * ldv + v], da);
            }
            As[t * ldc + s] = a;
            dAs[t * ldc + s] = da;
        }
        __syncthreads();
        // di
        for (int idx = tid; idx < C * dv; idx += blockDim.x) {
            int s = idx / dv, v = idx - s * dv;
            float acc = 0.0f;
            for (int t = s; t < C; ++t) acc = fmaf(As[t * ldc + s], Gs[t * ldv + v], acc);
            for (int j = 0; j < dk; ++j)
                acc = fmaf(Ks[s * ldk + j] * Es[s * ldk + j], dS[j * ldv + v], acc);
            if (s < n) dx[tok(b, c0 + s, h, T_, H, dv) + v] = from_f<T>(acc);
        }
        // dk
        for (int idx = tid; idx < C * dk; idx += blockDim.x) {
            int s = idx / dk, j = idx - s * dk;
            const float bs = Bs[s * ldk + j];
            float acc = 0.0f;
            for (int t = s; t < C; ++t)
                acc = fmaf(dAs[t * ldc + s] * Qs[t * ldk + j], expf(Bs[t * ldk + j] - bs), acc);
            float sv = 0.0f;
            for (int v = 0; v < dv; ++v) sv = fmaf(dS[j * ldv + v], Vs[s * ldv + v], sv);
            DKs[s * ldk + j] = fmaf(Es[s * ldk + j], sv, acc);
        }
        __syncthreads();
        // d log f: reverse cumulative sum inside the chunk plus the carry from later chunks
        for (int j = tid; j < dk; j += blockDim.x) {
            float rc = carry[j];
            for (int t = C - 1; t >= 0; --t) {
                const float dkt = DKs[t * ldk + j];
                rc += Qs[t * ldk + j] * Ds[t * ldk + j] - Ks[t * ldk + j] * dkt;
                const float bprev = t > 0 ? Bs[(t - 1) * ldk + j] : 0.0f;
                const float f = expf(Bs[t * ldk + j] - bprev);
                if (t < n) dlf[tok(b, c0 + t, h, T_, H, dk) + j] = from_f<T>(rc - f * dkt);
            }
            carry[j] = rc;
        }
        __syncthreads();
        for (int idx = tid; idx < C * dk; idx += blockDim.x) {
            int t = idx / dk, j = idx - t * dk;
            Qs[t * ldk + j] *= expf(Bs[t * ldk + j]);
        }
        __syncthreads();
        for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
            int j = idx / dv, v = idx - j * dv;
            float acc = expf(Bs[(C - 1) * ldk + j]) * dS[j * ldv + v];
            for (int t = 0; t < C; ++t) acc = fmaf(Qs[t * ldk + j], Gs[t * ldv + v], acc);
            dS[j * ldv + v] = acc;
        }
    }
    __syncthreads();
    if (dh0)
        for (int idx = tid; idx < dk * dv; idx += blockDim.x) {
            int j = idx / dv, v = idx - j * dv;
            dh0[sbase + idx] = dS[j * ldv + v];
        }
}


// ------------------------------------------------------------------ kernels (one CTA per (b,h))
// With cu (variable-length packed sequences: token tensors [total_T][H][D], sequence s at
// tokens cu[s] .. cu[s+1]-1), CTA (r,h) runs sequence s = perm[r] (r without perm) on pointers
// offset to the sequence's first token, with batch 0 and T = its length; its states are those
// of pair s*H+h.  cu values are clamped to [0, total_T].
struct SeqView {
    int b, h, T, sidx;
    size_t tok0;
};
__device__ __forceinline__ SeqView seq_view(const int *cu, const int *perm, int bid, int H, int T_) {
    SeqView v;
    v.h = bid % H;
    v.sidx = bid;
    if (cu) {
        const int s = packed_seq(perm, bid / H, gridDim.x / H);
        const int a = min(max(cu[s], 0), T_), e = min(max(cu[s + 1], a), T_);
        v.b = 0;
        v.T = e - a;
        v.tok0 = (size_t)a;
        v.sidx = s * H + v.h;
    } else {
        v.b = bid / H;
        v.T = T_;
        v.tok0 = 0;
    }
    return v;
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
simt_fwd_kernel(const T *__restrict__ q, const T *__restrict__ lf, const T *__restrict__ x,
                const float *__restrict__ h0, T *__restrict__ o, float *__restrict__ hT,
                int T_, int H, int dk, int dv, int C, const int *__restrict__ only, const int *__restrict__ cu,
                const int *__restrict__ perm) {
    if (only && only[blockIdx.x] == 0) return;
    extern __shared__ float sm[];
    const SeqView v = seq_view(cu, perm, blockIdx.x, H, T_);
    const size_t ok = v.tok0 * H * dk, ov = v.tok0 * H * dv;
    simt_fwd_body<T>(q + ok, lf + ok, x + ov, h0, o + ov, hT, v.T, H, dk, dv, C, sm, v.b, v.h, v.sidx);
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
simt_bwd_dq_kernel(const T *__restrict__ lf, const T *__restrict__ x, const float *__restrict__ h0,
                   const T *__restrict__ dO, const float *__restrict__ dhT, T *__restrict__ dq,
                   float *__restrict__ rs, T *dlf, T *dx, int T_, int H, int dk, int dv, int C,
                   const int *__restrict__ only, const int *__restrict__ cu, const int *__restrict__ perm) {
    if (only && only[blockIdx.x] == 0) return;
    extern __shared__ float sm[];
    const SeqView v = seq_view(cu, perm, blockIdx.x, H, T_);
    const size_t ok = v.tok0 * H * dk, ov = v.tok0 * H * dv;
    const bool st = sizeof(T) == 2 && dv >= dk && dlf;
    simt_bwd_dq_body<T>(lf + ok, x + ov, h0, dO + ov, dhT, dq + ok, rs, v.T, H, dk, dv, C, sm, v.b, v.h, v.sidx,
                        st ? dlf + ok : nullptr, st ? dx + ov : nullptr);
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
simt_bwd_rev_kernel(const T *__restrict__ q, const T *__restrict__ lf, const T *__restrict__ x,
                    const T *__restrict__ dO, const float *__restrict__ dhT, const T *__restrict__ dq,
                    const float *__restrict__ rs, T *__restrict__ dlf, T *__restrict__ dx,
                    float *__restrict__ dh0, int T_, int H, int dk, int dv, int C, const int *__restrict__ only,
                    const int *__restrict__ cu, const int *__restrict__ perm) {
    if (only && only[blockIdx.x] == 0) return;
    extern __shared__ float sm[];
    const SeqView v = seq_view(cu, perm, blockIdx.x, H, T_);
    const size_t ok = v.tok0 * H * dk, ov = v.tok0 * H * dv;
    simt_bwd_rev_body<T>(q + ok, lf + ok, x + ov, dO + ov, dhT, dq + ok, rs, dlf + ok, dx + ov, dh0, v.T, H, dk, dv, C,
                         sm, v.b, v.h, v.sidx, sizeof(T) == 2 && dv >= dk);
}

// ------------------------------------------------------------------ launchers
template <typename T>
static cudaError_t launch_simt_fwd_t(const SimtFwdArgs &a, cudaStream_t st) {
    size_t smem = simt_fwd_smem(a.C, a.dk, a.dv);
    auto *k = simt_fwd_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.B * a.H, kSimtThreads, smem, st>>>((const T *)a.q, (const T *)a.lf, (const T *)a.x, a.h0,
                                             (T *)a.o, a.hT, a.T, a.H, a.dk, a.dv, a.C, a.only, a.cu, a.perm);
    return cudaGetLastError();
}

cudaError_t launch_simt_fwd(const SimtFwdArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_simt_fwd_t<__nv_bfloat16>(a, st) : launch_simt_fwd_t<float>(a, st);
}

template <typename T>
static cudaError_t launch_simt_bwd_t(const SimtBwdArgs &a, cudaStream_t st) {
    size_t s1 = simt_bwd_dq_smem(a.C, a.dk, a.dv), s2 = simt_bwd_rev_smem(a.C, a.dk, a.dv);
    auto *k1 = simt_bwd_dq_kernel<T>;
    auto *k2 = simt_bwd_rev_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
    if (e != cudaSuccess) return e;
    k1<<<a.B * a.H, kSimtThreads, s1, st>>>((const T *)a.lf, (const T *)a.x, a.h0, (const T *)a.dO,
                                            a.dhT, (T *)a.dq, a.rs, (T *)a.dlf, (T *)a.dx, a.T, a.H, a.dk, a.dv,
                                            a.C, a.only, a.cu, a.perm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k2<<<a.B * a.H, kSimtThreads, s2, st>>>((const T *)a.q, (const T *)a.lf, (const T *)a.x,
                                            (const T *)a.dO, a.dhT, (const T *)a.dq, a.rs,
                                            (T *)a.dlf, (T *)a.dx, a.dh0, a.T, a.H, a.dk, a.dv, a.C, a.only, a.cu, a.perm);
    return cudaGetLastError();
}

cudaError_t launch_simt_bwd(const SimtBwdArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_simt_bwd_t<__nv_bfloat16>(a, st) : launch_simt_bwd_t<float>(a, st);
}

}  // namespace hgrn2
