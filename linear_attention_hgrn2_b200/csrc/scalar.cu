// scalar.cu -- the scalar-decay variant on CUDA cores (fp32 arithmetic).
//
// One decay per head and token and a key of its own (the per-head decay of models such
// as Mamba2 and RetNet, which "HGRN2: Gated Linear RNNs with State Expansion", §5,
// contrasts with its per-dimension decay):
//
//   S_t = g_t S_{t-1} + k_t v_t^T,      o_t = S_t^T q_t,      g_t = exp(log_g_t)
//
// With a decay shared by every key dim the chunkwise form factors exactly: inside a chunk
// with b_t = sum_{r<=t} log g_r (from the chunk start) and B = b at its last token,
//
//   o_t   = e^{b_t} q_t^T S_in + sum_{s<=t} e^{b_t - b_s} (q_t . k_s) v_s
//   S_out = e^{B} S_in + sum_s e^{B - b_s} k_s v_s^T
//
// and every exponent is <= 0 for log g <= 0, so no decay strength needs another route.
// Backward, per chunk with dS = dL/dS_out:
//
//   dq_t   = e^{b_t} S_in dO_t + sum_{s<=t} e^{b_t - b_s} (dO_t . v_s) k_s   (forward sweep)
//   dk_s   = sum_{t>=s} e^{b_t - b_s} (dO_t . v_s) q_t + e^{B - b_s} dS v_s
//   dv_s   = sum_{t>=s} e^{b_t - b_s} (q_t . k_s) dO_t + e^{B - b_s} dS^T k_s
//   dS_in  = e^{B} dS + sum_t e^{b_t} q_t dO_t^T
//   dlog g_t = sum_{t'>=t} (q_t' . dq_t' - k_t' . dk_t') + <dhT, hT>      (reverse sweep)
//
// The last line follows from o and hT being homogeneous in the decays; it runs as a reverse
// cumulative sum across chunks.  One thread block walks the chunks of one (batch, head); the
// state (or its gradient) stays in shared memory in fp32.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace hgrn2 {

namespace sd {

constexpr int kThreads = 256;
constexpr int kC = 32;   // tokens per chunk

// log g row of one (b, h): one value per token, [B][T][H]
__device__ __forceinline__ size_t gidx(int b, int t, int h, int T_, int H) {
    return ((size_t)b * T_ + t) * H + h;
}
__device__ __forceinline__ size_t tidx(int b, int t, int h, int T_, int H, int D) {
    return (((size_t)b * T_ + t) * H + h) * D;
}

// Loads rows t0 .. t0+kC-1 of one (b,h) of a [B][T][H][D] tensor into smem (row stride ld),
// zero past the end of the sequence.
template <typename T>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *src, int b, int h, int t0, int n, int T_,
                                          int H, int D) {
    for (int e = threadIdx.x; e < kC * D; e += blockDim.x) {
        const int t = e / D, j = e - t * D;
        dst[t * ld + j] = t < n ? to_f<T>(src[tidx(b, t0 + t, h, T_, H, D) + j]) : 0.0f;
    }
}

// Warp 0: b_t = inclusive cumsum of log g over the chunk (0 past its end, so b stays at the
// last token's value), e_t = e^{b_t}, w_t = e^{B - b_t}.
template <typename T>
__device__ __forceinline__ void gate_prefix(float *bs, float *es, float *ws, const T *lg, int b, int h, int t0,
                                            int n, int T_, int H) {
    if (threadIdx.x < 32) {
        const int t = threadIdx.x;
        float a = t < n ? to_f<T>(lg[gidx(b, t0 + t, h, T_, H)]) : 0.0f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, a, o);
            if (t >= o) a += y;
        }
        const float Bt = __shfl_sync(0xffffffffu, a, 31);
        bs[t] = a;
        es[t] = expf(a);
        ws[t] = expf(Bt - a);
    }
}

// M[t][s] = s <= t ? (X_t . Y_s) e^{b_t - b_s} : 0, for the chunk's kC x kC pairs.
__device__ __forceinline__ void decay_scores(float *M, const float *X, const float *Y, int ld, int D,
                                             const float *bs) {
    for (int e = threadIdx.x; e < kC * kC; e += blockDim.x) {
        const int t = e / kC, s = e - t * kC;
        float acc = 0.0f;
        if (s <= t) {
            for (int j = 0; j < D; ++j) acc = fmaf(X[t * ld + j], Y[s * ld + j], acc);
            acc *= expf(bs[t] - bs[s]);
        }
        M[t * (kC + 1) + s] = acc;
    }
}

constexpr size_t fwd_smem(int dk, int dv) {
    return sizeof(float) * ((size_t)dk * (dv + 1) + 2 * kC * (dk + 1) + kC * (dv + 1) + kC * (kC + 1) + 3 * kC);
}
size_t dq_smem(int dk, int dv) {
    return sizeof(float) * ((size_t)dk * (dv + 1) + 2 * kC * (dk + 1) + 2 * kC * (dv + 1) + kC * (kC + 1) + 4 * kC);
}
size_t rev_smem(int dk, int dv) {
    return sizeof(float) * ((size_t)dk * (dv + 1) + 3 * kC * (dk + 1) + 2 * kC * (dv + 1) + 2 * kC * (kC + 1) +
                            5 * kC);
}

// The forward of one (b, h) by the whole thread block (any multiple of 32 threads), in the shared
// memory at sm (fwd_smem bytes).  Kept out of line: the tensor-core forward calls it only for the
// pairs whose chunk decay leaves its factorised form's range.
template <typename T>
__device__ __noinline__ void fwd_body(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                                      const T *__restrict__ lg, const float *__restrict__ h0, T *__restrict__ o,
                                      float *__restrict__ hT, int T_, int H, int dk, int dv, float *sm, int b, int h,
                                      int bh) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lds = dv + 1, ldk = dk + 1, ldv = dv + 1, lda = kC + 1;
    float *S = sm, *Qs = S + dk * lds, *Ks = Qs + kC * ldk, *Vs = Ks + kC * ldk, *A = Vs + kC * ldv;
    float *bs = A + kC * lda, *es = bs + kC, *ws = es + kC;
    const size_t so = (size_t)bh * dk * dv;
    for (int e = tid; e < dk * dv; e += nt) S[(e / dv) * lds + e % dv] = h0 ? h0[so + e] : 0.0f;
    for (int t0 = 0; t0 < T_; t0 += kC) {
        const int n = min(kC, T_ - t0);
        __syncthreads();   // the previous chunk is done with every tile
        load_rows<T>(Qs, ldk, q, b, h, t0, n, T_, H, dk);
        load_rows<T>(Ks, ldk, k, b, h, t0, n, T_, H, dk);
        load_rows<T>(Vs, ldv, v, b, h, t0, n, T_, H, dv);
        gate_prefix<T>(bs, es, ws, lg, b, h, t0, n, T_, H);
        __syncthreads();
        decay_scores(A, Qs, Ks, ldk, dk, bs);
        __syncthreads();
        for (int e = tid; e < n * dv; e += nt) {   // o_t (reads S_in)
            const int t = e / dv, c = e - t * dv;
            float inter = 0.0f, intra = 0.0f;
            for (int j = 0; j < dk; ++j) inter = fmaf(Qs[t * ldk + j], S[j * lds + c], inter);
            for (int s = 0; s <= t; ++s) intra = fmaf(A[t * lda + s], Vs[s * ldv + c], intra);
            o[tidx(b, t0 + t, h, T_, H, dv) + c] = from_f<T>(fmaf(es[t], inter, intra));
        }
        __syncthreads();
        const float eB = es[kC - 1];
        for (int e = tid; e < dk * dv; e += nt) {   // S_out
            const int j = e / dv, c = e - j * dv;
            float acc = 0.0f;
            for (int s = 0; s < n; ++s) acc = fmaf(ws[s] * Ks[s * ldk + j], Vs[s * ldv + c], acc);
            S[j * lds + c] = fmaf(eB, S[j * lds + c], acc);
        }
    }
    __syncthreads();
    if (hT)
        for (int e = tid; e < dk * dv; e += nt) hT[so + e] = S[(e / dv) * lds + e % dv];
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
fwd_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ lg,
           const float *__restrict__ h0, T *__restrict__ o, float *__restrict__ hT, int T_, int H, int dk, int dv) {
    extern __shared__ float sm[];
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    fwd_body<T>(q, k, v, lg, h0, o, hT, T_, H, dk, dv, sm, b, h, bh);
}

// Forward sweep of the backward: dq of every token, q_t . dq_t in fp32 (for the reverse sweep's
// d log g, so that it does not read back the rounded dq), and rs = <dhT, hT>.
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_dq_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ lg,
              const float *__restrict__ h0, const T *__restrict__ dO, const float *__restrict__ dhT,
              T *__restrict__ dq, float *__restrict__ qdq, float *__restrict__ rs, int T_, int H, int dk, int dv,
              const int *only) {
    if (only && only[blockIdx.x] == 0) return;   // only the pairs the tensor-core route flagged
    extern __shared__ float sm[];
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H, tid = threadIdx.x;
    const int lds = dv + 1, ldk = dk + 1, ldv = dv + 1, lda = kC + 1;
    float *S = sm, *Ks = S + dk * lds, *Vs = Ks + kC * ldk, *Gs = Vs + kC * ldv, *dA = Gs + kC * ldv;
    float *bs = dA + kC * lda, *es = bs + kC, *ws = es + kC, *Qs = ws + kC;
    const size_t so = (size_t)bh * dk * dv;
    for (int e = tid; e < dk * dv; e += kThreads) S[(e / dv) * lds + e % dv] = h0 ? h0[so + e] : 0.0f;
    for (int t0 = 0; t0 < T_; t0 += kC) {
        const int n = min(kC, T_ - t0);
        __syncthreads();
        load_rows<T>(Qs, ldk, q, b, h, t0, n, T_, H, dk);
        load_rows<T>(Ks, ldk, k, b, h, t0, n, T_, H, dk);
        load_rows<T>(Vs, ldv, v, b, h, t0, n, T_, H, dv);
        load_rows<T>(Gs, ldv, dO, b, h, t0, n, T_, H, dv);
        gate_prefix<T>(bs, es, ws, lg, b, h, t0, n, T_, H);
        __syncthreads();
        decay_scores(dA, Gs, Vs, ldv, dv, bs);
        __syncthreads();
        for (int e = tid; e < n * dk; e += kThreads) {   // dq_t (reads S_in)
            const int t = e / dk, j = e - t * dk;
            float inter = 0.0f, intra = 0.0f;
            for (int c = 0; c < dv; ++c) inter = fmaf(Gs[t * ldv + c], S[j * lds + c], inter);
            for (int s = 0; s <= t; ++s) intra = fmaf(dA[t * lda + s], Ks[s * ldk + j], intra);
            const float g = fmaf(es[t], inter, intra);
            dq[tidx(b, t0 + t, h, T_, H, dk) + j] = from_f<T>(g);
            Qs[t * ldk + j] *= g;   // q dq per element (nothing else reads Qs in this phase)
        }
        __syncthreads();
        if (tid < n) {   // q_t . dq_t, summed in a fixed order
            float acc = 0.0f;
            for (int j = 0; j < dk; ++j) acc += Qs[tid * ldk + j];
            qdq[gidx(b, t0 + tid, h, T_, H)] = acc;
        }
        const float eB = es[kC - 1];
        for (int e = tid; e < dk * dv; e += kThreads) {
            const int j = e / dv, c = e - j * dv;
            float acc = 0.0f;
            for (int s = 0; s < n; ++s) acc = fmaf(ws[s] * Ks[s * ldk + j], Vs[s * ldv + c], acc);
            S[j * lds + c] = fmaf(eB, S[j * lds + c], acc);
        }
    }
    __syncthreads();
    // rs = <dhT, hT>: per-thread partial sums, then a block reduction through shared memory
    float part = 0.0f;
    if (dhT)
        for (int e = tid; e < dk * dv; e += kThreads) part = fmaf(dhT[so + e], S[(e / dv) * lds + e % dv], part);
    __syncthreads();
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) sm[tid >> 5] = part;
    __syncthreads();
    if (tid == 0) {
        float tot = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) tot += sm[w];
        rs[bh] = tot;
    }
}

// Reverse sweep: dk, dv, dlog g and dh0, chunks from last to first.
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_rev_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ lg,
               const T *__restrict__ dO, const float *__restrict__ dhT, const T *__restrict__ dq,
               const float *__restrict__ qdq, const float *__restrict__ rs, T *__restrict__ dk_out,
               T *__restrict__ dv_out,
               T *__restrict__ dlg, float *__restrict__ dh0, int T_, int H, int dk, int dv, const int *only) {
    if (only && only[blockIdx.x] == 0) return;
    extern __shared__ float sm[];
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H, tid = threadIdx.x;
    const int lds = dv + 1, ldk = dk + 1, ldv = dv + 1, lda = kC + 1;
    float *dS = sm, *Qs = dS + dk * lds, *Ks = Qs + kC * ldk, *DK = Ks + kC * ldk, *Vs = DK + kC * ldk;
    float *Gs = Vs + kC * ldv, *A = Gs + kC * ldv, *dA = A + kC * lda;
    float *bs = dA + kC * lda, *es = bs + kC, *ws = es + kC, *term = ws + kC, *misc = term + kC;
    const size_t so = (size_t)bh * dk * dv;
    for (int e = tid; e < dk * dv; e += kThreads) dS[(e / dv) * lds + e % dv] = dhT ? dhT[so + e] : 0.0f;
    if (tid == 0) misc[0] = dhT ? rs[bh] : 0.0f;   // carry of the reverse cumulative sum
    const int nch = (T_ + kC - 1) / kC;
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int t0 = ci * kC, n = min(kC, T_ - t0);
        __syncthreads();
        load_rows<T>(Qs, ldk, q, b, h, t0, n, T_, H, dk);
        load_rows<T>(Ks, ldk, k, b, h, t0, n, T_, H, dk);
        load_rows<T>(Vs, ldv, v, b, h, t0, n, T_, H, dv);
        load_rows<T>(Gs, ldv, dO, b, h, t0, n, T_, H, dv);
        gate_prefix<T>(bs, es, ws, lg, b, h, t0, n, T_, H);
        __syncthreads();
        decay_scores(A, Qs, Ks, ldk, dk, bs);
        decay_scores(dA, Gs, Vs, ldv, dv, bs);
        __syncthreads();
        for (int e = tid; e < n * dk; e += kThreads) {   // dk_s (reads dS = dL/dS_out)
            const int s = e / dk, j = e - s * dk;
            float intra = 0.0f, inter = 0.0f;
            for (int t = s; t < n; ++t) intra = fmaf(dA[t * lda + s], Qs[t * ldk + j], intra);
            for (int c = 0; c < dv; ++c) inter = fmaf(dS[j * lds + c], Vs[s * ldv + c], inter);
            const float g = fmaf(ws[s], inter, intra);
            DK[s * ldk + j] = g;
            dk_out[tidx(b, t0 + s, h, T_, H, dk) + j] = from_f<T>(g);
        }
        for (int e = tid; e < n * dv; e += kThreads) {   // dv_s
            const int s = e / dv, c = e - s * dv;
            float intra = 0.0f, inter = 0.0f;
            for (int t = s; t < n; ++t) intra = fmaf(A[t * lda + s], Gs[t * ldv + c], intra);
            for (int j = 0; j < dk; ++j) inter = fmaf(dS[j * lds + c], Ks[s * ldk + j], inter);
            dv_out[tidx(b, t0 + s, h, T_, H, dv) + c] = from_f<T>(fmaf(ws[s], inter, intra));
        }
        __syncthreads();
        if (tid < kC) {   // q_t . dq_t - k_t . dk_t
            const int t = tid;
            float acc = 0.0f;
            if (t < n) {
                if (std::is_same<T, float>::value) {   // dq is exact: pair the terms element by element
                    const size_t r = tidx(b, t0 + t, h, T_, H, dk);
                    for (int j = 0; j < dk; ++j)
                        acc += Qs[t * ldk + j] * to_f<T>(dq[r + j]) - Ks[t * ldk + j] * DK[t * ldk + j];
                } else {   // dq was rounded to bf16: q . dq from the forward sweep's fp32 sum
                    acc = qdq[gidx(b, t0 + t, h, T_, H)];
                    for (int j = 0; j < dk; ++j) acc -= Ks[t * ldk + j] * DK[t * ldk + j];
                }
            }
            term[t] = acc;
        }
        const float eB = es[kC - 1];
        for (int e = tid; e < dk * dv; e += kThreads) {   // dS_in
            const int j = e / dv, c = e - j * dv;
            float acc = 0.0f;
            for (int t = 0; t < n; ++t) acc = fmaf(es[t] * Qs[t * ldk + j], Gs[t * ldv + c], acc);
            dS[j * lds + c] = fmaf(eB, dS[j * lds + c], acc);
        }
        __syncthreads();
        if (tid < 32) {   // dlog g_t = suffix sum of term from t + carry (warp 0)
            const int t = tid;
            float a = term[kC - 1 - t];   // reversed, so a prefix sum gives the suffix sums
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, a, o);
                if (t >= o) a += y;
            }
            const float carry = misc[0];
            const int tt = kC - 1 - t;   // the token this lane's suffix sum starts at
            if (tt < n) dlg[gidx(b, t0 + tt, h, T_, H)] = from_f<T>(a + carry);
            const float tot = __shfl_sync(0xffffffffu, a, 31);
            __syncwarp();
            if (t == 0) misc[0] = carry + tot;
        }
    }
    __syncthreads();
    if (dh0)
        for (int e = tid; e < dk * dv; e += kThreads) dh0[so + e] = dS[(e / dv) * lds + e % dv];
}

}  // namespace sd

template <typename T>
static cudaError_t launch_sd_fwd_t(const ScalarArgs &a, cudaStream_t st) {
    const size_t smem = sd::fwd_smem(a.dk, a.dv);
    cudaError_t e = cudaFuncSetAttribute(sd::fwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sd::fwd_kernel<T><<<a.B * a.H, sd::kThreads, smem, st>>>((const T *)a.q, (const T *)a.k, (const T *)a.v,
                                                              (const T *)a.lg, a.h0, (T *)a.o, a.hT, a.T, a.H,
                                                              a.dk, a.dv);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_sd_bwd_t(const ScalarArgs &a, cudaStream_t st) {
    const size_t s1 = sd::dq_smem(a.dk, a.dv), s2 = sd::rev_smem(a.dk, a.dv);
    cudaError_t e = cudaFuncSetAttribute(sd::bwd_dq_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(sd::bwd_rev_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
    if (e != cudaSuccess) return e;
    sd::bwd_dq_kernel<T><<<a.B * a.H, sd::kThreads, s1, st>>>((const T *)a.q, (const T *)a.k, (const T *)a.v,
                                                               (const T *)a.lg, a.h0, (const T *)a.dO, a.dhT,
                                                               (T *)a.dq, a.qdq, a.rs, a.T, a.H, a.dk, a.dv, a.only);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sd::bwd_rev_kernel<T><<<a.B * a.H, sd::kThreads, s2, st>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.lg, (const T *)a.dO, a.dhT, (const T *)a.dq,
        a.qdq, a.rs, (T *)a.dk_out, (T *)a.dv_out, (T *)a.dlg, a.dh0, a.T, a.H, a.dk, a.dv, a.only);
    return cudaGetLastError();
}

cudaError_t launch_scalar_fwd(const ScalarArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_sd_fwd_t<__nv_bfloat16>(a, st) : launch_sd_fwd_t<float>(a, st);
}
cudaError_t launch_scalar_bwd(const ScalarArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_sd_bwd_t<__nv_bfloat16>(a, st) : launch_sd_bwd_t<float>(a, st);
}

}  // namespace hgrn2
