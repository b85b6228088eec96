// seqpar.cu -- the state maps of a token slice and their scan, for running one sequence
// across several GPUs (sequence parallelism).
//
// Over a slice of tokens the recurrence ("HGRN2: Gated Linear RNNs with State
// Expansion", §3.2: S_t = Diag(f_t) S_{t-1} + k_t i_t^T with k = 1 - f; §5: one decay
// per key dimension) is affine in the state that enters the slice:
//
//   S_out = Diag(g) S_in + U,    g = prod_t f_t,    U = sum_t (k_t * prod_{r>t} f_r) i_t^T
//
// and its backward is affine in the gradient that leaves it:
//
//   dL/dS_in = Diag(g) dL/dS_out + W,    W = sum_t (q_t * prod_{r<=t} f_r) dO_t^T
//
// (W is the slice's own contribution: o_t = S_t^T q_t reads S_in through prod_{r<=t} f_r).
// So a sequence cut into slices needs, per slice, (g, U) forward and (g, W) backward;
// an exchange of these maps; and a scan of them in slice order (forward) or reverse
// slice order (backward) to get every slice's boundary state.  Then each slice runs
// the ordinary chunkwise forward / backward from its boundary states.  This is the
// state passing of the chunkwise algorithm with slices in place of chunks; the pages
// cite linear-attention sequence parallelism (LASP) for running it across devices.
//
// state_map_kernel steps the recurrence token by token on CUDA cores in fp32, in the
// same order as the plain recurrence (every product of gates is <= 1: exact for any
// decay strength).  One block per (batch, head) and block of 32 value columns; thread
// (j, half) owns 16 consecutive columns of state row j.  Tokens are staged 32 at a time.
#include "common.cuh"
#include "kernels.h"

namespace hgrn2 {
namespace sp {

constexpr int kThreads = 256;
constexpr int kCols = 32;    // value columns per block
constexpr int kTB = 32;      // tokens staged per batch

// Bwd = false: (g, U) from log f and i.  Bwd = true: (g, W) from log f, q and dO.
template <typename T, bool Bwd>
__global__ void __launch_bounds__(kThreads)
state_map_kernel(const T *__restrict__ lf, const T *__restrict__ a, const T *__restrict__ v, float *__restrict__ g,
                 float *__restrict__ M, int T_, int H, int dk, int dv) {
    __shared__ float Cs[kTB][128];      // per token and key dim: f (forward) or q * prod f (backward)
    __shared__ float Ks[kTB][128];      // forward: k = 1 - f
    __shared__ float Vs[kTB][kCols];    // i (forward) or dO (backward), this block's columns
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int c0 = blockIdx.y * kCols;
    const int tid = threadIdx.x, j = tid >> 1, col = 16 * (tid & 1);
    float S[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) S[c] = 0.0f;
    float P = 1.0f;   // staging thread tid < dk: running product of f for key dim tid
    for (int t0 = 0; t0 < T_; t0 += kTB) {
        const int nt = min(kTB, T_ - t0);
        __syncthreads();   // the previous batch has been consumed
        // stage the gate terms: threads 0..dk-1 walk the batch for their key dim in order
        if (tid < dk) {
            for (int u = 0; u < nt; ++u) {
                const size_t off = (((size_t)b * T_ + t0 + u) * H + h) * dk + tid;
                const float la = to_f<T>(lf[off]);
                const float f = __expf(la);
                if constexpr (Bwd) {
                    P *= f;
                    Cs[u][tid] = to_f<T>(a[off]) * P;
                } else {
                    Cs[u][tid] = f;
                    Ks[u][tid] = one_minus_exp(la);
                    P *= f;
                }
            }
        }
        for (int idx = tid; idx < nt * kCols; idx += kThreads) {
            const int u = idx / kCols, c = idx - u * kCols;
            Vs[u][c] = c0 + c < dv ? to_f<T>(v[(((size_t)b * T_ + t0 + u) * H + h) * dv + c0 + c]) : 0.0f;
        }
        __syncthreads();
        if (j < dk) {
            for (int u = 0; u < nt; ++u) {
                if constexpr (Bwd) {
                    const float cq = Cs[u][j];
#pragma unroll
                    for (int c = 0; c < 16; ++c) S[c] = fmaf(cq, Vs[u][col + c], S[c]);
                } else {
                    const float f = Cs[u][j], k = Ks[u][j];
#pragma unroll
                    for (int c = 0; c < 16; ++c) S[c] = fmaf(f, S[c], k * Vs[u][col + c]);
                }
            }
        }
    }
    if (j < dk) {
        float *dst = M + ((size_t)bh * dk + j) * dv;
#pragma unroll
        for (int c = 0; c < 16; ++c)
            if (c0 + col + c < dv) dst[c0 + col + c] = S[c];
    }
    if (blockIdx.y == 0 && tid < dk) g[(size_t)bh * dk + tid] = P;   // the staging thread of key dim tid
}

// S = init (or 0), then for each of `count` maps r = first, first + step, ...:
// S <- Diag(g_r) S + M_r.  g: [R][B*H][dk], M: [R][B*H][dk][dv]; S may be init.
__global__ void __launch_bounds__(256)
affine_scan_kernel(const float *__restrict__ g, const float *__restrict__ M, const float *init, float *S,
                   size_t nbh, int dk, int dv, int first, int count, int step) {
    const size_t n = nbh * dk * dv;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / dv;   // (b,h,j)
        float s = init ? init[e] : 0.0f;
        for (int k = 0, r = first; k < count; ++k, r += step)
            s = fmaf(g[(size_t)r * nbh * dk + row], s, M[(size_t)r * n + e]);
        S[e] = s;
    }
}

}  // namespace sp

template <typename T>
static cudaError_t launch_state_map_t(const StateMapArgs &a, cudaStream_t st) {
    dim3 grid(a.B * a.H, (a.dv + sp::kCols - 1) / sp::kCols);
    if (a.backward)
        sp::state_map_kernel<T, true><<<grid, sp::kThreads, 0, st>>>((const T *)a.lf, (const T *)a.q, (const T *)a.v,
                                                                    a.g, a.M, a.T, a.H, a.dk, a.dv);
    else
        sp::state_map_kernel<T, false><<<grid, sp::kThreads, 0, st>>>((const T *)a.lf, nullptr, (const T *)a.v,
                                                                     a.g, a.M, a.T, a.H, a.dk, a.dv);
    return cudaGetLastError();
}

cudaError_t launch_state_map(const StateMapArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_state_map_t<__nv_bfloat16>(a, st) : launch_state_map_t<float>(a, st);
}

cudaError_t launch_affine_scan(const float *g, const float *M, const float *init, float *S, size_t nbh, int dk, int dv,
                               int first, int count, int step, cudaStream_t st) {
    const size_t n = nbh * dk * dv;
    if (n == 0) return cudaSuccess;
    const size_t want = (n + 255) / 256;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    sp::affine_scan_kernel<<<blocks, 256, 0, st>>>(g, M, init, S, nbh, dk, dv, first, count, step);
    return cudaGetLastError();
}

}  // namespace hgrn2
