// step.cu -- single-token recurrent decode step of HGRN2 (bandwidth-bound).
//
// For each (batch, head), in place on the fp32 state ("HGRN2: Gated Linear RNNs
// with State Expansion", §3.2 recurrence for one token; §1 linear-time
// recurrent inference without a KV cache):
//
//   S[j,:] <- f[j] * S[j,:] + k[j] * i          (f = exp(log f), k = 1 - f)
//   o      <- S^T q                             (from the updated state)
//
// The state is read and written exactly once: 2 * d_k * d_v * 4 bytes per
// (batch, head), versus (2 d_k + 2 d_v) token elements.  One thread block per
// (batch, head); each thread owns one 16-byte column group (4 values of d_v)
// of d_k * (d_v/4) / 256 rows, issues all its 16-byte streaming loads before
// any arithmetic (so that up to 64 KB per block are in flight), and writes the
// rows back with streaming stores: the state is touched once per step and is
// larger than L2 at serving batch sizes, so it should not displace other data.
// The d_k-long dot products for o are reduced across row groups in shared
// memory.
//
// Lower-bounded gate (the kLB instantiation): the call passes the raw gate logits g
// instead of log f, and f = lb + (1 - lb) sigmoid(g) ("HGRN2", §2.2: each layer's forget
// gate is kept above a lower bound lb in [0, 1)) is formed here, with
// k = 1 - f = (1 - lb) sigmoid(-g) taken directly, so neither f nor k loses precision and
// no separate pass writes log f.
#include "common.cuh"
#include "kernels.h"

namespace hgrn2 {

constexpr int kStepThreads = 256;
constexpr int kStepMaxRows = 16;   // ceil(128 * 32 / 256): d_k <= 128, d_v <= 128

template <typename T, bool kLB>
__global__ void __launch_bounds__(kStepThreads, 2)
step_kernel(const T *__restrict__ q, const T *__restrict__ lf, const T *__restrict__ x,
            float *__restrict__ S, T *__restrict__ o, int dk, int dv, float lb) {
    __shared__ float sq[128], sf[128], sk[128];
    __shared__ float4 red[kStepThreads];
    const int bh = blockIdx.x, tid = threadIdx.x;
    const int CG = dv >> 2;                    // 16-byte column groups per row
    const int RG = kStepThreads / CG;          // row groups
    const int cg = tid % CG, rg = tid / CG;
    const bool active = rg < RG;
    float4 *Sp = reinterpret_cast<float4 *>(S + (size_t)bh * dk * dv);

    float4 r[kStepMaxRows];
#pragma unroll
    for (int i = 0; i < kStepMaxRows; ++i) {
        const int j = rg + i * RG;
        if (active && j < dk) r[i] = __ldcs(Sp + (size_t)j * CG + cg);
    }
    for (int j = tid; j < dk; j += kStepThreads) {
        const float a = to_f<T>(lf[(size_t)bh * dk + j]);
        if (kLB) {   // a = g: sigmoid(|g|) and sigmoid(-|g|) from e^{-|g|} in (0, 1]
            const float e = expf(-fabsf(a)), sp = 1.0f / (1.0f + e), sn = e * sp;
            sf[j] = lb + (1.0f - lb) * (a >= 0.0f ? sp : sn);
            sk[j] = (1.0f - lb) * (a >= 0.0f ? sn : sp);
        } else {
            sf[j] = expf(a);
            sk[j] = one_minus_exp(a);
        }
        sq[j] = to_f<T>(q[(size_t)bh * dk + j]);
    }
    float4 xv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) {
        const T *xp = x + (size_t)bh * dv + 4 * cg;
        xv = make_float4(to_f<T>(xp[0]), to_f<T>(xp[1]), to_f<T>(xp[2]), to_f<T>(xp[3]));
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kStepMaxRows; ++i) {
        const int j = rg + i * RG;
        if (active && j < dk) {
            const float f = sf[j], k = sk[j], qj = sq[j];
            float4 s = r[i];
            s.x = fmaf(f, s.x, k * xv.x);
            s.y = fmaf(f, s.y, k * xv.y);
            s.z = fmaf(f, s.z, k * xv.z);
            s.w = fmaf(f, s.w, k * xv.w);
            __stcs(Sp + (size_t)j * CG + cg, s);
            acc.x = fmaf(qj, s.x, acc.x);
            acc.y = fmaf(qj, s.y, acc.y);
            acc.z = fmaf(qj, s.z, acc.z);
            acc.w = fmaf(qj, s.w, acc.w);
        }
    }
    red[tid] = acc;
    __syncthreads();
    if (tid < CG) {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int g = 0; g < RG; ++g) {
            const float4 p = red[g * CG + tid];
            s.x += p.x; s.y += p.y; s.z += p.z; s.w += p.w;
        }
        T *op = o + (size_t)bh * dv + 4 * tid;
        op[0] = from_f<T>(s.x);
        op[1] = from_f<T>(s.y);
        op[2] = from_f<T>(s.z);
        op[3] = from_f<T>(s.w);
    }
}

template <typename T>
static void launch_step_t(const void *q, const void *lf, const void *x, float *S, void *o, int grid, int dk, int dv,
                          bool gate_lb, float lb, cudaStream_t st) {
    if (gate_lb)
        step_kernel<T, true><<<grid, kStepThreads, 0, st>>>((const T *)q, (const T *)lf, (const T *)x, S, (T *)o, dk,
                                                            dv, lb);
    else
        step_kernel<T, false><<<grid, kStepThreads, 0, st>>>((const T *)q, (const T *)lf, (const T *)x, S, (T *)o, dk,
                                                             dv, 0.0f);
}

cudaError_t launch_step(const void *q, const void *lf, const void *x, float *S, void *o, int B, int H,
                        int dk, int dv, bool bf16, bool gate_lb, float lb, cudaStream_t st) {
    const int grid = B * H;
    if (bf16)
        launch_step_t<__nv_bfloat16>(q, lf, x, S, o, grid, dk, dv, gate_lb, lb, st);
    else
        launch_step_t<float>(q, lf, x, S, o, grid, dk, dv, gate_lb, lb, st);
    return cudaGetLastError();
}

}  // namespace hgrn2
