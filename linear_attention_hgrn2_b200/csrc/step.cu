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
#include <cooperative_groups.h>

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

// Backward of one step, for L(o, S_new) with dO = dL/do and dS = dL/dS_new (null: zero), from
// the state S the step read.  Per element, with G = dS + q dO^T the whole gradient at S_new:
//
//   dq[j]      = sum_v S_new[j,v] dO[v]              (S_new recomputed from S, f, k, i)
//   dL/df[j]   = sum_v G[j,v] (S[j,v] - i[v])        (k = 1 - f moves against f)
//   di[v]      = sum_j G[j,v] k[j]
//   dS_prev    = Diag(f) G
//
// and d log f = f dL/df, or, for the lower-bounded gate, dL/dg = dL/df (1 - lb) sigmoid(g)
// sigmoid(-g).  The two d_k x d_v fp32 reads and one write dominate: 3 * 4 * d_k * d_v bytes per
// (batch, head).  A cluster of two blocks shares one (batch, head), each block half of the rows,
// so that a thread holds at most 8 rows of S and dS (16-byte column groups, all loads issued
// first) and two blocks fit on an SM: one block's loads overlap the other's arithmetic and
// stores.  Row sums stay inside a block (padded shared memory); the column sum di crosses the
// pair once, through distributed shared memory.
// dS_prev may be dS itself (each element is read before its owner thread overwrites it), so
// neither pointer is declared restrict.
constexpr int kStepBwdRows = 8;   // ceil(64 * 32 / 256): half of d_k <= 128 rows, d_v <= 128

template <typename T, bool kLB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kStepThreads, 2)
step_bwd_kernel(const T *__restrict__ q, const T *__restrict__ lf, const T *__restrict__ x,
                const float *__restrict__ S, const T *__restrict__ dO, const float *dS, float *dSp,
                T *__restrict__ dq, T *__restrict__ dlf, T *__restrict__ dx, int dk, int dv, float lb) {
    __shared__ float sq[64], sf[64], sk[64], sd[64];
    __shared__ float rows[2][64][33];   // [dq | dL/df][row][column group], padded against conflicts
    __shared__ float4 red[kStepThreads];
    __shared__ float4 peer[32];         // the other block's di partials (block 0 only)
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int bh = blockIdx.x >> 1, tid = threadIdx.x;
    const int half = (dk + 1) >> 1, j0 = rank ? half : 0, nr = rank ? dk - half : half;
    const int CG = dv >> 2, RG = kStepThreads / CG;
    const int cg = tid % CG, rg = tid / CG;
    const bool active = rg < RG;
    const size_t so = ((size_t)bh * dk + j0) * dv;
    const float4 *Sp = reinterpret_cast<const float4 *>(S + so);
    const float4 *Dp = dS ? reinterpret_cast<const float4 *>(dS + so) : nullptr;
    float4 *Pp = dSp ? reinterpret_cast<float4 *>(dSp + so) : nullptr;

    float4 r[kStepBwdRows], d[kStepBwdRows];
#pragma unroll
    for (int i = 0; i < kStepBwdRows; ++i) {
        const int j = rg + i * RG;
        if (active && j < nr) {
            r[i] = __ldcs(Sp + (size_t)j * CG + cg);
            d[i] = Dp ? __ldcs(Dp + (size_t)j * CG + cg) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    const size_t vo = (size_t)bh * dk + j0;   // this block's first row in the [B,H,dk] vectors
    for (int j = tid; j < nr; j += kStepThreads) {
        const float a = to_f<T>(lf[vo + j]);
        if (kLB) {   // a = g; sp = sigmoid(|g|), sn = sigmoid(-|g|)
            const float e = expf(-fabsf(a)), sp = 1.0f / (1.0f + e), sn = e * sp;
            sf[j] = lb + (1.0f - lb) * (a >= 0.0f ? sp : sn);
            sk[j] = (1.0f - lb) * (a >= 0.0f ? sn : sp);
            sd[j] = (1.0f - lb) * sp * sn;   // df/dg
        } else {
            const float f = expf(a);
            sf[j] = f;
            sk[j] = one_minus_exp(a);
            sd[j] = f;                       // df/dlog f
        }
        sq[j] = to_f<T>(q[vo + j]);
    }
    float4 xv = make_float4(0.f, 0.f, 0.f, 0.f), gv = xv;
    if (active) {
        const T *xp = x + (size_t)bh * dv + 4 * cg, *gp = dO + (size_t)bh * dv + 4 * cg;
        xv = make_float4(to_f<T>(xp[0]), to_f<T>(xp[1]), to_f<T>(xp[2]), to_f<T>(xp[3]));
        gv = make_float4(to_f<T>(gp[0]), to_f<T>(gp[1]), to_f<T>(gp[2]), to_f<T>(gp[3]));
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);   // di partial over this thread's rows
#pragma unroll
    for (int i = 0; i < kStepBwdRows; ++i) {
        const int j = rg + i * RG;
        if (active && j < nr) {
            const float f = sf[j], k = sk[j], qj = sq[j];
            const float4 s = r[i];
            float4 G = d[i];
            G.x = fmaf(qj, gv.x, G.x);
            G.y = fmaf(qj, gv.y, G.y);
            G.z = fmaf(qj, gv.z, G.z);
            G.w = fmaf(qj, gv.w, G.w);
            const float pq = fmaf(f, s.x, k * xv.x) * gv.x + fmaf(f, s.y, k * xv.y) * gv.y +
                             fmaf(f, s.z, k * xv.z) * gv.z + fmaf(f, s.w, k * xv.w) * gv.w;
            const float pf = G.x * (s.x - xv.x) + G.y * (s.y - xv.y) + G.z * (s.z - xv.z) + G.w * (s.w - xv.w);
            acc.x = fmaf(G.x, k, acc.x);
            acc.y = fmaf(G.y, k, acc.y);
            acc.z = fmaf(G.z, k, acc.z);
            acc.w = fmaf(G.w, k, acc.w);
            if (Pp) __stcs(Pp + (size_t)j * CG + cg, make_float4(f * G.x, f * G.y, f * G.z, f * G.w));
            rows[0][j][cg] = pq;
            rows[1][j][cg] = pf;
        }
    }
    red[tid] = acc;
    __syncthreads();
    for (int t = tid; t < 2 * nr; t += kStepThreads) {
        const int w = t >= nr, j = t - w * nr;
        float sum = 0.0f;
        for (int c = 0; c < CG; ++c) sum += rows[w][j][c];
        if (w == 0)
            dq[vo + j] = from_f<T>(sum);
        else
            dlf[vo + j] = from_f<T>(sum * sd[j]);
    }
    float4 part = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < CG) {
        for (int g = 0; g < RG; ++g) {
            const float4 p = red[g * CG + tid];
            part.x += p.x; part.y += p.y; part.z += p.z; part.w += p.w;
        }
        if (rank == 1) cluster.map_shared_rank(peer, 0)[tid] = part;
    }
    cluster.sync();   // block 1's partials are in block 0's shared memory
    if (rank == 0 && tid < CG) {
        const float4 p = peer[tid];
        T *op = dx + (size_t)bh * dv + 4 * tid;
        op[0] = from_f<T>(part.x + p.x);
        op[1] = from_f<T>(part.y + p.y);
        op[2] = from_f<T>(part.z + p.z);
        op[3] = from_f<T>(part.w + p.w);
    }
}

template <typename T>
static void launch_step_bwd_t(const StepBwdArgs &a, int grid, cudaStream_t st) {
    if (a.gate_lb)
        step_bwd_kernel<T, true><<<grid, kStepThreads, 0, st>>>(
            (const T *)a.q, (const T *)a.lf, (const T *)a.x, a.S, (const T *)a.dO, a.dS, a.dS_prev, (T *)a.dq,
            (T *)a.dlf, (T *)a.dx, a.dk, a.dv, a.lb);
    else
        step_bwd_kernel<T, false><<<grid, kStepThreads, 0, st>>>(
            (const T *)a.q, (const T *)a.lf, (const T *)a.x, a.S, (const T *)a.dO, a.dS, a.dS_prev, (T *)a.dq,
            (T *)a.dlf, (T *)a.dx, a.dk, a.dv, 0.0f);
}

cudaError_t launch_step_bwd(const StepBwdArgs &a, bool bf16, cudaStream_t st) {
    const int grid = 2 * a.B * a.H;   // a cluster of two blocks per (batch, head)
    if (bf16)
        launch_step_bwd_t<__nv_bfloat16>(a, grid, st);
    else
        launch_step_bwd_t<float>(a, grid, st);
    return cudaGetLastError();
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
