// wide.cu -- heads wider than 128 (d_k, d_v <= 256) as blocks of the 128-wide path.
//
// Diag(f_t) acts on each key dim alone and the update k_t i_t^T on each value column alone, so
// with the key dims cut into blocks a and the value dims into blocks c, each state block
// S[a, c] is a recurrence of its own ("HGRN2: Gated Linear RNNs with State Expansion", §3.2
// outer-product state; §5 one decay per key dim):
//
//   S_t[a,c] = Diag(f_t[a]) S_{t-1}[a,c] + k_t[a] i_t[c]^T,     o_t[c] = sum_a S_t[a,c]^T q_t[a].
//
// Gradients split the same way: dq[a] and d log f[a] sum over c, di[c] over a, and dh0[a,c]
// comes from block (a,c) alone.  These kernels move state blocks between the full tensors and
// contiguous scratch, and add the partial outputs of the blocks in fp32.
#include "common.cuh"
#include "kernels.h"

namespace hgrn2 {
namespace {

constexpr int kWideThreads = 256;

// full [nmat][dk][dv] fp32, block rows ro .. ro+rw-1 and columns co .. co+cw-1, against the
// rw x cw matrices of blk, `bstride` elements apart; to_full = 1 writes the block into full, 0
// reads it out.
__global__ void __launch_bounds__(kWideThreads)
state_block_kernel(float *__restrict__ full, float *__restrict__ blk, size_t bstride, size_t nmat, int dk, int dv,
                   int ro, int rw, int co, int cw, int to_full) {
    const size_t n = nmat * rw * cw;
    for (size_t e = blockIdx.x * (size_t)kWideThreads + threadIdx.x; e < n; e += (size_t)gridDim.x * kWideThreads) {
        const size_t m = e / ((size_t)rw * cw), in = e - m * rw * cw;
        const int r = (int)(in / cw), c = (int)(in % cw);
        float *f = full + (m * dk + ro + r) * dv + co + c;
        float *b = blk + m * bstride + in;
        if (to_full) *f = *b;
        else *b = *f;
    }
}

// dst[r][off + c] = p0[r][c] + p1[r][c] (p1 null: p0 alone) for r < rows, c < w, added in fp32
// and rounded once; dst rows are `pitch` elements apart, p0 and p1 rows `spitch` apart.
template <typename T>
__global__ void __launch_bounds__(kWideThreads)
sum_blocks_kernel(T *__restrict__ dst, int pitch, int off, const T *__restrict__ p0, const T *__restrict__ p1,
                  int spitch, size_t rows, int w) {
    const size_t n = rows * w;
    for (size_t e = blockIdx.x * (size_t)kWideThreads + threadIdx.x; e < n; e += (size_t)gridDim.x * kWideThreads) {
        const size_t r = e / w;
        const int c = (int)(e - r * w);
        const size_t si = r * spitch + c;
        float v = to_f<T>(p0[si]);
        if (p1) v += to_f<T>(p1[si]);
        dst[r * pitch + off + c] = from_f<T>(v);
    }
}

int wide_grid(size_t n) {
    const size_t b = (n + kWideThreads - 1) / kWideThreads, cap = 148 * 8;
    return (int)(b < 1 ? 1 : b > cap ? cap : b);
}

}  // namespace

cudaError_t launch_state_block(float *full, float *blk, size_t bstride, size_t nmat, int dk, int dv, int ro, int rw,
                               int co, int cw, bool to_full, cudaStream_t st) {
    const size_t n = nmat * rw * cw;
    if (n == 0) return cudaSuccess;
    state_block_kernel<<<wide_grid(n), kWideThreads, 0, st>>>(full, blk, bstride, nmat, dk, dv, ro, rw, co, cw,
                                                              to_full ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_sum_blocks(void *dst, int pitch, int off, const void *p0, const void *p1, int spitch, size_t rows,
                              int w, bool bf16, cudaStream_t st) {
    const size_t n = rows * w;
    if (n == 0) return cudaSuccess;
    if (bf16)
        sum_blocks_kernel<__nv_bfloat16><<<wide_grid(n), kWideThreads, 0, st>>>(
            (__nv_bfloat16 *)dst, pitch, off, (const __nv_bfloat16 *)p0, (const __nv_bfloat16 *)p1, spitch, rows, w);
    else
        sum_blocks_kernel<float><<<wide_grid(n), kWideThreads, 0, st>>>(
            (float *)dst, pitch, off, (const float *)p0, (const float *)p1, spitch, rows, w);
    return cudaGetLastError();
}

}  // namespace hgrn2
