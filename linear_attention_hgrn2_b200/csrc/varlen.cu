// varlen.cu -- launch order of packed variable-length sequences.
//
// One CTA runs one (sequence, head) pair from its first chunk to its last, and
// CTAs start in blockIdx order as SMs free up.  Launching the sequences with
// the most 128-token chunks first (longest-processing-time-first list
// scheduling) keeps a long document that happens to sit late in the packing
// from running alone at the end of the grid.  The order is a counting sort
// on the chunk count (clamped to 1023 buckets) in one CTA; sequences with the
// same count may come in any order, which changes no result: every pair's
// outputs depend on its own inputs only.

#include "common.cuh"
#include "kernels.h"

namespace hgrn2 {

namespace {

constexpr int kOrderThreads = 1024;   // one bucket per thread

__global__ void __launch_bounds__(kOrderThreads)
lpt_order_kernel(const int *__restrict__ cu, int nseq, int T, int *__restrict__ perm) {
    __shared__ int base[kOrderThreads];
    __shared__ int wsum[kOrderThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // bucket 0 = most chunks: key = 1023 - min(chunks, 1023)
    auto key = [&](int s) -> int {
        const int a = min(max(cu[s], 0), T), e = min(max(cu[s + 1], a), T);
        return kOrderThreads - 1 - min((e - a + 127) >> 7, kOrderThreads - 1);
    };
    base[tid] = 0;
    __syncthreads();
    for (int s = tid; s < nseq; s += kOrderThreads) atomicAdd(&base[key(s)], 1);
    __syncthreads();
    // exclusive prefix sum of the bucket counts: warp scans, then a scan of the warp totals
    const int v = base[tid];
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;
    }
    __syncthreads();
    base[tid] = x - v + (warp > 0 ? wsum[warp - 1] : 0);
    __syncthreads();
    for (int s = tid; s < nseq; s += kOrderThreads) perm[atomicAdd(&base[key(s)], 1)] = s;
}

}  // namespace

cudaError_t launch_lpt_order(const int *cu, int nseq, int T, int *perm, cudaStream_t st) {
    lpt_order_kernel<<<1, kOrderThreads, 0, st>>>(cu, nseq, T, perm);
    return cudaGetLastError();
}

}  // namespace hgrn2
