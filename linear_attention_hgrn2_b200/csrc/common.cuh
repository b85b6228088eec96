// common.cuh -- small shared helpers of the HGRN2 CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hgrn2.h"

namespace hgrn2 {

// Device-side status word (HGRN2_OK / HGRN2_ERR_TIMEOUT / HGRN2_ERR_DEVICE) and
// diagnostic counters; read and cleared by hgrn2_get_device_status/_counters.
// (The library is a single translation unit, so these are defined here once.)
__device__ int g_status = 0;
__device__ unsigned long long g_counters[2] = {0ull, 0ull};

__device__ __forceinline__ void set_status(int s) { atomicCAS(&g_status, 0, s); }

// Packed sequences: the sequence that CTA row r runs, perm[r] (r without perm).  An entry out
// of [0, nseq) (a saved buffer that does not belong to this call) sets the status and maps to
// r, so no access leaves the caller's tensors.
__device__ __forceinline__ int packed_seq(const int *perm, int r, int nseq) {
    if (!perm) return r;
    const int s = perm[r];
    if ((unsigned)s < (unsigned)nseq) return s;
    set_status(HGRN2_ERR_DEVICE);
    return r;
}

// ---- element conversion -----------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// 1 - exp(a) for a <= 0, accurate when a is close to 0 (the tied input gate
// k = 1 - f of §2.1 with f = exp(a)).  For |a| < 0.25 it sums the Taylor series
// of -expm1(a) = -(a + a^2/2! + ... + a^9/9!) (truncation error below 1e-10
// relative); otherwise 1 - exp(a) loses no significant bits because
// exp(a) <= e^-0.25 < 0.78.
__device__ __forceinline__ float one_minus_exp(float a) {
    if (fabsf(a) < 0.25f) {
        float p = 1.0f / 362880.0f;             // 1/9!
        p = fmaf(p, a, 1.0f / 40320.0f);        // 1/8!
        p = fmaf(p, a, 1.0f / 5040.0f);
        p = fmaf(p, a, 1.0f / 720.0f);
        p = fmaf(p, a, 1.0f / 120.0f);
        p = fmaf(p, a, 1.0f / 24.0f);
        p = fmaf(p, a, 1.0f / 6.0f);
        p = fmaf(p, a, 0.5f);
        p = fmaf(p, a, 1.0f);
        return -a * p;
    }
    return 1.0f - expf(a);
}

__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

}  // namespace hgrn2
