// tc_common.cuh -- device and host helpers shared by the tensor-core kernels.
#pragma once

#include <climits>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace hgrn2 {
namespace tcc {

constexpr int kTile = 128;               // tokens per chunk (one M = 128 MMA tile)
constexpr int kTileBytes = 128 * 128 * 2;
constexpr int kBlk = 128 * 128;          // bytes of one 64-column block of a 128-row tile
// Factorisation range.  Inside a chunk the decay between tokens s <= t is split as
// e^{b_t - b_s} = e^{b_t - rho} e^{rho - b_s}, with b the cumulative log decay from the chunk
// start and the reference rho = B / 2, half the chunk's total B (per key dim).  Every factor
// then lies in [e^{B/2}, e^{-B/2}], so a chunk is on the tensor cores while B / 2 >= -kMaxRefLog:
// factors stay inside e^{+-75} (bf16 / fp32 overflow at e^{88.7}; a 128-term sum of products
// of such a factor with O(1) values stays below 1e37, and values down to e^{-75} |x| stay
// normal for |x| > 5e-6).  Beyond that span (an average log f below -1.17 over a 128-token
// chunk) the pair takes the exact route.
constexpr float kMaxRefLog = 75.0f;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
// 1 - exp(a) given f = exp(a): Taylor series of -expm1 for |a| < 0.25 (relative
// truncation error < 1.5e-6), 1 - f otherwise (no cancellation there).
__device__ __forceinline__ float k_from(float a, float f) {
    if (fabsf(a) < 0.25f) {
        float p = fmaf(a, 1.0f / 120.0f, 1.0f / 24.0f);
        p = fmaf(p, a, 1.0f / 6.0f);
        p = fmaf(p, a, 0.5f);
        p = fmaf(p, a, 1.0f);
        return -a * p;
    }
    return 1.0f - f;
}

// 2^x on the FMA pipe (keeps the MUFU unit free for the other half of the exponentials).
// Range reduction x = n + f with n = rint(x), |f| <= 1/2; 2^f = e^(f ln 2) by its Taylor
// series to degree 4 (relative error < 6e-5 over the range); 2^n placed in the exponent
// field.  x is clamped to [-126, 126] (no inf/denormal results).
__device__ __forceinline__ float exp2_fma(float x) {
    x = fminf(fmaxf(x, -126.0f), 126.0f);
    const float n = rintf(x);
    const float u = (x - n) * 0.69314718056f;
    float p = fmaf(u, 1.0f / 24.0f, 1.0f / 6.0f);
    p = fmaf(p, u, 0.5f);
    p = fmaf(p, u, 1.0f);
    p = fmaf(p, u, 1.0f);
    return p * __int_as_float(((int)n + 127) << 23);
}
constexpr float kLog2e = 1.4426950408889634f;

// k = 1 - f for the prep: -expm1(a) by its Taylor series to degree 4 in a when |a| < 1/4
// (relative truncation error < 3e-5, below bf16 rounding), else 1 - f with f = E_t / E_{t-1}
// supplied by the caller as `f` (no cancellation there: f <= e^-1/4).  Branch-free.
__device__ __forceinline__ float k_gate(float a, float f) {
    float p = fmaf(a, 1.0f / 24.0f, 1.0f / 6.0f);
    p = fmaf(p, a, 0.5f);
    p = fmaf(p, a, 1.0f);
    return fabsf(a) < 0.25f ? -a * p : 1.0f - f;
}

// Row j (lane) of a 64-column half of a TMEM tile -> bf16 row in a swizzled smem block.
__device__ __forceinline__ void store_row_bf16(uint8_t *blk, int row, const float (&r0)[32], const float (&r1)[32]) {
    uint8_t *base = blk + row * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float *src = c < 4 ? &r0[c * 8] : &r1[(c - 4) * 8];
        uint4 v;
        v.x = pack_bf2(src[0], src[1]);
        v.y = pack_bf2(src[2], src[3]);
        v.z = pack_bf2(src[4], src[5]);
        v.w = pack_bf2(src[6], src[7]);
        *reinterpret_cast<uint4 *>(base + ((c ^ (row & 7)) << 4)) = v;
    }
}


__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier over `count` threads that also ORs `pred` over them: every thread of the group
// gets the same answer, so a group can leave a loop together (a thread that gave up a wait on
// its own and skipped the next barrier would leave the others waiting there for good).
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ int ld_volatile(const int *p) { return *reinterpret_cast<const volatile int *>(p); }

// Waits for phase `parity` of `bar`, or returns false early once `*bad <= tile` (the
// pipeline stopped before that phase could complete) or after a bounded number of polls.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, const int *bad, int tile) {
    for (uint32_t it = 0; it < 20000000u; ++it) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if (ld_volatile(bad) <= tile) return false;
        if (it > (1u << 20)) __nanosleep(64);
    }
    set_status(HGRN2_ERR_TIMEOUT);
    return false;
}

// One 32-column chunk (c = 0..3) of a TMEM row -> bf16 into row `row` of a swizzled 128 x 128 tile.
// dst += src over rows t of batch b, half-head hv of [B][T][Hh][128] bf16 tensors (atomically: other
// CTAs add into the same rows).
__device__ __forceinline__ void add_rows_bf16(__nv_bfloat16 *dst, const __nv_bfloat16 *src, int b, int hv, int T,
                                              int Hh) {
    for (size_t idx = threadIdx.x; idx < (size_t)T * 64; idx += blockDim.x) {
        const size_t t = idx >> 6, cp = idx & 63;
        const size_t off = (((size_t)b * T + t) * Hh + hv) * 128 + 2 * cp;
        atomicAdd(reinterpret_cast<__nv_bfloat162 *>(dst + off), *reinterpret_cast<const __nv_bfloat162 *>(src + off));
    }
}

__device__ __forceinline__ void store_chunk_bf16(uint8_t *tile, int row, int c, const float (&r)[32]) {
    uint8_t *base = tile + (c >> 1) * kBlk + row * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int chunk = 4 * (c & 1) + q;
        uint4 v;
        v.x = pack_bf2(r[8 * q + 0], r[8 * q + 1]);
        v.y = pack_bf2(r[8 * q + 2], r[8 * q + 3]);
        v.z = pack_bf2(r[8 * q + 4], r[8 * q + 5]);
        v.w = pack_bf2(r[8 * q + 6], r[8 * q + 7]);
        *reinterpret_cast<uint4 *>(base + ((chunk ^ (row & 7)) << 4)) = v;
    }
}

// bf16 element (row, col) of a 128 x 128 tile in the two-block 128-byte-swizzled layout.
__device__ __forceinline__ __nv_bfloat16 *tile_elem(uint8_t *tile, int row, int col) {
    return reinterpret_cast<__nv_bfloat16 *>(tile + tc::sw128_off(row, col, 128));
}

}  // namespace tcc

// ------------------------------------------------------------------ host side
inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D map over a [B][T][H][D] bf16 tensor (D = 128 or 64): box = 64 features x 1 head x 128 tokens
// x 1 batch, so a 128 x 128 tile takes D / 64 boxes.
inline bool make_token_map(CUtensorMap *map, const void *ptr, int B, int T, int H, int D = 128) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t row = (cuuint64_t)D * 2;   // bytes of one (token, head) row: 256 or 128
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {row, (cuuint64_t)H * row, (cuuint64_t)T * H * row};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over fp32 [rows][128] (128 x 128 state matrices one after another): box = 32 columns x
// 128 rows, 128-byte swizzle, so a matrix takes 4 boxes of 16 KB.
inline bool make_state_map(CUtensorMap *map, const float *ptr, size_t rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128 * sizeof(float)};
    cuuint32_t box[2] = {32, 128};
    cuuint32_t es[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace hgrn2
