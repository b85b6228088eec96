// tc_fwd.cu -- chunkwise HGRN2 forward on 5th-generation tensor cores (sm_100a).
//
// One CTA walks the 128-token chunks of one (batch, head) (or of one segment of
// it); d_k = d_v = 128, bf16 token tensors, fp32 state.  Per chunk, with
// E_t = prod_{r<=t} f_r (cumulative inside the chunk, per key dim j),
// k = 1 - f, S_in the state entering the chunk and E_B = E at the chunk end
// ("HGRN2: Gated Linear RNNs with State Expansion", §3.2: gated linear attention
// with key 1 - f, value i, query q, so chunkwise; §5: per-dimension decay):
//
//   Qt = q * E,  Kt = k / E,  Kh = Kt * E_B = k * E_B / E     (all bf16 in smem)
//   A  = mask_{s<=t}(Qt Kt^T)                                  tcgen05, fp32 in TMEM
//   O  = Qt bf16(S_in) + bf16(A) V                             tcgen05, fp32 in TMEM
//   S  = Diag(E_B) S_in + Kh^T V                               fp32 state in TMEM
//
// Qt Kt^T realises sum_j q_t[j] k_s[j] exp(b_t[j] - b_s[j]) through factors
// referenced to the chunk start; it is valid while 1/E stays representable with
// margin, i.e. min_j E_B[j] >= 1e-26 (a cumulative log-decay span of about 60
// inside the chunk).  A (batch, head) meeting a chunk beyond that is flagged and
// recomputed afterwards by the exact CUDA-core route, which forms every
// exponent as a difference of cumulative sums.
//
// Data movement: q, log f, i tiles arrive by TMA (128-byte swizzle, two
// 64-column boxes per 128 x 128 tile) into a two-stage ring, so the next chunk
// loads while this one computes; o leaves by TMA store.  The state never leaves
// TMEM between chunks (d_k lanes x d_v fp32 columns); Diag(E_B) is a per-lane
// scale applied with tcgen05.ld/st.  The MMAs are issued by one thread;
// completion is tracked with tcgen05.commit on mbarriers.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace hgrn2 {
namespace tcf {

using namespace tc;
using namespace tcc;

constexpr int kThreads = 256;
constexpr uint32_t kColS = 0, kColO = 128, kColA = 256, kTmemCols = 512;

struct __align__(8) Misc {
    uint64_t full[2];
    uint64_t barA, barO1, barM;
    uint32_t tmem_base;
    int bad;
    float EB[128];
    float Ppart[4][128];
};

constexpr size_t kSmemBytes = 7 * (size_t)kTileBytes + sizeof(Misc);

struct Params {
    const float *h0;
    float *hT;
    int *flags;       // [B*H] set to 1 when the (b,h) must take the exact route
    const float *Sin; // [B*H][nseg-1][128][128] state entering segments 1.. (from the scan)
    int T, H, ntiles;
    int nseg, tps;    // sequence segments per (b,h) and chunks per segment
};

__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_lf,
           const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_o, Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *Qb[2] = {smem, smem + 3 * kTileBytes};
    uint8_t *Gb[2] = {smem + kTileBytes, smem + 4 * kTileBytes};
    uint8_t *Vb[2] = {smem + 2 * kTileBytes, smem + 5 * kTileBytes};
    uint8_t *X = smem + 6 * kTileBytes;
    Misc *m = reinterpret_cast<Misc *>(smem + 7 * kTileBytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / p.nseg, seg = blockIdx.x - bh * p.nseg, b = bh / p.H, h = bh - b * p.H;
    const int g0 = seg * p.tps;                                   // first chunk of this segment
    const int N = min(p.ntiles - g0, p.tps);                      // chunks of this segment
    if (smem_u32(smem) & 1023u) {   // the swizzled operand layout needs 1024-byte alignment
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    if (tid == 0) {
        mbar_init(&m->full[0], 1);
        mbar_init(&m->full[1], 1);
        mbar_init(&m->barA, 1);
        mbar_init(&m->barO1, 1);
        mbar_init(&m->barM, 1);
        fence_mbar_init();
        m->bad = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_lf);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;

    int issued = 0, waited = 0;   // chunks whose loads were issued / whose arrival was waited for
    auto issue_load = [&](int n) {
        const int s = n & 1;
        ++issued;
        mbar_arrive_expect_tx(&m->full[s], 3 * kTileBytes);
        for (int c = 0; c < 2; ++c) {
            tma_load_4d(Qb[s] + c * kBlk, &tm_q, &m->full[s], 64 * c, h, (g0 + n) * kTile, b);
            tma_load_4d(Gb[s] + c * kBlk, &tm_lf, &m->full[s], 64 * c, h, (g0 + n) * kTile, b);
            tma_load_4d(Vb[s] + c * kBlk, &tm_x, &m->full[s], 64 * c, h, (g0 + n) * kTile, b);
        }
    };
    if (tid == 0) {
        issue_load(0);
        if (N > 1) issue_load(1);
    }

    // TMEM lane quadrant and column half of this warp
    const int quad = warp & 3, ch = warp >> 2;
    const int lrow = 32 * quad + lane;                       // TMEM lane = row of the tile
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);

    // state init: S = h0 (or 0) for the first segment, the scanned incoming state otherwise;
    // rows j = lrow, columns 64ch .. 64ch+63
    {
        float r0[32], r1[32];
        const float *init = seg == 0 ? (p.h0 ? p.h0 + (size_t)bh * 16384 : nullptr)
                                     : p.Sin + ((size_t)bh * (p.nseg - 1) + seg - 1) * 16384;
        if (init) {
            const float4 *src = reinterpret_cast<const float4 *>(init + (size_t)lrow * 128 + 64 * ch);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float4 a = src[i], c = src[8 + i];
                r0[4 * i] = a.x; r0[4 * i + 1] = a.y; r0[4 * i + 2] = a.z; r0[4 * i + 3] = a.w;
                r1[4 * i] = c.x; r1[4 * i + 1] = c.y; r1[4 * i + 2] = c.z; r1[4 * i + 3] = c.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) r0[i] = r1[i] = 0.0f;
        }
        tmem_st32(tl + kColS + 64 * ch, r0);
        tmem_st32(tl + kColS + 64 * ch + 32, r1);
        tmem_wait_st();
    }

    const uint32_t id_kk = idesc_bf16(128, 128, false, false);
    const uint32_t id_kmn = idesc_bf16(128, 128, false, true);
    const uint32_t id_mnmn = idesc_bf16(128, 128, true, true);
    const int pc = tid & 63, rr = tid >> 6;                  // prep: column pair, 32-row range
    const int col0 = 2 * pc;
    const uint32_t poff_blk = (uint32_t)(col0 >> 6) * kBlk;
    const int pchunk = (col0 & 63) >> 3, pin = (col0 & 7) * 2;
    bool ok = true;
    int n = 0;

    for (n = 0; n < N; ++n) {
        const int s = n & 1;
        if (__syncthreads_or(!mbar_wait(&m->full[s], (n >> 1) & 1))) { ok = false; break; }
        waited = n + 1;

        // ---- prep pass 1: f = exp(log f) kept in registers, partial products per 32-row range
        float f0[32], f1[32];
        float P0 = 1.0f, P1 = 1.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int t = 32 * rr + i;
            const uint32_t off = poff_blk + t * 128 + (((uint32_t)pchunk ^ (t & 7)) << 4) + pin;
            const uint32_t w = *reinterpret_cast<const uint32_t *>(Gb[s] + off);
            f0[i] = __expf(bf_lo(w));
            f1[i] = __expf(bf_hi(w));
            P0 *= f0[i];
            P1 *= f1[i];
        }
        m->Ppart[rr][col0] = P0;
        m->Ppart[rr][col0 + 1] = P1;
        __syncthreads();
        // ---- prep pass 2: Qt = q E and Kt = k / E in place
        float E0 = 1.0f, E1 = 1.0f;
        for (int r2 = 0; r2 < rr; ++r2) {
            E0 *= m->Ppart[r2][col0];
            E1 *= m->Ppart[r2][col0 + 1];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int t = 32 * rr + i;
            const uint32_t off = poff_blk + t * 128 + (((uint32_t)pchunk ^ (t & 7)) << 4) + pin;
            uint32_t *gq = reinterpret_cast<uint32_t *>(Qb[s] + off);
            uint32_t *gg = reinterpret_cast<uint32_t *>(Gb[s] + off);
            const uint32_t wa = *gg, wq = *gq;
            E0 *= f0[i];
            E1 *= f1[i];
            const float k0 = k_from(bf_lo(wa), f0[i]), k1 = k_from(bf_hi(wa), f1[i]);
            *gq = pack_bf2(bf_lo(wq) * E0, bf_hi(wq) * E1);
            *gg = pack_bf2(k0 * __fdividef(1.0f, E0), k1 * __fdividef(1.0f, E1));
        }
        if (rr == 3) {
            m->EB[col0] = E0;
            m->EB[col0 + 1] = E1;
        }
        fence_proxy_async_smem();
        const int bad = __syncthreads_or(rr == 3 && !(E0 >= kMinEB && E1 >= kMinEB));
        if (bad) break;

        // ---- A = Qt Kt^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColA, sdesc_sw128(smem_u32(Qb[s]) + ko, 16, 1024),
                            sdesc_sw128(smem_u32(Gb[s]) + ko, 16, 1024), id_kk, kk > 0);
            }
            mma_commit(&m->barA);
            tma_store_wait_read0();   // the previous chunk's o store has finished reading X
        }
        __syncthreads();

        // ---- S phase: bf16 copy of S_in into X (B operand, MN-major) and S <- Diag(E_B) S
        {
            float r0[32], r1[32];
            tc_fence_after();
            tmem_ld32(tl + kColS + 64 * ch, r0);
            tmem_ld32(tl + kColS + 64 * ch + 32, r1);
            tmem_wait_ld();
            store_row_bf16(X + ch * kBlk, lrow, r0, r1);
            const float e = m->EB[lrow];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                r0[i] *= e;
                r1[i] *= e;
            }
            tmem_st32(tl + kColS + 64 * ch, r0);
            tmem_st32(tl + kColS + 64 * ch + 32, r1);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColO, sdesc_sw128(smem_u32(Qb[s]) + ko, 16, 1024),
                            sdesc_sw128(smem_u32(X) + kk * 2048, kBlk, 1024), id_kmn, kk > 0);
            }
            mma_commit(&m->barO1);
        }

        // ---- Kh = Kt * E_B in place (after the A MMA has read Kt)
        if (!mbar_wait(&m->barA, n & 1)) ok = false;
        tc_fence_after();
        {
            const float e0 = m->EB[col0], e1 = m->EB[col0 + 1];
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                const int t = 32 * rr + i;
                const uint32_t off = poff_blk + t * 128 + (((uint32_t)pchunk ^ (t & 7)) << 4) + pin;
                uint32_t *gg = reinterpret_cast<uint32_t *>(Gb[s] + off);
                const uint32_t w = *gg;
                *gg = pack_bf2(bf_lo(w) * e0, bf_hi(w) * e1);
            }
        }
        // ---- A phase: causal mask, bf16 into X (A operand, K-major) once the inter MMA is done with X
        {
            float r0[32], r1[32];
            tmem_ld32(tl + kColA + 64 * ch, r0);
            tmem_ld32(tl + kColA + 64 * ch + 32, r1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (64 * ch + i > lrow) r0[i] = 0.0f;
                if (64 * ch + 32 + i > lrow) r1[i] = 0.0f;
            }
            if (!mbar_wait(&m->barO1, n & 1)) { ok = false; }
            store_row_bf16(X + ch * kBlk, lrow, r0, r1);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) { ok = false; break; }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColO, sdesc_sw128(smem_u32(X) + ko, 16, 1024),
                            sdesc_sw128(smem_u32(Vb[s]) + kk * 2048, kBlk, 1024), id_kmn, true);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                mma_bf16_ss(tbase + kColS, sdesc_sw128(smem_u32(Gb[s]) + kk * 2048, kBlk, 1024),
                            sdesc_sw128(smem_u32(Vb[s]) + kk * 2048, kBlk, 1024), id_mnmn, true);
            }
            mma_commit(&m->barM);
        }
        if (__syncthreads_or(!mbar_wait(&m->barM, n & 1))) { ok = false; break; }
        tc_fence_after();
        if (tid == 0 && n + 2 < N) issue_load(n + 2);

        // ---- epilogue: O (fp32 TMEM) -> bf16 -> X -> TMA store
        {
            float r0[32], r1[32];
            tmem_ld32(tl + kColO + 64 * ch, r0);
            tmem_ld32(tl + kColO + 64 * ch + 32, r1);
            tmem_wait_ld();
            store_row_bf16(X + ch * kBlk, lrow, r0, r1);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_o, X, 0, h, (g0 + n) * kTile, b);
            tma_store_4d(&tm_o, X + kBlk, 64, h, (g0 + n) * kTile, b);
            tma_store_commit();
        }
    }

    const bool fell_back = ok && n < N;
    if (!ok && tid == 0) set_status(HGRN2_ERR_TIMEOUT);
    // drain: loads still landing in this CTA's shared memory, and the last o store
    if (tid == 0) {
        for (int k = waited; k < issued; ++k) mbar_wait(&m->full[k & 1], (k >> 1) & 1, 2000000u);
        tma_store_wait_all0();
    }
    if (ok && !fell_back && p.hT && seg == p.nseg - 1) {
        tc_fence_after();
        float r0[32], r1[32];
        tmem_ld32(tl + kColS + 64 * ch, r0);
        tmem_ld32(tl + kColS + 64 * ch + 32, r1);
        tmem_wait_ld();
        float4 *dst = reinterpret_cast<float4 *>(p.hT + ((size_t)bh * 128 + lrow) * 128 + 64 * ch);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            dst[i] = make_float4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
            dst[8 + i] = make_float4(r1[4 * i], r1[4 * i + 1], r1[4 * i + 2], r1[4 * i + 3]);
        }
    }
    if (tid == 0) {
        if (p.nseg == 1) p.flags[bh] = fell_back ? 1 : 0;   // sole writer
        else if (fell_back) p.flags[bh] = 1;                  // zeroed by the aggregate kernel
        if (fell_back) atomicAdd(&g_counters[0], 1ull);
        if (ok && !fell_back) atomicAdd(&g_counters[1], (unsigned long long)N);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}


// ------------------------------------------------------------------ sequence segments
// For few (batch, head) pairs, each sequence is cut into segments of `tps` chunks run by
// separate CTAs.  The state map of a segment started from zero is affine in its incoming
// state: S_out = Diag(g) S_in + U with g = prod of the chunks' E_B and U the state the
// segment reaches from S_in = 0.  agg_kernel computes (g, U) for every segment but the
// last, scan_kernel chains them in fp32 from h0, and fwd_kernel then runs each segment
// from its incoming state.  The aggregate uses Kh = k * prod_{r>t} f_r directly
// (suffix products inside the chunk), so it is exact for any decay strength.
struct AggMisc {
    uint64_t full[2];
    uint64_t barM;
    uint32_t tmem_base;
    int pad;
    float EB[128];
    float Ppart[4][128];
};
constexpr size_t kAggSmem = 4 * (size_t)kTileBytes + sizeof(AggMisc);

struct AggParams {
    float *U, *g;     // [B*H][nseg-1][128][128], [B*H][nseg-1][128]
    int *flags;       // zeroed here (segment 0) before fwd_kernel sets exact-route flags
    int H, nseg, tps;
};

__global__ void __launch_bounds__(kThreads, 1)
agg_kernel(const __grid_constant__ CUtensorMap tm_lf, const __grid_constant__ CUtensorMap tm_x, AggParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *Gb[2] = {smem, smem + 2 * kTileBytes};
    uint8_t *Vb[2] = {smem + kTileBytes, smem + 3 * kTileBytes};
    AggMisc *m = reinterpret_cast<AggMisc *>(smem + 4 * kTileBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nagg = p.nseg - 1;
    const int bh = blockIdx.x / nagg, seg = blockIdx.x - bh * nagg, b = bh / p.H, h = bh - b * p.H;
    const int g0 = seg * p.tps, N = p.tps;   // segments before the last are full
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    if (tid == 0) {
        mbar_init(&m->full[0], 1);
        mbar_init(&m->full[1], 1);
        mbar_init(&m->barM, 1);
        fence_mbar_init();
        if (seg == 0) p.flags[bh] = 0;
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;
    int issued = 0, waited = 0;
    auto issue_load = [&](int n) {
        const int s = n & 1;
        ++issued;
        mbar_arrive_expect_tx(&m->full[s], 2 * kTileBytes);
        for (int c = 0; c < 2; ++c) {
            tma_load_4d(Gb[s] + c * kBlk, &tm_lf, &m->full[s], 64 * c, h, (g0 + n) * kTile, b);
            tma_load_4d(Vb[s] + c * kBlk, &tm_x, &m->full[s], 64 * c, h, (g0 + n) * kTile, b);
        }
    };
    if (tid == 0) {
        issue_load(0);
        if (N > 1) issue_load(1);
    }
    const int quad = warp & 3, ch = warp >> 2, lrow = 32 * quad + lane;
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
    {
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.0f;
        tmem_st32(tl + 64 * ch, z);
        tmem_st32(tl + 64 * ch + 32, z);
        tmem_wait_st();
    }
    const uint32_t id_mnmn = idesc_bf16(128, 128, true, true);
    const int pc = tid & 63, rr = tid >> 6, col0 = 2 * pc;
    const uint32_t poff_blk = (uint32_t)(col0 >> 6) * kBlk;
    const int pchunk = (col0 & 63) >> 3, pin = (col0 & 7) * 2;
    float gprod = 1.0f;   // prod of E_B over the segment, key dim lrow (threads with ch == 0)
    bool ok = true;
    for (int n = 0; n < N; ++n) {
        const int s = n & 1;
        if (__syncthreads_or(!mbar_wait(&m->full[s], (n >> 1) & 1))) { ok = false; break; }
        waited = n + 1;
        float f0[32], f1[32];
        float P0 = 1.0f, P1 = 1.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int t = 32 * rr + i;
            const uint32_t off = poff_blk + t * 128 + (((uint32_t)pchunk ^ (t & 7)) << 4) + pin;
            const uint32_t w = *reinterpret_cast<const uint32_t *>(Gb[s] + off);
            f0[i] = __expf(bf_lo(w));
            f1[i] = __expf(bf_hi(w));
            P0 *= f0[i];
            P1 *= f1[i];
        }
        m->Ppart[rr][col0] = P0;
        m->Ppart[rr][col0 + 1] = P1;
        __syncthreads();
        float S0 = 1.0f, S1 = 1.0f;   // suffix products of f after this thread's rows
        for (int r2 = rr + 1; r2 < 4; ++r2) {
            S0 *= m->Ppart[r2][col0];
            S1 *= m->Ppart[r2][col0 + 1];
        }
        if (rr == 0) {
            m->EB[col0] = S0 * P0;
            m->EB[col0 + 1] = S1 * P1;
        }
#pragma unroll
        for (int i = 31; i >= 0; --i) {
            const int t = 32 * rr + i;
            const uint32_t off = poff_blk + t * 128 + (((uint32_t)pchunk ^ (t & 7)) << 4) + pin;
            uint32_t *gg = reinterpret_cast<uint32_t *>(Gb[s] + off);
            const uint32_t wa = *gg;
            *gg = pack_bf2(k_from(bf_lo(wa), f0[i]) * S0, k_from(bf_hi(wa), f1[i]) * S1);
            S0 *= f0[i];
            S1 *= f1[i];
        }
        fence_proxy_async_smem();
        __syncthreads();
        {   // S <- Diag(E_B) S
            float r0[32], r1[32];
            tc_fence_after();
            tmem_ld32(tl + 64 * ch, r0);
            tmem_ld32(tl + 64 * ch + 32, r1);
            tmem_wait_ld();
            const float e = m->EB[lrow];
            gprod *= e;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                r0[i] *= e;
                r1[i] *= e;
            }
            tmem_st32(tl + 64 * ch, r0);
            tmem_st32(tl + 64 * ch + 32, r1);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tbase, sdesc_sw128(smem_u32(Gb[s]) + kk * 2048, kBlk, 1024),
                            sdesc_sw128(smem_u32(Vb[s]) + kk * 2048, kBlk, 1024), id_mnmn, true);
            mma_commit(&m->barM);
        }
        if (__syncthreads_or(!mbar_wait(&m->barM, n & 1))) { ok = false; break; }
        tc_fence_after();
        if (tid == 0 && n + 2 < N) issue_load(n + 2);
    }
    if (!ok && tid == 0) {
        set_status(HGRN2_ERR_TIMEOUT);
        for (int k = waited; k < issued; ++k) mbar_wait(&m->full[k & 1], (k >> 1) & 1, 2000000u);
    }
    if (ok) {
        float r0[32], r1[32];
        tmem_ld32(tl + 64 * ch, r0);
        tmem_ld32(tl + 64 * ch + 32, r1);
        tmem_wait_ld();
        const size_t slot = (size_t)bh * nagg + seg;
        float4 *dst = reinterpret_cast<float4 *>(p.U + slot * 16384 + (size_t)lrow * 128 + 64 * ch);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            dst[i] = make_float4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
            dst[8 + i] = make_float4(r1[4 * i], r1[4 * i + 1], r1[4 * i + 2], r1[4 * i + 3]);
        }
        if (ch == 0) p.g[slot * 128 + lrow] = gprod;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 128);
}

// S_in(segment 0) = h0 (or 0); S_in(seg+1) = Diag(g_seg) S_in(seg) + U_seg, in fp32, written
// over U_seg.  One thread per 4 consecutive state elements of one (batch, head).
__global__ void __launch_bounds__(256)
scan_kernel(const float *__restrict__ h0, float *__restrict__ U, const float *__restrict__ g, int nseg) {
    const int bh = blockIdx.x >> 4;
    const int e = ((blockIdx.x & 15) * 256 + threadIdx.x) * 4;   // element offset in [0, 16384)
    const int jrow = e >> 7;
    const int nagg = nseg - 1;
    float4 S = h0 ? *reinterpret_cast<const float4 *>(h0 + (size_t)bh * 16384 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sg = 0; sg < nagg; ++sg) {
        const size_t slot = (size_t)bh * nagg + sg;
        float4 *u = reinterpret_cast<float4 *>(U + slot * 16384 + e);
        const float gj = g[slot * 128 + jrow];
        const float4 uv = *u;
        S = make_float4(fmaf(gj, S.x, uv.x), fmaf(gj, S.y, uv.y), fmaf(gj, S.z, uv.z), fmaf(gj, S.w, uv.w));
        *u = S;
    }
}

}  // namespace tcf

// ------------------------------------------------------------------ host side
static_assert(tcf::kSmemBytes <= 227 * 1024, "forward shared memory");
static_assert(tcf::kAggSmem <= 227 * 1024, "aggregate shared memory");

// Segments per (b,h): enough CTAs to cover the 148 SMs of a B200 once, at most one per chunk.
void tc_fwd_segments(int B, int T, int H, int *nseg, int *tps) {
    const int ntiles = (T + tcc::kTile - 1) / tcc::kTile;
    int ns = 148 / (B * H);
    if (ns < 1) ns = 1;
    if (ns > ntiles) ns = ntiles;
    if (ns < 1) ns = 1;
    const int t = (ntiles + ns - 1) / ns;
    *tps = t < 1 ? 1 : t;
    *nseg = ntiles > 0 ? (ntiles + *tps - 1) / *tps : 1;
}

size_t tc_fwd_workspace(int B, int T, int H) {
    int nseg, tps;
    tc_fwd_segments(B, T, H, &nseg, &tps);
    return (size_t)B * H * (nseg - 1) * (16384 + 128) * sizeof(float);
}

size_t tc_fwd_smem() { return tcf::kSmemBytes; }

cudaError_t launch_tc_fwd(const TcFwdArgs &a, cudaStream_t st) {
    CUtensorMap mq, ml, mx, mo;
    if (!make_token_map(&mq, a.q, a.B, a.T, a.H) || !make_token_map(&ml, a.lf, a.B, a.T, a.H) ||
        !make_token_map(&mx, a.x, a.B, a.T, a.H) || !make_token_map(&mo, a.o, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tcf::fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tcf::kSmemBytes);
    if (e != cudaSuccess) return e;
    int nseg, tps;
    tc_fwd_segments(a.B, a.T, a.H, &nseg, &tps);
    const int ntiles = (a.T + tcc::kTile - 1) / tcc::kTile;
    const int BH = a.B * a.H;
    float *U = a.seg_ws, *g = a.seg_ws ? a.seg_ws + (size_t)BH * (nseg - 1) * 16384 : nullptr;
    if (nseg > 1) {
        e = cudaFuncSetAttribute(tcf::agg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tcf::kAggSmem);
        if (e != cudaSuccess) return e;
        tcf::AggParams ap{U, g, a.flags, a.H, nseg, tps};
        tcf::agg_kernel<<<BH * (nseg - 1), tcf::kThreads, tcf::kAggSmem, st>>>(ml, mx, ap);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        tcf::scan_kernel<<<BH * 16, 256, 0, st>>>(a.h0, U, g, nseg);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    tcf::Params p{a.h0, a.hT, a.flags, U, a.T, a.H, ntiles, nseg, tps};
    tcf::fwd_kernel<<<BH * nseg, tcf::kThreads, tcf::kSmemBytes, st>>>(mq, ml, mx, mo, p);
    return cudaGetLastError();
}

}  // namespace hgrn2
