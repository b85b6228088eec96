// tc_bwd.cu -- chunkwise HGRN2 backward on 5th-generation tensor cores (sm_100a).
//
// Two sweeps per (batch, head), d_k = d_v = 128, bf16 token tensors, 128-token
// chunks, same factorisation as the forward: with b the cumulative log decay from
// the chunk start, B its chunk total and the balanced reference rho = B / 2 (per key
// dim), E_t = e^{b_t - rho}, Qt = q E, Kt = k / E, and H = e^{B - rho} = e^{rho} the
// scale of the state on either side of the chunk's MMAs (S_r = H S_in before them,
// S_out = H S' after them).
//
// Forward sweep (dq_kernel): the fp32 state is recomputed in TMEM and
//   dq = E * (dO S_r^T + mask(dO V^T) Kt)                                  (1)
// is formed transposed (TMEM lane = key dim j, column = token t), so the
// decay factor E[j][t] that finishes it sits in the same thread's lane.  The
// MMA accumulates S' = S_r + Kt^T V, and the next chunk multiplies its rows by
// both state scales before using it.  At the end it writes rowsum(dhT * hT) for
// the reverse sweep's carry.
//
// Reverse sweep (rev_kernel), chunks last to first, dS = dL/dS_out in TMEM:
//   dSh  = Diag(H) dS                                     (also the new dS)
//   di   = mask(A)^T dO + Kt dSh                            A = Qt Kt^T
//   dk^T = (Qt^T mask(dO V^T) + dSh V^T) / E               (lane j, column s)
//   dS   = Diag(H) (dSh + Qt^T dO)                          (dL/dS_in; the scale is
//                                                            applied with the next dSh)
//   dlog f_t = sum_{t'>=t} (q dq - k dk)_{t'} + rowsum(dhT hT) - f_t dk_t
// The last line is the gradient through both the decay and the tied input gate
// k = 1 - f ("HGRN2: Gated Linear RNNs with State Expansion", §2.1 tied gate,
// §3.2 outer-product state, §5 per-dimension decay); its reverse cumulative sum
// runs inside the chunk per key dim (thread-local, lane = j) and across chunks
// through a carry.  q, log f and dq for that line are read back from global
// memory (they were just streamed through L2) so that the next chunk's TMA
// load can start as soon as the MMAs are done.
//
// Validity and fallback are those of the forward: a (batch, head) whose chunk
// decay span exceeds the factorisation's range is flagged by the forward sweep,
// skipped by the reverse sweep, and recomputed by the exact route.
#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace hgrn2 {
namespace tcb {

using namespace tc;
using namespace tcc;

constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ void st_bar_expect(uint64_t *bar, uint32_t bytes) { mbar_arrive_expect_tx(bar, bytes); }

// ------------------------------------------------------------------ forward sweep: dq
// Warp roles (16 warps), coordinated by mbarriers:
//   warp 0      TMA producer: log f, i, dO tiles into a 2-stage ring
//   warp 1      TMEM allocator, MMA thread: dA = dO V^T as soon as a chunk lands, then
//               dq_pre^T = S_in dO^T + Kt^T mask(dA)^T and S' = S_in + Kt^T V
//   warps 4-7   TMEM warps: S phase (Diag(E_B) post-scale, bf16 copy), causal mask of
//               dA, dq = E * dq_pre epilogue (lane = key dim j) staged in smem, TMA store
//   warps 8-15  prep warps (thread = key dim j, half of the rows): Kt = k / E in place
//               of log f, and E into TMEM lane j for the epilogue
namespace fsw {
constexpr uint32_t kColS = 0, kColDA = 128, kColDQ = 256, kColE = 384;
constexpr int kDqThreads = 512;

struct __align__(8) Misc {
    uint64_t full[2], prepped[2], empty[2];
    uint64_t barDA, barQ1, barS, barQ;       // MMA completions (tcgen05.commit)
    uint64_t sdone, dadone, dqfree, efree;   // TMEM-warp arrivals (128 each)
    uint32_t tmem_base;
    int bad_tile;
    int waited_full;
    int pad;
    float EB[2][128];
    float Bpart[128];                        // sum of log f over rows 0..63, per key dim
    float Bpart2[128];                       // ... and over rows 64..127
    float rs_part[128];
};
constexpr size_t kSmemBytes = 7 * (size_t)kTileBytes + sizeof(Misc);
}  // namespace fsw

struct DqParams {
    const float *h0, *dhT;
    float *rs;       // [B*H*128] rowsum(dhT * hT)
    int *flags;      // [B*H]
    int T, H, ntiles;
    // for the in-kernel exact route
    const __nv_bfloat16 *q, *lf, *x, *dO;
    __nv_bfloat16 *dq, *dlf, *dx;
    float *dh0;
    int simt_chunk;
};

__global__ void __launch_bounds__(fsw::kDqThreads, 1)
dq_kernel(const __grid_constant__ CUtensorMap tm_lf, const __grid_constant__ CUtensorMap tm_x,
          const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_dq, DqParams p) {
    using namespace fsw;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *Gb[2] = {smem, smem + 3 * kTileBytes};
    uint8_t *Vb[2] = {smem + kTileBytes, smem + 4 * kTileBytes};
    uint8_t *Ob[2] = {smem + 2 * kTileBytes, smem + 5 * kTileBytes};
    uint8_t *X = smem + 6 * kTileBytes;
    Misc *m = reinterpret_cast<Misc *>(smem + 7 * kTileBytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / p.H, h = bh - b * p.H;
    const int N = p.ntiles;
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->full[s], 1);
            mbar_init(&m->prepped[s], 256);
            mbar_init(&m->empty[s], 1);
        }
        mbar_init(&m->barDA, 1);
        mbar_init(&m->barQ1, 1);
        mbar_init(&m->barS, 1);
        mbar_init(&m->barQ, 1);
        mbar_init(&m->sdone, 128);
        mbar_init(&m->dadone, 128);
        mbar_init(&m->dqfree, 128);
        mbar_init(&m->efree, 128);
        m->bad_tile = INT_MAX;
        m->waited_full = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_lf);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_do);
        tma_prefetch_desc(&tm_dq);
    }
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;
    int producer_issued = 0;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int n = 0; n < N; ++n) {
                const int s = n & 1;
                if (ld_volatile(&m->bad_tile) < n) break;
                if (n >= 2 && !wait_or_abort(&m->empty[s], ((n - 2) >> 1) & 1, &m->bad_tile, n - 2)) break;
                mbar_arrive_expect_tx(&m->full[s], 3 * kTileBytes);
                for (int c = 0; c < 2; ++c) {
                    tma_load_4d(Gb[s] + c * kBlk, &tm_lf, &m->full[s], 64 * c, h, n * kTile, b);
                    tma_load_4d(Vb[s] + c * kBlk, &tm_x, &m->full[s], 64 * c, h, n * kTile, b);
                    tma_load_4d(Ob[s] + c * kBlk, &tm_do, &m->full[s], 64 * c, h, n * kTile, b);
                }
                ++producer_issued;
                if (n + 2 < N)   // warm L2 for the chunk after next (its load waits for a free stage)
                    for (int c = 0; c < 2; ++c) {
                        tma_prefetch_l2_4d(&tm_lf, 64 * c, h, (n + 2) * kTile, b);
                        tma_prefetch_l2_4d(&tm_x, 64 * c, h, (n + 2) * kTile, b);
                        tma_prefetch_l2_4d(&tm_do, 64 * c, h, (n + 2) * kTile, b);
                    }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_kk = idesc_bf16(128, 128, false, false);
            const uint32_t id_mnk = idesc_bf16(128, 128, true, false);
            const uint32_t id_mnmn = idesc_bf16(128, 128, true, true);
            for (int n = 0; n < N; ++n) {
                const int s = n & 1;
                // dA = dO V^T (does not need the prep)
                if (!mbar_wait(&m->full[s], (n >> 1) & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                    mma_bf16_ss(tbase + kColDA, sdesc_add(sdesc_sw128(smem_u32(Ob[s]), 16, 1024), ko),
                                sdesc_add(sdesc_sw128(smem_u32(Vb[s]), 16, 1024), ko), id_kk, kk > 0);
                }
                mma_commit(&m->barDA);
                if (!mbar_wait(&m->prepped[s], (n >> 1) & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                if (ld_volatile(&m->bad_tile) <= n) {
                    mbar_wait(&m->barDA, n & 1);   // nothing left in flight
                    break;
                }
                // dq_pre^T = S_in dO^T (M = j, N = t); S' = S_in + Kt^T V
                if (!mbar_wait(&m->sdone, n & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                if (n >= 1 && !mbar_wait(&m->dqfree, (n - 1) & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                    mma_bf16_ss(tbase + kColDQ, sdesc_add(sdesc_sw128(smem_u32(X), 16, 1024), ko),
                                sdesc_add(sdesc_sw128(smem_u32(Ob[s]), 16, 1024), ko), id_kk, kk > 0);
                }
                mma_commit(&m->barQ1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tbase + kColS, sdesc_add(sdesc_sw128(smem_u32(Gb[s]), kBlk, 1024), kk * 2048),
                                sdesc_add(sdesc_sw128(smem_u32(Vb[s]), kBlk, 1024), kk * 2048), id_mnmn, true);
                mma_commit(&m->barS);
                // dq_pre^T += Kt^T mask(dA)^T (M = j, N = t, K = s)
                if (!mbar_wait(&m->dadone, n & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                    mma_bf16_ss(tbase + kColDQ, sdesc_add(sdesc_sw128(smem_u32(Gb[s]), kBlk, 1024), kk * 2048),
                                sdesc_add(sdesc_sw128(smem_u32(X), 16, 1024), ko), id_mnk, true);
                }
                mma_commit(&m->barQ);
                mma_commit(&m->empty[s]);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ TMEM warps
        const int quad = warp & 3, r = 32 * quad + lane;
        const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
        const uint32_t cblk = (uint32_t)(r >> 6) * kBlk, cch = (uint32_t)((r & 63) >> 3), cin = (uint32_t)(r & 7) * 2;
        {   // S = h0 (or 0)
            const float *init = p.h0 ? p.h0 + (size_t)bh * 16384 : nullptr;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[32];
                if (init) {
                    const float4 *src = reinterpret_cast<const float4 *>(init + (size_t)r * 128 + 32 * c);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 a = src[i];
                        v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                }
                tmem_st32(tl + kColS + 32 * c, v);
            }
            tmem_wait_st();
        }
        int n = 0;
        // a wait given up by a lane of this warp (warp-uniform: TMEM loads and stores are
        // warp-collective); the group leaves together at its next barrier
        bool fail = false;
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            fail = __any_sync(0xffffffffu, fail || !mbar_wait(bar, par));
        };
        float e_prev = 1.0f, e_cur = 1.0f;   // e^{B/2} of the previous and the current chunk
        for (; n < N; ++n) {
            const int s = n & 1;
            wait_all(&m->prepped[s], (n >> 1) & 1);
            if (n >= 1) {
                wait_all(&m->barS, (n - 1) & 1);
                if (r == 0) tma_store_wait_read0();   // the previous dq store has read X
            }
            if (named_bar_or(2, 128, fail || ld_volatile(&m->bad_tile) <= n)) break;
            e_prev = e_cur;
            e_cur = m->EB[s][r];
            // S phase: S_r = Diag(e^{B/2}) Diag(e^{B_prev/2}) S' of the previous chunk, one factor after
            // the other (their product can fall below the fp32 range; the first gives S_out, O(1))
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[32];
                tmem_ld32(tl + kColS + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = (v[i] * e_prev) * e_cur;
                store_chunk_bf16(X, r, c, v);
                tmem_st32(tl + kColS + 32 * c, v);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&m->sdone);
            // causal mask of dA (lane = t), bf16 -> X (rows t) once S_r dO^T has read X.  (After a
            // wait given up, this thread goes on with whatever TMEM holds; nothing it writes is used.)
            wait_all(&m->barDA, n & 1);
            wait_all(&m->barQ1, n & 1);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[32];
                tmem_ld32(tl + kColDA + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (32 * c + i > r) v[i] = 0.0f;
                store_chunk_bf16(X, r, c, v);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&m->dadone);
            // dq[t][j] = E[j][t] * dq_pre^T[j][t]  (lane j = r) -> X as the [t][j] tile
            wait_all(&m->barQ, n & 1);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float d[32], e[32];
                tmem_ld32(tl + kColDQ + 32 * c, d);
                tmem_ld32(tl + kColE + 32 * c, e);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = 32 * c + i;
                    *reinterpret_cast<__nv_bfloat16 *>(X + cblk + t * 128 + ((cch ^ (t & 7)) << 4) + cin) =
                        __float2bfloat16_rn(d[i] * e[i]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&m->dqfree);
            mbar_arrive(&m->efree);
            if (named_bar_or(2, 128, fail)) break;
            if (r == 0) {
                tma_store_4d(&tm_dq, X, 0, h, n * kTile, b);
                tma_store_4d(&tm_dq, X + kBlk, 64, h, n * kTile, b);
                tma_store_commit();
            }
        }
        if (fail) set_status(HGRN2_ERR_TIMEOUT);
        if (r == 0) tma_store_wait_all0();
        if (n >= 1) mbar_wait(&m->barS, (n - 1) & 1);
        tc_fence_after();
        if (n == N && !fail && p.dhT && p.rs) {
            // hT = Diag(e^{B/2} of the last chunk) S';  rs[j] = sum_v dhT[j,v] hT[j,v]
            const float *g = p.dhT + ((size_t)bh * 128 + r) * 128;
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[32];
                tmem_ld32(tl + kColS + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) acc = fmaf(g[32 * c + i], v[i] * e_cur, acc);
            }
            p.rs[(size_t)bh * 128 + r] = acc;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ prep warps
        // thread = key dim j (TMEM lane j, in this warp's lane quadrant) and 64 rows.
        const int j = 32 * (warp & 3) + lane, half = (warp - 8) >> 2;
        const uint32_t tl = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t cblk = (uint32_t)(j >> 6) * kBlk, cch = (uint32_t)((j & 63) >> 3), cin = (uint32_t)(j & 7) * 2;
        auto eoff = [&](int t) -> uint32_t { return cblk + t * 128 + ((cch ^ (t & 7)) << 4) + cin; };
        for (int n = 0; n < N; ++n) {
            const int s = n & 1;
            const bool landed = mbar_wait(&m->full[s], (n >> 1) & 1);
            if (warp == 8 && lane == 0 && landed) m->waited_full = n + 1;
            {   // half 1 sums rows 0..63 (its prefix), half 0 rows 64..127: with both, the chunk total
                float sum = 0.0f;
#pragma unroll 16
                for (int t = 0; t < 64; ++t)
                    sum += __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(Gb[s] + eoff(t + 64 * (1 - half))));
                (half ? m->Bpart : m->Bpart2)[j] = sum;
            }
            // every row of log f is read before either half overwrites it; the group leaves
            // together if a wait gave up
            if (named_bar_or(1, 256, !landed)) {
                if (!landed) set_status(HGRN2_ERR_TIMEOUT);
                break;
            }
            const float rho = 0.5f * (m->Bpart[j] + m->Bpart2[j]);   // the balanced reference
            float bsum = (half ? m->Bpart[j] : 0.0f) - rho;           // b - rho before this half
            float ev[64];
#pragma unroll
            for (int bt = 0; bt < 8; ++bt) {
                const int t0 = 64 * half + 8 * bt;
                float av[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    av[i] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(Gb[s] + eoff(t0 + i)));
                __nv_bfloat16 ok[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    bsum += av[i];
                    const float E = __expf(bsum), iE = __expf(-bsum);
                    ok[i] = __float2bfloat16_rn((1.0f - __expf(av[i])) * iE);
                    ev[8 * bt + i] = E;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) *reinterpret_cast<__nv_bfloat16 *>(Gb[s] + eoff(t0 + i)) = ok[i];
            }
            if (half == 1) {   // bsum = B - rho = B / 2
                m->EB[s][j] = __expf(bsum);
                if (!(bsum >= -kMaxRefLog)) atomicMin(&m->bad_tile, n);   // also NaN
            }
            fence_proxy_async_smem();
            // E -> TMEM lane j once the previous chunk's dq epilogue has read it
            const bool efree = __all_sync(0xffffffffu, n < 1 || mbar_wait(&m->efree, (n - 1) & 1));
            if (efree) {
                tmem_st32(tl + kColE + 64 * half, *reinterpret_cast<float(*)[32]>(ev));
                tmem_st32(tl + kColE + 64 * half + 32, *reinterpret_cast<float(*)[32]>(ev + 32));
                tmem_wait_st();
            }
            tc_fence_before();
            if (named_bar_or(1, 256, !efree)) {   // bad_tile settled, Bpart free
                if (!efree) set_status(HGRN2_ERR_TIMEOUT);
                break;
            }
            mbar_arrive(&m->prepped[s]);
            if (ld_volatile(&m->bad_tile) <= n) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool fell_back = m->bad_tile < N;
    if (warp == 0 && lane == 0)
        for (int k = m->waited_full; k < producer_issued; ++k) mbar_wait(&m->full[k & 1], (k >> 1) & 1, 2000000u);
    if (tid == 0) {
        p.flags[bh] = fell_back ? 1 : 0;
        if (fell_back) atomicAdd(&g_counters[0], 1ull);
        else atomicAdd(&g_counters[1], (unsigned long long)N);
    }
    __syncwarp();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
    // exact route for this (b,h): both sweeps on CUDA cores in the drained CTA (the reverse
    // tensor-core kernel skips flagged pairs)
    if (fell_back) {
        __syncthreads();
        float *sm = reinterpret_cast<float *>(smem);
        simt_bwd_dq_body<__nv_bfloat16>(p.lf, p.x, p.h0, p.dO, p.dhT, p.dq, p.rs, p.T, p.H, 128, 128,
                                        p.simt_chunk, sm, b, h, bh, p.dlf, p.dx);
        __syncthreads();
        simt_bwd_rev_body<__nv_bfloat16>(p.q, p.lf, p.x, p.dO, p.dhT, p.dq, p.rs, p.dlf, p.dx, p.dh0, p.T, p.H,
                                         128, 128, p.simt_chunk, sm, b, h, bh, true);
    }
}

// ------------------------------------------------------------------ reverse sweep
// 16 warps; every phase is spread over all of them.  TMEM lane quadrant = warp & 3,
// quarter = warp >> 2 selects 32 TMEM columns (or 32 rows of the chunk in the prep).
// Shared memory (7 tiles of 32 KB): Qb q -> Qt, Gb log f -> Kt, Vb v, Ob dO, D16 bf16(dSh)
// then the dq tile, AT mask(A)^T then di staging, DA mask(dA) then d log f staging.
//
// Phase 2 issues its two products that read bf16(dSh) first, under a commit of their own, so
// that D16 takes its next tile while the other two run.  Two modes.  Recompute mode (kSaved =
// false) follows the forward-sweep kernel: dq of this chunk (written by that kernel) lands in
// D16, v and dO of the next chunk in Vb, Ob once phase 2 is done; q and log f of the next chunk
// follow once the epilogue has read Qt and Kt.  Saved-state mode (kSaved = true) needs no
// forward sweep: the bf16 state entering each chunk, stored by the training forward, lands in
// D16 and a third MMA phase forms dq itself, transposed (lane j, tokens along the columns),
//     dq_pre^T = Kt^T mask(dA)^T + S_in dO^T,      dq = E * dq_pre,
// reusing the masked dA of this chunk; q dq = Qt dq_pre then enters d log f without
// reading dq back.  A (batch, head) that the forward flagged for the exact route runs
// both exact sweeps here, on CUDA cores.
namespace rsw {
constexpr uint32_t kColDS = 0, kColX1 = 128, kColX2 = 256, kColE = 384;
constexpr int kRevThreads = 512;
constexpr int kStoreTid = 256;   // issues the output TMA stores (thread 0 issues loads and MMAs)

struct __align__(8) Misc {
    uint64_t barIn, barVO, barDQ, barP1, barP2, barP3;   // barDQ: dq (recompute) or S_in (saved)
    uint64_t barDS;                                      // all 512 threads wrote dSh into TMEM
    uint64_t barD16;                                     // the phase-2 MMAs that read bf16(dSh) completed
    uint32_t tmem_base;
    int pad;
    int issued[3], waited[3];   // loads issued / arrivals waited for: [barIn, barVO, barDQ]
    float EB[128];
    float Bpart[3][128];   // per 32-row range sums of log f; in the epilogue, quarter suffix totals
    float carry[128];
};
constexpr size_t kSmemBytes = 7 * (size_t)kTileBytes + sizeof(Misc);
static_assert(offsetof(Misc, Bpart) == offsetof(Misc, EB) + sizeof(float) * 128,
              "the scalar-decay reduction uses EB and Bpart as one [4][128] array");
}  // namespace rsw

struct RevParams {
    const float *dhT;
    float *rs;           // rowsum(dhT * hT) from the forward sweep; exact-route workspace (saved mode)
    float *dh0;
    const int *flags;    // [B*H] 1: the (b,h) takes the exact route
    int T, H, ntiles;
    // saved-state mode
    const float *hTs;    // [B*H][128][128] final state saved by the forward
    const float *h0;
    const __nv_bfloat16 *q, *lf, *x, *dO;   // for the exact route
    __nv_bfloat16 *dq, *dlf, *dx;
    int simt_chunk;
    const int *cu;       // packed sequences (saved mode only), or null; B = their number
    const int *perm;     // with cu: CTA row r runs sequence perm[r]
    int D;               // head size d_k = d_v: 128, or 64 (saved mode; the second 64-column half of
                         // every operand tile is held at zero, which is exactly neutral)
    const __nv_bfloat16 *lgs;   // scalar decay: log g [B][T][H] (lf is then the key k, dlf its gradient)
    __nv_bfloat16 *dlg;         // scalar decay: d log g [B][T][H]
    // Heads of width 256 read in place (saved mode; nK = nV = 2): head h of the call is block pair
    // (a, c) of head h / (nK nV); q, log f at half-head (h / (nK nV)) nK + a and i, dO at * nV + c of
    // the caller's tensors viewed as [B][T][2 Hw][128].  Every block pair adds its shares of dq,
    // d log f (key-side half-heads) and di (value-side) into the outputs, zeroed by the host, by TMA
    // reduce-add; a flagged pair's exact route writes its shares into the partials (dq, d log f: the
    // value block's, [nV][B][T][Hw][256]; di: the key block's, [nK][B][T][Hw][256]) and adds them
    // from there.  nK = nV = 1 otherwise.
    int nK, nV, Bo;
    __nv_bfloat16 *dq_part, *dlf_part, *dx_part;   // heads read in place: the exact route's partials
    // Sequence segments (kSeg): [B*H][nseg] segments of tps chunks each; every segment's reverse
    // sweep starts from a zero gradient (the last from dhT) and writes its backward map: W, the
    // gradient it hands to the state entering it ([B*H][nseg][128][128]), and g, its decay product
    // ([B*H][nseg][128])
    int nseg, tps;
    float *Wseg, *gseg;
    // and sum_v |W[j,v]| over each quarter of the value dims ([B*H][nseg][128][4]; the fix-up's
    // bound on what the maps it leaves out could add)
    float *Wabs;
};

// kPacked (saved mode only): p.cu holds packed sequences; compiled apart so the dense path
// carries no row masks.
// kScalar (saved mode only): the scalar-decay variant S_t = g_t S_{t-1} + k_t v_t^T.  Its chunk
// math is this kernel's with Qt = q E_t, Kt = k / E_t for a decay E_t shared by every key dim:
// the prep scans the gate per row instead of forming k = 1 - f; the epilogue writes dk = dk_pre /
// E in place of d log f, has no tied-key term, and sums the per-dim reverse sums over d_k into
// d log g_t.  Flagged pairs return at once; the host recomputes them on the exact route.
// kWide (saved mode only): heads of width 256 read in place (p.nK = p.nV = 2), compiled apart so
// that the other instances carry none of its head arithmetic.
// kSeg (saved mode, dense, per-dim): one CTA per sequence segment (p.nseg per pair); a flagged
// pair is recomputed whole by its first segment's CTA.
template <bool kSaved, bool kPacked, bool kScalar = false, bool kWide = false, bool kSeg = false>
__global__ void __launch_bounds__(rsw::kRevThreads, 1)
rev_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_lf,
           const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_do,
           const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_di,
           const __grid_constant__ CUtensorMap tm_dlf, const __grid_constant__ CUtensorMap tm_st, RevParams p) {
    using namespace rsw;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *Qb = smem, *Gb = smem + kTileBytes, *Vb = smem + 2 * kTileBytes, *Ob = smem + 3 * kTileBytes;
    uint8_t *D16 = smem + 4 * kTileBytes, *AT = smem + 5 * kTileBytes, *DA = smem + 6 * kTileBytes;
    Misc *m = reinterpret_cast<Misc *>(smem + 7 * kTileBytes);

    // (kSeg: no early trigger of the dependent scan or fix-up, as in the forward's segments: the
    // fix-up scheduled at this kernel's start made the long-sequence backward slower, A/B on one
    // B200 240.4 -> 224.9 us without the trigger.)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    static_assert(!kSeg || (kSaved && !kPacked && !kScalar && !kWide), "segments: saved mode, dense, per-dim");
    const int seg = kSeg ? (int)blockIdx.x % p.nseg : 0;
    int bh = kSeg ? (int)blockIdx.x / p.nseg : (int)blockIdx.x;
    const int h = bh % p.H;
    // token of chunk n: tok0 + n * kTile of batch bc; saved-state slot: slot0 + n * sstride.
    // Packed sequences (saved mode only): rows from the sequence's end on (valid(n) < kTile)
    // are masked in the prep and not stored.
    int b = bh / p.H, bc = b, tok0 = 0, len = p.T, N = p.ntiles, slot0 = bh * p.ntiles, sstride = 1;
    if (kSeg) {   // this segment's chunks
        const int g0 = seg * p.tps;
        N = min(p.ntiles - g0, p.tps);
        tok0 = g0 * kTile;
        slot0 += g0;
    }
    // the sequence's last segment starts from dhT (and the carry rowsum(dhT * hT)); others from zero
    const bool from_dhT = !kSeg || seg == p.nseg - 1;
    static_assert(kSaved || !kPacked, "packed sequences need the saved states");
    if (kPacked) {
        const int sq = packed_seq(p.perm, bh / p.H, gridDim.x / p.H);
        bh = sq * p.H + h;   // the pair whose states, flag and gradients this CTA owns
        const int a = min(max(p.cu[sq], 0), p.T), e = min(max(p.cu[sq + 1], a), p.T);
        b = bc = 0;
        tok0 = a;
        len = e - a;
        N = (len + kTile - 1) / kTile;
        slot0 = ((a >> 7) + sq) * p.H + h;
        sstride = p.H;
    }
    auto valid_rows = [&](int n) -> int { return kPacked ? min(kTile, len - n * kTile) : kTile; };
    // head coordinates of the key-side (q, log f, dq, d log f) and value-side (i, dO, di) token
    // tensors and the batch coordinates of the partial outputs; h and bc unless heads are read in place
    static_assert(!kWide || (kSaved && !kPacked && !kScalar), "heads read in place: saved mode, dense, per-dim");
    const int nK = kWide ? p.nK : 1, nV = kWide ? p.nV : 1, nbk = nK * nV;
    const int hw = h / nbk, ka = (h - hw * nbk) / nV, vc = h - hw * nbk - ka * nV;
    const int hk = hw * nK + ka, hv = hw * nV + vc, kbc = vc * p.Bo + bc, vbc = ka * p.Bo + bc;
    if (p.flags[bh] != 0) {   // this (b,h) takes the exact route
        if (kSeg && seg != 0) return;   // recomputed whole by the first segment's CTA
        if (kSaved && !kScalar) {   // both sweeps here (recompute mode: in the forward-sweep kernel)
            float *sm = reinterpret_cast<float *>(smem);
            const size_t ok = (size_t)tok0 * p.H * p.D;   // 0 unless packed sequences
            const int Tl = kPacked ? len : p.T;
            if constexpr (!kWide) {
                simt_bwd_dq_body<__nv_bfloat16>(p.lf + ok, p.x + ok, p.h0, p.dO + ok, p.dhT, p.dq + ok, p.rs, Tl, p.H,
                                                p.D, p.D, p.simt_chunk, sm, b, h, bh, p.dlf + ok, p.dx + ok);
                __syncthreads();
                simt_bwd_rev_body<__nv_bfloat16>(p.q + ok, p.lf + ok, p.x + ok, p.dO + ok, p.dhT, p.dq + ok, p.rs,
                                                 p.dlf + ok, p.dx + ok, p.dh0, Tl, p.H, p.D, p.D, p.simt_chunk, sm,
                                                 b, h, bh, true);
            } else {
                // heads read in place (nK = nV): every token tensor viewed with Hw nK half-heads of 128,
                // indexed at the value-side half-head hv; key-side tensors shifted by hk - hv half-heads,
                // the partial outputs by their block
                // The shares go to the partials first (the reverse sweep reads its dq share back),
                // then are added into the outputs (other block pairs add theirs by TMA reduce-add)
                const int Hh = (p.H / nbk) * p.nV;
                const long long ks = (long long)(hk - hv) * p.D;
                const size_t part = (size_t)p.Bo * p.T * Hh * p.D;
                __nv_bfloat16 *dq = p.dq_part + vc * part + ks, *dlf = p.dlf_part + vc * part + ks;
                __nv_bfloat16 *dx = p.dx_part + ka * part;
                simt_bwd_dq_body<__nv_bfloat16>(p.lf + ks, p.x, p.h0, p.dO, p.dhT, dq, p.rs, p.T, Hh, p.D, p.D,
                                                p.simt_chunk, sm, b, hv, bh, dlf, dx);
                __syncthreads();
                simt_bwd_rev_body<__nv_bfloat16>(p.q + ks, p.lf + ks, p.x, p.dO, p.dhT, dq, p.rs, dlf, dx, p.dh0, p.T,
                                                 Hh, p.D, p.D, p.simt_chunk, sm, b, hv, bh, true);
                __syncthreads();
                add_rows_bf16(p.dq + ks, dq, b, hv, p.T, Hh);
                add_rows_bf16(p.dlf + ks, dlf, b, hv, p.T, Hh);
                add_rows_bf16(p.dx, dx, b, hv, p.T, Hh);
            }
            if (tid == 0) atomicAdd(&g_counters[0], 1ull);
        }
        return;
    }
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    const int quad = warp & 3, q4 = warp >> 2;
    const int j = 32 * quad + lane;      // TMEM lane / key dim / tile row
    const int c0 = 32 * q4;              // this thread's 32 TMEM columns (or rows, in the prep)
    const int nblk = p.D >> 6;   // 64-column blocks loaded and stored per tile
    int *issued = m->issued, *waited = m->waited;   // thread 0 issues; waits are recorded by thread 0
    // two token tiles of one side (q, log f: key side, hk; i, dO: value side, hv)
    auto issue2 = [&](uint8_t *d0, const CUtensorMap *t0, uint8_t *d1, const CUtensorMap *t1, uint64_t *bar,
                      int q, int n) {
        ++issued[q];
        const int hh = q == 0 ? hk : hv;
        mbar_arrive_expect_tx(bar, 2 * nblk * kBlk);
        for (int c = 0; c < nblk; ++c) {
            tma_load_4d(d0 + c * kBlk, t0, bar, 64 * c, hh, tok0 + n * kTile, bc);
            tma_load_4d(d1 + c * kBlk, t1, bar, 64 * c, hh, tok0 + n * kTile, bc);
        }
    };
    if (tid == 0) {
        mbar_init(&m->barIn, 1);
        mbar_init(&m->barVO, 1);
        mbar_init(&m->barDQ, 1);
        mbar_init(&m->barP1, 1);
        mbar_init(&m->barP2, 1);
        mbar_init(&m->barP3, 1);
        mbar_init(&m->barDS, kRevThreads);
        mbar_init(&m->barD16, 1);
        fence_mbar_init();
        for (int q = 0; q < 3; ++q) issued[q] = waited[q] = 0;
        // the last chunk's tiles before the TMEM allocation and the block barrier (the d = 64 zero
        // fill below writes only the tiles' upper halves, which TMA does not load)
        if (N > 0) {
            issue2(Qb, &tm_q, Gb, &tm_lf, &m->barIn, 0, N - 1);
            issue2(Vb, &tm_x, Ob, &tm_do, &m->barVO, 1, N - 1);
        }
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (nblk == 1) {             // d = 64: the unloaded halves of the input tiles stay zero
        for (int i = tid; i < 4 * (int)(kBlk / 16); i += kRevThreads) {
            const int t = i / (int)(kBlk / 16), o = i - t * (int)(kBlk / 16);
            uint8_t *base = t == 0 ? Qb : t == 1 ? Gb : t == 2 ? Vb : Ob;
            reinterpret_cast<uint4 *>(base + kBlk)[o] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);

    {   // dS = dhT (or 0); carry = rowsum(dhT * hT) (or 0)
        float v[32];
        float part = 0.0f;   // saved mode: this quarter's share of rowsum(dhT * hT)
        if (from_dhT && p.dhT && j < p.D && c0 < p.D) {   // d x d; zero outside for d = 64
            const float4 *src = reinterpret_cast<const float4 *>(p.dhT + ((size_t)bh * p.D + j) * p.D + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 a = src[i];
                v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
            }
            if (kSaved) {
                const float4 *hs = reinterpret_cast<const float4 *>(p.hTs + ((size_t)bh * p.D + j) * p.D + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 a = hs[i];
                    part += v[4 * i] * a.x + v[4 * i + 1] * a.y + v[4 * i + 2] * a.z + v[4 * i + 3] * a.w;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.0f;
        }
        tmem_st32(tl + kColDS + c0, v);
        tmem_wait_st();
        if (kSaved) {
            if (q4 < 3) m->Bpart[q4][j] = part;
            else m->EB[j] = part;
            __syncthreads();
            if (q4 == 0) m->carry[j] = m->Bpart[0][j] + m->Bpart[1][j] + m->Bpart[2][j] + m->EB[j];
        } else if (q4 == 0) {
            m->carry[j] = (from_dhT && p.dhT && p.rs) ? p.rs[(size_t)bh * 128 + j] : 0.0f;
        }
    }

    const uint32_t id_kk = idesc_bf16(128, 128, false, false);
    const uint32_t id_kmn = idesc_bf16(128, 128, false, true);
    const uint32_t id_mnmn = idesc_bf16(128, 128, true, true);
    const uint32_t id_mnk = idesc_bf16(128, 128, true, false);
    const uint32_t cblk = (uint32_t)(j >> 6) * kBlk, cch = (uint32_t)((j & 63) >> 3), cin = (uint32_t)(j & 7) * 2;
    auto eoff = [&](int t) -> uint32_t { return cblk + t * 128 + ((cch ^ (t & 7)) << 4) + cin; };
    auto bfat = [&](const uint8_t *tile, int t) -> float {
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + eoff(t)));
    };
    bool ok = true;
    int it = 0, n = N - 1;
    float g_later = 1.0f;   // e^{rho} of the chunk processed before this one (the later chunk), key dim j
    float gprod = 1.0f;     // segments: the product of this segment's chunk decays e^{B}, key dim j
    for (; n >= 0; --n, ++it) {
        const uint32_t par = it & 1;
        if (__syncthreads_or(!mbar_wait(&m->barIn, par))) { ok = false; break; }
        if (tid == 0) waited[0] = it + 1;
        float em1 = 1.0f;   // E of the row before the chunk, e^{-rho}
        float hh = 1.0f;    // the state scale e^{B - rho} = e^{rho} of this chunk, key dim j
        // ---- prep: column j, rows c0 .. c0+31: Qt = q E, Kt = k / E in place; E -> TMEM.
        // f = e^a directly, so k = 1 - f has an absolute error of a few 1e-8; E = e^{b - rho} is the
        // running product of f from the range start, 1/E = e^{rho - b}.
        {
            const int vr = valid_rows(n);   // rows from vr on: log f = 0 and q = 0 (no effect)
            float bsum = 0.0f;   // the running b - rho; after the prep B - rho = B / 2
            float ev[32];
            if constexpr (kScalar) {
                // b_t = cumulative log g from the chunk start (0 past the sequence end), threads 0..127
                float a = 0.0f;
                if (tid < kTile) {
                    const int t = tok0 + n * kTile + tid;
                    if (t < p.T) a = __bfloat162float(p.lgs[((size_t)bc * p.T + t) * p.H + h]);
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float y = __shfl_up_sync(0xffffffffu, a, o);
                        if (lane >= o) a += y;
                    }
                    if (lane == 31) m->Bpart[1][tid >> 5] = a;
                }
                __syncthreads();
                if (tid < kTile) {
                    for (int w = 0; w < (tid >> 5); ++w) a += m->Bpart[1][w];
                    m->Bpart[0][tid] = a;
                }
                __syncthreads();
                const float rho = 0.5f * m->Bpart[0][kTile - 1];   // the balanced reference
                em1 = __expf(-rho);
                bsum = rho;   // B - rho
                hh = __expf(rho);
#pragma unroll
                for (int bt = 0; bt < 4; ++bt) {   // Qt = q e^{b_t - rho}, Kt = k e^{rho - b_t}
                    const int t0 = c0 + 8 * bt;
                    float kv[8], qv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        kv[i] = bfat(Gb, t0 + i);
                        qv[i] = bfat(Qb, t0 + i);
                    }
                    __nv_bfloat16 oq[8], ok2[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float b = m->Bpart[0][t0 + i] - rho, E = __expf(b);
                        ok2[i] = __float2bfloat16_rn(kv[i] * __expf(-b));
                        oq[i] = __float2bfloat16_rn(qv[i] * E);
                        ev[8 * bt + i] = E;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        *reinterpret_cast<__nv_bfloat16 *>(Gb + eoff(t0 + i)) = ok2[i];
                        *reinterpret_cast<__nv_bfloat16 *>(Qb + eoff(t0 + i)) = oq[i];
                    }
                }
            } else {
            float sum = 0.0f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) sum += c0 + i < vr ? bfat(Gb, c0 + i) : 0.0f;
            // quarters 0..2 in Bpart, quarter 3 in EB (free from the start of the prep until the
            // epilogue: the dS phase takes e^{B/2} from a register)
            if (q4 < 3) m->Bpart[q4][j] = sum;
            else m->EB[j] = sum;
            __syncthreads();
            for (int r2 = 0; r2 < q4; ++r2) bsum += m->Bpart[r2][j];
            // the chunk total, summed in the same order by the four threads of key dim j
            const float Btot = ((m->Bpart[0][j] + m->Bpart[1][j]) + m->Bpart[2][j]) + m->EB[j];
            const float rho = 0.5f * Btot;   // the balanced reference
            em1 = __expf(-rho);
            hh = __expf(Btot - rho);
            bsum -= rho;
            float E = __expf(bsum);
#pragma unroll
            for (int bt = 0; bt < 4; ++bt) {
                const int t0 = c0 + 8 * bt;
                float av[8], qv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    av[i] = t0 + i < vr ? bfat(Gb, t0 + i) : 0.0f;
                    qv[i] = t0 + i < vr ? bfat(Qb, t0 + i) : 0.0f;
                }
                __nv_bfloat16 oq[8], ok2[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    bsum += av[i];
                    const float f = __expf(av[i]);
                    E *= f;
                    ok2[i] = __float2bfloat16_rn((1.0f - f) * __expf(-bsum));
                    oq[i] = __float2bfloat16_rn(qv[i] * E);
                    ev[8 * bt + i] = E;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    *reinterpret_cast<__nv_bfloat16 *>(Gb + eoff(t0 + i)) = ok2[i];
                    *reinterpret_cast<__nv_bfloat16 *>(Qb + eoff(t0 + i)) = oq[i];
                }
            }
            }   // per-dim prep
            tmem_st32(tl + kColE + c0, ev);
            tmem_wait_st();
            // the previous chunk's output stores have read their staging tiles (D16, AT, DA are
            // written next, from the dS phase on): waited for by the issuing thread before this barrier
            if (tid == kStoreTid) tma_store_wait_read0();
            fence_proxy_async_smem();
            tc_fence_before();
            // the forward passed this (b,h): its chunks are in range (a unit of margin for the
            // rounding of the two kernels' sums)
            if (__syncthreads_or(q4 == 3 && !(bsum >= -kMaxRefLog - 1.0f))) {
                if (tid == 0) set_status(HGRN2_ERR_DEVICE);
                ok = false;
                break;
            }
        }
        // ---- phase 1: A^T = Kt Qt^T (M = s, N = t), dA = dO V^T (M = t, N = s)
        if (tid == 0) {
            if (!mbar_wait(&m->barVO, par)) ok = false;
            else waited[1] = it + 1;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColX1, sdesc_add(sdesc_sw128(smem_u32(Gb), 16, 1024), ko),
                            sdesc_add(sdesc_sw128(smem_u32(Qb), 16, 1024), ko), id_kk, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColX2, sdesc_add(sdesc_sw128(smem_u32(Ob), 16, 1024), ko),
                            sdesc_add(sdesc_sw128(smem_u32(Vb), 16, 1024), ko), id_kk, kk > 0);
            }
            mma_commit(&m->barP1);
            // warm L2: this chunk's dq (or saved state), the next chunk's inputs.  Issued here,
            // where this thread would otherwise only wait: a prefetch holds up its issuing thread,
            // and at the top of the chunk that delayed every warp at the next block barrier.
            for (int c = 0; c < 2; ++c) {
                if (kSaved) tma_prefetch_l2_4d(&tm_st, 64 * c, 0, 0, slot0 + n * sstride);
                else tma_prefetch_l2_4d(&tm_dq, 64 * c, h, n * kTile, b);
                if (n > 0) {
                    tma_prefetch_l2_4d(&tm_q, 64 * c, hk, tok0 + (n - 1) * kTile, bc);
                    tma_prefetch_l2_4d(&tm_lf, 64 * c, hk, tok0 + (n - 1) * kTile, bc);
                    tma_prefetch_l2_4d(&tm_x, 64 * c, hv, tok0 + (n - 1) * kTile, bc);
                    tma_prefetch_l2_4d(&tm_do, 64 * c, hv, tok0 + (n - 1) * kTile, bc);
                }
            }
        }
        // ---- dS phase: dSh = Diag(e^{B - rho}) dL/dS_out -> TMEM (becomes the new dS) and bf16 into
        // D16, with dL/dS_out = Diag(e^{rho_later}) dS of the later chunk; thread 0 joins once it has
        // issued phase 1
        {
            float v[32];
            tc_fence_after();
            tmem_ld32(tl + kColDS + c0, v);
            tmem_wait_ld();
            // one factor after the other: their product can fall below the fp32 range, while the first
            // gives dL/dS_out of this chunk, O(1)
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = (v[i] * g_later) * hh;
            g_later = hh;   // e^{rho} = e^{B - rho} of this chunk
            if (kSeg) gprod = (gprod * hh) * hh;
            store_chunk_bf16(D16, j, q4, v);
            tmem_st32(tl + kColDS + c0, v);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&m->barDS);
        }
        if (tid == 0) {   // the recurrence step, issued as soon as dSh is in TMEM: dS = dSh + Qt^T dO
            if (!mbar_wait(&m->barDS, par)) ok = false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                mma_bf16_ss(tbase + kColDS, sdesc_add(sdesc_sw128(smem_u32(Qb), kBlk, 1024), kk * 2048),
                            sdesc_add(sdesc_sw128(smem_u32(Ob), kBlk, 1024), kk * 2048), id_mnmn, true);
            }
        }
        // ---- masks: A^T keeps t >= s (lane s), dA keeps s <= t (lane t)
        {
            if (!mbar_wait(&m->barP1, par)) ok = false;
            tc_fence_after();
            // this thread's 32 columns are all kept (q4 > quad), all dropped (q4 < quad) or the
            // diagonal block (q4 == quad, compare per element); the branch is warp-uniform
            float v[32];
            if (q4 >= quad) {
                tmem_ld32(tl + kColX1 + c0, v);
                tmem_wait_ld();
                if (q4 == quad) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < lane) v[i] = 0.0f;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            store_chunk_bf16(AT, j, q4, v);
            if (q4 <= quad) {
                tmem_ld32(tl + kColX2 + c0, v);
                tmem_wait_ld();
                if (q4 == quad) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i > lane) v[i] = 0.0f;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            store_chunk_bf16(DA, j, q4, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) { ok = false; break; }
        // ---- phase 2: the two products that read bf16(dSh) in D16 first, so that D16 can take the
        // next tile (the saved state, or dq) while the other two run
        if (tid == 0) {
            tc_fence_after();
            // di = Kt dSh + mask(A)^T dO          (M = s, N = v)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColX1, sdesc_add(sdesc_sw128(smem_u32(Gb), 16, 1024), ko),
                            sdesc_add(sdesc_sw128(smem_u32(D16), kBlk, 1024), kk * 2048), id_kmn, kk > 0);
            }
            // dk_pre^T = dSh V^T + Qt^T mask(dA)   (M = j, N = s)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColX2, sdesc_add(sdesc_sw128(smem_u32(D16), 16, 1024), ko),
                            sdesc_add(sdesc_sw128(smem_u32(Vb), 16, 1024), ko), id_kk, kk > 0);
            }
            mma_commit(&m->barD16);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + kColX1, sdesc_add(sdesc_sw128(smem_u32(AT), 16, 1024), ko),
                            sdesc_add(sdesc_sw128(smem_u32(Ob), kBlk, 1024), kk * 2048), id_kmn, true);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                mma_bf16_ss(tbase + kColX2, sdesc_add(sdesc_sw128(smem_u32(Qb), kBlk, 1024), kk * 2048),
                            sdesc_add(sdesc_sw128(smem_u32(DA), kBlk, 1024), kk * 2048), id_mnmn, true);
            }
            mma_commit(&m->barP2);   // also covers the recurrence step issued after the dS phase
            // D16 once the first two products have read it: the saved bf16 state entering this chunk
            // (saved mode) or dq of this chunk (recompute mode)
            if (!mbar_wait(&m->barD16, par)) {
                ok = false;
            } else {
                ++issued[2];
                mbar_arrive_expect_tx(&m->barDQ, kTileBytes);
                if (kSaved) {
                    tma_load_4d(D16, &tm_st, &m->barDQ, 0, 0, 0, slot0 + n * sstride);
                    tma_load_4d(D16 + kBlk, &tm_st, &m->barDQ, 64, 0, 0, slot0 + n * sstride);
                } else {
                    tma_load_4d(D16, &tm_dq, &m->barDQ, 0, h, n * kTile, b);
                    tma_load_4d(D16 + kBlk, &tm_dq, &m->barDQ, 64, h, n * kTile, b);
                }
            }
        }
        // Qt and Kt to registers for the epilogue while the phase-2 MMAs run
        uint32_t qk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t off = eoff(c0 + i);
            qk[i] = (uint32_t)*reinterpret_cast<const uint16_t *>(Qb + off) |
                    ((uint32_t)*reinterpret_cast<const uint16_t *>(Gb + off) << 16);
        }
        if (__syncthreads_or(!mbar_wait(&m->barP2, par) || !ok)) { ok = false; break; }
        tc_fence_after();
        // recompute mode: v and dO of the next chunk into Vb, Ob
        if (!kSaved && tid == 0 && n > 0) issue2(Vb, &tm_x, Ob, &tm_do, &m->barVO, 1, n - 1);
        // ---- di (lane s) -> AT (rows s) for the TMA store
        {
            float v[32];
            tmem_ld32(tl + kColX1 + c0, v);
            tmem_wait_ld();
            store_chunk_bf16(AT, j, q4, v);
        }
        // ---- d log f (lane j, tokens c0 .. c0+31): partial values kept in TMEM X1 (di has
        // been read out): d'_t = sum_{t<=t'<quarter end} (q dq - k dk)_{t'} - f_t dk_t with
        // q = Qt / E, k dk = Kt dk_pre, f_t dk_t = dk_pre_t / E_{t-1}.  Qt and Kt were copied to
        // registers, so that q and log f of the next chunk can load during the epilogue.
        if (kSaved) {
            // phase 3 once di has left X1: dq_pre^T = Kt^T mask(dA)^T + S_in dO^T   (M = j, N = t),
            // the product that needs no saved state first
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                    mma_bf16_ss(tbase + kColX1, sdesc_add(sdesc_sw128(smem_u32(Gb), kBlk, 1024), kk * 2048),
                                sdesc_add(sdesc_sw128(smem_u32(DA), 16, 1024), ko), id_mnk, kk > 0);
                }
                if (!mbar_wait(&m->barDQ, par)) {
                    ok = false;
                } else {
                    waited[2] = it + 1;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                        mma_bf16_ss(tbase + kColX1, sdesc_add(sdesc_sw128(smem_u32(D16), 16, 1024), ko),
                                    sdesc_add(sdesc_sw128(smem_u32(Ob), 16, 1024), ko), id_kk, true);
                    }
                }
                mma_commit(&m->barP3);   // also on a timeout: the waits below then end at once
            }
            if (__syncthreads_or(!mbar_wait(&m->barP3, par) || !ok)) { ok = false; break; }
            tc_fence_after();
            if (tid == 0 && n > 0) {   // every operand tile of this chunk has been read
                issue2(Vb, &tm_x, Ob, &tm_do, &m->barVO, 1, n - 1);
                issue2(Qb, &tm_q, Gb, &tm_lf, &m->barIn, 0, n - 1);
            }
        } else {
            __syncthreads();
            if (tid == 0 && n > 0) issue2(Qb, &tm_q, Gb, &tm_lf, &m->barIn, 0, n - 1);
            if (__syncthreads_or(!mbar_wait(&m->barDQ, par))) { ok = false; break; }
            if (tid == 0) waited[2] = it + 1;
        }
        float suf = 0.0f;
#pragma unroll
        for (int hh = 1; hh >= 0; --hh) {
            float dkp[16], e[16], dap[16];
            const int col = c0 + 16 * hh;
            tmem_ld16(tl + kColX2 + col, dkp);
            tmem_ld16(tl + kColE + col, e);
            if (kSaved) tmem_ld16(tl + kColX1 + col, dap);   // dq_pre of these tokens
            const float eprev = col > 0 ? tmem_ld1(tl + kColE + col - 1) : em1;
            tmem_wait_ld();
            float invE = __fdividef(1.0f, e[15]);
#pragma unroll
            for (int i = 15; i >= 0; --i) {
                const int t = col + i;
                const float qt = bf_lo(qk[16 * hh + i]), kt = bf_hi(qk[16 * hh + i]);
                const float invEm1 = __fdividef(1.0f, i > 0 ? e[i - 1] : eprev);
                if (kSaved) {   // dq = E dq_pre into D16 (row t); q dq = Qt dq_pre
                    *reinterpret_cast<__nv_bfloat16 *>(D16 + eoff(t)) = __float2bfloat16_rn(e[i] * dap[i]);
                    suf += qt * dap[i] - kt * dkp[i];
                } else {
                    suf += qt * invE * bfat(D16, t) - kt * dkp[i];
                }
                if (kScalar) {   // dk = dk_pre / E into DA (row t); no tied-key term
                    *reinterpret_cast<__nv_bfloat16 *>(DA + eoff(t)) = __float2bfloat16_rn(dkp[i] * __fdividef(1.0f, e[i]));
                    dap[i] = suf;
                } else {
                    dap[i] = suf - dkp[i] * invEm1;
                }
                invE = invEm1;
            }
            tmem_st16(tl + kColX1 + col, dap);
        }
        tmem_wait_st();
        // quarter totals: quarters 0..2 in Bpart, quarter 3 in EB (free until the next prep)
        if (q4 < 3) m->Bpart[q4][j] = suf;
        else m->EB[j] = suf;
        __syncthreads();
        {
            float carry = m->carry[j];   // from later chunks (and rowsum(dhT * hT))
            if (q4 < 3) carry += m->EB[j];
            for (int r2 = q4 + 1; r2 < 3; ++r2) carry += m->Bpart[r2][j];
            float dap[32];
            tmem_ld32(tl + kColX1 + c0, dap);
            tmem_wait_ld();
            if constexpr (kScalar) {
                // d log g_t = sum_j (d'_t[j] + carry_j): the warp's 32 key dims by a butterfly (lane l
                // ends with token c0 + l), then the four key-dim quarters through shared memory (EB and
                // Bpart, free once every thread has read its carry and the next carry is in a register)
                const float nc = m->carry[j] + m->Bpart[0][j] + m->Bpart[1][j] + m->Bpart[2][j] + m->EB[j];
#pragma unroll
                for (int i = 0; i < 32; ++i) dap[i] += carry;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    const bool up = (lane & o) != 0;
#pragma unroll
                    for (int i = 0; i < o; ++i) {
                        const float send = up ? dap[i] : dap[i + o];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, o);
                        dap[i] = (up ? dap[i + o] : dap[i]) + recv;
                    }
                }
                __syncthreads();
                if (q4 == 0) m->carry[j] = nc;
                float *red = m->EB;   // EB[128] and Bpart[3][128], contiguous: [key-dim quarter][token]
                red[quad * kTile + c0 + lane] = dap[0];
                __syncthreads();
                const int tok = n * kTile + tid;
                if (tid < kTile && tok < p.T)
                    p.dlg[((size_t)bc * p.T + tok) * p.H + h] =
                        __float2bfloat16_rn(red[tid] + red[kTile + tid] + red[2 * kTile + tid] + red[3 * kTile + tid]);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    *reinterpret_cast<__nv_bfloat16 *>(DA + eoff(c0 + i)) = __float2bfloat16_rn(dap[i] + carry);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (!kScalar && q4 == 0) m->carry[j] += m->Bpart[0][j] + m->Bpart[1][j] + m->Bpart[2][j] + m->EB[j];
        const int vr = valid_rows(n);
        if (vr == kTile) {
            if (tid == kStoreTid) {   // a thread of another warp than the one issuing loads and MMAs
                for (int c = 0; c < nblk; ++c) {
                    if constexpr (kWide) {   // this block pair's shares, added into the outputs
                        tma_reduce_add_4d(&tm_di, AT + c * kBlk, 64 * c, hv, tok0 + n * kTile, bc);
                        tma_reduce_add_4d(&tm_dlf, DA + c * kBlk, 64 * c, hk, tok0 + n * kTile, bc);
                        tma_reduce_add_4d(&tm_dq, D16 + c * kBlk, 64 * c, hk, tok0 + n * kTile, bc);
                    } else {
                        tma_store_4d(&tm_di, AT + c * kBlk, 64 * c, hv, tok0 + n * kTile, vbc);
                        tma_store_4d(&tm_dlf, DA + c * kBlk, 64 * c, hk, tok0 + n * kTile, kbc);
                        if (kSaved) tma_store_4d(&tm_dq, D16 + c * kBlk, 64 * c, hk, tok0 + n * kTile, kbc);
                    }
                }
                tma_store_commit();
            }
        } else {   // a packed sequence's last chunk: rows 0 .. vr-1 of the three tiles, 16 bytes a thread
            const int nch = 8 * nblk;   // 16-byte chunks per row
            for (int idx = tid; idx < 3 * vr * nch; idx += kRevThreads) {
                const int tsel = idx / (vr * nch), rem = idx - tsel * vr * nch, row = rem / nch, ch = rem - row * nch;
                const uint8_t *tile = tsel == 0 ? AT : tsel == 1 ? DA : D16;
                __nv_bfloat16 *out = tsel == 0 ? p.dx : tsel == 1 ? p.dlf : p.dq;
                const uint4 w = *reinterpret_cast<const uint4 *>(tile + (ch >> 3) * kBlk + row * 128 +
                                                                 (((ch & 7) ^ (row & 7)) << 4));
                *reinterpret_cast<uint4 *>(out + ((size_t)(tok0 + n * kTile + row) * p.H + h) * p.D + 8 * ch) = w;
            }
        }
    }
    if (!ok && tid == 0) set_status(HGRN2_ERR_TIMEOUT);
    if (tid == 0) {   // drain loads that may still be landing in this CTA's shared memory
        uint64_t *bars[3] = {&m->barIn, &m->barVO, &m->barDQ};
        for (int q = 0; q < 3; ++q)
            for (int k = waited[q]; k < issued[q]; ++k) mbar_wait(bars[q], k & 1, 2000000u);
    }
    if (tid == kStoreTid) tma_store_wait_all0();
    // dh0 (or, with segments, the segment's W; its g alongside)
    float *dhout = kSeg ? p.Wseg + ((size_t)bh * p.nseg + seg) * 16384 : p.dh0 ? p.dh0 + (size_t)bh * p.D * p.D : nullptr;
    if (kSeg && ok && n < 0 && q4 == 0) p.gseg[((size_t)bh * p.nseg + seg) * 128 + j] = gprod;
    if (ok && n < 0 && dhout && j < p.D && c0 < p.D) {   // warp-uniform
        tc_fence_after();
        float v[32];
        tmem_ld32(tl + kColDS + c0, v);
        tmem_wait_ld();
        const float e = g_later;   // dh0 = Diag(e^{rho}) dL/dS_r of the first chunk
        float4 *dst = reinterpret_cast<float4 *>(dhout + (size_t)j * p.D + c0);
        float wabs = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 w = make_float4(v[4 * i] * e, v[4 * i + 1] * e, v[4 * i + 2] * e, v[4 * i + 3] * e);
            wabs += (fabsf(w.x) + fabsf(w.y)) + (fabsf(w.z) + fabsf(w.w));
            dst[i] = w;
        }
        if (kSeg && p.Wabs) p.Wabs[(((size_t)bh * p.nseg + seg) * 128 + j) * 4 + q4] = wabs;
    }
    if (tid == 0 && ok && n < 0) atomicAdd(&g_counters[1], (unsigned long long)N);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ backward segments
// With segments, every segment's reverse sweep started from a zero gradient (the last from dhT):
// W_k is the gradient it hands to the state entering it, g_k its decay product.  The gradient
// carried into the last state of segment k from the segments after it is
//   D_{last-1} = W_last,     D_{k-1} = Diag(g_k) D_k + W_k,     dh0 = Diag(g_0) D_0 + W_0.
// In fp32, in place: slot k of W becomes D_{k-1} (k >= 1); slot 0 gives dh0.  Flagged pairs
// (recomputed whole on the exact route) are left alone.  One thread per 4 consecutive elements
// of one (batch, head); the maps are loaded 16 segments at a time.  A programmatic dependent of
// the segments' kernel.  Used beyond kBwdMergedMax segments per pair; with fewer, the fix-up
// sums what it needs of the maps itself.
__global__ void __launch_bounds__(256)
bwd_scan_kernel(float *__restrict__ W, const float *__restrict__ g, int nseg, const int *__restrict__ flags,
                float *__restrict__ dh0) {
    grid_dep_launch();
    grid_dep_wait();
    const int bh = blockIdx.x >> 4;
    if (flags[bh]) return;
    const int e = ((blockIdx.x & 15) * 256 + threadIdx.x) * 4;
    const int jrow = e >> 7;
    constexpr int kBatch = 16;
    float4 D = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = nseg - 1; s0 >= 0; s0 -= kBatch) {
        float4 wv[kBatch];
        float gj[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            if (s0 - i >= 0) {
                const size_t slot = (size_t)bh * nseg + s0 - i;
                wv[i] = *reinterpret_cast<const float4 *>(W + slot * 16384 + e);
                gj[i] = g[slot * 128 + jrow];
            }
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int sg = s0 - i;
            if (sg >= 0) {
                D = make_float4(fmaf(gj[i], D.x, wv[i].x), fmaf(gj[i], D.y, wv[i].y), fmaf(gj[i], D.z, wv[i].z),
                                fmaf(gj[i], D.w, wv[i].w));
                if (sg > 0) *reinterpret_cast<float4 *>(W + ((size_t)bh * nseg + sg) * 16384 + e) = D;
                else if (dh0) *reinterpret_cast<float4 *>(dh0 + (size_t)bh * 16384 + e) = D;
            }
        }
    }
}

// The gradient D carried into the last state of segment k < last from later segments reaches its
// tokens through the decays since: at token t of a chunk (b_t the cumulative log decay from the
// chunk start, B its total) the state gradient misses Diag(e^{B - b_t}) D.  So, per chunk from the
// segment's end (k_t = 1 - f_t, i_t the input, S_in the state entering the chunk):
//   di_t       += D^T (k_t * e^{B - b_t})
//   dK_t[j]     = e^{B - b_t[j]} (D i_t)[j]           (the missing part of dL/dk_t)
//   d log f_t  += e^{B} rowsum(S_in * D) + sum_{s<t} k_s dK_s - f_t dK_t
//   D          <- Diag(e^{B}) D                        (into the chunk before)
// (the d log f term is f_t rowsum(S_{t-1} * missing gradient of S_t), written with the forward
// state S_{t-1} expanded over the chunk; it decays with D, so nothing beyond the walked chunks
// changes).  The saved state holds bf16(e^{rho} S_in), rho = B/2, so e^{B} rowsum(S_in * D) =
// e^{B - rho} rowsum(S_r * D).  Two MMAs per chunk: DI = Kd bf16(D) (lane t) and
// Y^T = bf16(D) I^T (lane j), Kd = k e^{B - b}.  One CTA per segment k < last walks its chunks from
// the end while max_j decay_j max |D[j,:]| >= kFixStop (as the forward's fix-up); di and d log f are
// read, corrected and stored back.  8 warps: thread (row r, half) holds 64 columns of row r of D.
// D_k is the scan's, or, with up to kBwdMergedMax segments (merged), summed here from the maps,
// nearest first: D_k = sum_{m>k} Diag(w_m) W_m, w_m = prod_{k<l<m} g_l, each thread for its own
// row r while w_m (nseg - m) M[r] >= kStop, M[r] = max_{m>k} sum_v |W_m[r,v]| (the maps left out
// add less than that to any entry, as in the forward's fix-up).  Segment 0's CTA then writes
// dh0 = Diag(g_0) D_0 + W_0.
namespace bfx {
constexpr float kStop = 0x1p-24f;
constexpr int kBwdMergedMax = 18;   // segments per pair up to which the fix-up sums D itself
struct Misc {
    uint64_t fullA, fullB, barM;   // A: i and the saved state; B: log f, di, d log f
    uint32_t tmem_base;
    int pad;
    float Ppart[4][128];   // 32-row range sums of log f
    float BT[128];         // the chunk's total log decay B, key dim
    float Rp[2][128];      // halves of rowsum(S_r * D)
    float Pre0[128];       // the first 64 tokens' sum of k dK, key dim
};
// log f, i, saved state (then Kd), di, d log f, bf16(D)
constexpr size_t kSmem = 6 * (size_t)kTileBytes + sizeof(Misc);
}  // namespace bfx

struct BwdFixParams {
    const float *D;     // [B*H][nseg][128][128]: slot k+1 = the gradient carried into segment k's end
                        // (the scan's), or (merged) the segments' maps W
    const int *flags;
    int H, nseg, tps, ntiles;
    bool merged;
    const float *g;     // merged: [B*H][nseg][128] the segments' decay products
    const float *Wabs;  // merged: [B*H][nseg][128][4] quarter sums of |W| per row
    float *dh0;         // merged: dh0 [B*H][128][128] (may be null)
};

__global__ void __launch_bounds__(256, 1)
bwd_fixup_kernel(const __grid_constant__ CUtensorMap tm_lf, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_st, const __grid_constant__ CUtensorMap tm_di,
                 const __grid_constant__ CUtensorMap tm_dlf, BwdFixParams p) {
    using namespace bfx;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *Lb = smem, *Ib = smem + kTileBytes, *Sb = smem + 2 * kTileBytes, *DIb = smem + 3 * kTileBytes;
    uint8_t *DLb = smem + 4 * kTileBytes, *X = smem + 5 * kTileBytes;
    uint8_t *Kd = Sb;   // once rowsum(S_r * D) has been formed
    Misc *m = reinterpret_cast<Misc *>(smem + 6 * kTileBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nfix = p.nseg - 1;
    const int bh = blockIdx.x / nfix, seg = blockIdx.x - bh * nfix, b = bh / p.H, h = bh - b * p.H;
    const int g0 = seg * p.tps, N = p.tps;   // a segment before the last: tps whole chunks
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    if (tid == 0) {
        mbar_init(&m->fullA, 1);
        mbar_init(&m->fullB, 1);
        mbar_init(&m->barM, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_lf);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_st);
        tma_prefetch_desc(&tm_di);
        tma_prefetch_desc(&tm_dlf);
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;
    const int quad = warp & 3, ch = warp >> 2, r = 32 * quad + lane;
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
    const uint32_t id_kk = idesc_bf16(128, 128, false, false);
    const uint32_t id_kmn = idesc_bf16(128, 128, false, true);
    const int pc = tid & 63, rr = tid >> 6, col0 = 2 * pc;   // prep: column pair, 32-row range
    const uint32_t cblk = (uint32_t)(col0 >> 6) * kBlk, cch = (uint32_t)((col0 & 63) >> 3), cin = (uint32_t)(col0 & 7) * 2;
    auto eoff = [&](int t) -> uint32_t { return cblk + t * 128 + ((cch ^ (t & 7)) << 4) + cin; };
    // element (t, j) of a tile (lane j's column)
    const uint32_t jblk = (uint32_t)(r >> 6) * kBlk, jch = (uint32_t)((r & 63) >> 3), jin = (uint32_t)(r & 7) * 2;
    auto joff = [&](int t) -> uint32_t { return jblk + t * 128 + ((jch ^ (t & 7)) << 4) + jin; };
    // Loads per chunk, in two groups: A (i, the saved state) once the chunk before's MMAs have read
    // Ib and Sb; B (log f, di, d log f) once its epilogue and stores are done (prefetched to L2
    // while it is on the tensor cores).  Counted in chunks walked.
    int issuedA = 0, issuedB = 0, waited = 0;
    auto load_a = [&](int c) {   // thread 0: chunk g0 + c
        const int tok = (g0 + c) * kTile, slot = bh * p.ntiles + g0 + c;
        mbar_arrive_expect_tx(&m->fullA, 2 * kTileBytes);
        for (int k = 0; k < 2; ++k) {
            tma_load_4d(Ib + k * kBlk, &tm_x, &m->fullA, 64 * k, h, tok, b);
            tma_load_4d(Sb + k * kBlk, &tm_st, &m->fullA, 64 * k, 0, 0, slot);
        }
        ++issuedA;
    };
    auto load_b = [&](int c) {
        const int tok = (g0 + c) * kTile;
        mbar_arrive_expect_tx(&m->fullB, 3 * kTileBytes);
        for (int k = 0; k < 2; ++k) {
            tma_load_4d(Lb + k * kBlk, &tm_lf, &m->fullB, 64 * k, h, tok, b);
            tma_load_4d(DIb + k * kBlk, &tm_di, &m->fullB, 64 * k, h, tok, b);
            tma_load_4d(DLb + k * kBlk, &tm_dlf, &m->fullB, 64 * k, h, tok, b);
        }
        ++issuedB;
    };

    grid_dep_wait();   // the segments' outputs and the scan's gradients are complete from here on
    const bool flagged = p.flags[bh] != 0;
    if (!flagged && tid == 0) {   // the last chunk's tiles, while the carried gradient is read
        load_a(N - 1);
        load_b(N - 1);
    }
    float Dr[64];      // the carried gradient, row r, columns 64 ch .. 64 ch + 63
    float dmax = 0.0f, decay = 1.0f;
    const size_t s0 = (size_t)bh * p.nseg;
    if (!p.merged) {
        const float4 *src = reinterpret_cast<const float4 *>(p.D + (s0 + seg + 1) * 16384 + (size_t)r * 128 + 64 * ch);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 a = src[i];
            Dr[4 * i] = a.x; Dr[4 * i + 1] = a.y; Dr[4 * i + 2] = a.z; Dr[4 * i + 3] = a.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) Dr[i] = 0.0f;
    }
    if (p.merged && !flagged) {
        // map m = seg+1+i, row r: x[i] = sum_v |W_m[r,v]|, loaded at once (indices clamped to the
        // last segment, the extra values unused); M = max over the later segments (NaN kept); the
        // maps m' >= m add at most w_m (nseg - m) M to an entry of row r
        constexpr int kMaps = kBwdMergedMax - 1;
        const int nl = p.nseg - 1 - seg;   // later segments
        float xr[kMaps];
#pragma unroll
        for (int i = 0; i < kMaps; ++i) {
            const float4 a = *reinterpret_cast<const float4 *>(p.Wabs + ((s0 + (size_t)min(seg + 1 + i, p.nseg - 1)) * 128 + r) * 4);
            xr[i] = (a.x + a.y) + (a.z + a.w);
        }
        float M = 0.0f;
#pragma unroll
        for (int i = 0; i < kMaps; ++i)
            if (i < nl) M = (xr[i] > M || isnan(xr[i])) ? xr[i] : M;
        float w = 1.0f;
        for (int i = 0; i < nl; ++i) {
            if (w * ((float)(nl - i) * M) < kStop) break;   // false for NaN: the row walks on
            const size_t sl = s0 + seg + 1 + i;
            const float4 *src = reinterpret_cast<const float4 *>(p.D + sl * 16384 + (size_t)r * 128 + 64 * ch);
            const float gm = p.g[sl * 128 + r];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float4 a = src[k];
                Dr[4 * k] = fmaf(w, a.x, Dr[4 * k]); Dr[4 * k + 1] = fmaf(w, a.y, Dr[4 * k + 1]);
                Dr[4 * k + 2] = fmaf(w, a.z, Dr[4 * k + 2]); Dr[4 * k + 3] = fmaf(w, a.w, Dr[4 * k + 3]);
            }
            w *= gm;
        }
        if (seg == 0 && p.dh0) {   // dh0 = Diag(g_0) D_0 + W_0
            const float gz = p.g[s0 * 128 + r];
            const float4 *src = reinterpret_cast<const float4 *>(p.D + s0 * 16384 + (size_t)r * 128 + 64 * ch);
            float4 *dst = reinterpret_cast<float4 *>(p.dh0 + (size_t)bh * 16384 + (size_t)r * 128 + 64 * ch);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float4 a = src[i];
                dst[i] = make_float4(fmaf(gz, Dr[4 * i], a.x), fmaf(gz, Dr[4 * i + 1], a.y),
                                     fmaf(gz, Dr[4 * i + 2], a.z), fmaf(gz, Dr[4 * i + 3], a.w));
            }
        }
    }
    if (!flagged) {
#pragma unroll
        for (int i = 0; i < 64; ++i) dmax = fmaxf(dmax, fabsf(Dr[i]));
    }
    bool ok = true;
    bool go = !flagged && __syncthreads_or(dmax >= kStop);
    for (int c = N - 1; go && c >= 0; --c) {
        const int tok = (g0 + c) * kTile;
        // bf16(D) -> X (row r = key dim, columns = value dims)
        {
            float v[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = Dr[32 * hh + i];
                store_chunk_bf16(X, r, 2 * ch + hh, v);
            }
        }
        if (__syncthreads_or(!mbar_wait(&m->fullA, waited & 1) || !mbar_wait(&m->fullB, waited & 1))) {
            ok = false;
            break;
        }
        ++waited;
        // rowsum(S_r * D), this thread's half of row r
        {
            float acc = 0.0f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int cc = 2 * ch + hh;
                const uint8_t *base = Sb + (cc >> 1) * kBlk + r * 128;
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(base + (((4 * (cc & 1) + qd) ^ (r & 7)) << 4));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        acc = fmaf(bf_lo(ws[k]), Dr[32 * hh + 8 * qd + 2 * k], acc);
                        acc = fmaf(bf_hi(ws[k]), Dr[32 * hh + 8 * qd + 2 * k + 1], acc);
                    }
                }
            }
            m->Rp[ch][r] = acc;
        }
        // prep: range sums of log f; B (summed as the forward's prep sums it); Kd = k e^{B - b}
        // over the saved state's tile (read above)
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(Lb + eoff(32 * rr + i));
            s0 += bf_lo(w);
            s1 += bf_hi(w);
        }
        m->Ppart[rr][col0] = s0;
        m->Ppart[rr][col0 + 1] = s1;
        __syncthreads();   // Ppart complete; every thread has read S_r
        {
            float b0 = 0.0f, b1 = 0.0f;
            for (int r2 = 0; r2 < rr; ++r2) {
                b0 += m->Ppart[r2][col0];
                b1 += m->Ppart[r2][col0 + 1];
            }
            const float B0 = ((m->Ppart[0][col0] + m->Ppart[1][col0]) + m->Ppart[2][col0]) + m->Ppart[3][col0];
            const float B1 = ((m->Ppart[0][col0 + 1] + m->Ppart[1][col0 + 1]) + m->Ppart[2][col0 + 1]) +
                             m->Ppart[3][col0 + 1];
            if (rr == 0) {
                m->BT[col0] = B0;
                m->BT[col0 + 1] = B1;
            }
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                const int t = 32 * rr + i;
                const uint32_t wa = *reinterpret_cast<const uint32_t *>(Lb + eoff(t));
                b0 += bf_lo(wa);
                b1 += bf_hi(wa);
                const float k0 = 1.0f - __expf(bf_lo(wa)), k1 = 1.0f - __expf(bf_hi(wa));
                *reinterpret_cast<uint32_t *>(Kd + eoff(t)) = pack_bf2(k0 * __expf(B0 - b0), k1 * __expf(B1 - b1));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();   // Kd, X, B, rowsum halves complete
        if (tid == 0) {    // DI = Kd bf16(D) (cols 0..127, lane t); Y^T = bf16(D) I^T (cols 128..255, lane j)
            tc_fence_after();
            const uint64_t dK = sdesc_sw128(smem_u32(Kd), 16, 1024);
            const uint64_t dXm = sdesc_sw128(smem_u32(X), kBlk, 1024);
            const uint64_t dXk = sdesc_sw128(smem_u32(X), 16, 1024);
            const uint64_t dI = sdesc_sw128(smem_u32(Ib), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase, sdesc_add(dK, ko), sdesc_add(dXm, kk * 2048), id_kmn, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase + 128, sdesc_add(dXk, ko), sdesc_add(dI, ko), id_kk, kk > 0);
            }
            mma_commit(&m->barM);
            if (c > 0) {   // the chunk before's log f, di, d log f into L2 for its loads after the stores
                const int tp = (g0 + c - 1) * kTile;
                for (int k = 0; k < 2; ++k) {
                    tma_prefetch_l2_4d(&tm_lf, 64 * k, h, tp, b);
                    tma_prefetch_l2_4d(&tm_di, 64 * k, h, tp, b);
                    tma_prefetch_l2_4d(&tm_dlf, 64 * k, h, tp, b);
                }
            }
        }
        if (__syncthreads_or(!mbar_wait(&m->barM, (N - 1 - c) & 1))) { ok = false; break; }   // chunk N-1-c walked
        tc_fence_after();
        // whether the chunk before will be walked: the carried gradient after this chunk's decay
        const bool next = __syncthreads_or(decay * __expf(m->BT[r]) * dmax >= kStop) && c > 0;
        if (next && tid == 0) load_a(c - 1);   // Ib and Sb were read by the MMAs above
        // di row r (token) += DI row r: this half's 64 columns
#pragma unroll 1
        for (int cc = 2 * ch; cc < 2 * ch + 2; ++cc) {
            float v[32];
            tmem_ld32(tl + 32 * cc, v);
            tmem_wait_ld();
            const uint8_t *base = DIb + (cc >> 1) * kBlk + r * 128;
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
                const uint4 w = *reinterpret_cast<const uint4 *>(base + (((4 * (cc & 1) + qd) ^ (r & 7)) << 4));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[8 * qd + 2 * k] += bf_lo(ws[k]);
                    v[8 * qd + 2 * k + 1] += bf_hi(ws[k]);
                }
            }
            store_chunk_bf16(DIb, r, cc, v);
        }
        // d log f column r (key dim), this half's 64 tokens in order, 32 at a time: their log f and
        // d log f first, then the running sums in registers.  The second half's sum of k dK
        // starts from the first half's total, exchanged through shared memory.
        {
            const float Bt = m->BT[r];
            const float rho = 0.5f * Bt;
            const float base = __expf(Bt - rho) * (m->Rp[0][r] + m->Rp[1][r]);   // e^{B} rowsum(S_in * D)
            float bsum = ch ? m->Ppart[0][r] + m->Ppart[1][r] : 0.0f;   // log decay before the half
            float pre = 0.0f;
            float dv[64];   // d log f + this half's own terms
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int t0 = 64 * ch + 32 * cb;
                float y[32], av[32];
                tmem_ld32(tl + 128 + t0, y);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    av[i] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(Lb + joff(t0 + i)));
                    dv[32 * cb + i] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(DLb + joff(t0 + i)));
                }
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    bsum += av[i];
                    const float f = __expf(av[i]);
                    const float dK = __expf(Bt - bsum) * y[i];
                    dv[32 * cb + i] += pre - f * dK;
                    pre = fmaf(1.0f - f, dK, pre);
                }
            }
            if (ch == 0) m->Pre0[r] = pre;
            __syncthreads();
            const float off = base + (ch ? m->Pre0[r] : 0.0f);
#pragma unroll
            for (int i = 0; i < 64; ++i)
                *reinterpret_cast<__nv_bfloat16 *>(DLb + joff(64 * ch + i)) = __float2bfloat16_rn(dv[i] + off);
        }
        // the carried gradient into the chunk before
        const float eb = __expf(m->BT[r]);
        decay *= eb;
#pragma unroll
        for (int i = 0; i < 64; ++i) Dr[i] *= eb;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            for (int k = 0; k < 2; ++k) {
                tma_store_4d(&tm_di, DIb + k * kBlk, 64 * k, h, tok, b);
                tma_store_4d(&tm_dlf, DLb + k * kBlk, 64 * k, h, tok, b);
            }
            tma_store_commit();
            if (next) {   // log f, di, d log f tiles, once this chunk's stores have read them
                tma_store_wait_read0();
                load_b(c - 1);
            }
        }
        go = next;
    }
    if (tid == 0) {
        if (!ok) set_status(HGRN2_ERR_TIMEOUT);
        // loads still landing: the last chunk's when nothing was walked, or any after a timeout
        for (int k = waited; k < issuedA; ++k) mbar_wait(&m->fullA, k & 1, 2000000u);
        for (int k = waited; k < issuedB; ++k) mbar_wait(&m->fullB, k & 1, 2000000u);
        tma_store_wait_all0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

}  // namespace tcb

static_assert(tcb::fsw::kSmemBytes <= 227 * 1024, "forward-sweep shared memory");
static_assert(tcb::rsw::kSmemBytes <= 227 * 1024, "reverse-sweep shared memory");

static_assert(tcb::bfx::kSmem <= 227 * 1024, "backward fix-up shared memory");

size_t tc_bwd_workspace(int B, int T, int H) {
    int nseg, tps;
    tc_fwd_segments(B, T, H, &nseg, &tps);   // the forward's cut
    // per segment: W, g and the quarter sums of |W| per row
    return nseg > 1 ? (size_t)B * H * nseg * (16384 + 128 + 512) * sizeof(float) : 0;
}
int tc_bwd_launches(int B, int T, int H) {
    int nseg, tps;
    tc_fwd_segments(B, T, H, &nseg, &tps);
    return tc_bwd_workspace(B, T, H) ? (nseg <= tcb::bfx::kBwdMergedMax ? 2 : 3) : 1;
}

// Launches a kernel as a programmatic dependent of the previous work in the stream: it may be
// scheduled before that work completes, and waits for it with grid_dep_wait().
template <typename... Exp, typename... Act>
static cudaError_t launch_dependent_b(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      Act &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

size_t tc_bwd_smem() { return tcb::fsw::kSmemBytes > tcb::rsw::kSmemBytes ? tcb::fsw::kSmemBytes : tcb::rsw::kSmemBytes; }

cudaError_t launch_tc_bwd(const TcBwdArgs &a, cudaStream_t st) {
    const bool saved = a.st16 != nullptr;
    const bool packed = a.cu != nullptr;   // saved mode only; a.B is then the number of sequences
    if ((packed || a.D != 128 || a.lgs) && !saved) return cudaErrorInvalidValue;
    if (a.lgs && packed) return cudaErrorInvalidValue;
    const int nbk = a.nK * a.nV;
    const bool inplace = nbk > 1;
    if (inplace && (!saved || packed || a.lgs || a.D != 128 || a.nK != a.nV || a.H % nbk || !a.dq_part ||
                    !a.dlf_part || !a.dx_part))
        return cudaErrorInvalidValue;
    const int Hk = inplace ? a.H / nbk * a.nK : a.H, Hv = inplace ? a.H / nbk * a.nV : a.H;
    const int Bm = packed ? 1 : a.B, D = a.D;
    const int ntiles = (a.T + tcc::kTile - 1) / tcc::kTile;
    CUtensorMap mq, ml, mx, mdo, mdq, mdi, mdl, mst;
    if (!make_token_map(&mq, a.q, Bm, a.T, Hk, D) || !make_token_map(&ml, a.lf, Bm, a.T, Hk, D) ||
        !make_token_map(&mx, a.x, Bm, a.T, Hv, D) || !make_token_map(&mdo, a.dO, Bm, a.T, Hv, D) ||
        !make_token_map(&mdq, a.dq, Bm, a.T, Hk, D) || !make_token_map(&mdi, a.dx, Bm, a.T, Hv, D) ||
        !make_token_map(&mdl, a.dlf, Bm, a.T, Hk, D))
        return cudaErrorInvalidValue;
    // saved states: 128-row "token" tiles
    if (saved && !make_token_map(&mst, a.st16, tc_saved_slots(a.B, a.T, a.H, packed), 128, 1))
        return cudaErrorInvalidValue;
    if (!saved) mst = mq;   // unused
    tcb::RevParams p2{a.dhT, a.rs, a.dh0, a.flags, a.T, a.H, ntiles, a.hTs, a.h0,
                      (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.lf, (const __nv_bfloat16 *)a.x,
                      (const __nv_bfloat16 *)a.dO, (__nv_bfloat16 *)a.dq, (__nv_bfloat16 *)a.dlf,
                      (__nv_bfloat16 *)a.dx, a.simt_C, a.cu, a.perm, D, (const __nv_bfloat16 *)a.lgs,
                      (__nv_bfloat16 *)a.dlg, a.nK, a.nV, Bm, (__nv_bfloat16 *)a.dq_part,
                      (__nv_bfloat16 *)a.dlf_part, (__nv_bfloat16 *)a.dx_part, 1, ntiles, nullptr, nullptr};
    cudaError_t e;
    int nseg = 1, tps = ntiles;
    if (saved && !packed && !a.lgs && !inplace && D == 128 && a.seg_ws) tc_fwd_segments(a.B, a.T, a.H, &nseg, &tps);
    if (nseg > 1) {
        // sequence segments: every segment from a zero gradient (the last from dhT), the reverse
        // scan of their maps (and dh0) unless the fix-up sums them itself, then the carried
        // gradients added to each segment's last chunks
        const int BH = a.B * a.H;
        float *W = a.seg_ws, *g = a.seg_ws + (size_t)BH * nseg * 16384, *Wabs = g + (size_t)BH * nseg * 128;
        const bool merged = nseg <= tcb::bfx::kBwdMergedMax;
        p2.nseg = nseg;
        p2.tps = tps;
        p2.Wseg = W;
        p2.gseg = g;
        p2.Wabs = Wabs;
        size_t smem = tcb::rsw::kSmemBytes;
        if (simt_bwd_dq_smem(a.simt_C, D, D) > smem) smem = simt_bwd_dq_smem(a.simt_C, D, D);
        if (simt_bwd_rev_smem(a.simt_C, D, D) > smem) smem = simt_bwd_rev_smem(a.simt_C, D, D);
        auto kern = tcb::rev_kernel<true, false, false, false, true>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        kern<<<BH * nseg, tcb::rsw::kRevThreads, smem, st>>>(mq, ml, mx, mdo, mdq, mdi, mdl, mst, p2);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (!merged) {
            e = launch_dependent_b(tcb::bwd_scan_kernel, dim3(BH * 16), dim3(256), 0, st, W, (const float *)g, nseg,
                                   (const int *)a.flags, a.dh0);
            if (e != cudaSuccess) return e;
        }
        if ((e = cudaFuncSetAttribute(tcb::bwd_fixup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)tcb::bfx::kSmem)) != cudaSuccess)
            return e;
        tcb::BwdFixParams fp{W, a.flags, a.H, nseg, tps, ntiles, merged, g, Wabs, a.dh0};
        return launch_dependent_b(tcb::bwd_fixup_kernel, dim3(BH * (nseg - 1)), dim3(256), tcb::bfx::kSmem, st, ml,
                                  mx, mst, mdi, mdl, fp);
    }
    if (saved) {
        // one launch; the exact route of a flagged (b,h) runs in the same shared memory
        size_t smem = tcb::rsw::kSmemBytes;
        if (simt_bwd_dq_smem(a.simt_C, D, D) > smem) smem = simt_bwd_dq_smem(a.simt_C, D, D);
        if (simt_bwd_rev_smem(a.simt_C, D, D) > smem) smem = simt_bwd_rev_smem(a.simt_C, D, D);
        auto kern = packed ? tcb::rev_kernel<true, true>
                    : a.lgs ? tcb::rev_kernel<true, false, true>
                    : inplace ? tcb::rev_kernel<true, false, false, true> : tcb::rev_kernel<true, false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<a.B * a.H, tcb::rsw::kRevThreads, smem, st>>>(mq, ml, mx, mdo, mdq, mdi, mdl, mst, p2);
        return cudaGetLastError();
    }
    e = cudaFuncSetAttribute(tcb::dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tcb::fsw::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tcb::rev_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tcb::rsw::kSmemBytes);
    if (e != cudaSuccess) return e;
    tcb::DqParams p1{a.h0, a.dhT, a.rs, a.flags, a.T, a.H, ntiles,
                     (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.lf, (const __nv_bfloat16 *)a.x,
                     (const __nv_bfloat16 *)a.dO, (__nv_bfloat16 *)a.dq, (__nv_bfloat16 *)a.dlf,
                     (__nv_bfloat16 *)a.dx, a.dh0, a.simt_C};
    tcb::dq_kernel<<<a.B * a.H, tcb::fsw::kDqThreads, tcb::fsw::kSmemBytes, st>>>(ml, mx, mdo, mdq, p1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    tcb::rev_kernel<false, false><<<a.B * a.H, tcb::rsw::kRevThreads, tcb::rsw::kSmemBytes, st>>>(mq, ml, mx, mdo, mdq, mdi,
                                                                                           mdl, mst, p2);
    return cudaGetLastError();
}

}  // namespace hgrn2
