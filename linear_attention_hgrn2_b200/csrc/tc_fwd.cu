// tc_fwd.cu -- chunkwise HGRN2 forward on 5th-generation tensor cores (sm_100a).
//
// One CTA walks the 128-token chunks of one (batch, head) (or of one segment of
// it); d_k = d_v = 128, bf16 token tensors, fp32 state.  Per chunk and key dim j,
// with b_t the cumulative log decay from the chunk start, B = b at the chunk end,
// the reference rho = B / 2, E_t = e^{b_t - rho}, k = 1 - f and S_in the state
// entering the chunk ("HGRN2: Gated Linear RNNs with State Expansion", §3.2: gated
// linear attention with key 1 - f, value i, query q, so chunkwise; §5:
// per-dimension decay):
//
//   Qt = q * E,  Kt = k / E                                    (bf16 in smem)
//   S_r = Diag(e^rho) S_in                                     fp32 state in TMEM
//   A  = mask_{s<=t}(Qt Kt^T)                                  tcgen05, fp32 in TMEM
//   O  = Qt bf16(S_r) + bf16(A) V                              tcgen05, fp32 in TMEM
//   S' = S_r + Kt^T V,   S_out = Diag(e^{B - rho}) S'          fp32 state in TMEM
//
// Qt Kt^T realises sum_j q_t[j] k_s[j] e^{b_t[j] - b_s[j]} through factors referenced
// to rho, and Qt S_r realises sum_j q_t[j] e^{b_t[j]} S_in[j, :].  With rho = B / 2 (a
// balanced reference, the stabilising second level of the chunk form: the decay is
// split at the middle of its range instead of at the chunk start) every factor lies
// in [e^{B/2}, e^{-B/2}], which halves the exponent range of the start-referenced
// form.  A chunk is valid while B / 2 >= -75 for every key dim (an average log f of
// -1.17 per token over the chunk; a first layer with lower bound 0 sums to about
// -103 +- 6); a (batch, head) meeting a chunk beyond that is flagged and
// recomputed afterwards by the exact CUDA-core route, which forms every exponent
// as a difference of cumulative sums.
//
// For training, the forward can also keep what the backward needs: bf16(S_r) of every
// chunk (the operand it builds anyway for the inter-chunk MMA, written out by a TMA store)
// and the fp32 final state.
//
// The two state scales of consecutive chunks are applied together: the next chunk's S
// phase multiplies the rows by e^{B_n - rho_n} e^{rho_{n+1}} = e^{(B_n + B_{n+1}) / 2} <= 1
// before building its operand (the products of Kt with these scales are never formed in
// bf16 at all).
//
// Warp roles (16 warps), coordinated by mbarriers only:
//   warp 0      TMA producer: q, log f, i tiles (128-byte swizzle) into a 2-stage ring; q and
//               log f of a stage are refilled as soon as the state MMA has read Qt and Kt,
//               i once the last MMA of the chunk has read it
//   warp 1      TMEM allocator and the single MMA-issuing thread
//   warps 4-7   TMEM warps (one thread per TMEM lane): S phase (bf16 copy of S_in,
//               Diag(E_B) scale), causal mask of A (bf16 pairs back into TMEM: the intra
//               MMA reads its A operand from TMEM), o epilogue (staged in smem, TMA store)
//   warps 8-15  prep warps: f, E, k, Qt, Kt for the next chunk while the current one
//               is on the tensor cores
// Every wait is bounded; a wait that gives up records HGRN2_ERR_TIMEOUT.
#include <climits>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace hgrn2 {
namespace tcf {

using namespace tc;
using namespace tcc;

constexpr int kThreads = 256;        // aggregate kernel
constexpr int kFwdThreads = 512;     // forward kernel: 16 warps
constexpr uint32_t kColS = 0, kColO = 128, kColA = 256, kColP = 384, kTmemCols = 512;   // P: bf16 mask(A)

struct __align__(8) Misc {
    uint64_t fullQG[2], fullV[2], prepped[2];   // stage s: q and log f / i landed; prep done
    uint64_t emptyQG[2], emptyV[2];             // stage s: Qt, Kt / v read by every MMA of its chunk
    uint64_t barA, barO1, barS, barO2;      // MMA completions (tcgen05.commit)
    uint64_t sdone, adone, ofree;           // TMEM-warp arrivals (128 each)
    uint32_t tmem_base;
    int bad_tile;                           // first chunk whose decay span is too wide
    int waited_full;                        // q / log f arrivals the prep warps consumed
    int waited_v;                           // v arrivals the MMA thread consumed
    float EB[2][128];                       // E_B ring: read by the TMEM warps while that chunk is current
    float Ppart[3][128];                    // per 32-row range sums of log f (ranges 0..2; range 3's
                                            // sums go to the stage's EB slot until the prep ends)
};

constexpr size_t kSmemBytes = 7 * (size_t)kTileBytes + sizeof(Misc);

struct Params {
    const float *h0;
    float *hT;
    __nv_bfloat16 *o;
    const __nv_bfloat16 *q, *lf, *x;   // for the in-kernel exact route
    int simt_chunk;
    int *flags;       // [B*H] set to 1 when the (b,h) must take the exact route
    float *Useg;      // with segments: [B*H][nseg][128][128] every segment's final state from its start
                      // state (zero; h0 for segment 0), for the scan
    float *gseg;      // with segments: [B*H][nseg][128] every segment's decay product (0 for segment 0)
    int T, H, ntiles;
    int nseg, tps;    // sequence segments per (b,h) and chunks per segment
    bool save;        // store bf16(S_in) of every chunk through tm_st
    float *hTs;       // with save: the final state [B*H][128][128]
    const int *cu;    // packed sequences (or null): sequence s at tokens cu[s] .. cu[s+1]-1 of a
                      // [1][T][H][128] tensor; CTA (r,h) runs sequence perm[r]; no segments
    const int *perm;
    int D;            // head size d_k = d_v: 128, or 64 (the second 64-column half of every operand
                      // tile is held at zero: log f = 0, q = i = 0 there, exactly neutral)
    const __nv_bfloat16 *lgs;   // scalar-decay variant: log g [B][T][H]; tm_lf then maps the key k
    int *seg_done;    // with segments: [B*H] segments of the pair finished (zeroed before the launch)
    // Heads of width 256 read in place: head h of the call is block pair (a, c) of head
    // h / (nK nV) of the caller's [B][T][Hw][256] tensors, a = key block, c = value block.  Those
    // are read as [B][T][Hw nK][128] (q, log f: half-head Hw-index * nK + a) and [B][T][Hw nV][128]
    // (i: * nV + c).  Every block pair adds its share of o into o ([B][T][Hw nV][128], zeroed by the
    // host) by TMA reduce-add; a flagged pair's exact route writes its share into its key block's
    // partial of opart ([nK][B][T][Hw nV][128]) and adds it from there.  nK = nV = 1 otherwise.
    int nK, nV, Bo;   // Bo: the batch count of one o partial
    // With segments, for the carried-state fix-up of segments k >= 1: bf16(q e^{b}) of the
    // segment's first chunk ([B*H][nseg][128][128], b the cumulative log f from the chunk start)
    // and that chunk's total log decay B ([B*H][nseg][128])
    __nv_bfloat16 *qtil;
    float *bseg;
    __nv_bfloat16 *opart;   // heads read in place: the exact route's partial outputs
    // Final states (hT, the saved final state, or a segment's U) leave through shared memory by
    // TMA: tm_h1 / tm_h2 map them as fp32 [rows][128] (bit 0 / bit 1 of hmaps set when mapped;
    // d = 128 only); h1row0 / h2row0: this CTA's first row = its slot times 128.
    int hmaps;
    int hslot1, hslot2;   // 0: the pair's index; 1: the segment slot (b,h) nseg + seg
    // With segments: [B*H][nseg][128] sum_v |U[j,v]| of every segment's U, row j (the fix-up's
    // bound on what the maps it leaves out could add; a sum, so that inf and NaN carry into it)
    float *uabs;
};

// kPacked: p.cu holds packed sequences (compiled apart so the dense path carries no row masks).
// kScalar: the scalar-decay variant S_t = g_t S_{t-1} + k_t v_t^T (one decay per head and token,
// key k loaded in place of log f).  The same chunk form with a decay shared by the key dims:
// b_t = cumulative log g from the chunk start, rho = B / 2, Qt = q e^{b_t - rho}, Kt = k e^{rho - b_t}
// (per-row factors), the state scales e^{B/2} for every state row.  A chunk with B / 2 < -kMaxRefLog
// sends the pair to the exact CUDA-core forward (its flag also routes the backward).
// kSeg: dense launches with sequence segments (the first chunk's q e^{b} and B are written for the
// fix-up), compiled apart from the one-CTA-per-pair instance.
template <bool kPacked, bool kScalar = false, bool kSeg = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_lf,
           const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_o,
           const __grid_constant__ CUtensorMap tm_st, const __grid_constant__ CUtensorMap tm_h1,
           const __grid_constant__ CUtensorMap tm_h2, Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *Qb[2] = {smem, smem + 3 * kTileBytes};
    uint8_t *Gb[2] = {smem + kTileBytes, smem + 4 * kTileBytes};
    uint8_t *Vb[2] = {smem + 2 * kTileBytes, smem + 5 * kTileBytes};
    uint8_t *X = smem + 6 * kTileBytes;
    Misc *m = reinterpret_cast<Misc *>(smem + 7 * kTileBytes);

    // (kSeg: no early trigger of the dependent scan or fix-up; it launches as this grid's CTAs
    // exit.  Triggered at this kernel's start, the fix-up's CTAs took the SMs this grid leaves free
    // and waited there, and the calls measured slower: A/B on one B200, forward layer 48.4 -> 45.8
    // us, long sequence 128.1 -> 119.9 us without the trigger.)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int bh = blockIdx.x / p.nseg;
    const int seg = blockIdx.x - bh * p.nseg, h = bh % p.H;
    const int g0 = seg * p.tps;                                   // first chunk of this segment
    // token of chunk n: tok0 + n * kTile of batch bc; saved-state slot: slot0 + n * sstride.
    // Packed sequences: rows from the sequence's end on (valid(n) < kTile) are masked in the
    // prep and not stored; a sequence may start at any token.
    int b = bh / p.H, bc = b, tok0 = g0 * kTile, len = p.T, N = min(p.ntiles - g0, p.tps);
    int slot0 = bh * p.ntiles + g0, sstride = 1;
    if (kPacked) {
        const int sq = packed_seq(p.perm, bh / p.H, gridDim.x / p.H);
        bh = sq * p.H + h;   // the pair whose states and flag this CTA owns
        const int a = min(max(p.cu[sq], 0), p.T), e = min(max(p.cu[sq + 1], a), p.T);
        b = 0;
        bc = 0;
        tok0 = a;
        len = e - a;
        N = (len + kTile - 1) / kTile;
        slot0 = ((a >> 7) + sq) * p.H + h;
        sstride = p.H;
    }
    auto valid_rows = [&](int n) -> int { return kPacked ? min(kTile, len - n * kTile) : kTile; };
    // head coordinates of the key-side (q, log f) and value-side (i, o) token tensors, and the
    // batch coordinate of o (the key block's partial); all h and bc unless heads are read in place
    const int nbk = p.nK * p.nV, hw = h / nbk, ka = (h - hw * nbk) / p.nV, vc = h - hw * nbk - ka * p.nV;
    const int hk = hw * p.nK + ka, hv = hw * p.nV + vc, obc = ka * p.Bo + bc;
    if (smem_u32(smem) & 1023u) {   // the swizzled operand layout needs 1024-byte alignment
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    const int nblk = p.D >> 6;   // 64-column blocks loaded and stored per tile
    int issued_qg = 0, issued_v = 0;   // producer (thread 0): loads issued per barrier pair
    // chunk n's q and log f into stage n & 1, and its i (thread 0)
    auto load_qg = [&](int n) {
        const int s = n & 1;
        mbar_arrive_expect_tx(&m->fullQG[s], 2 * nblk * kBlk);
        for (int c = 0; c < nblk; ++c) {
            tma_load_4d(Qb[s] + c * kBlk, &tm_q, &m->fullQG[s], 64 * c, hk, tok0 + n * kTile, bc);
            tma_load_4d(Gb[s] + c * kBlk, &tm_lf, &m->fullQG[s], 64 * c, hk, tok0 + n * kTile, bc);
        }
        ++issued_qg;
    };
    auto load_v = [&](int n) {
        const int s = n & 1;
        mbar_arrive_expect_tx(&m->fullV[s], nblk * kBlk);
        for (int c = 0; c < nblk; ++c)
            tma_load_4d(Vb[s] + c * kBlk, &tm_x, &m->fullV[s], 64 * c, hv, tok0 + n * kTile, bc);
        ++issued_v;
    };
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->fullQG[s], 1);
            mbar_init(&m->fullV[s], 1);
            mbar_init(&m->prepped[s], 256);
            mbar_init(&m->emptyQG[s], 1);
            mbar_init(&m->emptyV[s], 1);
        }
        mbar_init(&m->barA, 1);
        mbar_init(&m->barO1, 1);
        mbar_init(&m->barS, 1);
        mbar_init(&m->barO2, 1);
        mbar_init(&m->sdone, 128);
        mbar_init(&m->adone, 128);
        mbar_init(&m->ofree, 128);
        m->bad_tile = INT_MAX;
        m->waited_full = 0;
        m->waited_v = 0;
        fence_mbar_init();
        // the first chunk's tiles before the TMEM allocation and the block barrier (the d = 64
        // zero fill below writes only the tiles' upper halves, which TMA does not load)
        if (N > 0) {
            load_qg(0);
            load_v(0);
        }
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_lf);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_o);
    }
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (nblk == 1) {             // d = 64: the unloaded halves of the input tiles stay zero
        for (int i = tid; i < 6 * (int)(kBlk / 16); i += kFwdThreads) {
            const int t = i / (int)(kBlk / 16), o = i - t * (int)(kBlk / 16);
            uint8_t *base = t < 2 ? Qb[t] : t < 4 ? Gb[t - 2] : Vb[t - 4];
            reinterpret_cast<uint4 *>(base + kBlk)[o] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int n = 1; n < N; ++n) {   // chunk 0's loads went out with the set-up
                const int s = n & 1;
                if (ld_volatile(&m->bad_tile) < n) break;
                // q and log f once the state MMA of chunk n-2 has read Qt, Kt; i once its last
                // MMA has read v
                if (n >= 2 && !wait_or_abort(&m->emptyQG[s], ((n - 2) >> 1) & 1, &m->bad_tile, n - 2)) break;
                load_qg(n);
                if (n >= 2 && !wait_or_abort(&m->emptyV[s], ((n - 2) >> 1) & 1, &m->bad_tile, n - 2)) break;
                load_v(n);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_kk = idesc_bf16(128, 128, false, false);
            const uint32_t id_kmn = idesc_bf16(128, 128, false, true);
            const uint32_t id_mnmn = idesc_bf16(128, 128, true, true);
            const uint64_t dXm = sdesc_sw128(smem_u32(X), kBlk, 1024);   // bf16(S_in), MN-major
            for (int n = 0; n < N; ++n) {
                const int s = n & 1;
                if (!mbar_wait(&m->prepped[s], (n >> 1) & 1)) {
                    set_status(HGRN2_ERR_TIMEOUT);
                    break;
                }
                if (ld_volatile(&m->bad_tile) <= n) break;
                tc_fence_after();
                // operand descriptors of this stage: K-major (for A, O) and MN-major (for S, O2) views
                const uint64_t dQ = sdesc_sw128(smem_u32(Qb[s]), 16, 1024);
                const uint64_t dG = sdesc_sw128(smem_u32(Gb[s]), 16, 1024);
                const uint64_t dGm = sdesc_sw128(smem_u32(Gb[s]), kBlk, 1024);
                const uint64_t dVm = sdesc_sw128(smem_u32(Vb[s]), kBlk, 1024);
                // A = Qt Kt^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                    mma_bf16_ss(tbase + kColA, sdesc_add(dQ, ko), sdesc_add(dG, ko), id_kk, kk > 0);
                }
                mma_commit(&m->barA);
                // O = Qt bf16(S_in) once the S phase wrote it and the last epilogue read O;
                // S' = S_in + Kt^T V
                if (!mbar_wait(&m->sdone, n & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                if (n >= 1 && !mbar_wait(&m->ofree, (n - 1) & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                    mma_bf16_ss(tbase + kColO, sdesc_add(dQ, ko), sdesc_add(dXm, kk * 2048), id_kmn, kk > 0);
                }
                mma_commit(&m->barO1);
                if (!mbar_wait(&m->fullV[s], (n >> 1) & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                m->waited_v = n + 1;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tbase + kColS, sdesc_add(dGm, kk * 2048), sdesc_add(dVm, kk * 2048), id_mnmn, true);
                mma_commit(&m->barS);
                mma_commit(&m->emptyQG[s]);   // Qt and Kt of stage s are free once the MMAs above completed
                // O += bf16(mask(A)) V once the TMEM warps wrote it (A operand in TMEM)
                if (!mbar_wait(&m->adone, n & 1)) { set_status(HGRN2_ERR_TIMEOUT); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tbase + kColO, tbase + kColP + 8 * kk, sdesc_add(dVm, kk * 2048), id_kmn, true);
                mma_commit(&m->barO2);
                mma_commit(&m->emptyV[s]);   // v of stage s is free once every MMA above completed
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ TMEM warps
        const int quad = warp & 3, r = 32 * quad + lane;             // TMEM lane = tile row
        const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
        {   // S = h0 for a sequence's first segment, else 0 (d x d, zero outside for d = 64): with
            // segments, the carried state is added afterwards (fixup_kernel)
            const float *init = seg == 0 && p.h0 ? p.h0 + (size_t)bh * p.D * p.D : nullptr;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[32];
                if (init && r < p.D && 32 * c < p.D) {
                    const float4 *src = reinterpret_cast<const float4 *>(init + (size_t)r * p.D + 32 * c);
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
        // a wait given up by a lane of this warp (warp-uniform, since the TMEM loads and stores
        // are warp-collective): the group leaves together at its next barrier
        bool fail = false;
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            fail = __any_sync(0xffffffffu, fail || !mbar_wait(bar, par));
        };
        // e^{B - rho} of the previous and the current chunk, key dim r (e^{B/2} for both scales)
        float e_prev = 1.0f, e_cur = 1.0f;
        float gprod = 1.0f;   // with segments: the segment's decay product, prod of e^{B} = (e^{B/2})^2
        for (; n < N; ++n) {
            const int s = n & 1;
            wait_all(&m->prepped[s], (n >> 1) & 1);
            // the previous chunk's state MMA completed, and its o store has read X
            if (n >= 1) {
                wait_all(&m->barS, (n - 1) & 1);
                if (r == 0) tma_store_wait_read0();
            }
            // one decision for the whole group: a wait given up anywhere in it, or a flagged chunk
            if (named_bar_or(2, 128, fail || ld_volatile(&m->bad_tile) <= n)) break;
            e_prev = e_cur;
            e_cur = m->EB[s][kScalar ? 0 : r];   // the prep warps rewrite this slot only after this chunk's stage is released
            gprod = (gprod * e_cur) * e_cur;
            // S phase: S_r = Diag(e^{rho}) Diag(e^{B_prev - rho_prev}) S' of the previous chunk (both
            // factors e^{B/2}); bf16(S_r) -> X (B operand).  The two factors are applied one after
            // the other: the first gives S_out of the previous chunk, O(1), while their product can
            // fall below the fp32 range (two strongly decaying chunks: e^{-52} e^{-52}).
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
            if (p.save) {   // bf16(S_r) of this chunk, kept for the backward
                named_bar_sync(2, 128);   // no thread of the group has left since the barrier above
                if (r == 0) {
                    const int slot = slot0 + n * sstride;
                    tma_store_4d(&tm_st, X, 0, 0, 0, slot);
                    tma_store_4d(&tm_st, X + kBlk, 64, 0, 0, slot);
                    tma_store_commit();
                }
            }
            // causal mask of A -> bf16 pairs in TMEM columns P (the A operand of the intra MMA),
            // as soon as A is complete.  Column block c is kept (c < quad), dropped (c > quad) or
            // diagonal (per element).  The MMA that read the previous chunk's P completed before A.
            // (After a wait given up, this thread goes on with whatever TMEM holds; nothing it
            // writes is used, and the group leaves at its next barrier.)
            wait_all(&m->barA, n & 1);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[32], pk[16];
                if (c <= quad) {
                    tmem_ld32(tl + kColA + 32 * c, v);
                    tmem_wait_ld();
                    if (c == quad) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i > lane) v[i] = 0.0f;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = __uint_as_float(pack_bf2(v[2 * i], v[2 * i + 1]));
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0.0f;
                }
                tmem_st16(tl + kColP + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&m->adone);
            // o epilogue: O -> bf16 rows in X (free: the last MMA of the chunk completed, and the
            // state store has read it) -> TMA store; the next S phase waits until the store has read X
            wait_all(&m->barO2, n & 1);
            if (p.save) {
                if (r == 0) tma_store_wait_read0();
                if (named_bar_or(2, 128, fail)) break;
            }
            tc_fence_after();
            const int vr = valid_rows(n);
            if (vr == kTile) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float v[32];
                    tmem_ld32(tl + kColO + 32 * c, v);
                    tmem_wait_ld();
                    store_chunk_bf16(X, r, c, v);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&m->ofree);
                if (named_bar_or(2, 128, fail)) break;
                if (r == 0) {
                    if (nbk > 1) {   // heads read in place: this block pair's share, added into o
                        tma_reduce_add_4d(&tm_o, X, 0, hv, tok0 + n * kTile, bc);
                        tma_reduce_add_4d(&tm_o, X + kBlk, 64, hv, tok0 + n * kTile, bc);
                    } else {
                        tma_store_4d(&tm_o, X, 0, hv, tok0 + n * kTile, obc);
                        if (nblk == 2) tma_store_4d(&tm_o, X + kBlk, 64, hv, tok0 + n * kTile, obc);
                    }
                    tma_store_commit();
                }
            } else if (!fail) {   // a packed sequence's last chunk: its rows only, stored by their threads
                uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((size_t)(tok0 + n * kTile + r) * p.H + h) * p.D);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (32 * c >= p.D) break;
                    float v[32];
                    tmem_ld32(tl + kColO + 32 * c, v);
                    tmem_wait_ld();
                    if (r < vr) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq)
                            dst[4 * c + qq] = make_uint4(pack_bf2(v[8 * qq], v[8 * qq + 1]),
                                                         pack_bf2(v[8 * qq + 2], v[8 * qq + 3]),
                                                         pack_bf2(v[8 * qq + 4], v[8 * qq + 5]),
                                                         pack_bf2(v[8 * qq + 6], v[8 * qq + 7]));
                    }
                }
                tc_fence_before();
                mbar_arrive(&m->ofree);
            }
        }
        if (fail) set_status(HGRN2_ERR_TIMEOUT);
        if (r == 0) {
            tma_store_wait_all0();
            fence_proxy_async_global();   // the stores are ordered before the segment count below
        }
        // the last state MMA must be complete before hT is read or TMEM is released
        if (n >= 1) mbar_wait(&m->barS, (n - 1) & 1);
        tc_fence_after();
        if (p.nseg > 1 && n == N && !fail) {   // with segments: this segment's map (g, U) for the scan
            if (r < p.D) p.gseg[((size_t)bh * p.nseg + seg) * 128 + r] = seg == 0 ? 0.0f : gprod;
        }
        if (n == N && !fail && (p.nseg > 1 || ((p.hT || p.hTs) && seg == p.nseg - 1)) && r < p.D) {   // warp-uniform
            const float e = e_cur;   // hT (or the segment's U) = Diag(e^{B - rho}) S' of the last chunk
            if (p.hmaps) {
                // d = 128: every row into four swizzled 32-column boxes of fp32 in the (now idle) first
                // two ring tiles, then TMA stores (the group's condition here is uniform: all 128
                // threads finished the loop together, and r < 128)
                uint8_t *stg = smem;
                float rabs = 0.0f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float v[32];
                    tmem_ld32(tl + kColS + 32 * c, v);
                    tmem_wait_ld();
                    uint8_t *row = stg + (size_t)c * 16384 + r * 128;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float4 w = make_float4(v[4 * k] * e, v[4 * k + 1] * e, v[4 * k + 2] * e, v[4 * k + 3] * e);
                        rabs += (fabsf(w.x) + fabsf(w.y)) + (fabsf(w.z) + fabsf(w.w));
                        *reinterpret_cast<float4 *>(row + ((k ^ (r & 7)) << 4)) = w;
                    }
                }
                if (p.nseg > 1 && p.uabs) p.uabs[((size_t)bh * p.nseg + seg) * 128 + r] = rabs;
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                if (r == 0) {
                    const int seg_slot = bh * p.nseg + seg;
                    for (int c = 0; c < 4; ++c) {
                        if (p.hmaps & 1) tma_store_2d(&tm_h1, stg + (size_t)c * 16384, 32 * c, (p.hslot1 ? seg_slot : bh) * 128);
                        if (p.hmaps & 2) tma_store_2d(&tm_h2, stg + (size_t)c * 16384, 32 * c, (p.hslot2 ? seg_slot : bh) * 128);
                    }
                    tma_store_commit();
                    tma_store_wait_all0();
                }
            } else {
                float *dst = p.nseg > 1 ? p.Useg + (((size_t)bh * p.nseg + seg) * 128 + r) * 128
                                        : p.hT ? p.hT + ((size_t)bh * p.D + r) * p.D : nullptr;
                float *dsv = p.nseg > 1 ? nullptr : p.hTs ? p.hTs + ((size_t)bh * p.D + r) * p.D : nullptr;
                float rabs = 0.0f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (32 * c >= p.D) break;
                    float v[32];
                    tmem_ld32(tl + kColS + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 w = make_float4(v[4 * i] * e, v[4 * i + 1] * e, v[4 * i + 2] * e, v[4 * i + 3] * e);
                        rabs += (fabsf(w.x) + fabsf(w.y)) + (fabsf(w.z) + fabsf(w.w));
                        if (dst) reinterpret_cast<float4 *>(dst + 32 * c)[i] = w;
                        if (dsv) reinterpret_cast<float4 *>(dsv + 32 * c)[i] = w;
                    }
                }
                if (p.nseg > 1 && p.uabs) p.uabs[((size_t)bh * p.nseg + seg) * 128 + r] = rabs;
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ prep warps
        // thread = one column pair (2 key dims, 4-byte smem accesses) and one 32-row range.
        // Each range first sums its own rows of log f; ranges exchange sums through shared
        // memory, which also gives the chunk total B and the reference rho = B / 2.  Then
        // f = e^a directly (so k = 1 - f has an absolute error of a few 1e-8), E = e^{b - rho}
        // as the running product of f from the range start, 1/E = e^{rho - b} with b the
        // running sum of log f.  Rows go in batches of 8: all loads, then the arithmetic, then
        // all stores.
        const int ptid = tid - 256;
        const int pc = ptid & 63, rr = ptid >> 6, col0 = 2 * pc;
        const uint32_t cblk = (uint32_t)(col0 >> 6) * kBlk, cch = (uint32_t)((col0 & 63) >> 3), cin = (uint32_t)(col0 & 7) * 2;
        auto eoff = [&](int t) -> uint32_t { return cblk + t * 128 + ((cch ^ (t & 7)) << 4) + cin; };
        float gnx[4];   // scalar decay: log g of rows 4 lane .. 4 lane + 3 of the next chunk
        auto load_lg = [&](int n) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = tok0 + n * kTile + 4 * lane + j;
                gnx[j] = n < N && t < p.T ? __bfloat162float(p.lgs[((size_t)bc * p.T + t) * p.H + h]) : 0.0f;
            }
        };
        if (kScalar) load_lg(0);
        for (int n = 0; n < N; ++n) {
            const int s = n & 1;
            const bool landed = mbar_wait(&m->fullQG[s], (n >> 1) & 1);
            if (ptid == 0 && landed) m->waited_full = n + 1;
            if constexpr (kScalar) {
                if (!__all_sync(0xffffffffu, landed)) {   // no group barrier here: each warp may leave alone
                    set_status(HGRN2_ERR_TIMEOUT);
                    break;
                }
                // b_t = cumulative log g from the chunk start (0 past the sequence end): every prep
                // warp scans all 128 rows itself (rows 4l .. 4l+3 in lane l), so this prep needs no
                // block barrier
                float bl[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) bl[j] = gnx[j];
                load_lg(n + 1);
                bl[1] += bl[0];
                bl[2] += bl[1];
                bl[3] += bl[2];
                float x = bl[3];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                const float ex = x - bl[3];   // sum over the lanes before this one
                const float Bt = __shfl_sync(0xffffffffu, x, 31);   // the chunk total B
                const float rho = 0.5f * Bt;                         // the balanced reference
                float eq[4], ek[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    bl[j] += ex - rho;
                    eq[j] = __expf(bl[j]);
                    ek[j] = __expf(-bl[j]);
                }
                const bool bad = !(rho >= -kMaxRefLog);   // also NaN
                // Qt = q e^{b_t - rho}, Kt = k e^{rho - b_t}, rows in batches of 8: row t = 32 rr + 8 bt + i
                // has its factors in lane 8 rr + 2 bt + i / 4, slot i % 4
#pragma unroll 1
                for (int bt = 0; bt < 4; ++bt) {
                    const int t0 = 32 * rr + 8 * bt;
                    uint32_t wq[8], wk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        wq[i] = *reinterpret_cast<const uint32_t *>(Qb[s] + eoff(t0 + i));
                        wk[i] = *reinterpret_cast<const uint32_t *>(Gb[s] + eoff(t0 + i));
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int src = 8 * rr + 2 * bt + (i >> 2);
                        const float et = __shfl_sync(0xffffffffu, eq[i & 3], src);
                        const float kt = __shfl_sync(0xffffffffu, ek[i & 3], src);
                        wq[i] = pack_bf2(bf_lo(wq[i]) * et, bf_hi(wq[i]) * et);
                        wk[i] = pack_bf2(bf_lo(wk[i]) * kt, bf_hi(wk[i]) * kt);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        *reinterpret_cast<uint32_t *>(Qb[s] + eoff(t0 + i)) = wq[i];
                        *reinterpret_cast<uint32_t *>(Gb[s] + eoff(t0 + i)) = wk[i];
                    }
                }
                if (ptid == 0) {   // read after prepped[s] completes (this thread arrives after these)
                    m->EB[s][0] = __expf(Bt - rho);
                    if (bad) atomicMin(&m->bad_tile, n);
                }
                fence_proxy_async_smem();
                mbar_arrive(&m->prepped[s]);
                if (bad) break;
                continue;
            }
            const int vr = valid_rows(n);   // rows from vr on: log f = 0 and q = 0 (no effect)
            float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                uint32_t w = *reinterpret_cast<const uint32_t *>(Gb[s] + eoff(32 * rr + i));
                if (32 * rr + i >= vr) w = 0u;
                s0 += bf_lo(w);
                s1 += bf_hi(w);
            }
            // ranges 0..2 in Ppart, range 3 in this stage's E_B slot (free until the end of this
            // prep: the TMEM warps read it only after prepped[s], and its last reader, two chunks
            // back, released the stage before these rows were loaded)
            float *p3 = m->EB[s];
            if (rr < 3) {
                m->Ppart[rr][col0] = s0;
                m->Ppart[rr][col0 + 1] = s1;
            } else {
                p3[col0] = s0;
                p3[col0 + 1] = s1;
            }

            // the whole prep group leaves together if any of its waits gave up (its later barriers
            // would otherwise wait for the leavers)
            if (named_bar_or(1, 256, !landed)) {
                if (!landed) set_status(HGRN2_ERR_TIMEOUT);
                break;
            }
            float b0 = 0.0f, b1 = 0.0f;   // sum of log f over the rows before this range
            for (int r2 = 0; r2 < rr; ++r2) {
                b0 += m->Ppart[r2][col0];
                b1 += m->Ppart[r2][col0 + 1];
            }
            // the chunk total, summed in the same order by the four threads of a column
            const float Bt0 = ((m->Ppart[0][col0] + m->Ppart[1][col0]) + m->Ppart[2][col0]) + p3[col0];
            const float Bt1 = ((m->Ppart[0][col0 + 1] + m->Ppart[1][col0 + 1]) + m->Ppart[2][col0 + 1]) + p3[col0 + 1];
            // relative to the balanced reference rho = B / 2
            b0 -= 0.5f * Bt0;
            b1 -= 0.5f * Bt1;
            float E0 = __expf(b0), E1 = __expf(b1);   // E = e^{b - rho} of the row before the range
            // a later segment's first chunk: bf16(q e^{b}) and B, for the fix-up
            uint32_t *qt_out = nullptr;
            float er0 = 0.0f, er1 = 0.0f;
            if (kSeg && n == 0 && seg > 0 && p.qtil) {
                const size_t slot = (size_t)bh * p.nseg + seg;
                qt_out = reinterpret_cast<uint32_t *>(p.qtil + slot * 16384 + col0);
                er0 = __expf(0.5f * Bt0);
                er1 = __expf(0.5f * Bt1);
                if (rr == 0) {
                    p.bseg[slot * 128 + col0] = Bt0;
                    p.bseg[slot * 128 + col0 + 1] = Bt1;
                }
            }
#pragma unroll 1
            for (int bt = 0; bt < 4; ++bt) {
                const int t0 = 32 * rr + 8 * bt;
                uint32_t wa[8], wq[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    wa[i] = *reinterpret_cast<const uint32_t *>(Gb[s] + eoff(t0 + i));
                    wq[i] = *reinterpret_cast<const uint32_t *>(Qb[s] + eoff(t0 + i));
                    if (t0 + i >= vr) wa[i] = wq[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float a0 = bf_lo(wa[i]), a1 = bf_hi(wa[i]);
                    b0 += a0;
                    b1 += a1;
                    const float f0 = __expf(a0), f1 = __expf(a1);
                    E0 *= f0;
                    E1 *= f1;
                    wq[i] = pack_bf2(bf_lo(wq[i]) * E0, bf_hi(wq[i]) * E1);
                    wa[i] = pack_bf2((1.0f - f0) * __expf(-b0), (1.0f - f1) * __expf(-b1));
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    *reinterpret_cast<uint32_t *>(Qb[s] + eoff(t0 + i)) = wq[i];
                    *reinterpret_cast<uint32_t *>(Gb[s] + eoff(t0 + i)) = wa[i];
                }
            }
            if (qt_out) {   // q e^{b} = Qt e^{rho}, from this thread's Qt rows (rounded to bf16 twice)
#pragma unroll 4
                for (int i = 0; i < 32; ++i) {
                    const int t = 32 * rr + i;
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(Qb[s] + eoff(t));
                    qt_out[(size_t)t * 64] = pack_bf2(bf_lo(w) * er0, bf_hi(w) * er1);
                }
            }
            // b = B - rho = B / 2 now: the scale e^{B/2} of both state factors
            if (rr == 3 && !(b0 >= -kMaxRefLog && b1 >= -kMaxRefLog)) atomicMin(&m->bad_tile, n);   // also NaN
            fence_proxy_async_smem();
            named_bar_sync(1, 256);   // bad_tile settled; Ppart and the range-3 sums read by all
            if (rr == 3) {   // before this thread's arrival, which publishes it to the TMEM warps
                m->EB[s][col0] = __expf(b0);
                m->EB[s][col0 + 1] = __expf(b1);
            }
            mbar_arrive(&m->prepped[s]);
            if (ld_volatile(&m->bad_tile) <= n) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int bad = m->bad_tile;
    const bool fell_back = bad < N;
    if (warp == 0 && lane == 0)   // drain loads still landing in this CTA's shared memory
    {
        for (int k = m->waited_full; k < issued_qg; ++k) mbar_wait(&m->fullQG[k & 1], (k >> 1) & 1, 2000000u);
        for (int k = m->waited_v; k < issued_v; ++k) mbar_wait(&m->fullV[k & 1], (k >> 1) & 1, 2000000u);
    }
    if (tid == 0) {
        if (p.nseg == 1) { if (p.flags) p.flags[bh] = fell_back ? 1 : 0; }   // sole writer
        else if (fell_back) p.flags[bh] = 1;                  // zeroed before the launch
        if (fell_back) atomicAdd(&g_counters[0], 1ull);
        else atomicAdd(&g_counters[1], (unsigned long long)N);
    }
    __syncwarp();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
    // With segments, the last segment of the pair to finish runs the exact route for the whole
    // sequence if any segment flagged the pair (every other segment's flag, o and hT stores are
    // complete before its count: its stores were waited for, then the fence and the atomic)
    bool exact = fell_back && p.nseg == 1;
    if (p.nseg > 1) {
        if (tid == 0) {
            fence_proxy_async_global();   // this CTA's bulk-async o stores before the count
            __threadfence();
            const int prev = atomicAdd(&p.seg_done[bh], 1);
            __threadfence();
            m->waited_v = (prev == p.nseg - 1 && ld_volatile(&p.flags[bh]) != 0) ? 1 : 0;
        }
        __syncthreads();
        exact = m->waited_v != 0;
    }
    // exact route for this (b,h): the pipeline is drained, so the CTA's shared memory is free for
    // the CUDA-core chunkwise forward of the whole sequence
    if (exact) {
        __syncthreads();
        if constexpr (kScalar) {   // the scalar-decay exact forward (key k in p.lf, value v in p.x)
            sd::fwd_body<__nv_bfloat16>(p.q, p.lf, p.x, p.lgs, p.h0, p.o, p.hT, p.T, p.H, p.D, p.D,
                                        reinterpret_cast<float *>(smem), b, h, bh);
        } else {
            // the whole sequence from its first token: a packed sequence's offset (a segmented
            // launch's tok0 is its segment's first token, not the sequence's)
            const size_t ok = kPacked ? (size_t)tok0 * p.H * p.D : 0;
            if (nbk == 1) {
                simt_fwd_body<__nv_bfloat16>(p.q + ok, p.lf + ok, p.x + ok, p.h0, p.o + ok, p.hT, kPacked ? len : p.T,
                                             p.H, p.D, p.D, p.simt_chunk, reinterpret_cast<float *>(smem), b, h, bh);
            } else {
                // heads read in place (nK = nV): every token tensor is viewed with Hw nK half-heads of
                // 128 and indexed at the value-side half-head hv; the key-side tensors are shifted by
                // the half-heads between hk and hv.  The share goes to the key block's partial, then
                // is added into o (other block pairs add theirs by TMA reduce-add, in any order)
                const int Hh = (p.H / nbk) * p.nV;   // half-heads of the token tensors
                const long long kshift = (long long)(hk - hv) * p.D;
                const size_t opart = (size_t)ka * p.Bo * p.T * Hh * p.D;
                simt_fwd_body<__nv_bfloat16>(p.q + kshift, p.lf + kshift, p.x, p.h0, p.opart + opart, p.hT, p.T, Hh,
                                             p.D, p.D, p.simt_chunk, reinterpret_cast<float *>(smem), b, hv, bh);
                __syncthreads();
                add_rows_bf16(p.o, p.opart + opart, b, hv, p.T, Hh);
            }
        }
    }
}

// ------------------------------------------------------------------ sequence segments
// For few (batch, head) pairs, each sequence is cut into segments of `tps` chunks run by
// separate CTAs.  The state map of a segment is affine in its incoming state:
// S_out = Diag(g) S_in + U with g = prod of the chunks' e^{B} and U the state the segment
// reaches from S_in = 0.  fwd_kernel runs every segment from zero (the first from h0) and
// writes its (g, U); scan_kernel chains them in fp32 (the states entering the segments, and
// hT); fixup_kernel adds the carried states to the segments' outputs.
//
// agg_kernel computes (g, U) of a run of chunks without its outputs, on the tensor cores, with
// Kh = k * prod_{r>t} f_r directly (suffix products inside the chunk): exact for any decay
// strength.  It serves hgrn2_state_map (one segment = a whole slice).
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
    int *flags;       // zeroed here (segment 0) before fwd_kernel sets exact-route flags (or null)
    int *seg_done;    // zeroed here (segment 0): fwd_kernel's finished-segment counts (or null)
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
        if (seg == 0 && p.flags) p.flags[bh] = 0;
        if (seg == 0 && p.seg_done) p.seg_done[bh] = 0;
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
        // the previous chunk's MMA ran under this prep: it must be done before S is scaled, and
        // before its stage takes the chunk after this one
        if (n >= 1) {
            if (__syncthreads_or(!mbar_wait(&m->barM, (n - 1) & 1))) { ok = false; break; }
            tc_fence_after();
            if (tid == 0 && n + 1 < N) issue_load(n + 1);
        } else {
            __syncthreads();
        }
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
        if (tid == 0) {   // S += Kh^T V, completing under the next chunk's prep
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tbase, sdesc_add(sdesc_sw128(smem_u32(Gb[s]), kBlk, 1024), kk * 2048),
                            sdesc_add(sdesc_sw128(smem_u32(Vb[s]), kBlk, 1024), kk * 2048), id_mnmn, true);
            mma_commit(&m->barM);
        }
    }
    if (ok && N > 0 && __syncthreads_or(!mbar_wait(&m->barM, (N - 1) & 1))) ok = false;   // the last MMA
    tc_fence_after();
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

// With segments: every segment ran from a zero state (segment 0 from h0), so its final state is
// U_seg and the state entering segment k is the scan of the maps of segments 0..k-1 (segment 0's
// g is 0: h0 is inside its U).  In fp32, over the U slots: slot k-1 becomes the state entering
// segment k; the sequence's final state goes to hT (and the saved final state).  Pairs the exact
// route recomputed whole (flagged) are left alone.  One thread per 4 consecutive state elements
// of one (batch, head); the maps are loaded kScanBatch segments at a time, so that one memory
// latency covers a batch rather than each segment.  Launched as a programmatic dependent of the segments' kernel.
constexpr int kScanBatch = 16;
__global__ void __launch_bounds__(256)
scan_kernel(float *__restrict__ U, const float *__restrict__ g, int nseg, const int *__restrict__ flags,
            float *__restrict__ hT, float *__restrict__ hTs) {
    grid_dep_launch();   // the fix-up may be scheduled now; it waits for this grid itself
    grid_dep_wait();     // the segments' maps and flags are complete
    const int bh = blockIdx.x >> 4;
    if (flags[bh]) return;
    const int e = ((blockIdx.x & 15) * 256 + threadIdx.x) * 4;   // element offset in [0, 16384)
    const int jrow = e >> 7;
    float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nseg; s0 += kScanBatch) {
        float4 uv[kScanBatch];
        float gj[kScanBatch];
#pragma unroll
        for (int i = 0; i < kScanBatch; ++i) {
            if (s0 + i < nseg) {
                const size_t slot = (size_t)bh * nseg + s0 + i;
                uv[i] = *reinterpret_cast<const float4 *>(U + slot * 16384 + e);
                gj[i] = g[slot * 128 + jrow];
            }
        }
#pragma unroll
        for (int i = 0; i < kScanBatch; ++i) {
            const int sg = s0 + i;
            if (sg < nseg) {
                S = make_float4(fmaf(gj[i], S.x, uv[i].x), fmaf(gj[i], S.y, uv[i].y), fmaf(gj[i], S.z, uv[i].z),
                                fmaf(gj[i], S.w, uv[i].w));
                if (sg < nseg - 1) {
                    *reinterpret_cast<float4 *>(U + ((size_t)bh * nseg + sg) * 16384 + e) = S;
                } else {
                    if (hT) *reinterpret_cast<float4 *>(hT + (size_t)bh * 16384 + e) = S;
                    if (hTs) *reinterpret_cast<float4 *>(hTs + (size_t)bh * 16384 + e) = S;
                }
            }
        }
    }
}

// ------------------------------------------------------------------ carried-state fix-up
// With segments, segment k >= 1 of a pair ran from a zero state; its outputs lack the state S_in
// that enters it, carried through its chunks with no new input:
//   o_t += (q_t * e^{b_t})^T S_c,      S_{c+1} = Diag(e^{B_c}) S_c,      S_0 = S_in
// (b_t the cumulative log decay from chunk c's start, B_c its total; every factor <= 1), and,
// when the chunk states are kept for the backward, the chunk's saved bf16(e^{rho} S_in) lacks
// e^{rho_c} S_c.  One CTA per segment walks its chunks from the start while
// max_j decay_j max_v |S_c[j,v]| >= kFixStop (decay_j the carried decay of key dim j so far): a
// term left out is below 128 |q| kFixStop, 2^-15 of the relative rounding of the bf16 copy of the
// state that every inter-chunk product reads.  Per chunk: q e^{b} (the first chunk's from the
// segments' kernel, later ones from q and log f), o (and the saved state) in; one MMA
// O = (q e^{b}) bf16(S_c) into TMEM; o += O; the saved state corrected; the carried state scaled.
// 8 warps; thread (row r, half) holds 64 columns of row r of the carried state in registers.
// Without saved states two stages: the next chunk's tiles load while this one is on the tensor
// cores and in the epilogue (the decision to walk it is taken from this chunk's e^{B}, before
// they are requested).
// S_in is the scan kernel's (slot k-1 of Sin), or, with up to kMergedScanMax segments (merged),
// summed here from the segments' maps, nearest first: S_in = sum_{m<k} Diag(w_m) U_m with
// w_m = prod_{m<l<k} g_l.  The walk ends at the first m where max_j w_m[j] (m + 1) M[j] <
// kFixStop, M[j] = max_{m'<k} sum_v |U_m'[j,v]|: the maps m' <= m left out add less than that to
// any entry (w only shrinks further back), the bar the carried state itself is held to.  The last
// segment's CTA then also writes hT = Diag(g_k) S_in + U_k.  A programmatic dependent of the
// kernel before it: only its set-up runs before grid_dep_wait().
constexpr float kFixStop = 0x1p-24f;

struct FixMisc {
    uint64_t fullQG[2], fullO[2], barM, fullU[2];   // fullU: the segments' state slots
    uint32_t tmem_base;
    int nmaps;            // merged: the segments' maps the walk takes
    float EB[128];        // e^{B} of the chunk, key dim
    float ER[128];        // e^{rho} = e^{B/2} of the chunk, key dim (the saved states' scale)
    float Ppart[3][128];  // per 32-row range sums of log f (ranges 0..2)
};
// one stage (q, log f, o, saved state) + X, or two stages (q, log f, o) + X
constexpr size_t fix_smem(bool save) { return (save ? 5 : 7) * (size_t)kTileBytes + sizeof(FixMisc); }
constexpr int kMergedScanMax = 18;   // segments per pair up to which the fix-up sums S_in itself

struct FixParams {
    const float *U;     // [B*H][nseg][128][128]: the segments' U, or (after the scan kernel) slot k-1 =
                        // the state entering segment k
    const float *g;     // [B*H][nseg][128]: the segments' decay products (merged)
    const float *uabs;  // [B*H][nseg][128]: sum_v |U[j,v]| of the segments' U, row j (merged)
    const float *B0;    // [B*H][nseg][128]: each segment's first-chunk total log decay
    const int *flags;   // [B*H] nonzero: recomputed whole by the exact route (skipped)
    float *hT, *hTs;    // merged: the final state (either may be null)
    int H, nseg, tps, ntiles;
    bool save;          // saved bf16 chunk states (slot bh * ntiles + chunk) to correct
    bool merged;        // S_in summed here (else read from the scan's slots)
};

__global__ void __launch_bounds__(kThreads, 1)
fixup_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_lf,
             const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_st,
             const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_u, FixParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int NS = p.save ? 1 : 2;   // stages
    // stage s: q, log f, o at smem + 3 s tiles (s = 0 with one stage)
    auto Qb = [&](int s) { return smem + (size_t)s * 3 * kTileBytes; };
    auto Gb = [&](int s) { return smem + ((size_t)s * 3 + 1) * kTileBytes; };
    auto Ob = [&](int s) { return smem + ((size_t)s * 3 + 2) * kTileBytes; };
    uint8_t *Sb = smem + 3 * kTileBytes;                              // one stage only
    uint8_t *X = smem + (NS == 2 ? 6 : 4) * kTileBytes;
    FixMisc *m = reinterpret_cast<FixMisc *>(smem + (NS == 2 ? 7 : 5) * kTileBytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nfix = p.nseg - 1;
    const int bh = blockIdx.x / nfix, seg = 1 + blockIdx.x - bh * nfix, b = bh / p.H, h = bh - b * p.H;
    const int g0 = seg * p.tps, N = min(p.ntiles - g0, p.tps);
    const size_t myslot = (size_t)bh * p.nseg + seg;
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_status(HGRN2_ERR_DEVICE);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->fullQG[s], 1);
            mbar_init(&m->fullO[s], 1);
            mbar_init(&m->fullU[s], 1);
        }
        mbar_init(&m->barM, 1);
        m->nmaps = 1;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_lf);
        tma_prefetch_desc(&tm_o);
        tma_prefetch_desc(&tm_qt);
        tma_prefetch_desc(&tm_u);
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m->tmem_base;
    const int quad = warp & 3, ch = warp >> 2, r = 32 * quad + lane;   // carried-state row / token row r
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
    const uint32_t id_kmn = idesc_bf16(128, 128, false, true);
    const int pc = tid & 63, rr = tid >> 6, col0 = 2 * pc;   // prep: column pair, 32-row range
    const uint32_t cblk = (uint32_t)(col0 >> 6) * kBlk, cch = (uint32_t)((col0 & 63) >> 3), cin = (uint32_t)(col0 & 7) * 2;
    auto eoff = [&](int t) -> uint32_t { return cblk + t * 128 + ((cch ^ (t & 7)) << 4) + cin; };
    // loads issued (thread 0) and waited for (every thread), per barrier kind, counted in chunks
    int issued_qg = 0, issued_o = 0, waited_qg = 0, waited_o = 0;
    auto load_qg = [&](int c) {   // thread 0; the first chunk: q e^{b} into the q tile
        const int s = NS == 2 ? (c & 1) : 0, tok = (g0 + c) * kTile;
        mbar_arrive_expect_tx(&m->fullQG[s], (c == 0 ? 1 : 2) * kTileBytes);
        for (int k = 0; k < 2; ++k) {
            if (c == 0) {
                tma_load_4d(Qb(s) + k * kBlk, &tm_qt, &m->fullQG[s], 64 * k, 0, 0, (int)myslot);
            } else {
                tma_load_4d(Qb(s) + k * kBlk, &tm_q, &m->fullQG[s], 64 * k, h, tok, b);
                tma_load_4d(Gb(s) + k * kBlk, &tm_lf, &m->fullQG[s], 64 * k, h, tok, b);
            }
        }
        ++issued_qg;
    };
    auto load_o = [&](int c) {    // thread 0
        const int s = NS == 2 ? (c & 1) : 0, tok = (g0 + c) * kTile, slot = bh * p.ntiles + g0 + c;
        mbar_arrive_expect_tx(&m->fullO[s], (p.save ? 2 : 1) * kTileBytes);
        for (int k = 0; k < 2; ++k) {
            tma_load_4d(Ob(s) + k * kBlk, &tm_o, &m->fullO[s], 64 * k, h, tok, b);
            if (p.save) tma_load_4d(Sb + k * kBlk, &tm_st, &m->fullO[s], 64 * k, 0, 0, slot);
        }
        ++issued_o;
    };
    // prep of stage s (chunks after the first): b = cumulative log f from the chunk start;
    // Qt = q e^{b} in place; e^{B} and e^{B/2}, B summed as the forward's prep sums it
    // (((P0 + P1) + P2) + P3, Pk the 32-row range totals)
    auto prep = [&](int s) {
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(Gb(s) + eoff(32 * rr + i));
            s0 += bf_lo(w);
            s1 += bf_hi(w);
        }
        if (rr < 3) {
            m->Ppart[rr][col0] = s0;
            m->Ppart[rr][col0 + 1] = s1;
        }
        __syncthreads();
        float b0 = 0.0f, b1 = 0.0f;
        for (int r2 = 0; r2 < rr; ++r2) {
            b0 += m->Ppart[r2][col0];
            b1 += m->Ppart[r2][col0 + 1];
        }
        if (rr == 3) {
            const float B0 = b0 + s0, B1 = b1 + s1;
            m->EB[col0] = __expf(B0);
            m->EB[col0 + 1] = __expf(B1);
            m->ER[col0] = __expf(0.5f * B0);
            m->ER[col0 + 1] = __expf(0.5f * B1);
        }
        float E0 = __expf(b0), E1 = __expf(b1);
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const int t = 32 * rr + i;
            const uint32_t wa = *reinterpret_cast<const uint32_t *>(Gb(s) + eoff(t));
            uint32_t *wq = reinterpret_cast<uint32_t *>(Qb(s) + eoff(t));
            E0 *= __expf(bf_lo(wa));
            E1 *= __expf(bf_hi(wa));
            *wq = pack_bf2(bf_lo(*wq) * E0, bf_hi(*wq) * E1);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();   // Qt, e^{B}, e^{B/2} complete
    };

    grid_dep_wait();   // the segments' outputs (and the scan's) are complete from here on
    bool ok = true, go = false;
    float S[64];          // the carried state, row r, columns 64 ch .. 64 ch + 63
    float smax = 0.0f;    // max |S| of the row's 64 columns as entered
    float decay = 1.0f;   // the carried decay of row r so far
    const bool flagged = p.flags[bh] != 0;
    const bool want_hT = p.merged && seg == p.nseg - 1 && (p.hT || p.hTs);
    // The segments' state slots it reads, 64 KB each, staged through shared memory by TMA (tiles
    // the first chunk does not use yet): merged, segments seg-1, seg-2, ... (nmaps of them) and its
    // own for hT; else the scan's slot seg-1.  Two buffers with two stages, one with one.
    const int nbuf = NS;
    auto ubox = [&](int buf, int bx) -> uint8_t * {   // 32 columns x 128 rows of fp32, swizzled
        if (NS == 2) return smem + (size_t)(3 + 2 * buf) * kTileBytes + (size_t)bx * 16384;
        return smem + (size_t)(bx < 2 ? 1 : 4) * kTileBytes + (size_t)(bx & 1) * 16384;
    };
    int nmaps = 1;   // slots i < nmaps: segment seg-1-i (merged); i = nmaps: its own (hT)
    auto slot_of = [&](int i) {
        return (size_t)bh * p.nseg + (!p.merged ? seg - 1 : i < nmaps ? seg - 1 - i : seg);
    };
    int issuedU = 0, waitedU = 0;
    auto load_u = [&](int i) {   // thread 0: slot i into buffer i % nbuf
        const int buf = i % nbuf;
        mbar_arrive_expect_tx(&m->fullU[buf], 4 * 16384);
        for (int bx = 0; bx < 4; ++bx) tma_load_2d(ubox(buf, bx), &tm_u, &m->fullU[buf], 32 * bx, (int)slot_of(i) * 128);
        ++issuedU;
    };
    if (tid == 0 && !flagged) load_u(0);   // segment seg-1 (merged) or the scan's slot: always read
    if (!flagged) {
        if (tid == 0) {   // the first chunk's tiles
            fence_proxy_async_global();
            load_qg(0);
            load_o(0);
        }
        if (tid < 128) {  // the first chunk's e^{B}, e^{B/2}
            const float B = p.B0[myslot * 128 + tid];
            m->EB[tid] = __expf(B);
            m->ER[tid] = __expf(0.5f * B);
        }
    }
    if (p.merged && !flagged) {   // how far back the walk goes, from this thread's row r
        // map m = seg-1-i, row r: x[i] = sum_v |U_m[r,v]| and g_m[r], all loaded at once (indices
        // clamped to segment 0, the extra values unused).  M = max_{i<seg} x[i] (NaN kept): the maps
        // m' <= m add at most w_m (m + 1) M to an entry of row r.
        const size_t s0 = (size_t)bh * p.nseg;
        constexpr int kMaps = kMergedScanMax - 1;
        float xr[kMaps], gr[kMaps];
#pragma unroll
        for (int i = 0; i < kMaps; ++i) {
            const size_t sl = s0 + (size_t)max(seg - 1 - i, 0);
            xr[i] = p.uabs[sl * 128 + r];
            gr[i] = p.g[sl * 128 + r];
        }
        float M = 0.0f;
#pragma unroll
        for (int i = 0; i < kMaps; ++i)
            if (i < seg) M = (xr[i] > M || isnan(xr[i])) ? xr[i] : M;
        float w = 1.0f;
        int n = 0;
        bool on = true;
#pragma unroll
        for (int i = 0; i < kMaps; ++i) {   // "not below" is true for NaN: such a row walks on
            on = on && i < seg && !(w * ((float)(seg - i) * M) < kFixStop);
            if (on) {
                ++n;
                w *= gr[i];
            }
        }
        n = __reduce_max_sync(0xffffffffu, n);
        if (lane == 0 && n > 1) atomicMax(&m->nmaps, n);
        __syncthreads();
        nmaps = m->nmaps;
    }
    const int nslots = flagged ? 0 : p.merged ? nmaps + (want_hT ? 1 : 0) : 1;
    if (tid == 0)
        for (int i = 1; i < nslots && i < nbuf; ++i) load_u(i);
#pragma unroll
    for (int i = 0; i < 64; ++i) S[i] = 0.0f;
    float wr = 1.0f;   // merged: the weight of the next map, row r
    for (int i = 0; i < nslots; ++i) {
        const int buf = i % nbuf;
        const float gi = p.merged ? p.g[slot_of(i) * 128 + r] : 0.0f;   // issued before the wait
        if (__syncthreads_or(!mbar_wait(&m->fullU[buf], (i / nbuf) & 1))) { ok = false; break; }
        waitedU = i + 1;
        float u[64];   // row r, columns 64 ch .. 64 ch + 63 of the slot
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            const uint8_t *row = ubox(buf, 2 * ch + hb) + r * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 a = *reinterpret_cast<const float4 *>(row + ((k ^ (r & 7)) << 4));
                u[32 * hb + 4 * k] = a.x; u[32 * hb + 4 * k + 1] = a.y;
                u[32 * hb + 4 * k + 2] = a.z; u[32 * hb + 4 * k + 3] = a.w;
            }
        }
        if (!p.merged) {          // the scan's state entering this segment
#pragma unroll
            for (int k = 0; k < 64; ++k) S[k] = u[k];
        } else if (i < nmaps) {   // S_in += Diag(w) U_m, m = seg-1-i; then w *= g_m
#pragma unroll
            for (int k = 0; k < 64; ++k) S[k] = fmaf(wr, u[k], S[k]);
            wr *= gi;
        } else {                  // the sequence's final state: Diag(g_k) S_in + U_k
            const float gk = gi;
            const size_t rowoff = (size_t)bh * 16384 + (size_t)r * 128 + 64 * ch;
            float4 *d1 = p.hT ? reinterpret_cast<float4 *>(p.hT + rowoff) : nullptr;
            float4 *d2 = p.hTs ? reinterpret_cast<float4 *>(p.hTs + rowoff) : nullptr;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float4 w = make_float4(fmaf(gk, S[4 * k], u[4 * k]), fmaf(gk, S[4 * k + 1], u[4 * k + 1]),
                                             fmaf(gk, S[4 * k + 2], u[4 * k + 2]), fmaf(gk, S[4 * k + 3], u[4 * k + 3]));
                if (d1) d1[k] = w;
                if (d2) d2[k] = w;
            }
        }
        __syncthreads();   // the buffer has been read
        if (tid == 0 && i + nbuf < nslots) load_u(i + nbuf);
    }
    if (!flagged && ok) {
#pragma unroll
        for (int i = 0; i < 64; ++i) smax = fmaxf(smax, fabsf(S[i]));
        go = __syncthreads_or(smax >= kFixStop);
    }
    for (int c = 0; go && c < N; ++c) {
        const int s = NS == 2 ? (c & 1) : 0, par = (c / NS) & 1;
        const int tok = (g0 + c) * kTile, slot = bh * p.ntiles + g0 + c;
        if (__syncthreads_or(!mbar_wait(&m->fullQG[s], par))) { ok = false; break; }
        waited_qg = c + 1;
        if (c > 0) prep(s);   // the first chunk's q e^{b} came ready-made
        // bf16(S_c) -> X, the MN-major B operand (row r = key dim, columns = value dims)
        {
            float v[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = S[32 * hh + i];
                store_chunk_bf16(X, r, 2 * ch + hh, v);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        // whether the carried state still matters after this chunk
        const bool next = __syncthreads_or(decay * m->EB[r] * smax >= kFixStop) && c + 1 < N;
        if (tid == 0) {   // O = Qt bf16(S_c): M = tokens, N = value dims, K = key dims
            tc_fence_after();
            const uint64_t dQ = sdesc_sw128(smem_u32(Qb(s)), 16, 1024);
            const uint64_t dXm = sdesc_sw128(smem_u32(X), kBlk, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kBlk + (kk & 3) * 32;
                mma_bf16_ss(tbase, sdesc_add(dQ, ko), sdesc_add(dXm, kk * 2048), id_kmn, kk > 0);
            }
            mma_commit(&m->barM);
            if (next && NS == 2) {   // the other stage: chunk c-1's MMA is complete, its stores read
                tma_store_wait_read0();
                load_qg(c + 1);
                load_o(c + 1);
            } else if (next) {   // one stage: the next chunk's tiles into L2 for its loads after the stores
                const int tn = (g0 + c + 1) * kTile, sn = bh * p.ntiles + g0 + c + 1;
                for (int k = 0; k < 2; ++k) {
                    tma_prefetch_l2_4d(&tm_q, 64 * k, h, tn, b);
                    tma_prefetch_l2_4d(&tm_lf, 64 * k, h, tn, b);
                    tma_prefetch_l2_4d(&tm_o, 64 * k, h, tn, b);
                    tma_prefetch_l2_4d(&tm_st, 64 * k, 0, 0, sn);
                }
            }
        }
        if (__syncthreads_or(!mbar_wait(&m->fullO[s], par) || !mbar_wait(&m->barM, c & 1))) { ok = false; break; }
        waited_o = c + 1;
        tc_fence_after();
        // the saved state of this chunk, row r (key dim): + e^{rho} S_c
        if (p.save) {
            const float er = m->ER[r];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float v[32];
                const int cc = 2 * ch + hh;
                uint8_t *base = Sb + (cc >> 1) * kBlk + r * 128;
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(base + (((4 * (cc & 1) + qd) ^ (r & 7)) << 4));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        v[8 * qd + 2 * k] = bf_lo(ws[k]) + er * S[32 * hh + 8 * qd + 2 * k];
                        v[8 * qd + 2 * k + 1] = bf_hi(ws[k]) + er * S[32 * hh + 8 * qd + 2 * k + 1];
                    }
                }
                store_chunk_bf16(Sb, r, cc, v);
            }
        }
        // o row r (token) += O row r
        {
            float v[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int cc = 2 * ch + hh;
                tmem_ld32(tl + 32 * cc, v);
                tmem_wait_ld();
                uint8_t *base = Ob(s) + (cc >> 1) * kBlk + r * 128;
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
                store_chunk_bf16(Ob(s), r, cc, v);
            }
        }
        // the carried state to the next chunk
        const float eb = m->EB[r];
        decay *= eb;
#pragma unroll
        for (int i = 0; i < 64; ++i) S[i] *= eb;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            for (int k = 0; k < 2; ++k) {
                tma_store_4d(&tm_o, Ob(s) + k * kBlk, 64 * k, h, tok, b);
                if (p.save) tma_store_4d(&tm_st, Sb + k * kBlk, 64 * k, 0, 0, slot);
            }
            tma_store_commit();
            if (next && NS == 1) {   // the single stage, once this chunk's stores have read it
                tma_store_wait_read0();
                load_qg(c + 1);
                load_o(c + 1);
            }
        }
        go = next;
    }
    if (tid == 0) {
        if (!ok) set_status(HGRN2_ERR_TIMEOUT);
        // loads still in flight: the first chunk's when the carried state was negligible, or
        // any after a timeout
        for (int k = waitedU; k < issuedU; ++k) mbar_wait(&m->fullU[k % nbuf], (k / nbuf) & 1, 2000000u);
        for (int k = waited_qg; k < issued_qg; ++k) mbar_wait(&m->fullQG[NS == 2 ? (k & 1) : 0], (k / NS) & 1, 2000000u);
        for (int k = waited_o; k < issued_o; ++k) mbar_wait(&m->fullO[NS == 2 ? (k & 1) : 0], (k / NS) & 1, 2000000u);
        tma_store_wait_all0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 128);
}

}  // namespace tcf

// ------------------------------------------------------------------ host side
static_assert(tcf::kSmemBytes <= 227 * 1024, "forward shared memory");
static_assert(tcf::kAggSmem <= 227 * 1024, "aggregate shared memory");
static_assert(tcf::fix_smem(false) <= 227 * 1024 && tcf::fix_smem(true) <= 227 * 1024, "fix-up shared memory");
static_assert(sd::fwd_smem(128, 128) <= tcf::kSmemBytes, "scalar-decay exact forward inside the forward kernel");

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
    if (nseg <= 1) return 0;
    // per segment: U, g, the first chunk's B, the row sums of |U| (fp32) and q e^{b} (bf16); then
    // the per-pair finished-segment counts
    return (size_t)B * H * nseg * ((16384 + 3 * 128) * sizeof(float) + 16384 * sizeof(__nv_bfloat16)) +
           (size_t)B * H * sizeof(int);
}

size_t tc_fwd_smem() { return tcf::kSmemBytes; }

// segments, then the fix-up, with the scan between them beyond kMergedScanMax segments
int tc_fwd_launches(int nseg) { return nseg <= 1 ? 1 : nseg <= tcf::kMergedScanMax ? 2 : 3; }

// Slots of the saved bf16 chunk states: [B*H*ntiles] (slot bh * ntiles + n), or for packed
// sequences [(T / 128 + nseq) * H] (slot ((cu[s] / 128) + s + n) * H + h: sequence s's chunks
// never reach sequence s+1's first slot, whatever the lengths).
int tc_saved_slots(int B, int T, int H, bool packed) {
    return packed ? ((T >> 7) + B) * H : B * H * ((T + tcc::kTile - 1) / tcc::kTile);
}

// The whole slice as one segment: (g, U) of every (b,h), [B*H][128] and [B*H][128][128].
cudaError_t launch_tc_state_map(const void *lf, const void *x, int B, int T, int H, float *g, float *U,
                                cudaStream_t st) {
    CUtensorMap ml, mx;
    if (!make_token_map(&ml, lf, B, T, H, 128) || !make_token_map(&mx, x, B, T, H, 128)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tcf::agg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tcf::kAggSmem);
    if (e != cudaSuccess) return e;
    const int ntiles = (T + tcc::kTile - 1) / tcc::kTile;
    tcf::AggParams ap{U, g, nullptr, nullptr, H, 2, ntiles};
    tcf::agg_kernel<<<B * H, tcf::kThreads, tcf::kAggSmem, st>>>(ml, mx, ap);
    return cudaGetLastError();
}

// Launches a kernel as a programmatic dependent of the previous work in the stream: it may be
// scheduled before that work completes, and waits for it with grid_dep_wait().
template <typename... Exp, typename... Act>
static cudaError_t launch_dependent(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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

cudaError_t launch_tc_fwd(const TcFwdArgs &a, cudaStream_t st) {
    const bool packed = a.cu != nullptr;   // a.B is then the number of sequences
    const int Bm = packed ? 1 : a.B;
    const int nbk = a.nK * a.nV;
    const bool inplace = nbk > 1;
    if (inplace && (packed || a.lgs || a.D != 128 || a.nK != a.nV || a.H % nbk || !a.opart)) return cudaErrorInvalidValue;
    const int Hk = inplace ? a.H / nbk * a.nK : a.H, Hv = inplace ? a.H / nbk * a.nV : a.H;
    CUtensorMap mq, ml, mx, mo, mst;
    if (!make_token_map(&mq, a.q, Bm, a.T, Hk, a.D) || !make_token_map(&ml, a.lf, Bm, a.T, Hk, a.D) ||
        !make_token_map(&mx, a.x, Bm, a.T, Hv, a.D) || !make_token_map(&mo, a.o, Bm, a.T, Hv, a.D))
        return cudaErrorInvalidValue;
    // saved states: 128-row "token" tiles
    if (a.st16 && !make_token_map(&mst, a.st16, tc_saved_slots(a.B, a.T, a.H, packed), 128, 1))
        return cudaErrorInvalidValue;
    if (!a.st16) mst = mo;   // unused
    const bool scalar = a.lgs != nullptr;   // the scalar-decay variant (a.lf is then the key k)
    const int ntiles = (a.T + tcc::kTile - 1) / tcc::kTile;
    int nseg = 1, tps = ntiles;
    if (!packed && !scalar && !inplace && a.D == 128) tc_fwd_segments(a.B, a.T, a.H, &nseg, &tps);   // else one CTA per (b,h)
    auto kern = packed ? tcf::fwd_kernel<true>
                : scalar ? tcf::fwd_kernel<false, true>
                : nseg > 1 ? tcf::fwd_kernel<false, false, true>
                : tcf::fwd_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tcf::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int BH = a.B * a.H;
    // segment workspace: U [BH][nseg][128][128], g, the first chunk's B and the row sums of |U|
    // [BH][nseg][128] (fp32), the first chunk's q e^{b} [BH][nseg][128][128] (bf16), the
    // finished-segment counts [BH]
    const size_t nsl = (size_t)BH * nseg;
    float *U = a.seg_ws, *g = a.seg_ws ? U + nsl * 16384 : nullptr, *bs = a.seg_ws ? g + nsl * 128 : nullptr;
    float *uabs = a.seg_ws ? bs + nsl * 128 : nullptr;
    __nv_bfloat16 *qtil = a.seg_ws ? reinterpret_cast<__nv_bfloat16 *>(uabs + nsl * 128) : nullptr;
    int *seg_done = a.seg_ws ? reinterpret_cast<int *>(qtil + nsl * 16384) : nullptr;
    if (nseg > 1) {
        // pass 1 only raises the exact-route flags and counts finished segments: both start at zero
        if (!a.seg_ws || !a.flags) return cudaErrorInvalidValue;
        if ((e = cudaMemsetAsync(a.flags, 0, sizeof(int) * (size_t)BH, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(seg_done, 0, sizeof(int) * (size_t)BH, st)) != cudaSuccess) return e;
    }
    tcf::Params p{a.h0, a.hT, (__nv_bfloat16 *)a.o, (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.lf,
                  (const __nv_bfloat16 *)a.x, a.simt_C, a.flags, U, g, a.T, a.H, ntiles, nseg, tps,
                  a.st16 != nullptr, a.st16 ? a.hTs : nullptr, a.cu, a.perm, a.D,
                  (const __nv_bfloat16 *)a.lgs, seg_done, a.nK, a.nV, Bm,
                  nseg > 1 ? qtil : nullptr, nseg > 1 ? bs : nullptr, (__nv_bfloat16 *)a.opart, 0, 0, 0};
    // the segments' final states U leave through shared memory by TMA (measured: U stores 4 us
    // sooner on the long sequence; for one CTA per pair the row stores of hT, whose drain does not
    // hold the CTA, measured 1 us faster than the TMA store and its wait)
    p.uabs = nseg > 1 ? uabs : nullptr;
    CUtensorMap mh1 = mo, mh2 = mo;
    if (a.D == 128 && nseg > 1 && U && make_state_map(&mh1, U, (size_t)BH * nseg * 128)) {
        p.hmaps = 1;
        p.hslot1 = 1;
    }
    kern<<<BH * nseg, tcf::kFwdThreads, tcf::kSmemBytes, st>>>(mq, ml, mx, mo, mst, mh1, mh2, p);
    if ((e = cudaGetLastError()) != cudaSuccess || nseg == 1) return e;
    // segments: the states entering them (and hT), then the carried states' contributions.  With
    // up to kMergedScanMax segments the fix-up sums the states it needs itself, nearest first;
    // else the scan kernel chains them first.
    // Each launch is a programmatic dependent of the one before it, so that its start-up overlaps
    // that kernel's end.
    const bool merged = nseg <= tcf::kMergedScanMax;
    if (!merged) {
        e = launch_dependent(tcf::scan_kernel, dim3(BH * 16), dim3(256), 0, st, U, (const float *)g, nseg,
                             (const int *)a.flags, a.hT, a.st16 ? a.hTs : nullptr);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mqt, mu;   // the first chunks' q e^{b}: 128-row tiles, one per segment slot; the state slots
    if (!make_token_map(&mqt, qtil, (int)nsl, 128, 1) || !make_state_map(&mu, U, nsl * 128)) return cudaErrorInvalidValue;
    const size_t fsm = tcf::fix_smem(a.st16 != nullptr);
    e = cudaFuncSetAttribute(tcf::fixup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm);
    if (e != cudaSuccess) return e;
    tcf::FixParams fp{U, g, uabs, bs, a.flags, merged ? a.hT : nullptr, merged && a.st16 ? a.hTs : nullptr,
                      a.H, nseg, tps, ntiles, a.st16 != nullptr, merged};
    e = launch_dependent(tcf::fixup_kernel, dim3(BH * (nseg - 1)), dim3(tcf::kThreads), fsm, st, mq, ml, mo, mst,
                         mqt, mu, fp);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace hgrn2
