// pair_attention.cu -- the fused chunk attention at head_dim 128 on a CTA
// pair: a cluster of two CTAs on two SMs whose tensor cores run each MMA
// together (tcgen05 cta_group::2, M = 256).
//
// What it computes is the plain definition (no causal mask): for every valid
// query row i of a (session, head),
//     O_i = sum_j softmax_j(scale * q_i . k_j) v_j,   LSE_i = ln sum_j e^{scale q_i.k_j}
// over every valid slot j of every KV segment.  Sources: "StreamRender-H3"
// (molayo1419.me) -- streaming context section (bidirectional attention
// inside the window; the moving part sees the whole window) and inference
// acceleration section (FlashAttention on Blackwell tuned to the streaming
// shapes; persistent KV in the kernel's layout); "AlayaRenderer-Flash"
// (aitrends.kr) -- methodology (past chunks as clean tokens; persistent
// style-prompt KV in every self-attention layer).
//
// Why a pair.  With one SM per 256 query rows, S = Q K^T reads both operands
// from shared memory at the SM's full shared-memory bandwidth, and the
// tensor memory (two S tiles, two O tiles = 512 columns) leaves no room to
// compute the next S while the softmax of the current one runs, so the
// tensor core waits for the softmax every tile.  In a pair each SM owns 128
// query rows and holds only half of every K and V tile (the hardware
// exchanges the halves), which halves the operand traffic per SM and frees
// tensor memory for:
//     S buffers 0, 1   columns [0, 128), [128, 256)   S(j) in buffer j % 2
//     O_lo, O_hi       columns [256, 384), [384, 512)
// S(j + 2) is computed into the buffer of S(j) as soon as P(j) has been
// consumed, i.e. while the softmax works on S(j + 1).
//
// Softmax split by keys.  Warpgroup h (h = 0, 1) handles keys [64h, 64h + 64)
// of every KV tile for all 128 rows, with its own running max m_h and sum
// l_h, and its own accumulator O_h += P_h V[64h .. 64h + 64).  The two halves
// never exchange anything during the loop; the epilogue merges them:
//     M = max(m_lo, m_hi),  a_h = 2^(m_h - M),
//     O = (a_lo O_lo + a_hi O_hi) / (a_lo l_lo + a_hi l_hi),  LSE = M + log2(...)
// (log2 domain).  This is exact: each half is an ordinary online softmax over
// its keys and the merge is the usual combination of partial softmaxes.  A
// running max moves only when it grows by more than 2^8 (lazy rescale; the
// final normalisation uses the same stale max).
//
// Roles per CTA (384 threads):
//   warps 0-3   softmax, keys 0-63 of each tile; warps 4-7 keys 64-127: read
//               their half S row from TMEM, mask the segment tail, write P
//               (bf16 pairs) back over the first 32 columns of their half,
//               rescale O_h when the max moved (waiting for PV_h(j-1) only
//               then), then signal the MMA issuer.
//   warp 8      TMA producer: this CTA's 128 query rows, then its half of
//               every K tile (64 keys, all 128 dims) and of every V tile (all
//               128 keys, 64 of the dims) into 4-stage rings.
//   warp 9      even CTA: the single thread that issues every pair MMA;
//               odd CTA: forwards the completion of its own loads to the even
//               CTA (each CTA's loads complete on its own barriers, so each
//               can wait for its own copies in flight).
//   warps 8-11  after the loop: the epilogue (merge, normalise, bf16 store).
// MMA order: S(0), S(1), then per tile j: PV_lo(j), PV_hi(j), S(j + 2).
//
// Every wait is bounded (sr_device.cuh).  When one gives up, the CTA raises
// its abort flag and the peer's, sets the status word, and every role leaves
// its loop; then the producer waits (bounded) for its loads in flight, the
// issuer commits and waits (bounded) for its MMAs, and only after both CTAs
// have met at a cluster barrier is the tensor memory released.
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_device.cuh"
#include "sr_internal.h"

namespace sr {

namespace {

// Tuning parameters (the values built by default were chosen by measurement).
#ifndef SR_PAIR_STAGES
#define SR_PAIR_STAGES 4
#endif
#ifndef SR_PAIR_EXP2_FMA_EVERY
#define SR_PAIR_EXP2_FMA_EVERY 0
#endif
constexpr int kRows = 128;              // query rows per CTA
constexpr int kKeys = 128;              // keys per KV tile
constexpr int kStages = SR_PAIR_STAGES;  // depth of the K and V rings
// every kExpFmaEvery-th column's exponential runs on the FMA pipe (exp2_fma)
// instead of the MUFU pipe, whose 16 results per clock per SM equal the
// tensor core's pace at this tile shape; 0 = all on MUFU
constexpr int kExpFmaEvery = SR_PAIR_EXP2_FMA_EVERY;
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8, kWarpIssuer = 9;
constexpr int kPanel = 64;              // bf16 elements per 128-byte swizzle row
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

__host__ __device__ constexpr uint32_t tmem_s(int buf) { return static_cast<uint32_t>(buf) * 128u; }
__host__ __device__ constexpr uint32_t tmem_o(int h) { return 256u + static_cast<uint32_t>(h) * 128u; }

struct PairParams {
    __nv_bfloat16 *o;
    float *lse;
    const int32_t *kv_len;   // [B][n_seg]
    const int32_t *q_len;    // [B]
    int32_t *status;
    int32_t seg_start[SR_MAX_SEG];
    int32_t seg_cap[SR_MAX_SEG];
    int32_t n_seg;
    int32_t n_heads;
    int32_t q_cap;
    float scale_log2;        // softmax_scale * log2(e)
    int32_t qb_per_head;     // 256-row query blocks per (session, head)
    int32_t n_full;          // items [0, n_full) are whole units
    int32_t split;           // KV parts per tail unit
    float *ws_o;             // [slot][2][128][128] unnormalised partial O
    float *ws_ml;            // [slot][m | l][2][128]
    uint64_t wait_limit_ns;
    int32_t withheld_tile;   // test hook: the K tile whose load is withheld (-1: none)
};

struct Layout {
    static constexpr int kQBytes = 2 * kRows * 128;      // 128 rows x 128 dims: two 64-dim panels
    static constexpr int kKBytes = 2 * (kKeys / 2) * 128;  // 64 keys x 128 dims: two panels
    static constexpr int kVBytes = kKeys * 128;          // 128 keys x 64 dims: one panel
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQBytes;
    static constexpr int kV = kK + kStages * kKBytes;
    static constexpr int kBar = kV + kStages * kVBytes;
    // q_full, q_peer, k_full[S], k_peer[S], v_full[S], v_peer[S], k_empty[S],
    // v_empty[S], s_full[2], p_full[2], pv_done[2][2], o_final, stats_ready, drain
    static constexpr int kNumBars = 2 + 6 * kStages + 8 + 3;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kRow = kMisc + 32 + 16 * SR_MAX_SEG;   // m[2][128], l[2][128]
    static constexpr int kEnd = kRow + 4 * kRows * 4;
    static constexpr int kAlloc = kEnd + 1024;   // slack for manual 1024-byte alignment
};
static_assert(Layout::kAlloc <= 227 * 1024, "shared memory");

// Walks the valid 128-token tiles of every segment in buffer order.
struct TileWalk {
    int s, t;
    __device__ void next(const int *ntile, int n_seg) {
        if (++t == ntile[s]) {
            t = 0;
            ++s;
            while (s < n_seg && ntile[s] == 0) ++s;
        }
    }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    pair_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const PairParams p) {
    using L = Layout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    // ---- work item (one per pair) -> (unit, KV part)
    const int item = static_cast<int>(blockIdx.x >> 1);
    int unit, part = 0, split = 1;
    if (item < p.n_full) {
        unit = item;
    } else {
        split = p.split;
        unit = p.n_full + (item - p.n_full) / split;
        part = (item - p.n_full) % split;
    }
    const int qb = unit % p.qb_per_head;
    const int bh = unit / p.qb_per_head;
    const int h = bh % p.n_heads, b = bh / p.n_heads;
    // q_len is caller data on the device: clamped to [0, q_cap]
    const int q_len = min(max(p.q_len[b], 0), p.q_cap);
    const int q_unit = qb * 2 * kRows;
    if (q_unit >= q_len) return;   // the same for both CTAs of the pair
    const int q0 = q_unit + static_cast<int>(rank) * kRows;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *q_full = bars;                   // this CTA's query rows landed
    uint64_t *q_peer = bars + 1;               // even CTA: the odd CTA's query rows landed
    uint64_t *k_full = bars + 2;               // [S] this CTA's K half landed
    uint64_t *k_peer = k_full + kStages;       // [S] even CTA: the odd CTA's K half landed
    uint64_t *v_full = k_peer + kStages;
    uint64_t *v_peer = v_full + kStages;
    uint64_t *k_empty = v_peer + kStages;      // [S] S MMA done with the stage (both CTAs)
    uint64_t *v_empty = k_empty + kStages;     // [S] PV MMAs done with the stage (both CTAs)
    uint64_t *s_full = v_empty + kStages;      // [2] S buffer computed (both CTAs)
    uint64_t *p_full = s_full + 2;             // [2] even CTA: P_h written by the 8 warps of half h
    uint64_t *pv_done = p_full + 2;            // [2][2] PV_h(j) complete, by h and j % 2 (both CTAs)
    uint64_t *o_final = pv_done + 4;           // last PV complete (both CTAs)
    uint64_t *stats_ready = o_final + 1;       // the 8 softmax warps stored their row statistics
    uint64_t *drain = stats_ready + 1;         // every MMA issued so far is complete (both CTAs)
    // Every waiter consumes each phase of its barrier in order, so parity
    // waits never alias (pv_done: see the softmax).
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    int *n_tiles_s = reinterpret_cast<int *>(smem + L::kMisc + 8);
    int *walk_start = reinterpret_cast<int *>(smem + L::kMisc + 16);   // (segment, tile) of the first tile
    int *seg_ntile = reinterpret_cast<int *>(smem + L::kMisc + 32);
    int *seg_len = seg_ntile + SR_MAX_SEG;
    int *seg_start = seg_len + SR_MAX_SEG;
    float *row_m = reinterpret_cast<float *>(smem + L::kRow);   // [2][128]
    float *row_l = row_m + 2 * kRows;                           // [2][128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_peer, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_peer[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_peer[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 8);   // 4 warps of half i in each CTA
            mbar_init(&pv_done[2 * i], 1);
            mbar_init(&pv_done[2 * i + 1], 1);
        }
        mbar_init(o_final, 1);
        mbar_init(stats_ready, 8);
        mbar_init(drain, 1);
        *abort_flag = 0;
        int total = 0;
#pragma unroll
        for (int s = 0; s < SR_MAX_SEG; ++s) {   // static indices keep the param arrays out of local memory
            int len = s < p.n_seg ? p.kv_len[b * p.n_seg + s] : 0;
            len = len < 0 ? 0 : (len > p.seg_cap[s] ? p.seg_cap[s] : len);
            seg_len[s] = len;
            seg_ntile[s] = (len + kKeys - 1) / kKeys;
            seg_start[s] = p.seg_start[s];
            total += seg_ntile[s];
        }
        const int tile0 = static_cast<int>((static_cast<int64_t>(part) * total) / split);
        const int tile1 = static_cast<int>((static_cast<int64_t>(part + 1) * total) / split);
        int s0 = 0, k = tile0;
        while (s0 < p.n_seg && (seg_ntile[s0] == 0 || k >= seg_ntile[s0])) {
            k -= seg_ntile[s0];
            ++s0;
        }
        n_tiles_s[0] = tile1 - tile0;
        walk_start[0] = s0;
        walk_start[1] = k;
        fence_mbarrier_init();
    }
    if (warp == kWarpIssuer) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs: barriers initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = *n_tiles_s;
    const int n_seg = p.n_seg;
    const float sl2 = p.scale_log2;
    const uint64_t limit = p.wait_limit_ns;
    const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int *>(abort_flag)), rank ^ 1u);
    // give up: raise the peer's abort flag too (this CTA's is already raised)
    auto fail = [&]() {
        st_cluster_u32(peer_abort, 1u);
        return false;
    };
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        return mbar_wait(bar, parity, abort_flag, p.status, limit) || fail();
    };
    auto wait_cluster = [&](uint64_t *bar, uint32_t parity) {
        return mbar_wait<true>(bar, parity, abort_flag, p.status, limit) || fail();
    };

    if (warp < 8) {
        // ================================================================ softmax, key half hf
        const int hf = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t p_full_addr = mapa_shared(smem_u32(&p_full[hf]), 0);   // in the even CTA
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int seen0 = 0, seen1 = 0;   // phases of pv_done[hf][0 / 1] consumed so far (registers)
        auto consume_pv = [&](int par, int upto) {
            int seen = par ? seen1 : seen0;
            bool good = true;
            while (good && seen <= upto) {
                good = wait(&pv_done[2 * hf + par], seen & 1);
                seen += good ? 1 : 0;
            }
            if (par)
                seen1 = seen;
            else
                seen0 = seen;
            return good;
        };
        TileWalk w;
        w.s = walk_start[0];
        w.t = walk_start[1];
        for (int j = 0; j < n_tiles; ++j, w.next(seg_ntile, n_seg)) {
            const int valid = min(max(min(kKeys, seg_len[w.s] - w.t * kKeys) - hf * 64, 0), 64);
            if (!(ok = __all_sync(0xffffffffu, wait(&s_full[j & 1], (j >> 1) & 1)))) break;
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + tmem_s(j & 1) + hf * 64;
            float s[64];
            {
                uint32_t r[2][32];
                tmem_ld32(s_addr, r[0]);
                tmem_ld32(s_addr + 32, r[1]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[c][e]);
            }
            if (valid < 64) {
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] = c < valid ? s[c] : -INFINITY;
            }
            // row max over eight independent chains, then a tree
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                mx8[i] = fmax3(s[i], s[8 + i], s[16 + i]);
                mx8[i] = fmax3(mx8[i], s[24 + i], s[32 + i]);
                mx8[i] = fmax3(mx8[i], s[40 + i], s[48 + i]);
                mx8[i] = fmaxf(mx8[i], s[56 + i]);
            }
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float m_new = fmaxf(m_run, mx * sl2);
            const bool need = m_new > m_run + kRescaleThreshold;
            const float m_use = need ? m_new : m_run;
            const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
            // a half that has seen no valid key yet keeps m = -inf: subtract 0
            // there (every score is -inf, every weight 0) instead of -inf
            const float m_sub = m_use == -INFINITY ? 0.f : m_use;
            float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float x = fmaf(s[c], sl2, -m_sub);
                s[c] = (kExpFmaEvery > 0 && c % (kExpFmaEvery > 0 ? kExpFmaEvery : 1) == kExpFmaEvery - 1)
                           ? exp2_fma(x)
                           : fast_exp2(x);
                sum8[c & 7] += s[c];
            }
            const float sum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
            l_run = l_run * alpha + sum;
            m_run = m_use;
            {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(s[2 * e], s[2 * e + 1]);
                tmem_st32(s_addr, pk);
            }
            // PV_hf(i) completes a phase of pv_done[hf][i & 1].  Every iteration
            // consumes PV(j-2) (long complete: S(j) was issued after it), and a
            // rescale of O_hf, which needs PV(j-1) complete, consumes that one
            // first; so no waiter falls two phases behind its barrier (PV(j)
            // cannot complete before this P is handed over) and parity waits
            // never alias, while the common path never waits on the tensor core.
            if (j >= 2 && !(ok = __all_sync(0xffffffffu, consume_pv(j & 1, (j - 2) >> 1)))) break;
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                if (!(ok = __all_sync(0xffffffffu, consume_pv((j - 1) & 1, (j - 1) >> 1)))) break;
                {
                    tc_fence_after();
                    const uint32_t o_addr = tmem + lane_base + tmem_o(hf);
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld32(o_addr + c * 32, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(o_addr + c * 32, r);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(&p_full[hf]);
                else
                    mbar_arrive_remote(p_full_addr);
            }
        }
        row_m[hf * kRows + row] = m_run;
        row_l[hf * kRows + row] = l_run;
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(stats_ready);
    } else {
        if (warp == kWarpProducer && lane == 0 && n_tiles > 0) {
            // ============================================================ TMA producer
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_expect_tx(q_full, L::kQBytes);
#pragma unroll
            for (int pn = 0; pn < 2; ++pn)
                tma_load_3d(smem + L::kQ + pn * (L::kQBytes / 2), &tmQ, pn * kPanel, q0, bh, q_full);
            int k_last[kStages], v_last[kStages];   // last tile loaded into each stage (for the drain)
#pragma unroll
            for (int i = 0; i < kStages; ++i) k_last[i] = v_last[i] = -1;
            TileWalk wk, wv;
            wk.s = wv.s = walk_start[0];
            wk.t = wv.t = walk_start[1];
            int kt = 0;   // next K tile to load
            auto load_k = [&]() {
                const int st = kt % kStages;
                if (!wait(&k_empty[st], ((kt / kStages) & 1) ^ 1)) return false;
                if (kt != p.withheld_tile) {
                    const int row0 = seg_start[wk.s] + wk.t * kKeys + static_cast<int>(rank) * (kKeys / 2);
                    mbar_expect_tx(&k_full[st], L::kKBytes);
#pragma unroll
                    for (int pn = 0; pn < 2; ++pn)
                        tma_load_3d(smem + L::kK + st * L::kKBytes + pn * (L::kKBytes / 2), &tmK, pn * kPanel, row0,
                                    bh, &k_full[st]);
                    k_last[st] = kt;
                }
                ++kt;
                wk.next(seg_ntile, n_seg);
                return true;
            };
            bool ok = load_k() && (n_tiles < 2 || load_k());
            for (int j = 0; ok && j < n_tiles; ++j, wv.next(seg_ntile, n_seg)) {
                const int st = j % kStages;
                if (!(ok = wait(&v_empty[st], ((j / kStages) & 1) ^ 1))) break;
                mbar_expect_tx(&v_full[st], L::kVBytes);
                tma_load_3d(smem + L::kV + st * L::kVBytes, &tmV, static_cast<int>(rank) * kPanel,
                            seg_start[wv.s] + wv.t * kKeys, bh, &v_full[st]);
                v_last[st] = j;
                if (j + 2 < n_tiles) ok = load_k();
            }
            if (*abort_flag) {
                // wait, bounded, for this CTA's own loads still in flight
                mbar_drain(q_full, 0, limit);
                for (int i = 0; i < kStages; ++i) {
                    if (k_last[i] >= 0) mbar_drain(&k_full[i], (k_last[i] / kStages) & 1, limit);
                    if (v_last[i] >= 0) mbar_drain(&v_full[i], (v_last[i] / kStages) & 1, limit);
                }
            }
        } else if (warp == kWarpIssuer && lane == 0 && n_tiles > 0) {
            if (leader) {
                // ======================================================== pair MMA issuer
                constexpr uint32_t idesc_s = umma_idesc_bf16(2 * kRows, kKeys, false, false);
                constexpr uint32_t idesc_pv = umma_idesc_bf16(2 * kRows, 128, false, true);
                const uint64_t desc_q = umma_desc_sw128(smem_u32(smem + L::kQ), 16, 1024);
                const uint64_t desc_k = umma_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
                const uint64_t desc_v = umma_desc_sw128(smem_u32(smem + L::kV), L::kVBytes, 1024);
                constexpr uint16_t kBoth = 3;
                auto issue_s = [&](int buf, int st) {
                    const uint64_t b0 = umma_desc_advance(desc_k, st * L::kKBytes);
                    const uint32_t d = tmem + tmem_s(buf);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_pair_ss(d, umma_desc_advance(desc_q, (kk >> 2) * (L::kQBytes / 2) + (kk & 3) * 32),
                                     umma_desc_advance(b0, (kk >> 2) * (L::kKBytes / 2) + (kk & 3) * 32), idesc_s,
                                     kk > 0 ? 1u : 0u);
                    umma_commit_pair(&s_full[buf], kBoth);
                    umma_commit_pair(&k_empty[st], kBoth);
                };
                auto issue_pv = [&](int hf, int buf, int st, bool acc) {
                    const uint64_t b0 = umma_desc_advance(desc_v, st * L::kVBytes + hf * (L::kVBytes / 2));
                    const uint32_t d = tmem + tmem_o(hf);
                    const uint32_t a = tmem + tmem_s(buf) + hf * 64;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_pair_ts(d, a + kk * 8, umma_desc_advance(b0, kk * 2048), idesc_pv,
                                     (acc || kk > 0) ? 1u : 0u);
                    umma_commit_pair(&pv_done[2 * hf + (buf & 1)], kBoth);
                };
                auto wait_k = [&](int t) {
                    const int st = t % kStages;
                    const uint32_t ph = (t / kStages) & 1;
                    return wait(&k_full[st], ph) && wait_cluster(&k_peer[st], ph);
                };
                bool ok = wait(q_full, 0) && wait_cluster(q_peer, 0) && wait_k(0);
                if (ok) {
                    tc_fence_after();
                    issue_s(0, 0);
                    if (n_tiles > 1) {
                        if ((ok = wait_k(1))) {
                            tc_fence_after();
                            issue_s(1, 1);
                        }
                    }
                }
                for (int j = 0; ok && j < n_tiles; ++j) {
                    const int st = j % kStages;
                    const uint32_t ph = (j / kStages) & 1;
                    if (!(ok = wait(&v_full[st], ph) && wait_cluster(&v_peer[st], ph))) break;
                    if (!(ok = wait_cluster(&p_full[0], j & 1))) break;
                    tc_fence_after();
                    issue_pv(0, j & 1, st, j > 0);
                    if (!(ok = wait_cluster(&p_full[1], j & 1))) break;
                    tc_fence_after();
                    issue_pv(1, j & 1, st, j > 0);
                    umma_commit_pair(&v_empty[st], kBoth);
                    if (j + 2 < n_tiles) {
                        if (!(ok = wait_k(j + 2))) break;
                        tc_fence_after();
                        issue_s(j & 1, (j + 2) % kStages);
                    }
                }
                if (ok) umma_commit_pair(o_final, kBoth);
                // every MMA issued so far complete (in both CTAs) before anyone
                // may release shared or tensor memory
                umma_commit_pair(drain, kBoth);
                mbar_drain(drain, 0, limit);
            } else {
                // ======================================================== forwarder (odd CTA)
                const uint32_t rq = mapa_shared(smem_u32(q_peer), 0);
                const uint32_t rk = mapa_shared(smem_u32(k_peer), 0);
                const uint32_t rv = mapa_shared(smem_u32(v_peer), 0);
                auto fwd_k = [&](int t) {
                    const int st = t % kStages;
                    if (!wait(&k_full[st], (t / kStages) & 1)) return false;
                    mbar_arrive_remote(rk + st * 8);
                    return true;
                };
                bool ok = wait(q_full, 0);
                if (ok) mbar_arrive_remote(rq);
                ok = ok && fwd_k(0) && (n_tiles < 2 || fwd_k(1));
                for (int j = 0; ok && j < n_tiles; ++j) {
                    const int st = j % kStages;
                    if (!(ok = wait(&v_full[st], (j / kStages) & 1))) break;
                    mbar_arrive_remote(rv + st * 8);
                    if (j + 2 < n_tiles) ok = fwd_k(j + 2);
                }
                // the even CTA's MMAs read this CTA's shared memory and write its
                // tensor memory: wait (bounded) until they are all complete
                mbar_drain(drain, 0, limit);
            }
        }
        __syncwarp();
        // ================================================================ epilogue (warps 8-11)
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int grow = q0 + row;
        const bool row_ok = grow < q_len;
        bool ok = n_tiles == 0 || (__all_sync(0xffffffffu, wait(stats_ready, 0)) &&
                                   __all_sync(0xffffffffu, wait(o_final, 0)));
        if (ok) {
            tc_fence_after();
            float a_lo = 0.f, a_hi = 0.f, M = -INFINITY, Lsum = 0.f;
            if (n_tiles > 0) {
                const float m_lo = row_m[row], m_hi = row_m[kRows + row];
                M = fmaxf(m_lo, m_hi);
                a_lo = m_lo == -INFINITY ? 0.f : fast_exp2(m_lo - M);
                a_hi = m_hi == -INFINITY ? 0.f : fast_exp2(m_hi - M);
                Lsum = a_lo * row_l[row] + a_hi * row_l[kRows + row];
            }
            if (split == 1) {
                __nv_bfloat16 *orow = p.o + ((static_cast<size_t>(b) * p.q_cap + grow) * p.n_heads + h) * 128;
                const float inv = Lsum > 0.f ? 1.0f / Lsum : 0.f;
                const float w_lo = a_lo * inv, w_hi = a_hi * inv;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t lo[32], hi[32];
                    if (n_tiles > 0) {
                        tmem_ld32(tmem + lane_base + tmem_o(0) + c * 32, lo);
                        tmem_ld32(tmem + lane_base + tmem_o(1) + c * 32, hi);
                        tmem_wait_ld();
                    }
                    if (row_ok) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f[i] = n_tiles > 0 ? __uint_as_float(lo[e + i]) * w_lo + __uint_as_float(hi[e + i]) * w_hi
                                                   : 0.f;
                            uint4 v;
                            v.x = pack_bf16x2(f[0], f[1]);
                            v.y = pack_bf16x2(f[2], f[3]);
                            v.z = pack_bf16x2(f[4], f[5]);
                            v.w = pack_bf16x2(f[6], f[7]);
                            *reinterpret_cast<uint4 *>(orow + c * 32 + e) = v;
                        }
                    }
                }
                if (row_ok && p.lse)
                    p.lse[static_cast<size_t>(bh) * p.q_cap + grow] =
                        Lsum > 0.f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
            } else {
                // split unit: this part's unnormalised (O, m, l) for the merge kernel
                const int slot = item - p.n_full;
                float *o_part = p.ws_o + (static_cast<size_t>(slot) * 2 + rank) * kRows * 128 +
                                static_cast<size_t>(row) * 128;
                float *ws_m = p.ws_ml + static_cast<size_t>(slot) * 4 * kRows;
#pragma unroll 1
                for (int c = 0; c < 4 && n_tiles > 0; ++c) {
                    uint32_t lo[32], hi[32];
                    tmem_ld32(tmem + lane_base + tmem_o(0) + c * 32, lo);
                    tmem_ld32(tmem + lane_base + tmem_o(1) + c * 32, hi);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        __stcg(reinterpret_cast<float4 *>(o_part + c * 32 + e),
                               make_float4(__uint_as_float(lo[e]) * a_lo + __uint_as_float(hi[e]) * a_hi,
                                           __uint_as_float(lo[e + 1]) * a_lo + __uint_as_float(hi[e + 1]) * a_hi,
                                           __uint_as_float(lo[e + 2]) * a_lo + __uint_as_float(hi[e + 2]) * a_hi,
                                           __uint_as_float(lo[e + 3]) * a_lo + __uint_as_float(hi[e + 3]) * a_hi));
                }
                __stcg(ws_m + rank * kRows + row, M);
                __stcg(ws_m + (2 + rank) * kRows + row, Lsum);
            }
        }
    }

    // ---- teardown: every role of this CTA is done (including the drains);
    // then both CTAs meet, so neither touches the other's memory afterwards,
    // and only then is the tensor memory of the pair released
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == kWarpIssuer) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// Pair slots the GPU can hold at once (clusters of two co-resident CTAs).
int pair_slots() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 74;
    if (!cached[dev]) {
        int n = 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 148, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = Layout::kAlloc;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaFuncSetAttribute(pair_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::kAlloc) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, pair_attention_kernel, &cfg) != cudaSuccess || n <= 0) {
            int sms = 0;
            if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 1) sms = 148;
            n = sms / 2;
        }
        cudaGetLastError();   // a failed query leaves no sticky error behind
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace

int attention_pair_slots() { return pair_slots(); }

int launch_pair_attention(const AttnLaunch &a, const AttnSchedule &sc) {
    CUtensorMap tq, tk, tv;
    const uint64_t bh = static_cast<uint64_t>(a.n_batch) * a.n_heads;
    int rc = make_tmap_bf16_3d(&tq, a.q, 128, static_cast<uint64_t>(a.q_cap), bh, kPanel, kRows);
    if (rc == SR_OK) rc = make_tmap_bf16_3d(&tk, a.k, 128, static_cast<uint64_t>(a.kv_tokens), bh, kPanel, kKeys / 2);
    if (rc == SR_OK) rc = make_tmap_bf16_3d(&tv, a.v, 128, static_cast<uint64_t>(a.kv_tokens), bh, kPanel, kKeys);
    if (rc != SR_OK) return rc;
    PairParams p{};
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.kv_len = a.kv_len;
    p.q_len = a.q_len;
    p.status = a.status;
    int acc = 0;
    for (int s = 0; s < SR_MAX_SEG; ++s) {
        p.seg_start[s] = acc;
        p.seg_cap[s] = s < a.n_seg ? a.cap[s] : 0;
        acc += p.seg_cap[s];
    }
    p.n_seg = a.n_seg;
    p.n_heads = a.n_heads;
    p.q_cap = a.q_cap;
    p.scale_log2 = static_cast<float>(static_cast<double>(a.softmax_scale) * 1.4426950408889634);
    p.qb_per_head = sc.qb_per_head;
    p.n_full = sc.n_full;
    p.split = 1;
    p.wait_limit_ns = a.wait_limit_ns;
    p.withheld_tile = a.withheld_tile;
    int64_t items = sc.units;
    if (sc.split > 1 && a.workspace && a.workspace_bytes >= sc.workspace_bytes) {
        uint8_t *ws = static_cast<uint8_t *>(a.workspace);
        p.split = sc.split;
        p.ws_o = reinterpret_cast<float *>(ws);
        p.ws_ml = reinterpret_cast<float *>(ws + sc.o_bytes);
        items = sc.n_full + static_cast<int64_t>(sc.tail_units) * sc.split;
    } else {
        p.n_full = static_cast<int32_t>(sc.units);
    }
    static bool attr_set[64] = {};   // the shared-memory opt-in is per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(pair_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::kAlloc);
        if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(pair_attention)", e);
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    if (items > 0x3fffffff) return set_error(SR_ERR_INVALID_ARG, "chunk_attention: too many work items");
    pair_attention_kernel<<<static_cast<unsigned>(2 * items), kThreads, Layout::kAlloc, a.stream>>>(tq, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("pair_attention launch", e);
    if (p.split > 1)
        return launch_split_combine(p.ws_o, p.ws_ml, p.o, p.lse, p.q_len, p.n_full, p.split, sc.tail_units,
                                    p.qb_per_head, p.n_heads, p.q_cap, 128, a.stream);
    return SR_OK;
}

}  // namespace sr
