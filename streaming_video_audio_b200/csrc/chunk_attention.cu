// chunk_attention.cu -- fused chunk attention over [prompt | context | chunk]
// KV segments on sm_100a (tcgen05 tensor cores, TMEM accumulators, TMA).
//
// What it computes (plain definition, no causal mask): for every valid query
// row i of a (session, head),
//     O_i = sum_j softmax_j(scale * q_i . k_j) v_j,   LSE_i = ln sum_j e^{scale q_i.k_j}
// over every valid slot j of every KV segment.  Sources: "StreamRender-H3"
// (molayo1419.me) -- streaming context section (bidirectional attention
// inside the window; the moving part sees the whole window) and inference
// acceleration section (FlashAttention on Blackwell tuned to the streaming
// shapes with a single KV split; persistent KV kept in the kernel's layout);
// "AlayaRenderer-Flash" (aitrends.kr) -- methodology (past chunks as clean
// tokens; persistent style-prompt KV in every self-attention layer).
//
// Design (one CTA = two 128-row query tiles Q0, Q1 of one (session, head),
// sharing every K/V tile; 16 warps):
//   warps 0-3   softmax of Q0, warps 4-7 softmax of Q1 (one thread per query
//               row): read the S row from TMEM, mask the segment tail, keep an
//               fp32 running max/sum in the log2 domain, write P (bf16 pairs)
//               back into TMEM over the S columns.  The max only moves when it
//               grows by more than 2^8 (lazy rescale: exact, the final
//               normalisation uses the same stale max).
//               When a row's max does move, the softmax warp rescales its O_t
//               row in TMEM itself: S_t(j) is issued after PV_t(j-1) and its
//               commit tracks every earlier MMA, so once S_t(j) has landed
//               PV_t(j-1) has too, and PV_t(j) waits for this warp's P.
//   warps 8-11  epilogue: O / l -> bf16 token-major output and LSE, staged in
//               Q_t's shared memory and stored by tiled copies (or the
//               unnormalised partials of a split unit).
//   warp 12     TMA producer: Q0, Q1 once, then K and V tiles (128 tokens) into
//               a two-stage ring (stage i: K(i) and V(i-1), one barrier pair),
//               walking only the segments' valid tiles.
//   warp 13     TMEM owner + single-thread tcgen05.mma issuer, ping-pong order
//                 PV0(j), S0(j+1) = Q0 K(j+1)^T, PV1(j), S1(j+1)
//               so the tensor core works on one tile while the other tile's
//               softmax runs.  S = Q K^T reads both operands from shared memory;
//               O += P V reads P from TMEM (A operand) and V from shared memory.
// TMEM: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512) (fp32 columns); P_t
// aliases the first 64 columns of S_t.  Every wait is bounded
// (sr_device.cuh): a stuck pipeline sets the status word and the CTA returns
// instead of hanging.
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_device.cuh"
#include "sr_internal.h"

namespace sr {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kQTiles = 2;               // query tiles per CTA
constexpr int kStages = 2;
constexpr int kThreads = 512;
constexpr int kWarpTma = 12, kWarpMma = 13;
constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16), one swizzle-128B panel
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
// The producer's waits for a free stage are never on the critical path (loads
// run a stage ahead): it polls with a suspend-time hint, leaving the issue
// slots of its SM sub-partition to the softmax warps there.
constexpr uint32_t kProducerSuspend = 5000;


// Registers per thread after reallocation (launch: 65536 / 512 = 128 each):
// 2 x 128 x 160 + 128 x 88 + 128 x 104 = 65536 (the launch total; no spills).
constexpr int kRegSoftmax = 160, kRegCorrection = 88, kRegOther = 104;

// Byte offset of 16-byte chunk k of row `row` in a tile of 64-column bf16
// panels (128 rows x 128 bytes each) laid out with the 128-byte swizzle.
__device__ __forceinline__ int sw128_offset(int row, int k) {
    return (k >> 3) * kPanelBytes + row * 128 + (((k & 7) ^ (row & 7)) << 4);
}

__host__ __device__ constexpr uint32_t tmem_s(int t) { return static_cast<uint32_t>(t) * 128u; }
__host__ __device__ constexpr uint32_t tmem_o(int t) { return 256u + static_cast<uint32_t>(t) * 128u; }

struct AttnParams {
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
    // work list: items [0, n_full) are whole units (one per CTA); the
    // remaining units are each split into `split` KV ranges whose partial
    // results meet in the workspace
    int32_t qb_per_head;     // 256-row query blocks per (session, head)
    int32_t n_full;
    int32_t split;
    float *ws_o;             // [slot][2][D/4][128][4] unnormalised partial O (column blocks of 4)
    float *ws_ml;            // [slot][m | l][2][128]
    uint64_t wait_limit_ns;
    int32_t withheld_tile;   // test hook: the K tile whose load is withheld (-1: none)
};

template <int D>
struct Smem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQTiles * kTileBytes;
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kBar = kV + kStages * kTileBytes;
    // q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2],
    // stats_ready[2], drain
    static constexpr int kNumBars = 1 + 2 * kStages + 4 * kQTiles + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kRow = kMisc + 16 + 12 * SR_MAX_SEG + 16;   // float l[2][128], m[2][128]
    static constexpr int kEnd = kRow + 2 * kQTiles * kTileM * 4;
    static constexpr int kAlloc = kEnd + 1024;   // slack for manual 1024-byte alignment
};

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



__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status, uint64_t limit, uint32_t suspend_ns = 0) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, limit, suspend_ns));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                           const AttnParams p) {
    using L = Smem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    // ---- work item -> (unit, KV part)
    const int item = blockIdx.x;
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
    // q_len is caller data on the device: clamped to [0, q_cap] so that no
    // row past the o / lse buffers is ever written, whatever it holds
    const int q_len = min(max(p.q_len[b], 0), p.q_cap);
    const int q0 = qb * kQTiles * kTileM;
    if (q0 >= q_len) return;   // uniform for the whole CTA

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *q_full = bars;
    // Stage i % kStages holds K(i) and V(i-1): the two tiles the MMAs of one
    // period read (PV(i-1) and S(i)), loaded and released under one barrier
    // pair, so that the issuing thread makes one load wait and one release
    // commit per KV tile.
    uint64_t *kv_full = bars + 1;
    uint64_t *kv_empty = kv_full + kStages;
    uint64_t *s_full = kv_empty + kStages;       // [2] MMA -> softmax t
    uint64_t *p_full = s_full + kQTiles;         // [2] softmax t -> MMA (P_t written, O_t rescaled)
    uint64_t *o_done = p_full + kQTiles;         // [2] MMA (PV_t) -> epilogue
    uint64_t *stats_ready = o_done + kQTiles;    // [2] softmax t -> epilogue: final row max / sum
    uint64_t *drain = stats_ready + kQTiles;     // every MMA issued so far is complete
    // Every waiter consumes each phase of its barrier in order, so parity
    // waits never alias: a barrier is never more than one phase ahead of the
    // phase its waiter asks for.
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    int *n_tiles_s = reinterpret_cast<int *>(smem + L::kMisc + 8);
    int *seg_ntile = reinterpret_cast<int *>(smem + L::kMisc + 16);
    int *seg_len = seg_ntile + SR_MAX_SEG;
    int *seg_start = seg_len + SR_MAX_SEG;
    int *walk_start = seg_start + SR_MAX_SEG;   // (segment, tile) of this item's first tile
    float *row_l = reinterpret_cast<float *>(smem + L::kRow);   // [2][128]
    float *row_m = row_l + kQTiles * kTileM;                     // [2][128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == kWarpTma && lane == 0) {
        // The producer thread sets the CTA up, and sends the Q loads on their
        // way before it reads the segment lengths (their latency overlaps).
        mbar_init(q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);        // the four softmax warps of tile t
            mbar_init(&o_done[t], 1);
            mbar_init(&stats_ready[t], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_expect_tx(q_full, kQTiles * L::kTileBytes);
#pragma unroll
        for (int t = 0; t < kQTiles; ++t)
#pragma unroll
            for (int pn = 0; pn < L::kPanels; ++pn)
                tma_load_3d(smem + L::kQ + t * L::kTileBytes + pn * kPanelBytes, &tmQ, pn * 64, q0 + t * kTileM, bh,
                            q_full);
        int total = 0;
#pragma unroll
        for (int s = 0; s < SR_MAX_SEG; ++s) {   // static indices keep the param arrays out of local memory
            int len = s < p.n_seg ? p.kv_len[b * p.n_seg + s] : 0;
            len = len < 0 ? 0 : (len > p.seg_cap[s] ? p.seg_cap[s] : len);
            seg_len[s] = len;
            seg_ntile[s] = (len + kTileN - 1) / kTileN;
            seg_start[s] = p.seg_start[s];
            total += seg_ntile[s];
        }
        // this item's share of the valid tiles, and where its walk starts
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
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = *n_tiles_s;
    const int n_seg = p.n_seg;
    const float sl2 = p.scale_log2;
    const uint64_t limit = p.wait_limit_ns;

    if (warp < 4 * kQTiles) {
        // ================================================================ softmax of tile t
        regs_increase<kRegSoftmax>();
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_base + tmem_s(t);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        // O_t *= alpha (lazy rescale).  PV_t(j-1) is complete: S_t(j), whose
        // completion this warp waited for, was issued after it; PV_t(j) waits
        // for this warp's hand-off.
        auto rescale_o = [&](float alpha) {
            const uint32_t o_addr = tmem + lane_base + tmem_o(t);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(o_addr + c * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                tmem_st32(o_addr + c * 32, r);
            }
        };
        TileWalk w;
        w.s = walk_start[0];
        w.t = walk_start[1];
        for (int j = 0; j < n_tiles; ++j, w.next(seg_ntile, n_seg)) {
            const int valid = min(kTileN, seg_len[w.s] - w.t * kTileN);
            if (!(ok = warp_wait(&s_full[t], j & 1, abort_flag, p.status, limit))) break;
            tc_fence_after();
            float s[kTileN];
            {
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[c][e]);
            }
            if (valid < kTileN) {
#pragma unroll
                for (int c = 0; c < kTileN; ++c) s[c] = c < valid ? s[c] : -INFINITY;
            }
            // row max over eight independent chains, then a tree: scores 0-7
            // start the chains, 8-119 join them in pairs of eights, 120-127 alone
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
            for (int c = 8; c + 16 <= kTileN; c += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], s[c + i], s[c + 8 + i]);
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], s[kTileN - 8 + i]);
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float m_new = fmaxf(m_run, mx * sl2);
            const bool need = m_new > m_run + kRescaleThreshold;
            const float m_use = need ? m_new : m_run;
            const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
            // exponentials, their row sum (eight partial sums), P as bf16 pairs
            // over the first 64 columns of S_t
            float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kTileN; ++c) {
                s[c] = fast_exp2(fmaf(s[c], sl2, -m_use));
                sum8[c & 7] += s[c];
            }
            const float sum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
            l_run = l_run * alpha + sum;
            m_run = m_use;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(s[half * 64 + 2 * e], s[half * 64 + 2 * e + 1]);
                tmem_st32(s_addr + half * 32, pk);
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) rescale_o(alpha);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t]);
        }
        // hand the row statistics to the epilogue
        row_l[t * kTileM + row] = l_run;
        row_m[t * kTileM + row] = m_run;
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(&stats_ready[t]);
    } else if (warp < 4 * kQTiles + 4) {
        // ================================================================ epilogue
        regs_decrease<kRegCorrection>();
        constexpr int kRowChunks = D / 8;   // 16-byte chunks in one bf16 row of O
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        bool ok = true;
        // ---------------------------------------------------------------- epilogue
        if (split == 1) {
#pragma unroll
            for (int t = 0; t < kQTiles; ++t) {
                const int grow = q0 + t * kTileM + row;
                const bool row_ok = grow < q_len;
                if (n_tiles == 0) {
                    __nv_bfloat16 *orow = p.o + ((static_cast<size_t>(b) * p.q_cap + grow) * p.n_heads + h) * D;
                    if (row_ok) {
                        for (int d = 0; d < D; d += 8) *reinterpret_cast<uint4 *>(orow + d) = make_uint4(0, 0, 0, 0);
                        if (p.lse) p.lse[static_cast<size_t>(bh) * p.q_cap + grow] = -INFINITY;
                    }
                    continue;
                }
                if (!ok) break;
                if (!(ok = warp_wait(&stats_ready[t], 0, abort_flag, p.status, limit, 20000u))) break;
                if (!(ok = warp_wait(&o_done[t], 0, abort_flag, p.status, limit, 20000u))) break;
                tc_fence_after();
                const float l_row = row_l[t * kTileM + row];
                const float inv_l = 1.0f / l_row;
                // This warp's 32 rows of O_t, normalised and packed to bf16, are
                // staged in Q_t's shared memory (no MMA reads Q_t once O_t is
                // final) in the copy engine's 128-byte swizzled layout (64-column
                // panels, 16-byte chunks XOR-ed with the row: no bank conflicts),
                // then stored by one tiled copy per panel when all 32 rows are
                // valid, else by whole-row coalesced stores of the valid rows: a
                // thread per row would touch 32 lines per store instruction.
                uint8_t *stage = smem + L::kQ + t * L::kTileBytes;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + tmem_o(t) + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(r[e + 0]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                        v.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
                        v.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
                        v.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
                        const int k = c * 4 + e / 8;   // 16-byte chunk of the row
                        *reinterpret_cast<uint4 *>(stage + sw128_offset(row, k)) = v;
                    }
                }
                const int r0 = q0 + t * kTileM + quarter * 32;   // this warp's first row
                if (r0 + 32 <= q_len) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
#pragma unroll
                        for (int pn = 0; pn < L::kPanels; ++pn)
                            tma_store_4d(&tmO, stage + pn * kPanelBytes + quarter * 32 * 128, pn * 64, h, r0, b);
                        bulk_commit_group();
                    }
                } else {
                    __syncwarp();
                    const int sub = lane / kRowChunks, k = lane % kRowChunks;
#pragma unroll 4
                    for (int i = 0; i < 32; i += 32 / kRowChunks) {
                        const int r = quarter * 32 + i + sub;
                        const int g = q0 + t * kTileM + r;
                        const uint4 v = *reinterpret_cast<const uint4 *>(stage + sw128_offset(r, k));
                        if (g < q_len)
                            *reinterpret_cast<uint4 *>(
                                p.o + ((static_cast<size_t>(b) * p.q_cap + g) * p.n_heads + h) * D + k * 8) = v;
                    }
                }
                if (row_ok && p.lse)
                    p.lse[static_cast<size_t>(bh) * p.q_cap + grow] =
                        (row_m[t * kTileM + row] + log2f(l_row)) * 0.69314718055994531f;
            }
            // the tiled stores have read their shared-memory source before the
            // CTA's shared memory is released
            if (lane == 0) bulk_wait_group_read0();
        } else {
            // Split unit: publish this part's unnormalised (O, m, l); the
            // combine kernel that follows on the stream merges the parts.
            const int slot = item - p.n_full;
            float *ws_m = p.ws_ml + static_cast<size_t>(slot) * 4 * kTileM;
#pragma unroll 1
            for (int t = 0; t < kQTiles; ++t) {
                // column blocks of 4 floats, rows inner: a warp's store is 512
                // contiguous bytes
                float *o_part = p.ws_o + (static_cast<size_t>(slot) * kQTiles + t) * kTileM * D + row * 4;
                float m_part = -INFINITY, l_part = 0.f;
                if (n_tiles > 0) {
                    if (!ok) break;
                    if (!(ok = warp_wait(&stats_ready[t], 0, abort_flag, p.status, limit))) break;
                    if (!(ok = warp_wait(&o_done[t], 0, abort_flag, p.status, limit))) break;
                    tc_fence_after();
                    m_part = row_m[t * kTileM + row];
                    l_part = row_l[t * kTileM + row];
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tmem + lane_base + tmem_o(t) + c * 32, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            __stcg(reinterpret_cast<float4 *>(o_part + (c * 8 + e / 4) * kTileM * 4),
                                   make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                               __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3])));
                    }
                }
                __stcg(ws_m + t * kTileM + row, m_part);
                __stcg(ws_m + (2 + t) * kTileM + row, l_part);
            }
        }
    } else {
        regs_decrease<kRegOther>();
        if (warp == kWarpTma) {
            // ============================================================ TMA producer
            // (Q is on its way since the set-up)
            if (lane == 0 && n_tiles == 0) mbar_drain(q_full, 0, limit);   // no tile: only Q to see land
            if (lane == 0 && n_tiles > 0) {
                int kv_last[kStages];   // last stage fill issued into each stage (for the drain)
#pragma unroll
                for (int i = 0; i < kStages; ++i) kv_last[i] = -1;
                TileWalk w;
                w.s = walk_start[0];
                w.t = walk_start[1];
                int row_v = 0;
                // fill i: K(i) (i < n_tiles) and V(i-1) (i > 0)
                for (int i = 0; i <= n_tiles; ++i) {
                    const int st = i % kStages;
                    const uint32_t ph = (i / kStages) & 1;
                    const bool has_k = i < n_tiles, has_v = i > 0;
                    const int row_k = has_k ? seg_start[w.s] + w.t * kTileN : 0;
                    if (!mbar_wait(&kv_empty[st], ph ^ 1, abort_flag, p.status, limit, kProducerSuspend)) break;
                    if (!(has_k && i == p.withheld_tile)) {
                        mbar_expect_tx(&kv_full[st], (has_k && has_v ? 2 : 1) * L::kTileBytes);
                        if (has_k) {
#pragma unroll
                            for (int pn = 0; pn < L::kPanels; ++pn)
                                tma_load_3d(smem + L::kK + st * L::kTileBytes + pn * kPanelBytes, &tmK, pn * 64,
                                            row_k, bh, &kv_full[st]);
                        }
                        if (has_v) {
#pragma unroll
                            for (int pn = 0; pn < L::kPanels; ++pn)
                                tma_load_3d(smem + L::kV + st * L::kTileBytes + pn * kPanelBytes, &tmV, pn * 64,
                                            row_v, bh, &kv_full[st]);
                        }
                        kv_last[st] = i;
                    }
                    row_v = row_k;
                    if (has_k) w.next(seg_ntile, n_seg);
                }
                if (*abort_flag) {
                    // wait, bounded, for the loads still in flight into this CTA
                    mbar_drain(q_full, 0, limit);
                    for (int i = 0; i < kStages; ++i)
                        if (kv_last[i] >= 0) mbar_drain(&kv_full[i], (kv_last[i] / kStages) & 1, limit);
                }
            }
        } else if (warp == kWarpMma) {
            // ============================================================ MMA issuer
            if (lane == 0 && n_tiles > 0) {
                constexpr uint32_t idesc_qk = umma_idesc_bf16(kTileM, kTileN, false, false);
                constexpr uint32_t idesc_pv = umma_idesc_bf16(kTileM, D, false, true);
                // Descriptors are built once; each instruction only advances the
                // start address (one add): the issuing thread shares its SM
                // sub-partition with busy softmax warps, so its instruction
                // count matters.
                const uint64_t desc_q = umma_desc_sw128(smem_u32(smem + L::kQ), 16, 1024);
                const uint64_t desc_k = umma_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
                const uint64_t desc_v = umma_desc_sw128(smem_u32(smem + L::kV), kPanelBytes, 1024);
                auto issue_qk = [&](int t, int st) {
                    const uint64_t a0 = umma_desc_advance(desc_q, t * L::kTileBytes);
                    const uint64_t b0 = umma_desc_advance(desc_k, st * L::kTileBytes);
                    const uint32_t d = tmem + tmem_s(t);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
                        umma_bf16_ss(d, umma_desc_advance(a0, off), umma_desc_advance(b0, off), idesc_qk,
                                     kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[t]);
                };
                auto issue_pv = [&](int t, int st, bool acc, bool last) {
                    const uint64_t b0 = umma_desc_advance(desc_v, st * L::kTileBytes);
                    const uint32_t d = tmem + tmem_o(t);
                    const uint32_t a = tmem + tmem_s(t);
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk)
                        umma_bf16_ts(d, a + kk * 8, umma_desc_advance(b0, kk * 2048), idesc_pv,
                                     (acc || kk > 0) ? 1u : 0u);
                    if (last) umma_commit(&o_done[t]);   // the epilogue reads only the final O
                };
                // P_t(j) -> O_t once the softmax of tile t has handed P_t(j) over
                auto pv_step = [&](int t, int st, int j, bool last) -> bool {
                    if (!mbar_wait(&p_full[t], j & 1, abort_flag, p.status, limit)) return false;
                    tc_fence_after();
                    issue_pv(t, st, j > 0, last);
                    return true;
                };
                bool ok = mbar_wait(q_full, 0, abort_flag, p.status, limit) &&
                          mbar_wait(&kv_full[0], 0, abort_flag, p.status, limit);
                if (ok) {
                    tc_fence_after();
                    issue_qk(0, 0);
                    issue_qk(1, 0);
                    umma_commit(&kv_empty[0]);
                }
                for (int j = 0; ok && j < n_tiles; ++j) {
                    // stage st holds V(j) and K(j+1)
                    const int st = (j + 1) % kStages;
                    const bool more = j + 1 < n_tiles;
                    // the load wait first (the tiles landed long ago): once P arrives,
                    // the MMAs follow each other without a wait that would idle the pipe
                    if (!(ok = mbar_wait(&kv_full[st], ((j + 1) / kStages) & 1, abort_flag, p.status, limit))) break;
                    if (!(ok = pv_step(0, st, j, !more))) break;
                    if (more) issue_qk(0, st);
                    if (!(ok = pv_step(1, st, j, !more))) break;
                    if (more) issue_qk(1, st);
                    umma_commit(&kv_empty[st]);
                }
                // every MMA issued so far complete before the tensor and shared
                // memory may be released (matters after an abort)
                umma_commit(drain);
                mbar_drain(drain, 0, limit);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merges the KV parts of every split unit: for each query row,
//   M = max_q m_q,  L = sum_q l_q 2^(m_q - M),  O = sum_q 2^(m_q - M) O_q / L
// (O_q unnormalised, m in log2 units).  One thread per (unit, row, 8 columns);
// a warp takes 8 rows x 4 column chunks, so that its reads of the partials
// (column blocks, rows inner) and its writes of O (rows, columns inner) both
// cover whole runs of 64 to 128 bytes.
struct CombineParams {
    const float *ws_o;
    const float *ws_ml;
    __nv_bfloat16 *o;
    float *lse;
    const int32_t *q_len;
    int32_t n_full, split, tail_units, qb_per_head, n_heads, q_cap;
};

template <int D>
__global__ void __launch_bounds__(256) split_combine_kernel(const CombineParams c) {
    constexpr int kChunks = D / 8;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t total = static_cast<int64_t>(c.tail_units) * kQTiles * kTileM * kChunks;
    if (idx >= total) return;
    static_assert(kChunks % 4 == 0, "4 column chunks per warp");
    const int lane = static_cast<int>(idx & 31);
    const int64_t wg = idx >> 5;   // (tail, 8-row block, 4-chunk block), chunk blocks fastest
    const int r2 = static_cast<int>((wg / (kChunks / 4)) % (kQTiles * kTileM / 8)) * 8 + (lane & 7);   // row in the 256-row block
    const int chunk = static_cast<int>(wg % (kChunks / 4)) * 4 + (lane >> 3);
    const int tail = static_cast<int>(wg / ((kChunks / 4) * (kQTiles * kTileM / 8)));
    const int t = r2 / kTileM, row = r2 % kTileM;
    const int unit = c.n_full + tail;
    const int qb = unit % c.qb_per_head, bh = unit / c.qb_per_head;
    const int h = bh % c.n_heads, b = bh / c.n_heads;
    const int grow = qb * kQTiles * kTileM + r2;
    if (grow >= min(max(c.q_len[b], 0), c.q_cap)) return;   // clamped as in the attention kernel
    float mmax = -INFINITY;
    for (int q = 0; q < c.split; ++q)
        mmax = fmaxf(mmax, c.ws_ml[static_cast<size_t>(tail * c.split + q) * 4 * kTileM + t * kTileM + row]);
    float lsum = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int q = 0; q < c.split; ++q) {
        const float *mq = c.ws_ml + static_cast<size_t>(tail * c.split + q) * 4 * kTileM;
        const float lq = mq[(2 + t) * kTileM + row];
        if (!(lq > 0.f)) continue;
        const float w = fast_exp2(mq[t * kTileM + row] - mmax);
        lsum += lq * w;
        const float *oq = c.ws_o + (static_cast<size_t>(tail * c.split + q) * kQTiles + t) * kTileM * D +
                          (2 * chunk * kTileM + row) * 4;
        const float4 x0 = *reinterpret_cast<const float4 *>(oq);
        const float4 x1 = *reinterpret_cast<const float4 *>(oq + kTileM * 4);
        acc[0] += w * x0.x; acc[1] += w * x0.y; acc[2] += w * x0.z; acc[3] += w * x0.w;
        acc[4] += w * x1.x; acc[5] += w * x1.y; acc[6] += w * x1.z; acc[7] += w * x1.w;
    }
    const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
    uint4 v;
    v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4 *>(c.o + ((static_cast<size_t>(b) * c.q_cap + grow) * c.n_heads + h) * D + chunk * 8) = v;
    if (chunk == 0 && c.lse)
        c.lse[static_cast<size_t>(bh) * c.q_cap + grow] =
            lsum > 0.f ? (mmax + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
}

int sm_count() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

template <int D>
int launch(const AttnLaunch &a) {
    using L = Smem<D>;
    CUtensorMap tq, tk, tv, to;
    const uint64_t bh = static_cast<uint64_t>(a.n_batch) * a.n_heads;
    int rc = make_tmap_bf16_3d(&tq, a.q, D, static_cast<uint64_t>(a.q_cap), bh, 64, kTileM);
    if (rc == SR_OK) rc = make_tmap_bf16_3d(&tk, a.k, D, static_cast<uint64_t>(a.kv_tokens), bh, 64, kTileN);
    if (rc == SR_OK) rc = make_tmap_bf16_3d(&tv, a.v, D, static_cast<uint64_t>(a.kv_tokens), bh, 64, kTileN);
    // o [n_batch][q_cap][n_heads][D], stored in boxes of 32 rows x 64 columns
    if (rc == SR_OK)
        rc = make_tmap_bf16_4d(&to, a.o, D, static_cast<uint64_t>(a.n_heads), static_cast<uint64_t>(a.q_cap),
                               static_cast<uint64_t>(a.n_batch), 64, 32);
    if (rc != SR_OK) return rc;
    AttnParams p{};
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
    p.wait_limit_ns = a.wait_limit_ns;
    p.withheld_tile = a.withheld_tile;
    const AttnSchedule sc = attention_schedule(a.n_batch, a.n_heads, D, a.q_cap, sm_count());
    p.qb_per_head = sc.qb_per_head;
    p.n_full = sc.n_full;
    p.split = 1;
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
        e = cudaFuncSetAttribute(chunk_attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(chunk_attention)", e);
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    if (items > 0x7fffffff) return set_error(SR_ERR_INVALID_ARG, "chunk_attention: too many work items");
    chunk_attention_kernel<D><<<static_cast<unsigned>(items), kThreads, L::kAlloc, a.stream>>>(tq, tk, tv, to, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("chunk_attention launch", e);
    if (p.split > 1)
        return launch_split_combine(p.ws_o, p.ws_ml, p.o, p.lse, p.q_len, p.n_full, p.split, sc.tail_units,
                                    p.qb_per_head, p.n_heads, p.q_cap, D, a.stream);
    return SR_OK;
}

std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};
std::atomic<int32_t> g_withheld_tile{-1};

}  // namespace

uint64_t attention_wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
int32_t attention_withheld_tile() { return g_withheld_tile.load(std::memory_order_relaxed); }

int launch_split_combine(const float *ws_o, const float *ws_ml, void *o, float *lse, const int32_t *q_len,
                         int32_t n_full, int32_t split, int32_t tail_units, int32_t qb_per_head, int32_t n_heads,
                         int32_t q_cap, int32_t head_dim, cudaStream_t stream) {
    CombineParams c{ws_o, ws_ml, static_cast<__nv_bfloat16 *>(o), lse, q_len, n_full, split, tail_units,
                    qb_per_head, n_heads, q_cap};
    const int64_t threads = static_cast<int64_t>(tail_units) * kQTiles * kTileM * (head_dim / 8);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    if (head_dim == 128)
        split_combine_kernel<128><<<blocks, 256, 0, stream>>>(c);
    else
        split_combine_kernel<64><<<blocks, 256, 0, stream>>>(c);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SR_OK : set_cuda_error("split_combine launch", e);
}

AttnSchedule attention_schedule(int32_t n_batch, int32_t n_heads, int32_t head_dim, int32_t q_cap, int32_t sms) {
    AttnSchedule sc{};
    sc.qb_per_head = (q_cap + kQTiles * kTileM - 1) / (kQTiles * kTileM);
    sc.units = static_cast<int64_t>(n_batch) * n_heads * sc.qb_per_head;
    const int64_t P = sms > 0 ? sms : 148;
    const int64_t full = (sc.units / P) * P;
    const int64_t rem = sc.units - full;
    sc.split = 1;
    sc.n_full = static_cast<int32_t>(sc.units);
    if (rem > 0) {
        int64_t s = P / rem;
        if (s > 8) s = 8;
        if (s >= 2) {
            sc.split = static_cast<int32_t>(s);
            sc.n_full = static_cast<int32_t>(full);
            sc.tail_units = static_cast<int32_t>(rem);
        }
    }
    const int64_t slots = static_cast<int64_t>(sc.tail_units) * sc.split;
    sc.o_bytes = static_cast<size_t>(slots) * kQTiles * kTileM * head_dim * sizeof(float);
    sc.ml_bytes = static_cast<size_t>(slots) * 4 * kTileM * sizeof(float);
    sc.workspace_bytes = sc.split > 1 ? sc.o_bytes + sc.ml_bytes : 0;
    return sc;
}

int attention_sm_count() { return sm_count(); }

int launch_chunk_attention(const AttnLaunch &a) {
    if (a.head_dim == 128) return launch<128>(a);
    if (a.head_dim == 64) return launch<64>(a);
    return set_error(SR_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
}

// ============================================================================
// Allocation-free variant of sr_chunk_attention_fwd.
//
// Some callers cannot allocate device memory at the moment they run the
// attention: a plugin living inside another runtime that is handed only its
// input and output buffers, a real-time frame loop in which cudaMalloc (which
// may synchronise the whole device) is forbidden, or an application whose
// device memory is entirely owned by its own allocator.  For them the scratch
// that the split-KV schedule needs lives in this file-scope device array,
// which exists once per GPU that loads the library and stays there until the
// process exits.  Nothing in it has to start at zero: every partial result the
// merge step reads is written earlier in the same call.  All calls on a device
// share it, so calls that could run at the same time on that device (other
// streams, other host threads) race and must be ordered by the caller.
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[SR_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[64] = {};                  // device address of g_noalloc_scratch, per device
unsigned long long g_noalloc_ctx[64] = {};     // id of the context that address belongs to

// Unique id of the calling thread's current CUDA context (0 if there is none
// yet, or the driver does not offer the query).  Ids are never reused within
// a process, so a changed id means the device's context was re-created (for
// instance after cudaDeviceReset) and the module, with its static array, was
// loaded again at a possibly different address.
unsigned long long current_context_id() {
    using GetCurrentFn = CUresult (*)(CUcontext *);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long *);
    static std::once_flag once;
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    std::call_once(once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(fn);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(fn);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in for the symbol; the address a
// kernel may use comes from cudaGetSymbolAddress, resolved with that device
// current the first time a device is used, and again whenever the device's
// context has changed since (the cached address would point into a module
// that no longer exists).
int noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
    if (dev < 0 || dev >= 64) return set_error(SR_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> guard(g_noalloc_mutex);
    const unsigned long long ctx = current_context_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return set_cuda_error("cudaGetSymbolAddress(static attention scratch)", e);
        g_noalloc_ptr[dev] = ptr;
        g_noalloc_ctx[dev] = current_context_id();   // the lookup itself may have created the context
    }
    *out = g_noalloc_ptr[dev];
    return SR_OK;
}

}  // namespace

}  // namespace sr

extern "C" int sr_chunk_attention_fwd_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                               const sr_kv_layout *layout, const int32_t *kv_len_dev,
                                               const int32_t *q_len_dev, int32_t n_batch, int32_t n_heads,
                                               int32_t head_dim, int32_t q_cap, float softmax_scale,
                                               int32_t *status_dev, void *stream) {
    const size_t need = sr_chunk_attention_workspace_bytes(n_batch, n_heads, head_dim, q_cap);
    if (need > SR_NOALLOC_SCRATCH_BYTES)
        return sr::set_error(SR_ERR_UNSUPPORTED,
                             "chunk_attention_noalloc: this problem needs %zu bytes of scratch, the static scratch "
                             "holds %zu",
                             need, static_cast<size_t>(SR_NOALLOC_SCRATCH_BYTES));
    void *scratch = nullptr;
    const int rc = sr::noalloc_scratch(&scratch);
    if (rc != SR_OK) return rc;
    return sr_chunk_attention_fwd(q, k, v, o, lse, layout, kv_len_dev, q_len_dev, n_batch, n_heads, head_dim, q_cap,
                                  softmax_scale, scratch, SR_NOALLOC_SCRATCH_BYTES, status_dev, stream);
}

extern "C" int sr_set_wait_limit_ns(uint64_t limit_ns) {
    sr::g_wait_limit_ns.store(limit_ns ? limit_ns : sr::kWaitLimitNs, std::memory_order_relaxed);
    return SR_OK;
}

extern "C" int sr_set_withheld_kv_tile(int32_t tile) {
    if (tile < -1) return sr::set_error(SR_ERR_INVALID_ARG, "withheld tile must be >= -1");
    sr::g_withheld_tile.store(tile, std::memory_order_relaxed);
    return SR_OK;
}
