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
// Design (one CTA = one 128-row query tile of one (session, head)):
//   warp 0      TMA producer: Q once, then K and V tiles (128 tokens) into a
//               2-stage ring each, walking the segments' valid tiles only.
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer:
//                 S_j = Q K_j^T   (M=128, N=128, K=D; S double-buffered in TMEM)
//                 O  += P_j V_j   (M=128, N=D, K=128; O resident in TMEM)
//               S_{j+1} is issued before waiting for P_j so QK^T overlaps
//               the softmax of the previous tile.
//   warps 2..5  softmax: one thread per query row reads its S row from TMEM,
//               masks the segment tail, keeps an fp32 running max/sum in the
//               log2 domain, writes P (bf16) into a 128B-swizzled shared
//               tile and rescales O in TMEM only when the row max grew by
//               more than 2^8 (lazy rescale; exact because the final
//               normalisation uses the same stale max).  Epilogue: O / l ->
//               bf16 token-major output, LSE.
// Every wait is bounded (sr_device.cuh): a stuck pipeline sets the status word
// and the CTA returns instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_device.cuh"
#include "sr_internal.h"

namespace sr {

namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16), one swizzle-128B panel
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

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
};

template <int D>
struct Smem {
    static constexpr int kPanels = D / 64;
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kTileBytes;
    static constexpr int kV = kK + kStages * kTileBytes;
    static constexpr int kP = kV + kStages * kTileBytes;
    static constexpr int kBar = kP + 2 * kPanelBytes;
    static constexpr int kNumBars = 1 + 4 * kStages + 2 + 1 + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kEnd = kMisc + 16 + 12 * SR_MAX_SEG;
    static constexpr int kAlloc = kEnd + 1024;   // slack for manual 1024-byte alignment
};

// Walks the valid 128-token tiles of every segment in buffer order.
struct TileWalk {
    int s, t;
    __device__ void first(const int *ntile, int n_seg) {
        s = 0;
        t = 0;
        while (s < n_seg && ntile[s] == 0) ++s;
    }
    __device__ void next(const int *ntile, int n_seg) {
        if (++t == ntile[s]) {
            t = 0;
            ++s;
            while (s < n_seg && ntile[s] == 0) ++s;
        }
    }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using L = Smem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int q_len = p.q_len[b];
    const int q0 = qt * kTileM;
    if (q0 >= q_len) return;   // uniform for the whole CTA
    const int bh = b * p.n_heads + h;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + kStages;
    uint64_t *v_full = k_empty + kStages;
    uint64_t *v_empty = v_full + kStages;
    uint64_t *s_full = v_empty + kStages;   // [2]
    uint64_t *p_full = s_full + 2;
    uint64_t *o_done = p_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    int *n_tiles_s = reinterpret_cast<int *>(smem + L::kMisc + 8);
    int *seg_ntile = reinterpret_cast<int *>(smem + L::kMisc + 16);
    int *seg_len = seg_ntile + SR_MAX_SEG;
    int *seg_start = seg_len + SR_MAX_SEG;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(p_full, 4);   // one arrival per softmax warp
        mbar_init(o_done, 1);
        *abort_flag = 0;
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
        *n_tiles_s = total;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = *n_tiles_s;
    const int n_seg = p.n_seg;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_expect_tx(q_full, L::kTileBytes);
#pragma unroll
            for (int pn = 0; pn < L::kPanels; ++pn)
                tma_load_3d(smem + L::kQ + pn * kPanelBytes, &tmQ, pn * 64, q0, bh, q_full);
            TileWalk w;
            w.first(seg_ntile, n_seg);
            for (int j = 0; j < n_tiles; ++j, w.next(seg_ntile, n_seg)) {
                const int st = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                const int row0 = seg_start[w.s] + w.t * kTileN;
                if (!mbar_wait(&k_empty[st], ph ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(&k_full[st], L::kTileBytes);
#pragma unroll
                for (int pn = 0; pn < L::kPanels; ++pn)
                    tma_load_3d(smem + L::kK + st * L::kTileBytes + pn * kPanelBytes, &tmK, pn * 64, row0, bh,
                                &k_full[st]);
                if (!mbar_wait(&v_empty[st], ph ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(&v_full[st], L::kTileBytes);
#pragma unroll
                for (int pn = 0; pn < L::kPanels; ++pn)
                    tma_load_3d(smem + L::kV + st * L::kTileBytes + pn * kPanelBytes, &tmV, pn * 64, row0, bh,
                                &v_full[st]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(kTileM, kTileN, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kTileM, D, false, true);
            const uint32_t q_base = smem_u32(smem + L::kQ);
            const uint32_t k_base = smem_u32(smem + L::kK);
            const uint32_t v_base = smem_u32(smem + L::kV);
            const uint32_t p_base = smem_u32(smem + L::kP);
            auto issue_qk = [&](int j) {
                const int st = j % kStages;
                const uint32_t s_col = (j & 1) ? kTmemS1 : kTmemS0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
                    const uint64_t a = umma_desc_sw128(q_base + off, 16, 1024);
                    const uint64_t bdesc = umma_desc_sw128(k_base + st * L::kTileBytes + off, 16, 1024);
                    umma_bf16_ss(tmem + s_col, a, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&k_empty[st]);
                umma_commit(&s_full[j & 1]);
            };
            bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
            if (ok) ok = mbar_wait(&k_full[0], 0, abort_flag, p.status);
            if (ok) {
                tc_fence_after();
                issue_qk(0);
            }
            for (int j = 0; ok && j < n_tiles; ++j) {
                if (j + 1 < n_tiles) {
                    if (!(ok = mbar_wait(&k_full[(j + 1) % kStages], ((j + 1) / kStages) & 1, abort_flag,
                                         p.status)))
                        break;
                    tc_fence_after();
                    issue_qk(j + 1);
                }
                if (!(ok = mbar_wait(p_full, j & 1, abort_flag, p.status))) break;
                const int st = j % kStages;
                if (!(ok = mbar_wait(&v_full[st], (j / kStages) & 1, abort_flag, p.status))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk) {
                    const uint64_t a =
                        umma_desc_sw128(p_base + (kk >> 2) * kPanelBytes + (kk & 3) * 32, 16, 1024);
                    const uint64_t bdesc =
                        umma_desc_sw128(v_base + st * L::kTileBytes + kk * 2048, kPanelBytes, 1024);
                    umma_bf16_ss(tmem + kTmemO, a, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&v_empty[st]);
                umma_commit(o_done);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quarter = warp & 3;   // TMEM lanes this warp may access
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t p_base = smem_u32(smem + L::kP);
        const float sl2 = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        TileWalk w;
        w.first(seg_ntile, n_seg);
        for (int j = 0; j < n_tiles; ++j, w.next(seg_ntile, n_seg)) {
            const int valid = min(kTileN, seg_len[w.s] - w.t * kTileN);
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag, p.status));
            if (!ok) break;   // warp-uniform: the TMEM loads below are warp-collective
            tc_fence_after();
            float s[kTileN];
            {
                uint32_t r[4][32];
                const uint32_t s_addr = tmem + lane_base + ((j & 1) ? kTmemS1 : kTmemS0);
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[c][e]);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kTileN; ++c) mx = fmaxf(mx, c < valid ? s[c] : -INFINITY);
            const float m_new = fmaxf(m_run, mx * sl2);
            const bool need = m_new > m_run + kRescaleThreshold;
            const float m_use = need ? m_new : m_run;
            const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < kTileN; ++c) {
                const float pc = c < valid ? fast_exp2(fmaf(s[c], sl2, -m_use)) : 0.f;
                s[c] = pc;
                sum += pc;
            }
            l_run = l_run * alpha + sum;
            m_run = m_use;
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
            }
            // P row -> swizzled shared tile: panel c/64, 16-byte chunk index XOR (row % 8)
#pragma unroll
            for (int ch = 0; ch < kTileN / 8; ++ch) {
                const uint32_t addr =
                    p_base + (ch >> 3) * kPanelBytes + row * 128 + ((((ch & 7) ^ (row & 7))) << 4);
                st_shared_v4(addr, pack_bf16x2(s[8 * ch + 0], s[8 * ch + 1]), pack_bf16x2(s[8 * ch + 2], s[8 * ch + 3]),
                             pack_bf16x2(s[8 * ch + 4], s[8 * ch + 5]), pack_bf16x2(s[8 * ch + 6], s[8 * ch + 7]));
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    const uint32_t o_addr = tmem + lane_base + kTmemO + c * 32;
                    tmem_ld32(o_addr, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    tmem_st32(o_addr, r);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ---------------------------------------------------------------- epilogue
        const int grow = q0 + row;
        const bool row_ok = grow < q_len;
        __nv_bfloat16 *orow = p.o + ((static_cast<size_t>(b) * p.q_cap + grow) * p.n_heads + h) * D;
        if (n_tiles == 0) {
            if (row_ok) {
                for (int d = 0; d < D; d += 8) *reinterpret_cast<uint4 *>(orow + d) = make_uint4(0, 0, 0, 0);
                if (p.lse) p.lse[static_cast<size_t>(bh) * p.q_cap + grow] = -INFINITY;
            }
        } else if (ok && __all_sync(0xffffffffu, mbar_wait(o_done, (n_tiles - 1) & 1, abort_flag, p.status))) {
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + kTmemO + c * 32, r);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(r[e + 0]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                        v.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
                        v.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
                        v.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + e) = v;
                    }
                }
            }
            if (row_ok && p.lse)
                p.lse[static_cast<size_t>(bh) * p.q_cap + grow] = (m_run + log2f(l_run)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
int launch(const AttnLaunch &a) {
    using L = Smem<D>;
    CUtensorMap tq, tk, tv;
    const uint64_t bh = static_cast<uint64_t>(a.n_batch) * a.n_heads;
    int rc = make_tmap_bf16_3d(&tq, a.q, D, static_cast<uint64_t>(a.q_cap), bh, 64, kTileM);
    if (rc == SR_OK) rc = make_tmap_bf16_3d(&tk, a.k, D, static_cast<uint64_t>(a.kv_tokens), bh, 64, kTileN);
    if (rc == SR_OK) rc = make_tmap_bf16_3d(&tv, a.v, D, static_cast<uint64_t>(a.kv_tokens), bh, 64, kTileN);
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
    static bool attr_set[64] = {};   // the shared-memory opt-in is per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(chunk_attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(chunk_attention)", e);
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    dim3 grid((a.q_cap + kTileM - 1) / kTileM, a.n_heads, a.n_batch);
    chunk_attention_kernel<D><<<grid, kThreads, L::kAlloc, a.stream>>>(tq, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error("chunk_attention launch", e);
    return SR_OK;
}

}  // namespace

int launch_chunk_attention(const AttnLaunch &a) {
    if (a.head_dim == 128) return launch<128>(a);
    if (a.head_dim == 64) return launch<64>(a);
    return set_error(SR_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
}

}  // namespace sr
