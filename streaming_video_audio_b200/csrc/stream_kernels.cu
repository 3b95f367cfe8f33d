// stream_kernels.cu -- the HBM-bound steps of the streaming attention layer:
// 3-D RoPE + re-layout (QK-prep), history-tier pooling and KV append.
//
// All three move 16-byte vectors (8 bf16) per thread; a warp covers whole
// 256-byte head rows (D = 128) so every DRAM sector it touches is used
// completely.  They do no tensor-core work: their roofline is HBM bandwidth.
#include <cmath>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_device.cuh"
#include "sr_internal.h"

namespace sr {

namespace {

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(h[i]);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]);
    u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]);
    u.w = pack_bf16x2(f[6], f[7]);
    return u;
}

// ============================================================== 3-D RoPE
// Per pair p of the head vector: its axis (0 = t, 1 = h, 2 = w) and
// theta_p = base^(-2j/d_a) (j = index of the pair inside its axis block),
// computed on the host in double.
struct RopeTable {
    double theta[64];
    int32_t pairs_t, pairs_th;   // pairs of the t block, of the t and h blocks together
};

struct RopeArgs {
    const __nv_bfloat16 *__restrict__ x;
    __nv_bfloat16 *__restrict__ y;
    const float *__restrict__ pos;
    const int32_t *__restrict__ n_valid;
    int32_t n_heads;
    float out_scale;
    int64_t xb, xt, xh, yb, yt, yh, pb;
    // QK normalisation (norm kernels only): per-head RMSNorm with gain
    // gamma[D]; y_raw (optional) receives the normalised vector before RoPE
    // (without normalisation: the input itself, a plain copy)
    const float *__restrict__ gamma;
    float eps;
    __nv_bfloat16 *__restrict__ y_raw;
    int64_t rb, rt, rh;
    // optional fp64 offset added to every token's t (the stream clock)
    const double *__restrict__ t_origin;
    // optional second tensor copied unrotated with the strides of x -> y (V
    // rows that travel with their K rows)
    const __nv_bfloat16 *__restrict__ vx;
    __nv_bfloat16 *__restrict__ vy;
};

// (cos, sin) * scale of one pair: the angle p * theta is formed in double and
// reduced to [-pi, pi] in double, so its error does not grow with the
// position's magnitude; the small remainder goes through fp32 sincosf.
__device__ __forceinline__ float2 pair_rotation(const RopeTable &tab, int pair, double pt, float ph, float pw,
                                                float scale) {
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
    const double pa = pair < tab.pairs_t ? pt : (pair < tab.pairs_th ? ph : pw);
    const double phi = pa * tab.theta[pair];
    const double r = fma(-rint(phi * kInvTwoPi), kTwoPi, phi);
    float s, co;
    sincosf(static_cast<float>(r), &s, &co);
    return make_float2(co * scale, s * scale);
}

// The token's four (cos, sin) pairs of chunk c (pairs 4c .. 4c+3), computed
// as pair_rotation does; s_theta: the per-pair theta in shared memory.
__device__ __forceinline__ void token_rotation(const double *s_theta, const RopeTable &tab, int c, double pt,
                                               float ph, float pw, float scale, float (&cs)[4], float (&sn)[4]) {
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int pair = c * 4 + k;
        const double pa = pair < tab.pairs_t ? pt : (pair < tab.pairs_th ? ph : pw);
        const double phi = pa * s_theta[pair];
        const double r = fma(-rint(phi * kInvTwoPi), kTwoPi, phi);
        float s, co;
        sincosf(static_cast<float>(r), &s, &co);
        cs[k] = co * scale;
        sn[k] = s * scale;
    }
}

__device__ __forceinline__ uint4 rotate8(const uint4 &u, const float (&cs)[4], const float (&sn)[4]) {
    float f[8], r[8];
    unpack8(u, f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        r[2 * k] = f[2 * k] * cs[k] - f[2 * k + 1] * sn[k];
        r[2 * k + 1] = f[2 * k] * sn[k] + f[2 * k + 1] * cs[k];
    }
    return pack8(r);
}

RopeTable make_rope_table(const sr_rope_cfg &cfg) {
    RopeTable tab{};
    const int widths[3] = {cfg.d_t, cfg.d_h, cfg.d_w};
    int pair = 0;
    for (int ax = 0; ax < 3; ++ax)
        for (int j = 0; j < widths[ax] / 2; ++j, ++pair)
            tab.theta[pair] = std::pow(static_cast<double>(cfg.base), -2.0 * static_cast<double>(j) / widths[ax]);
    tab.pairs_t = cfg.d_t / 2;
    tab.pairs_th = (cfg.d_t + cfg.d_h) / 2;
    return tab;
}

// One CTA per (token, batch).  Thread t handles the 16-byte chunk
// c = t % (D/8) of heads t/(D/8), t/(D/8) + 128/(D/8), ... (kPasses heads,
// a compile-time count so that only the registers in use are allocated).  It
// first issues the loads of all its heads, then derives the token's four
// (cos, sin) pairs -- they depend on (token, pair) only and are reused for
// every head -- and finally rotates and stores.  The angle p * theta is
// formed in double and reduced to [-pi, pi] in double, so its error does not
// grow with the position's magnitude; the small remainder goes through fp32
// sincosf.  The rotation itself runs in fp32.
// kNorm: RMSNorm of each head vector first (QK normalisation): the D/8
// threads holding one head row reduce its sum of squares with shuffles --
// the reductions of all passes side by side, so their latencies overlap --
// then scale by rsqrt(mean + eps) * gamma before rotating.  Needs n_heads <=
// kPasses * (128 / (D/8)) so every thread runs the same shuffles.
template <int D, bool kNorm, int kPasses>
__global__ void __launch_bounds__(128, kPasses <= 5 ? 8 : 4) rope3d_kernel(const RopeArgs a, const RopeTable tab) {
    constexpr int kChunks = D / 8;
    constexpr int kHeadsPerPass = 128 / kChunks;
    const int n = blockIdx.x, b = blockIdx.y;
    if (a.n_valid && n >= a.n_valid[b]) return;   // uniform per CTA (before the barrier below)
    const int c = threadIdx.x % kChunks;
    const int hp = threadIdx.x / kChunks;
    const __nv_bfloat16 *xt = a.x + b * a.xb + n * a.xt + c * 8;
    __nv_bfloat16 *yt = a.y + b * a.yb + n * a.yt + c * 8;
    uint4 u[kPasses];
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int h = hp + i * kHeadsPerPass;
        u[i] = h < a.n_heads ? __ldg(reinterpret_cast<const uint4 *>(xt + h * a.xh)) : make_uint4(0, 0, 0, 0);
    }
    // The token's D/2 (cos, sin) pairs, one per thread of the first D/2, shared
    // through shared memory: every head-row group of the CTA needs the same
    // pairs of its chunk, so each is evaluated once per token.
    __shared__ __align__(16) float2 s_rot[D / 2];
    __shared__ __align__(16) float s_gamma[kNorm ? D : 1];   // gains, read per pass (keeps registers free)
    if (threadIdx.x < D / 2) {
        double pt = a.t_origin ? *a.t_origin : 0.0;
        float ph = 0.f, pw = 0.f;
        if (a.pos) {
            const float *pp = a.pos + b * a.pb + 3 * static_cast<int64_t>(n);
            pt += static_cast<double>(pp[0]);
            ph = pp[1];
            pw = pp[2];
        }
        s_rot[threadIdx.x] = pair_rotation(tab, threadIdx.x, pt, ph, pw, a.out_scale);
    }

    if constexpr (kNorm) {
        if (threadIdx.x < D) s_gamma[threadIdx.x] = a.gamma[threadIdx.x];
    }
    __syncthreads();
    float cs[4], sn[4];
    {
        const float4 r01 = *reinterpret_cast<const float4 *>(s_rot + c * 4);
        const float4 r23 = *reinterpret_cast<const float4 *>(s_rot + c * 4 + 2);
        cs[0] = r01.x; sn[0] = r01.y; cs[1] = r01.z; sn[1] = r01.w;
        cs[2] = r23.x; sn[2] = r23.y; cs[3] = r23.z; sn[3] = r23.w;
    }
    float inv[kPasses];
    if constexpr (kNorm) {
#pragma unroll
        for (int i = 0; i < kPasses; ++i) {
            float f[8];
            unpack8(u[i], f);
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
            inv[i] = ss;
        }
#pragma unroll
        for (int off = kChunks / 2; off > 0; off >>= 1)
#pragma unroll
            for (int i = 0; i < kPasses; ++i) inv[i] += __shfl_xor_sync(0xffffffffu, inv[i], off);
#pragma unroll
        for (int i = 0; i < kPasses; ++i) inv[i] = rsqrtf(inv[i] * (1.0f / D) + a.eps);
    }
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int h = hp + i * kHeadsPerPass;
        if (h >= a.n_heads) continue;
        float f[8], r[8];
        unpack8(u[i], f);
        if constexpr (kNorm) {
            const float4 g0 = *reinterpret_cast<const float4 *>(s_gamma + c * 8);
            const float4 g1 = *reinterpret_cast<const float4 *>(s_gamma + c * 8 + 4);
            const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = f[e] * inv[i] * g[e];
            if (a.y_raw)
                *reinterpret_cast<uint4 *>(a.y_raw + b * a.rb + n * a.rt + h * a.rh + c * 8) = pack8(f);
        }
        if constexpr (!kNorm) {
            if (a.y_raw) *reinterpret_cast<uint4 *>(a.y_raw + b * a.rb + n * a.rt + h * a.rh + c * 8) = u[i];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            r[2 * k] = f[2 * k] * cs[k] - f[2 * k + 1] * sn[k];
            r[2 * k + 1] = f[2 * k] * sn[k] + f[2 * k + 1] * cs[k];
        }
        *reinterpret_cast<uint4 *>(yt + h * a.yh) = pack8(r);
    }
    if constexpr (!kNorm) {   // with normalisation the host guarantees n_heads fits the passes above
        for (int h = hp + kPasses * kHeadsPerPass; h < a.n_heads; h += kHeadsPerPass) {   // very many heads
            const uint4 x8 = __ldg(reinterpret_cast<const uint4 *>(xt + h * a.xh));
            if (a.y_raw) *reinterpret_cast<uint4 *>(a.y_raw + b * a.rb + n * a.rt + h * a.rh + c * 8) = x8;
            *reinterpret_cast<uint4 *>(yt + h * a.yh) = rotate8(x8, cs, sn);
        }
    }
    if (!kNorm && a.vx) {
        // rows that travel unrotated with their K rows (V into the window):
        // after the K rows, in the registers they used
        const __nv_bfloat16 *vt = a.vx + b * a.xb + n * a.xt + c * 8;
        __nv_bfloat16 *vo = a.vy + b * a.yb + n * a.yt + c * 8;
        uint4 w[kPasses];
#pragma unroll
        for (int i = 0; i < kPasses; ++i) {
            const int h = hp + i * kHeadsPerPass;
            w[i] = h < a.n_heads ? __ldg(reinterpret_cast<const uint4 *>(vt + h * a.xh)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kPasses; ++i) {
            const int h = hp + i * kHeadsPerPass;
            if (h < a.n_heads) *reinterpret_cast<uint4 *>(vo + h * a.yh) = w[i];
        }
        for (int h = hp + kPasses * kHeadsPerPass; h < a.n_heads; h += kHeadsPerPass)   // very many heads
            *reinterpret_cast<uint4 *>(vo + h * a.yh) = __ldg(reinterpret_cast<const uint4 *>(vt + h * a.xh));
    }
}

// ============================================================== pooling
struct PoolArgs {
    const __nv_bfloat16 *__restrict__ k_in;
    const __nv_bfloat16 *__restrict__ v_in;
    __nv_bfloat16 *__restrict__ k_out;
    __nv_bfloat16 *__restrict__ v_out;
    int32_t n_frames, n_heads, grid_h, grid_w, pool_h, pool_w, cells_w, cells;
    int64_t ib, i_f, it, ih, ob, o_f, ot, oh;
    const float *__restrict__ frame_t;
    float *__restrict__ pos_out;
    int64_t pos_b;
    int64_t total;   // threads doing work per (batch, frame)
    // optional fused RoPE of the pooled K (as rounded to bf16) into k_rot
    // (strides of k_out) at rot_pos (layout of pos_out) + t_origin on t
    __nv_bfloat16 *__restrict__ k_rot;
    const float *__restrict__ rot_pos;
    int64_t rot_pos_b;
    const double *__restrict__ t_origin;
    float rot_scale;
};

// One thread per (batch, frame, cell, head, 16-byte chunk); chunk fastest so a
// warp reads whole 256-byte head rows of each member token.  PH, PW > 0 fix
// the window at compile time so that all member loads of a tensor are in
// flight together (members outside the grid are skipped); PH = PW = 0 reads
// the window from the arguments.
template <int D, int PH, int PW>
__global__ void __launch_bounds__(256) pool_kernel(const PoolArgs a, const RopeTable tab) {
    constexpr int kChunks = D / 8;
    const uint32_t idx = blockIdx.x * blockDim.x + threadIdx.x;   // (cell, head, chunk) of one frame
    if (idx >= static_cast<uint32_t>(a.total)) return;
    const int f = blockIdx.y, b = blockIdx.z;
    const int c = static_cast<int>(idx % kChunks);
    const uint32_t hj = idx / kChunks;
    const int h = static_cast<int>(hj % static_cast<uint32_t>(a.n_heads));
    const int j = static_cast<int>(hj / static_cast<uint32_t>(a.n_heads));
    const int ph = PH > 0 ? PH : a.pool_h, pw = PW > 0 ? PW : a.pool_w;
    const int r = j / a.cells_w, cc = j % a.cells_w;
    const int r0 = r * ph, r1 = min(r0 + ph, a.grid_h);
    const int c0 = cc * pw, c1 = min(c0 + pw, a.grid_w);
    const float count = static_cast<float>((r1 - r0) * (c1 - c0));
    const int64_t in_off = b * a.ib + f * a.i_f + h * a.ih + c * 8;
    const int64_t out_off = b * a.ob + f * a.o_f + j * a.ot + h * a.oh + c * 8;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
        const __nv_bfloat16 *src = which ? a.v_in : a.k_in;
        __nv_bfloat16 *dst = which ? a.v_out : a.k_out;
        if (!src) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if constexpr (PH > 0 && PW > 0) {
            uint4 u[PH * PW];
#pragma unroll
            for (int m = 0; m < PH * PW; ++m) {
                const int rr = r0 + m / PW, ci = c0 + m % PW;
                u[m] = (rr < r1 && ci < c1)
                           ? __ldg(reinterpret_cast<const uint4 *>(src + in_off +
                                                                   static_cast<int64_t>(rr * a.grid_w + ci) * a.it))
                           : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int m = 0; m < PH * PW; ++m) {
                float v[8];
                unpack8(u[m], v);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] += v[e];
            }
        } else {
            for (int rr = r0; rr < r1; ++rr) {
#pragma unroll 4
                for (int ci = c0; ci < c1; ++ci) {
                    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                        src + in_off + static_cast<int64_t>(rr * a.grid_w + ci) * a.it));
                    float v[8];
                    unpack8(u, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] += v[e];
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = acc[e] / count;
        const uint4 pooled = pack8(acc);
        *reinterpret_cast<uint4 *>(dst + out_off) = pooled;
        if (which == 0 && a.k_rot) {
            // the pooled key enters its slot rotated once, from its bf16 value
            const float *pp = a.rot_pos + b * a.rot_pos_b + 3 * (static_cast<int64_t>(f) * a.cells + j);
            const double pt = (a.t_origin ? *a.t_origin : 0.0) + static_cast<double>(pp[0]);
            float cs[4], sn[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 r = pair_rotation(tab, c * 4 + k, pt, pp[1], pp[2], a.rot_scale);
                cs[k] = r.x;
                sn[k] = r.y;
            }
            *reinterpret_cast<uint4 *>(a.k_rot + out_off) = rotate8(pooled, cs, sn);
        }
    }
    if (a.pos_out && h == 0 && c == 0) {
        float *pp = a.pos_out + b * a.pos_b + 3 * (static_cast<int64_t>(f) * a.cells + j);
        pp[0] = a.frame_t[static_cast<int64_t>(b) * a.n_frames + f];
        pp[1] = 0.5f * static_cast<float>(r0 + r1 - 1);
        pp[2] = 0.5f * static_cast<float>(c0 + c1 - 1);
    }
}

__global__ void slot_map_kernel(int32_t *slot, int n_frames, int grid_h, int grid_w, int pool_h, int pool_w,
                                int cells_w, int cells) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t per = static_cast<int64_t>(grid_h) * grid_w;
    if (idx >= per * n_frames) return;
    const int f = static_cast<int>(idx / per);
    const int i = static_cast<int>(idx % per);
    const int r = i / grid_w, c = i % grid_w;
    slot[idx] = f * cells + (r / pool_h) * cells_w + c / pool_w;
}

// ============================================================== KV append
struct AppendArgs {
    __nv_bfloat16 *__restrict__ k_buf;
    __nv_bfloat16 *__restrict__ v_buf;
    float *__restrict__ pos_buf;
    const __nv_bfloat16 *__restrict__ k_src;
    const __nv_bfloat16 *__restrict__ v_src;
    const float *__restrict__ pos_src;
    const int32_t *__restrict__ n_valid;
    int32_t n_heads, n_tokens, buf_tokens, dst_token;
    int64_t sb, st, sh, psb;
    int64_t total;
};

// One thread per (batch, token, head, 16-byte chunk), chunk then head
// fastest: reads follow the token-major source, writes are whole 256-byte
// head rows of the head-major buffer.
template <int D>
__global__ void __launch_bounds__(256) append_kernel(const AppendArgs a) {
    constexpr int kChunks = D / 8;
    const uint32_t idx = blockIdx.x * blockDim.x + threadIdx.x;   // (token, head, chunk) of one session
    if (idx >= static_cast<uint32_t>(a.total)) return;
    const int b = blockIdx.y;
    const int c = static_cast<int>(idx % kChunks);
    const uint32_t hn = idx / kChunks;
    const int h = static_cast<int>(hn % static_cast<uint32_t>(a.n_heads));
    const int n = static_cast<int>(hn / static_cast<uint32_t>(a.n_heads));
    if (a.n_valid && n >= a.n_valid[b]) return;
    const int64_t s_off = b * a.sb + n * a.st + h * a.sh + c * 8;
    const int64_t d_off =
        ((static_cast<int64_t>(b) * a.n_heads + h) * a.buf_tokens + a.dst_token + n) * D + c * 8;
    if (a.k_src)
        *reinterpret_cast<uint4 *>(a.k_buf + d_off) = __ldg(reinterpret_cast<const uint4 *>(a.k_src + s_off));
    if (a.v_src)
        *reinterpret_cast<uint4 *>(a.v_buf + d_off) = __ldg(reinterpret_cast<const uint4 *>(a.v_src + s_off));
    if (a.pos_src && h == 0 && c == 0) {
        const float *ps = a.pos_src + b * a.psb + 3 * static_cast<int64_t>(n);
        float *pd = a.pos_buf + (static_cast<int64_t>(b) * a.buf_tokens + a.dst_token + n) * 3;
        pd[0] = ps[0];
        pd[1] = ps[1];
        pd[2] = ps[2];
    }
}

// ============================================================== index gather / scatter
// Token rows move between a token list and a slotted layout (window-major
// buffers, ring slots).  One thread per (batch, slot, head, 16-byte chunk).
struct GatherArgs {
    void *__restrict__ dst;
    const void *__restrict__ src;
    const int32_t *__restrict__ idx;   // [n_batch][n_slots]: source token, or < 0
    const float *__restrict__ src_pos; // gather only: [tokens][3] or null (required for RoPE)
    float *__restrict__ dst_pos;       // gather only: [n_batch][n_slots][3] or null
    int32_t n_slots, n_heads;
    int64_t src_t, src_h, dst_b, dst_s, dst_h, pos_b;
    int64_t total;                     // threads per batch entry: slots x D/8
    float out_scale;                   // RoPE gather only
    const double *__restrict__ t_origin;   // RoPE gather only: optional offset added to every t
};

constexpr int kGatherHeads = 8;   // head rows a thread keeps in flight

// One thread per (batch, slot, 16-byte chunk), chunk fastest: half a warp
// covers one 256-byte head row of a token.  The thread walks the token's
// heads 8 at a time with all 8 loads in flight.
// Gather: dst[b][s][h][:] = idx >= 0 ? src[idx][h][:] : 0 (positions likewise);
// kRope: the row is rotated by the position src_pos[idx] on the way (the
// cache write and the RoPE in one pass), the token's (cos, sin) pairs
// computed once for all its heads.
template <int D, bool kRope>
__global__ void __launch_bounds__(256, 4) gather_kernel(const GatherArgs a, const RopeTable tab) {
    constexpr int kChunks = D / 8;
    __shared__ double s_theta[kRope ? D / 2 : 1];
    if constexpr (kRope) {
        if (threadIdx.x < D / 2) s_theta[threadIdx.x] = tab.theta[threadIdx.x];
        __syncthreads();
    }
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= static_cast<uint32_t>(a.total)) return;
    const int b = blockIdx.y;
    const int c = static_cast<int>(i % kChunks);
    const int sl = static_cast<int>(i / kChunks);
    const int t = a.idx[static_cast<int64_t>(b) * a.n_slots + sl];
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.dst) + b * a.dst_b + sl * a.dst_s + c * 8;
    if (a.dst_pos && c == 0) {
        float *pd = a.dst_pos + b * a.pos_b + 3 * static_cast<int64_t>(sl);
        for (int e = 0; e < 3; ++e) pd[e] = t >= 0 ? a.src_pos[3 * static_cast<int64_t>(t) + e] : 0.f;
    }
    if (t < 0) {
        for (int h = 0; h < a.n_heads; ++h) *reinterpret_cast<uint4 *>(dst + h * a.dst_h) = make_uint4(0, 0, 0, 0);
        return;
    }
    const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(a.src) + t * a.src_t + c * 8;
    float cs[4], sn[4];
    if constexpr (kRope) {
        const float *pp = a.src_pos + 3 * static_cast<int64_t>(t);
        const double pt = (a.t_origin ? *a.t_origin : 0.0) + static_cast<double>(pp[0]);
        token_rotation(s_theta, tab, c, pt, pp[1], pp[2], a.out_scale, cs, sn);
    }
    for (int h0 = 0; h0 < a.n_heads; h0 += kGatherHeads) {
        uint4 u[kGatherHeads];
#pragma unroll
        for (int j = 0; j < kGatherHeads; ++j)
            u[j] = h0 + j < a.n_heads ? __ldg(reinterpret_cast<const uint4 *>(src + (h0 + j) * a.src_h))
                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kGatherHeads; ++j) {
            if (h0 + j >= a.n_heads) break;
            uint4 v = u[j];
            if constexpr (kRope) v = rotate8(v, cs, sn);
            *reinterpret_cast<uint4 *>(dst + (h0 + j) * a.dst_h) = v;
        }
    }
}

// dst[idx][h][:] = src[b][s][h][:] for idx >= 0 (dst/src roles of GatherArgs:
// src is the slotted layout here, dst the token list); same thread layout.
template <int D>
__global__ void __launch_bounds__(256) scatter_kernel(const GatherArgs a) {
    constexpr int kChunks = D / 8;
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= static_cast<uint32_t>(a.total)) return;
    const int b = blockIdx.y;
    const int c = static_cast<int>(i % kChunks);
    const int sl = static_cast<int>(i / kChunks);
    const int t = a.idx[static_cast<int64_t>(b) * a.n_slots + sl];
    if (t < 0) return;
    const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(a.src) + b * a.dst_b + sl * a.dst_s + c * 8;
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.dst) + t * a.src_t + c * 8;
    for (int h0 = 0; h0 < a.n_heads; h0 += kGatherHeads) {
        uint4 u[kGatherHeads];
#pragma unroll
        for (int j = 0; j < kGatherHeads; ++j)
            u[j] = h0 + j < a.n_heads ? __ldg(reinterpret_cast<const uint4 *>(src + (h0 + j) * a.dst_h))
                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kGatherHeads; ++j) {
            if (h0 + j >= a.n_heads) break;
            *reinterpret_cast<uint4 *>(dst + (h0 + j) * a.src_h) = u[j];
        }
    }
}

template <int D>
int gather_launch(const GatherLaunch &l) {
    GatherArgs a{l.dst, l.src, l.idx, l.src_pos, l.dst_pos, l.n_slots, l.n_heads,
                 l.src_t, l.src_h, l.dst_b, l.dst_s, l.dst_h, l.pos_b,
                 static_cast<int64_t>(l.n_slots) * (D / 8), l.out_scale, l.t_origin};
    if (a.total > 0x7fffffff || l.n_batch > 65535)
        return set_error(SR_ERR_INVALID_ARG, "gather/scatter: too many slots or batch entries");
    const dim3 grid(static_cast<unsigned>((a.total + 255) / 256), l.n_batch);
    if (l.scatter) {
        scatter_kernel<D><<<grid, 256, 0, l.stream>>>(a);
    } else if (l.rope) {
        gather_kernel<D, true><<<grid, 256, 0, l.stream>>>(a, make_rope_table(l.cfg));
    } else {
        gather_kernel<D, false><<<grid, 256, 0, l.stream>>>(a, RopeTable{});
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SR_OK : set_cuda_error("gather/scatter launch", e);
}

template <int D, bool kNorm>
int rope_launch(const RopeLaunch &l) {
    const RopeTable tab = make_rope_table(l.cfg);
    RopeArgs a{static_cast<const __nv_bfloat16 *>(l.x), static_cast<__nv_bfloat16 *>(l.y), l.pos, l.n_valid,
               l.n_heads, l.out_scale, l.xb, l.xt, l.xh, l.yb, l.yt, l.yh, l.pb,
               l.gamma, l.eps, static_cast<__nv_bfloat16 *>(l.y_raw), l.rb, l.rt, l.rh,
               l.t_origin, static_cast<const __nv_bfloat16 *>(l.vx), static_cast<__nv_bfloat16 *>(l.vy)};
    dim3 grid(l.n_tokens, l.n_batch);
    // passes of 128 / (D/8) heads each: instantiated for 1..8 (more heads run
    // the extra passes in a loop, without normalisation only)
    const int passes = (l.n_heads + 128 / (D / 8) - 1) / (128 / (D / 8));
    switch (passes < 8 ? passes : 8) {
        case 1: rope3d_kernel<D, kNorm, 1><<<grid, 128, 0, l.stream>>>(a, tab); break;
        case 2: rope3d_kernel<D, kNorm, 2><<<grid, 128, 0, l.stream>>>(a, tab); break;
        case 3: rope3d_kernel<D, kNorm, 3><<<grid, 128, 0, l.stream>>>(a, tab); break;
        case 4: rope3d_kernel<D, kNorm, 4><<<grid, 128, 0, l.stream>>>(a, tab); break;
        case 5: rope3d_kernel<D, kNorm, 5><<<grid, 128, 0, l.stream>>>(a, tab); break;
        case 6: rope3d_kernel<D, kNorm, 6><<<grid, 128, 0, l.stream>>>(a, tab); break;
        case 7: rope3d_kernel<D, kNorm, 7><<<grid, 128, 0, l.stream>>>(a, tab); break;
        default: rope3d_kernel<D, kNorm, 8><<<grid, 128, 0, l.stream>>>(a, tab); break;
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SR_OK : set_cuda_error("rope3d launch", e);
}

template <int D>
int pool_launch(const PoolLaunch &l) {
    PoolArgs a{};
    a.k_in = static_cast<const __nv_bfloat16 *>(l.k_in);
    a.v_in = static_cast<const __nv_bfloat16 *>(l.v_in);
    a.k_out = static_cast<__nv_bfloat16 *>(l.k_out);
    a.v_out = static_cast<__nv_bfloat16 *>(l.v_out);
    a.n_frames = l.n_frames;
    a.n_heads = l.n_heads;
    a.grid_h = l.cfg.grid_h;
    a.grid_w = l.cfg.grid_w;
    a.pool_h = l.cfg.pool_h;
    a.pool_w = l.cfg.pool_w;
    a.cells_w = (l.cfg.grid_w + l.cfg.pool_w - 1) / l.cfg.pool_w;
    a.cells = a.cells_w * ((l.cfg.grid_h + l.cfg.pool_h - 1) / l.cfg.pool_h);
    a.ib = l.ib; a.i_f = l.i_f; a.it = l.it; a.ih = l.ih;
    a.ob = l.ob; a.o_f = l.o_f; a.ot = l.ot; a.oh = l.oh;
    a.frame_t = l.frame_t;
    a.pos_out = l.pos_out;
    a.pos_b = l.pos_b;
    a.k_rot = static_cast<__nv_bfloat16 *>(l.k_rot);
    a.rot_pos = l.rot_pos;
    a.rot_pos_b = l.rot_pos_b;
    a.t_origin = l.t_origin;
    a.rot_scale = l.rot_scale;
    a.total = static_cast<int64_t>(a.cells) * l.n_heads * (D / 8);   // threads per frame
    if (a.total > 0x7fffffff || l.n_frames > 65535 || l.n_batch > 65535)
        return set_error(SR_ERR_INVALID_ARG, "history_compress: too many cells, frames or sessions");
    if (a.total > 0) {
        const dim3 blocks(static_cast<unsigned>((a.total + 255) / 256), l.n_frames, l.n_batch);
        const RopeTable tab = l.k_rot ? make_rope_table(l.rot_cfg) : RopeTable{};
        if (a.pool_h == 2 && a.pool_w == 2)
            pool_kernel<D, 2, 2><<<blocks, 256, 0, l.stream>>>(a, tab);
        else if (a.pool_h == 4 && a.pool_w == 4)
            pool_kernel<D, 4, 4><<<blocks, 256, 0, l.stream>>>(a, tab);
        else
            pool_kernel<D, 0, 0><<<blocks, 256, 0, l.stream>>>(a, tab);
    }
    if (l.slot_of_src) {
        const int64_t n = static_cast<int64_t>(l.n_frames) * l.cfg.grid_h * l.cfg.grid_w;
        if (n > 0)
            slot_map_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, l.stream>>>(
                l.slot_of_src, l.n_frames, l.cfg.grid_h, l.cfg.grid_w, l.cfg.pool_h, l.cfg.pool_w, a.cells_w,
                a.cells);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SR_OK : set_cuda_error("history_compress launch", e);
}

template <int D>
int append_launch(const AppendLaunch &l) {
    if (l.k_rot) {
        // K rotated into k_rot (and copied raw into k_buf if given), V copied:
        // the RoPE kernel, one CTA per token, head-major destination rows
        const int64_t hb = static_cast<int64_t>(l.buf_tokens) * D;   // head stride of the buffers
        const int64_t bb = static_cast<int64_t>(l.n_heads) * hb;      // batch stride
        const int64_t off = static_cast<int64_t>(l.dst_token) * D;
        RopeLaunch r{l.k_src, static_cast<__nv_bfloat16 *>(l.k_rot) + off, l.rot_pos, l.n_valid, l.n_batch,
                     l.n_tokens, l.n_heads, D, l.rot_cfg, l.rot_scale, l.sb, l.st, l.sh, bb, D, hb,
                     l.rot_pos_b, l.stream};
        r.y_raw = l.k_buf && l.k_src ? static_cast<__nv_bfloat16 *>(l.k_buf) + off : nullptr;
        r.rb = bb;
        r.rt = D;
        r.rh = hb;
        r.t_origin = l.t_origin;
        if (l.v_src) {
            r.vx = l.v_src;
            r.vy = static_cast<__nv_bfloat16 *>(l.v_buf) + off;
        }
        int rc = rope_launch<D, false>(r);
        if (rc != SR_OK || !l.pos_src) return rc;
        AppendLaunch pl = l;   // positions only, by the plain copy
        pl.k_src = pl.v_src = nullptr;
        pl.k_rot = nullptr;
        return append_launch<D>(pl);
    }
    AppendArgs a{};
    a.k_buf = static_cast<__nv_bfloat16 *>(l.k_buf);
    a.v_buf = static_cast<__nv_bfloat16 *>(l.v_buf);
    a.pos_buf = l.pos_buf;
    a.k_src = static_cast<const __nv_bfloat16 *>(l.k_src);
    a.v_src = static_cast<const __nv_bfloat16 *>(l.v_src);
    a.pos_src = l.pos_src;
    a.n_valid = l.n_valid;
    a.n_heads = l.n_heads;
    a.n_tokens = l.n_tokens;
    a.buf_tokens = l.buf_tokens;
    a.dst_token = l.dst_token;
    a.sb = l.sb; a.st = l.st; a.sh = l.sh; a.psb = l.psb;
    a.total = static_cast<int64_t>(l.n_tokens) * l.n_heads * (D / 8);   // threads per session
    if (a.total > 0x7fffffff || l.n_batch > 65535)
        return set_error(SR_ERR_INVALID_ARG, "kv_append: too many tokens or sessions");
    const dim3 blocks(static_cast<unsigned>((a.total + 255) / 256), l.n_batch);
    append_kernel<D><<<blocks, 256, 0, l.stream>>>(a);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SR_OK : set_cuda_error("kv_append launch", e);
}

__global__ void clock_advance_kernel(double *clock, double frames) { *clock += frames; }

}  // namespace

int launch_clock_advance(double *clock, double frames, cudaStream_t stream) {
    clock_advance_kernel<<<1, 1, 0, stream>>>(clock, frames);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SR_OK : set_cuda_error("stream_clock_advance launch", e);
}

int launch_rope3d(const RopeLaunch &l) {
    if (l.gamma) return l.head_dim == 128 ? rope_launch<128, true>(l) : rope_launch<64, true>(l);
    return l.head_dim == 128 ? rope_launch<128, false>(l) : rope_launch<64, false>(l);
}
int rope_norm_max_heads(int head_dim) { return 8 * (128 / (head_dim / 8)); }
int launch_gather(const GatherLaunch &l) { return l.head_dim == 128 ? gather_launch<128>(l) : gather_launch<64>(l); }
int launch_history_compress(const PoolLaunch &l) {
    return l.head_dim == 128 ? pool_launch<128>(l) : pool_launch<64>(l);
}
int launch_kv_append(const AppendLaunch &l) {
    return l.head_dim == 128 ? append_launch<128>(l) : append_launch<64>(l);
}

}  // namespace sr
