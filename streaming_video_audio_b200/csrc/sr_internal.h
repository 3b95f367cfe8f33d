// sr_internal.h -- host-side declarations shared by the libsr.so sources.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sr.h"

namespace sr {

// Record a thread-local error message and return `code`.
int set_error(int code, const char *fmt, ...);
int set_cuda_error(const char *what, cudaError_t e);

// 3-D bf16 tensor map over [outer][rows][inner] (inner contiguous), box
// {box_inner, box_rows, 1}, 128-byte swizzle, zero fill out of bounds.
int make_tmap_bf16_3d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t rows, uint64_t outer,
                      uint32_t box_inner, uint32_t box_rows);

// 4-D bf16 tensor map over a dense [d3][d2][d1][d0] tensor (d0 contiguous),
// box {box0, 1, box2, 1}, 128-byte swizzle (used for tiled stores).
int make_tmap_bf16_4d(CUtensorMap *tm, void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                      uint32_t box0, uint32_t box2);

struct AttnLaunch {
    const void *q, *k, *v;
    void *o;
    float *lse;
    const int32_t *kv_len, *q_len;
    int32_t *status;
    int32_t cap[SR_MAX_SEG];
    int32_t n_seg, n_batch, n_heads, head_dim, q_cap;
    int64_t kv_tokens;
    float softmax_scale;
    void *workspace;
    size_t workspace_bytes;
    cudaStream_t stream;
    uint64_t wait_limit_ns;    // bound of every pipeline wait inside the kernels
    int32_t withheld_tile;     // test hook: K tile whose load is withheld (-1: none)
};
int launch_chunk_attention(const AttnLaunch &a);

// Library-wide settings of the attention launches (sr_set_wait_limit_ns,
// sr_set_withheld_kv_tile): read at every launch.
uint64_t attention_wait_limit_ns();
int32_t attention_withheld_tile();

// Work list of the attention kernel: units are (session, head, 256-row query
// block); whole waves of units run one per CTA, and the units of a last
// partial wave are split into `split` KV ranges that fill the idle SMs.
struct AttnSchedule {
    int32_t qb_per_head;
    int64_t units;
    int32_t n_full;        // items that are whole units
    int32_t split;         // parts per tail unit (1 = no split)
    int32_t tail_units;
    size_t o_bytes, ml_bytes, workspace_bytes;
};
AttnSchedule attention_schedule(int32_t n_batch, int32_t n_heads, int32_t head_dim, int32_t q_cap, int32_t sms);
int attention_sm_count();
// Merge of the KV parts of split units (fp32 partials in the workspace).
int launch_split_combine(const float *ws_o, const float *ws_ml, void *o, float *lse, const int32_t *q_len,
                         int32_t n_full, int32_t split, int32_t tail_units, int32_t qb_per_head, int32_t n_heads,
                         int32_t q_cap, int32_t head_dim, cudaStream_t stream);

struct RopeLaunch {
    const void *x;
    void *y;
    const float *pos;
    const int32_t *n_valid;
    int32_t n_batch, n_tokens, n_heads, head_dim;
    sr_rope_cfg cfg;
    float out_scale;
    int64_t xb, xt, xh, yb, yt, yh, pb;
    cudaStream_t stream;
    const float *gamma = nullptr;   // non-null: RMSNorm each head vector first
    float eps = 0.f;
    void *y_raw = nullptr;          // optional unrotated copy (normalised when gamma is set)
    int64_t rb = 0, rt = 0, rh = 0;
    const double *t_origin = nullptr;   // optional device offset added to every t
    const void *vx = nullptr;       // optional rows copied unrotated, strides of x -> y
    void *vy = nullptr;
};
int launch_rope3d(const RopeLaunch &a);
int rope_norm_max_heads(int head_dim);

struct GatherLaunch {
    void *dst;
    const void *src;
    const int32_t *idx;
    const float *src_pos;
    float *dst_pos;
    int32_t n_batch, n_slots, n_heads, head_dim;
    int64_t src_t, src_h, dst_b, dst_s, dst_h, pos_b;
    bool scatter;
    bool rope;           // gather only: rotate each row by src_pos[idx] on the way
    sr_rope_cfg cfg;
    float out_scale;
    cudaStream_t stream;
    const double *t_origin = nullptr;   // RoPE gather: optional offset added to every t
};
int launch_gather(const GatherLaunch &l);

struct PoolLaunch {
    const void *k_in, *v_in;
    void *k_out, *v_out;
    int32_t n_batch, n_frames, n_heads, head_dim;
    sr_pool_cfg cfg;
    int64_t ib, i_f, it, ih, ob, o_f, ot, oh;
    const float *frame_t;
    float *pos_out;
    int64_t pos_b;
    int32_t *slot_of_src;
    cudaStream_t stream;
    void *k_rot = nullptr;          // optional fused RoPE output of the pooled K
    const float *rot_pos = nullptr;
    int64_t rot_pos_b = 0;
    const double *t_origin = nullptr;
    sr_rope_cfg rot_cfg{};
    float rot_scale = 1.f;
};
int launch_history_compress(const PoolLaunch &a);

struct AppendLaunch {
    void *k_buf, *v_buf;
    float *pos_buf;
    int32_t n_batch, n_heads, head_dim, buf_tokens, dst_token;
    const void *k_src, *v_src;
    const float *pos_src;
    int32_t n_tokens;
    const int32_t *n_valid;
    int64_t sb, st, sh, psb;
    cudaStream_t stream;
    void *k_rot = nullptr;          // optional: K rotated into this buffer (layout of k_buf)
    const float *rot_pos = nullptr;
    int64_t rot_pos_b = 0;
    const double *t_origin = nullptr;
    sr_rope_cfg rot_cfg{};
    float rot_scale = 1.f;
};
int launch_kv_append(const AppendLaunch &a);
int launch_clock_advance(double *clock, double frames, cudaStream_t stream);

}  // namespace sr
