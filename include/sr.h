/*
 * sr.h -- C ABI of libsr.so: the chunk-streaming joint video+audio
 * self-attention step on one NVIDIA B200 (sm_100a).
 *
 * The step (one DiT layer, all heads) is four calls launched back to back on
 * one CUDA stream:
 *   sr_history_compress  pool history frames into coarser tiers
 *   sr_kv_append         write token K/V (and positions) into the window
 *   sr_rope3d_apply      3-D (t, h, w) RoPE + re-layout of Q and window K
 *   sr_chunk_attention_fwd  softmax attention of the chunk queries over the
 *                        prompt, context and chunk KV segments
 *
 * Conventions shared by every call
 *   - Every function returns an int status (SR_OK or an SR_ERR_* code).  On
 *     error nothing is launched and sr_get_last_error() (thread-local) holds
 *     a one-line reason.
 *   - Every tensor pointer is DEVICE memory owned by the caller.  The library
 *     never allocates, frees or synchronises; launches are asynchronous on the
 *     caller's stream (`stream` is a cudaStream_t passed as void*; NULL means
 *     the legacy default stream).
 *   - Tensors are bf16 unless stated; positions are fp32 triples (t, h, w).
 *     Strides are in ELEMENTS.  The head dimension is contiguous (stride 1).
 *     Pointers to bf16 tensors must be 16-byte aligned and every stride a
 *     multiple of 8 elements (16 bytes); violations return SR_ERR_INVALID_ARG.
 *   - Sizes are int32/int64 counts; a call with zero work returns SR_OK and
 *     launches nothing.
 */
#ifndef SR_H_
#define SR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SR_VERSION 1

#define SR_OK 0
#define SR_ERR_INVALID_ARG 1
#define SR_ERR_UNSUPPORTED 2
#define SR_ERR_CUDA 3
#define SR_ERR_DEVICE_TIMEOUT 4

#define SR_MAX_SEG 8   /* KV segments per window */
#define SR_TILE 128    /* KV tile (tokens); every segment capacity is a multiple */

/* Library version (SR_VERSION of the build). */
int sr_version(void);

/* Reason for the last non-OK status returned on this thread ("" if none). */
const char *sr_get_last_error(void);

/* ------------------------------------------------------------------------ */
/* 3-D multimodal RoPE.
 *
 * Defined by: "MiniMax-H3 deep dive" (fiv.co.kr), H3-Omni-Transformer row of
 * the components table and the tensor-name paragraph (3D MM-RoPE on the
 * shared single-stream attention); the fused rotate-and-write-cache idea is
 * from "StreamRender-H3" (molayo1419.me), causal VAE section (qk-norm, RoPE
 * and KV-cache write fused in one kernel).
 *
 * Reading (the pages give no formula): the head vector is split into
 * contiguous sub-blocks [t: d_t | h: d_h | w: d_w]; inside the sub-block of
 * axis a (width d_a) the interleaved pair (x[2j], x[2j+1]) turns
 * counter-clockwise by phi = pos_a * base^(-2j/d_a).
 *
 *   y = out_scale * R(pos) x            (computed in fp32, stored bf16 RNE)
 *
 * x   element (b, n, h, d) at x + b*x_batch_stride + n*x_token_stride + h*x_head_stride + d
 * y   element (b, n, h, d) at y + b*y_batch_stride + n*y_token_stride + h*y_head_stride + d
 * pos fp32 (t, h, w) of token (b, n) at pos + b*pos_batch_stride + 3*n; NULL = all zero
 *     (a pure re-layout, optionally scaled).
 * t_origin_dev  optional fp64 on the device added to every token's t before
 *     the angle is formed (in fp64): the stream clock of a streaming session,
 *     so that keys rotated at different steps share one time axis.  NULL = 0.
 *     8-byte aligned.
 * n_valid_dev  optional int32[n_batch] on the device: tokens n >= n_valid[b]
 *     are skipped (neither read nor written).  NULL = all n_tokens.
 * Layouts: any strides, e.g. token-major [B, N, H, D] in, head-major
 * [B, H, N, D] out (the attention layout).  x and y must not overlap.
 * Requirements: head_dim in {64, 128}; d_t + d_h + d_w == head_dim, each even
 * and a multiple of 8; n_heads >= 1.
 */
typedef struct {
    float base;                 /* 10000 */
    int32_t d_t, d_h, d_w;      /* sub-block widths */
} sr_rope_cfg;

int sr_rope3d_apply(const void *x, void *y, const float *pos,
                    int32_t n_batch, int32_t n_tokens, int32_t n_heads, int32_t head_dim,
                    const int32_t *n_valid_dev, sr_rope_cfg cfg, float out_scale,
                    int64_t x_batch_stride, int64_t x_token_stride, int64_t x_head_stride,
                    int64_t y_batch_stride, int64_t y_token_stride, int64_t y_head_stride,
                    int64_t pos_batch_stride, const double *t_origin_dev, void *stream);

/* QK normalisation fused with the 3-D RoPE and the cache write.
 *
 * Defined by: "MiniMax-H3 deep dive" (fiv.co.kr), tensor-name paragraph
 * (norm_q / norm_k beside to_q / to_k: QK normalisation in the shared
 * attention); "StreamRender-H3" (molayo1419.me), causal VAE section (qk-norm,
 * RoPE and KV-cache write fused in one kernel).
 *
 * Reading: per head vector (length D), RMSNorm with a learned gain, then the
 * rotation of sr_rope3d_apply:
 *   u = x / sqrt(mean_d(x[d]^2) + eps) * gamma      (fp32)
 *   y = out_scale * R(pos) u                         (bf16 RNE)
 *   y_raw = u                                        (bf16 RNE, optional)
 * Arguments as in sr_rope3d_apply, plus gamma: fp32 [head_dim] on the device
 * (16-byte aligned); eps >= 0; t_origin_dev as for sr_rope3d_apply; y_raw:
 * optional output with its own strides
 * (element (b, n, h, d) at y_raw + b*yraw_batch_stride + n*yraw_token_stride
 * + h*yraw_head_stride + d), NULL = not written.
 * Requires n_heads <= 64 at head_dim 128 (<= 128 at head_dim 64).
 */
int sr_qknorm_rope3d_apply(const void *x, void *y, void *y_raw, const float *gamma, float eps,
                           const float *pos, int32_t n_batch, int32_t n_tokens, int32_t n_heads,
                           int32_t head_dim, const int32_t *n_valid_dev, sr_rope_cfg cfg, float out_scale,
                           int64_t x_batch_stride, int64_t x_token_stride, int64_t x_head_stride,
                           int64_t y_batch_stride, int64_t y_token_stride, int64_t y_head_stride,
                           int64_t yraw_batch_stride, int64_t yraw_token_stride, int64_t yraw_head_stride,
                           int64_t pos_batch_stride, const double *t_origin_dev, void *stream);

/* Fused rotation of the K that a call writes into the window (optional
 * argument of sr_kv_append and sr_history_compress): the key enters its slot
 * rotated once, as sr_rope3d_apply would rotate it,
 *     k_rot[...] = out_scale * R(pos + (*t_origin_dev, 0, 0)) k
 * with the bf16 value k the call writes (or would write) as its K output.
 * k_rot has the layout of that K output; pos is documented per call. */
typedef struct {
    void *k_rot;                 /* bf16 destination; NULL = no rotation */
    const float *pos;            /* fp32 (t, h, w) per token (4-byte aligned) */
    int64_t pos_batch_stride;    /* elements between sessions in pos */
    const double *t_origin_dev;  /* device fp64 added to every t, or NULL */
    sr_rope_cfg cfg;             /* sub-blocks multiples of 8 summing to head_dim */
    float out_scale;
} sr_rope_out;

/* Stream clock of a streaming session: *clock_dev += frames, on the stream
 * (one-thread kernel, so that a step replayed from a CUDA graph sees the new
 * value).  The clock is the t offset (sr_rope3d_apply's t_origin_dev) of the
 * current chunk's first latent frame; a window slide of n frames advances it
 * by n.  Defined by: "StreamRender-H3" (molayo1419.me), streaming context
 * section (the fixed position template of the window; positions differ only
 * by the step's shift, so each key is rotated once on entry).  clock_dev:
 * 8-byte aligned device double. */
int sr_stream_clock_advance(double *clock_dev, double frames, void *stream);

/* ------------------------------------------------------------------------ */
/* History-tier pooling.
 *
 * Defined by: "AlayaRenderer-Flash" (aitrends.kr), key contributions and
 * technical details: past history is kept in three tiers by temporal
 * distance, recent at full resolution, older at progressively lower spatial
 * resolution.
 *
 * Reading: per frame, cell (r, c) of a pool_h x pool_w ceil-mode pooling is
 * the mean of the source tokens in rows [r*ph, min((r+1)*ph, Gh)) x cols
 * [c*pw, min((c+1)*pw, Gw)), counting valid members only, for K and V
 * separately and per head (fp32 accumulation, bf16 RNE result).  The pooled
 * position is (frame_t[f], mean member row, mean member col).
 *
 * Source token (b, f, i = row*Gw + col, h, d) at
 *   in + b*in_batch_stride + f*in_frame_stride + i*in_token_stride + h*in_head_stride + d
 * Pooled token (b, f, j = r*ceil(Gw/pw) + c, h, d) at
 *   out + b*out_batch_stride + f*out_frame_stride + j*out_token_stride + h*out_head_stride + d
 * k_in/k_out or v_in/v_out may both be NULL (that tensor is skipped).
 * frame_t   fp32 [n_batch][n_frames] (device) -- required when pos_out != NULL
 * pos_out   fp32 (t, h, w) of pooled token (b, f, j) at
 *           pos_out + b*pos_batch_stride + 3*(f*cells + j); NULL = not written
 * slot_of_src int32 [n_frames*Gh*Gw] (device): slot_of_src[f*Gh*Gw + i] =
 *           f*cells + (cell of i); the same for every batch; NULL = not written
 * rot       optional fused rotation of the pooled K (as rounded to bf16):
 *           rot->k_rot has the strides of k_out; the position of pooled token
 *           (b, f, j) is read at rot->pos + b*rot->pos_batch_stride + 3*(f*cells + j)
 *           (the layout of pos_out).  NULL = none.
 * Input and output must not overlap.  head_dim in {64, 128};
 * pool_h, pool_w in [1, 8].
 */
typedef struct {
    int32_t grid_h, grid_w;     /* source token grid (rows, cols) per frame */
    int32_t pool_h, pool_w;     /* pooling window = stride */
} sr_pool_cfg;

int sr_history_compress(const void *k_in, const void *v_in, void *k_out, void *v_out,
                        int32_t n_batch, int32_t n_frames, int32_t n_heads, int32_t head_dim,
                        sr_pool_cfg cfg,
                        int64_t in_batch_stride, int64_t in_frame_stride,
                        int64_t in_token_stride, int64_t in_head_stride,
                        int64_t out_batch_stride, int64_t out_frame_stride,
                        int64_t out_token_stride, int64_t out_head_stride,
                        const float *frame_t, float *pos_out, int64_t pos_batch_stride,
                        int32_t *slot_of_src, const sr_rope_out *rot, void *stream);

/* ------------------------------------------------------------------------ */
/* KV append into the persistent window buffer.
 *
 * Defined by: "StreamRender-H3" (molayo1419.me), inference acceleration
 * section: a per-layer persistent KV buffer kept in the layout the attention
 * kernel reads, with only the dynamic region updated in place (no
 * reallocation, no relocation of history); streaming context section: only
 * the recent history and the current chunk are recomputed.
 *
 * The window buffers are head-major [n_batch][n_heads][buf_tokens][head_dim]
 * (contiguous) for K and V, and fp32 [n_batch][buf_tokens][3] for positions.
 * Token n of the source lands in slot dst_token + n:
 *   k_buf[b][h][dst_token + n][:] = k_src + b*src_batch_stride + n*src_token_stride + h*src_head_stride
 * (likewise V and pos_src -> pos_buf; pos_src token stride 3, batch stride
 * pos_src_batch_stride).  Bytes are copied exactly.
 * Any of k_src / v_src / pos_src may be NULL (that buffer is left alone).
 * n_valid_dev: optional int32[n_batch]; tokens n >= n_valid[b] are skipped.
 * rot: optional fused rotation of K on its way in (the cache write and the
 * RoPE in one pass): rot->k_rot is a buffer of k_buf's layout whose slots
 * [dst_token, dst_token + n_tokens) receive the rotated K; the position of
 * token n of session b is read at rot->pos + b*rot->pos_batch_stride + 3*n.
 * With rot, k_buf may be NULL (only the rotated K is kept).  NULL = none.
 * Requires dst_token + n_tokens <= buf_tokens; head_dim in {64, 128}.
 */
int sr_kv_append(void *k_buf, void *v_buf, float *pos_buf,
                 int32_t n_batch, int32_t n_heads, int32_t head_dim, int32_t buf_tokens,
                 int32_t dst_token,
                 const void *k_src, const void *v_src, const float *pos_src,
                 int32_t n_tokens, const int32_t *n_valid_dev,
                 int64_t src_batch_stride, int64_t src_token_stride, int64_t src_head_stride,
                 int64_t pos_src_batch_stride, const sr_rope_out *rot, void *stream);

/* ------------------------------------------------------------------------ */
/* Index gather / scatter of token rows (window partition and merge).
 *
 * Defined by: "StreamRender-H3" (molayo1419.me), causal VAE section: the
 * decoder's attention uses non-overlapping 16x16 token windows, shifted by
 * half a window every other layer, with each window's KV in a preallocated
 * ring buffer; window partition and merge are done by index gathers.
 *
 * Gather:  dst[b][s][h][:] = idx[b][s] >= 0 ? src[idx[b][s]][h][:] : 0
 *   src element (t, h, d) at src + t*src_token_stride + h*src_head_stride + d
 *   dst element (b, s, h, d) at dst + b*dst_batch_stride + s*dst_slot_stride + h*dst_head_stride + d
 *   src_pos / dst_pos (optional, together): fp32 (t, h, w) triples, src_pos
 *   [tokens][3], dst_pos[b][s] at dst_pos + b*dst_pos_batch_stride + 3*s
 *   (zero for idx < 0).
 * Scatter: dst[idx[b][s]][h][:] = src[b][s][h][:] for every idx[b][s] >= 0
 *   (the slotted layout is the source; indices must not repeat).
 * idx: int32 [n_batch][n_slots] on the device.  head_dim in {64, 128}.
 */
int sr_gather_tokens(void *dst, const void *src, const int32_t *idx, int32_t n_batch, int32_t n_slots,
                     int32_t n_heads, int32_t head_dim, int64_t src_token_stride, int64_t src_head_stride,
                     int64_t dst_batch_stride, int64_t dst_slot_stride, int64_t dst_head_stride,
                     const float *src_pos, float *dst_pos, int64_t dst_pos_batch_stride, void *stream);
int sr_scatter_tokens(void *dst, const void *src, const int32_t *idx, int32_t n_batch, int32_t n_slots,
                      int32_t n_heads, int32_t head_dim, int64_t dst_token_stride, int64_t dst_head_stride,
                      int64_t src_batch_stride, int64_t src_slot_stride, int64_t src_head_stride, void *stream);

/* Gather with RoPE: the gather above with every copied row rotated by its
 * source token's position on the way, i.e. the positional encoding and the
 * cache write of the windowed KV ring in one pass.
 *
 * Defined by: "StreamRender-H3" (molayo1419.me), causal VAE section: the
 * position encoding and the cache write happen once, when a frame enters the
 * ring, and partition is an index gather; the rotation is the one of
 * sr_rope3d_apply (3-D RoPE, interleaved pairs in t/h/w sub-blocks).
 *
 *   dst[b][s][h][:] = idx[b][s] >= 0 ? R(src_pos[idx[b][s]]) src[idx[b][s]][h][:] * out_scale : 0
 * Strides as for sr_gather_tokens; src_pos: fp32 [tokens][3] (t, h, w),
 * required; t_origin_dev: optional device fp64 added to every t (the
 * absolute frame index of the call, so that the positions stay a fixed
 * table), NULL = 0.  cfg as for sr_rope3d_apply (sub-blocks multiples of 8 summing
 * to head_dim).  head_dim in {64, 128}.  Returns SR_ERR_INVALID_ARG (nothing
 * launched) for bad sizes, strides, alignment or a missing src_pos.
 */
int sr_gather_rope3d_tokens(void *dst, const void *src, const int32_t *idx, const float *src_pos, int32_t n_batch,
                            int32_t n_slots, int32_t n_heads, int32_t head_dim, sr_rope_cfg cfg, float out_scale,
                            int64_t src_token_stride, int64_t src_head_stride, int64_t dst_batch_stride,
                            int64_t dst_slot_stride, int64_t dst_head_stride, const double *t_origin_dev,
                            void *stream);

/* ------------------------------------------------------------------------ */
/* Fused chunk attention over [prompt | context | chunk] KV segments.
 *
 * Defined by: "StreamRender-H3" (molayo1419.me), streaming context section
 * (the window is attended bidirectionally; the moving part sees the whole
 * window) and inference acceleration section (FlashAttention on Blackwell
 * tuned to the streaming shapes with one KV split; lengths and offsets reused
 * without host-device synchronisation; persistent KV in the kernel's
 * layout); "AlayaRenderer-Flash" (aitrends.kr), methodology (past chunks as
 * clean tokens in self-attention; persistent style-prompt KV in every
 * self-attention layer).
 *
 *   O[b, i, h] = sum_j softmax_j(softmax_scale * q_i . k_j) v_j
 *   over every VALID slot j of every segment; LSE = ln sum_j exp(scale q.k_j)
 *
 * No causal mask.  Padded slots (beyond a segment's valid length) are masked.
 *
 * q    [n_batch][n_heads][q_cap][head_dim]      (head-major, after RoPE)
 * k, v [n_batch][n_heads][kv_tokens][head_dim]  kv_tokens = sum(layout->cap)
 *      segment s occupies slots [start_s, start_s + cap_s), start_s = sum_{t<s} cap_t;
 *      its valid tokens are the first kv_len[b][s] slots.
 *      Padded V slots must hold finite values (zero-fill the buffer once).
 * o    [n_batch][q_cap][n_heads][head_dim]      (token-major, bf16)
 * lse  fp32 [n_batch][n_heads][q_cap] natural-log LSE, or NULL
 * kv_len_dev int32 [n_batch][layout->n_seg] (device), 0 <= len <= cap
 * q_len_dev  int32 [n_batch] (device), 1 <= q_len <= q_cap; rows >= q_len are
 *      neither computed into o nor lse.  The host cannot check device values,
 *      so the kernels clamp q_len to [0, q_cap]: an out-of-range value never
 *      writes outside o or lse.
 * workspace  optional caller-owned device scratch of workspace_bytes >=
 *      sr_chunk_attention_workspace_bytes(n_batch, n_heads, head_dim, q_cap)
 *      bytes (16-byte aligned), or NULL.  With it, when the (session, head,
 *      256-row query block) units do not fill whole waves of the GPU's SMs,
 *      the units of the last partial wave are split along the KV tiles and
 *      their fp32 partial results are merged by a second kernel on the same
 *      stream; without it every unit runs whole.  Calls that share one
 *      workspace must be ordered (same stream).  Results of the two schedules
 *      agree to fp32 rounding.
 * status_dev optional int32 (device): left untouched on success; set to
 *      SR_ERR_DEVICE_TIMEOUT if a pipeline wait inside the kernel gave up
 *      (bounded waits; the kernel then returns early and its outputs are
 *      undefined).  Read it after synchronising the stream.
 * A session whose segments are all empty is a caller error: its rows are
 * written as zero with lse = -inf.
 * Requirements: head_dim in {64, 128}; 1 <= n_seg <= SR_MAX_SEG; every cap a
 * positive multiple of SR_TILE; q_cap >= 1.
 */
typedef struct {
    int32_t n_seg;
    int32_t cap[SR_MAX_SEG];    /* tokens, multiples of SR_TILE */
} sr_kv_layout;

int sr_chunk_attention_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                           const sr_kv_layout *layout, const int32_t *kv_len_dev,
                           const int32_t *q_len_dev, int32_t n_batch, int32_t n_heads,
                           int32_t head_dim, int32_t q_cap, float softmax_scale,
                           void *workspace, size_t workspace_bytes,
                           int32_t *status_dev, void *stream);

/* Bytes of workspace sr_chunk_attention_fwd can use for this problem on the
 * current device (0 if it would never split, or on invalid sizes).  Host
 * only; reads the device's SM count (no allocation, no synchronisation). */
size_t sr_chunk_attention_workspace_bytes(int32_t n_batch, int32_t n_heads, int32_t head_dim, int32_t q_cap);

/* Bound of every pipeline wait inside the attention kernels, for the launches
 * that follow on any thread (library-wide; default 1 s; 0 restores the
 * default).  A wait that runs out raises SR_ERR_DEVICE_TIMEOUT in status_dev:
 * the kernel then waits, again at most this long, for its own copies and
 * tensor-core operations still in flight, releases its tensor memory and
 * returns, leaving the context usable.  Not part of the method (the pages
 * have no counterpart): the failure detection of this library. */
int sr_set_wait_limit_ns(uint64_t limit_ns);

/* Test hook of that failure path, not for production use (the pages have no
 * counterpart): from the next attention launch on, the load of K tile `tile`
 * (counted from each work item's first tile), and of the V tile that shares
 * its pipeline stage, is withheld, so the pipeline
 * wait for it runs out after the limit above and the launch reports
 * SR_ERR_DEVICE_TIMEOUT.  Nothing faults or hangs.  -1 (the default) turns it
 * off; < -1 is rejected. */
int sr_set_withheld_kv_tile(int32_t tile);

/* Allocation-free variant of sr_chunk_attention_fwd (the pages have no
 * counterpart; this is a packaging option of this library).
 *
 * For callers that cannot allocate device memory when they run the
 * attention -- a plugin inside another runtime that only receives its input
 * and output buffers, a real-time frame loop where cudaMalloc (which may
 * synchronise the device) is not allowed, or an application whose device
 * memory is all owned by its own allocator.  Arguments, layouts and results
 * are those of sr_chunk_attention_fwd; the split-KV scratch comes from a
 * static device array of SR_NOALLOC_SCRATCH_BYTES (24 MiB) that every GPU
 * loading the library holds until the process exits.  The call allocates
 * nothing and frees nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is looked up again when the
 *     device's context has been re-created since (e.g. after
 *     cudaDeviceReset), so the first call after such a reset must also come
 *     before any capture.
 *   - Problems whose schedule needs more scratch than the array holds
 *     (sr_chunk_attention_workspace_bytes > SR_NOALLOC_SCRATCH_BYTES) are
 *     rejected with SR_ERR_UNSUPPORTED and nothing is launched.  On a 148-SM
 *     B200 the largest need is about 19.7 MB, so no problem is rejected there.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls that could
 *     execute concurrently on the same device (different streams or host
 *     threads) race on it: order them.
 */
#define SR_NOALLOC_SCRATCH_BYTES (24u * 1024u * 1024u)

int sr_chunk_attention_fwd_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                   const sr_kv_layout *layout, const int32_t *kv_len_dev,
                                   const int32_t *q_len_dev, int32_t n_batch, int32_t n_heads,
                                   int32_t head_dim, int32_t q_cap, float softmax_scale,
                                   int32_t *status_dev, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SR_H_ */
