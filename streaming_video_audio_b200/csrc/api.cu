// api.cu -- extern "C" entry points of libsr.so: argument validation,
// tensor-map creation and dispatch to the sm_100a kernels.  Nothing here
// allocates device memory or synchronises with the device.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "sr_internal.h"

namespace sr {

namespace {
thread_local char g_last_error[512] = "";

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t s) { return s % 8 == 0; }
}  // namespace

int set_error(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return code;
}

int set_cuda_error(const char *what, cudaError_t e) {
    return set_error(SR_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

namespace {
// cuTensorMapEncodeTiled from the driver, resolved once (nullptr if absent)
EncodeTiledFn encode_fn() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode;
}
}  // namespace

int make_tmap_bf16_3d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t rows, uint64_t outer,
                      uint32_t box_inner, uint32_t box_rows) {
    const EncodeTiledFn enc = encode_fn();
    if (!enc) return set_error(SR_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[3] = {inner, rows, outer};
    const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    const cuuint32_t box[3] = {box_inner, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(SR_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return SR_OK;
}

int make_tmap_bf16_4d(CUtensorMap *tm, void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                      uint32_t box0, uint32_t box2) {
    const EncodeTiledFn enc = encode_fn();
    if (!enc) return set_error(SR_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {box0, 1, box2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(SR_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return SR_OK;
}

}  // namespace sr

using namespace sr;

extern "C" {

int sr_version(void) { return SR_VERSION; }

const char *sr_get_last_error(void) { return g_last_error; }

int sr_rope3d_apply(const void *x, void *y, const float *pos, int32_t n_batch, int32_t n_tokens, int32_t n_heads,
                    int32_t head_dim, const int32_t *n_valid_dev, sr_rope_cfg cfg, float out_scale,
                    int64_t x_batch_stride, int64_t x_token_stride, int64_t x_head_stride, int64_t y_batch_stride,
                    int64_t y_token_stride, int64_t y_head_stride, int64_t pos_batch_stride,
                    const double *t_origin_dev, void *stream) {
    g_last_error[0] = 0;
    if (n_batch < 0 || n_tokens < 0 || n_heads < 1 || n_batch > 65535)
        return set_error(SR_ERR_INVALID_ARG, "rope3d: bad sizes (batch %d, tokens %d, heads %d)", n_batch,
                         n_tokens, n_heads);
    if (head_dim != 64 && head_dim != 128) return set_error(SR_ERR_UNSUPPORTED, "rope3d: head_dim must be 64 or 128");
    if (cfg.d_t < 0 || cfg.d_h < 0 || cfg.d_w < 0 || cfg.d_t % 8 || cfg.d_h % 8 || cfg.d_w % 8 ||
        cfg.d_t + cfg.d_h + cfg.d_w != head_dim)
        return set_error(SR_ERR_INVALID_ARG, "rope3d: sub-blocks %d/%d/%d must be multiples of 8 summing to %d",
                         cfg.d_t, cfg.d_h, cfg.d_w, head_dim);
    if (!(cfg.base > 0.f)) return set_error(SR_ERR_INVALID_ARG, "rope3d: base must be positive");
    if (n_batch == 0 || n_tokens == 0) return SR_OK;
    if (!x || !y) return set_error(SR_ERR_INVALID_ARG, "rope3d: null tensor");
    if (!aligned16(x) || !aligned16(y))
        return set_error(SR_ERR_INVALID_ARG, "rope3d: x and y must be 16-byte aligned");
    if (!stride_ok(x_batch_stride) || !stride_ok(x_token_stride) || !stride_ok(x_head_stride) ||
        !stride_ok(y_batch_stride) || !stride_ok(y_token_stride) || !stride_ok(y_head_stride))
        return set_error(SR_ERR_INVALID_ARG, "rope3d: strides must be multiples of 8 elements");
    if (pos && (reinterpret_cast<uintptr_t>(pos) & 3u))
        return set_error(SR_ERR_INVALID_ARG, "rope3d: pos must be 4-byte aligned");
    if (t_origin_dev && (reinterpret_cast<uintptr_t>(t_origin_dev) & 7u))
        return set_error(SR_ERR_INVALID_ARG, "rope3d: t_origin must be 8-byte aligned");
    RopeLaunch l{x, y, pos, n_valid_dev, n_batch, n_tokens, n_heads, head_dim, cfg, out_scale,
                 x_batch_stride, x_token_stride, x_head_stride, y_batch_stride, y_token_stride, y_head_stride,
                 pos_batch_stride, static_cast<cudaStream_t>(stream)};
    l.t_origin = t_origin_dev;
    return launch_rope3d(l);
}

int sr_qknorm_rope3d_apply(const void *x, void *y, void *y_raw, const float *gamma, float eps, const float *pos,
                           int32_t n_batch, int32_t n_tokens, int32_t n_heads, int32_t head_dim,
                           const int32_t *n_valid_dev, sr_rope_cfg cfg, float out_scale, int64_t x_batch_stride,
                           int64_t x_token_stride, int64_t x_head_stride, int64_t y_batch_stride,
                           int64_t y_token_stride, int64_t y_head_stride, int64_t yraw_batch_stride,
                           int64_t yraw_token_stride, int64_t yraw_head_stride, int64_t pos_batch_stride,
                           const double *t_origin_dev, void *stream) {
    g_last_error[0] = 0;
    if (!gamma) return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: gamma is NULL");
    if (reinterpret_cast<uintptr_t>(gamma) & 15u)
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: gamma must be 16-byte aligned");
    if (!(eps >= 0.f)) return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: eps must be >= 0");
    if ((head_dim == 64 || head_dim == 128) && n_heads > rope_norm_max_heads(head_dim))
        return set_error(SR_ERR_UNSUPPORTED, "qknorm_rope3d: at most %d heads of %d", rope_norm_max_heads(head_dim),
                         head_dim);
    if (y_raw && (!aligned16(y_raw) || !stride_ok(yraw_batch_stride) || !stride_ok(yraw_token_stride) ||
                  !stride_ok(yraw_head_stride)))
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: y_raw must be 16-byte aligned with strides of 8");
    // the rest of the validation is that of sr_rope3d_apply
    if (n_batch < 0 || n_tokens < 0 || n_heads < 1 || n_batch > 65535)
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: bad sizes (batch %d, tokens %d, heads %d)", n_batch,
                         n_tokens, n_heads);
    if (head_dim != 64 && head_dim != 128)
        return set_error(SR_ERR_UNSUPPORTED, "qknorm_rope3d: head_dim must be 64 or 128");
    if (cfg.d_t < 0 || cfg.d_h < 0 || cfg.d_w < 0 || cfg.d_t % 8 || cfg.d_h % 8 || cfg.d_w % 8 ||
        cfg.d_t + cfg.d_h + cfg.d_w != head_dim)
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: sub-blocks %d/%d/%d must be multiples of 8 summing to %d",
                         cfg.d_t, cfg.d_h, cfg.d_w, head_dim);
    if (!(cfg.base > 0.f)) return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: base must be positive");
    if (n_batch == 0 || n_tokens == 0) return SR_OK;
    if (!x || !y) return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: null tensor");
    if (!aligned16(x) || !aligned16(y))
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: x and y must be 16-byte aligned");
    if (!stride_ok(x_batch_stride) || !stride_ok(x_token_stride) || !stride_ok(x_head_stride) ||
        !stride_ok(y_batch_stride) || !stride_ok(y_token_stride) || !stride_ok(y_head_stride))
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: strides must be multiples of 8 elements");
    if (pos && (reinterpret_cast<uintptr_t>(pos) & 3u))
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: pos must be 4-byte aligned");
    RopeLaunch l{x, y, pos, n_valid_dev, n_batch, n_tokens, n_heads, head_dim, cfg, out_scale,
                 x_batch_stride, x_token_stride, x_head_stride, y_batch_stride, y_token_stride, y_head_stride,
                 pos_batch_stride, static_cast<cudaStream_t>(stream)};
    if (t_origin_dev && (reinterpret_cast<uintptr_t>(t_origin_dev) & 7u))
        return set_error(SR_ERR_INVALID_ARG, "qknorm_rope3d: t_origin must be 8-byte aligned");
    l.t_origin = t_origin_dev;
    l.gamma = gamma;
    l.eps = eps;
    l.y_raw = y_raw;
    l.rb = yraw_batch_stride;
    l.rt = yraw_token_stride;
    l.rh = yraw_head_stride;
    return launch_rope3d(l);
}

// Checks of an optional fused rotation (sr_rope_out) of a call whose K
// output has head_dim elements per row.
static int rope_out_check(const char *name, const sr_rope_out *rot, int32_t head_dim) {
    if (!rot || !rot->k_rot) return SR_OK;
    const sr_rope_cfg &c = rot->cfg;
    if (c.d_t < 0 || c.d_h < 0 || c.d_w < 0 || c.d_t % 8 || c.d_h % 8 || c.d_w % 8 || c.d_t + c.d_h + c.d_w != head_dim)
        return set_error(SR_ERR_INVALID_ARG, "%s: rotation sub-blocks %d/%d/%d must be multiples of 8 summing to %d",
                         name, c.d_t, c.d_h, c.d_w, head_dim);
    if (!(c.base > 0.f)) return set_error(SR_ERR_INVALID_ARG, "%s: rotation base must be positive", name);
    if (!aligned16(rot->k_rot)) return set_error(SR_ERR_INVALID_ARG, "%s: k_rot must be 16-byte aligned", name);
    if (!rot->pos || (reinterpret_cast<uintptr_t>(rot->pos) & 3u))
        return set_error(SR_ERR_INVALID_ARG, "%s: the rotation needs positions (4-byte aligned)", name);
    if (rot->t_origin_dev && (reinterpret_cast<uintptr_t>(rot->t_origin_dev) & 7u))
        return set_error(SR_ERR_INVALID_ARG, "%s: t_origin must be 8-byte aligned", name);
    return SR_OK;
}

static int gather_common(const char *name, void *dst, const void *src, const int32_t *idx, int32_t n_batch,
                         int32_t n_slots, int32_t n_heads, int32_t head_dim, int64_t tok_t, int64_t tok_h,
                         int64_t slot_b, int64_t slot_s, int64_t slot_h, GatherLaunch &l) {
    if (n_batch < 0 || n_slots < 0 || n_heads < 1 || n_batch > 65535)
        return set_error(SR_ERR_INVALID_ARG, "%s: bad sizes", name);
    if (head_dim != 64 && head_dim != 128) return set_error(SR_ERR_UNSUPPORTED, "%s: head_dim must be 64 or 128", name);
    if (n_batch == 0 || n_slots == 0) return -1;   // nothing to do
    if (!dst || !src || !idx) return set_error(SR_ERR_INVALID_ARG, "%s: null pointer", name);
    if (!aligned16(dst) || !aligned16(src)) return set_error(SR_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", name);
    for (int64_t st : {tok_t, tok_h, slot_b, slot_s, slot_h})
        if (!stride_ok(st)) return set_error(SR_ERR_INVALID_ARG, "%s: strides must be multiples of 8", name);
    l.idx = idx;
    l.n_batch = n_batch;
    l.n_slots = n_slots;
    l.n_heads = n_heads;
    l.head_dim = head_dim;
    l.src_t = tok_t;
    l.src_h = tok_h;
    l.dst_b = slot_b;
    l.dst_s = slot_s;
    l.dst_h = slot_h;
    return SR_OK;
}

int sr_gather_tokens(void *dst, const void *src, const int32_t *idx, int32_t n_batch, int32_t n_slots,
                     int32_t n_heads, int32_t head_dim, int64_t src_token_stride, int64_t src_head_stride,
                     int64_t dst_batch_stride, int64_t dst_slot_stride, int64_t dst_head_stride,
                     const float *src_pos, float *dst_pos, int64_t dst_pos_batch_stride, void *stream) {
    g_last_error[0] = 0;
    GatherLaunch l{};
    int rc = gather_common("gather_tokens", dst, src, idx, n_batch, n_slots, n_heads, head_dim, src_token_stride,
                           src_head_stride, dst_batch_stride, dst_slot_stride, dst_head_stride, l);
    if (rc != SR_OK) return rc < 0 ? SR_OK : rc;
    if ((src_pos == nullptr) != (dst_pos == nullptr))
        return set_error(SR_ERR_INVALID_ARG, "gather_tokens: src_pos and dst_pos go together");
    l.dst = dst;
    l.src = src;
    l.src_pos = src_pos;
    l.dst_pos = dst_pos;
    l.pos_b = dst_pos_batch_stride;
    l.scatter = false;
    l.stream = static_cast<cudaStream_t>(stream);
    return launch_gather(l);
}

int sr_scatter_tokens(void *dst, const void *src, const int32_t *idx, int32_t n_batch, int32_t n_slots,
                      int32_t n_heads, int32_t head_dim, int64_t dst_token_stride, int64_t dst_head_stride,
                      int64_t src_batch_stride, int64_t src_slot_stride, int64_t src_head_stride, void *stream) {
    g_last_error[0] = 0;
    GatherLaunch l{};
    int rc = gather_common("scatter_tokens", dst, src, idx, n_batch, n_slots, n_heads, head_dim, dst_token_stride,
                           dst_head_stride, src_batch_stride, src_slot_stride, src_head_stride, l);
    if (rc != SR_OK) return rc < 0 ? SR_OK : rc;
    l.dst = dst;
    l.src = src;
    l.scatter = true;
    l.stream = static_cast<cudaStream_t>(stream);
    return launch_gather(l);
}

int sr_gather_rope3d_tokens(void *dst, const void *src, const int32_t *idx, const float *src_pos, int32_t n_batch,
                            int32_t n_slots, int32_t n_heads, int32_t head_dim, sr_rope_cfg cfg, float out_scale,
                            int64_t src_token_stride, int64_t src_head_stride, int64_t dst_batch_stride,
                            int64_t dst_slot_stride, int64_t dst_head_stride, const double *t_origin_dev,
                            void *stream) {
    g_last_error[0] = 0;
    GatherLaunch l{};
    int rc = gather_common("gather_rope3d_tokens", dst, src, idx, n_batch, n_slots, n_heads, head_dim,
                           src_token_stride, src_head_stride, dst_batch_stride, dst_slot_stride, dst_head_stride, l);
    if (rc != SR_OK) return rc < 0 ? SR_OK : rc;
    if (cfg.d_t < 0 || cfg.d_h < 0 || cfg.d_w < 0 || cfg.d_t % 8 || cfg.d_h % 8 || cfg.d_w % 8 ||
        cfg.d_t + cfg.d_h + cfg.d_w != head_dim)
        return set_error(SR_ERR_INVALID_ARG, "gather_rope3d_tokens: sub-blocks %d/%d/%d must be multiples of 8 "
                         "summing to %d", cfg.d_t, cfg.d_h, cfg.d_w, head_dim);
    if (!(cfg.base > 0.f)) return set_error(SR_ERR_INVALID_ARG, "gather_rope3d_tokens: base must be positive");
    if (!src_pos || (reinterpret_cast<uintptr_t>(src_pos) & 3u))
        return set_error(SR_ERR_INVALID_ARG, "gather_rope3d_tokens: src_pos (4-byte aligned) is required");
    l.dst = dst;
    l.src = src;
    l.src_pos = src_pos;
    l.scatter = false;
    if (t_origin_dev && (reinterpret_cast<uintptr_t>(t_origin_dev) & 7u))
        return set_error(SR_ERR_INVALID_ARG, "gather_rope3d_tokens: t_origin must be 8-byte aligned");
    l.rope = true;
    l.cfg = cfg;
    l.out_scale = out_scale;
    l.t_origin = t_origin_dev;
    l.stream = static_cast<cudaStream_t>(stream);
    return launch_gather(l);
}

int sr_history_compress(const void *k_in, const void *v_in, void *k_out, void *v_out, int32_t n_batch,
                        int32_t n_frames, int32_t n_heads, int32_t head_dim, sr_pool_cfg cfg, int64_t in_batch_stride,
                        int64_t in_frame_stride, int64_t in_token_stride, int64_t in_head_stride,
                        int64_t out_batch_stride, int64_t out_frame_stride, int64_t out_token_stride,
                        int64_t out_head_stride, const float *frame_t, float *pos_out, int64_t pos_batch_stride,
                        int32_t *slot_of_src, const sr_rope_out *rot, void *stream) {
    g_last_error[0] = 0;
    if (n_batch < 0 || n_frames < 0 || n_heads < 1)
        return set_error(SR_ERR_INVALID_ARG, "history_compress: bad sizes");
    if (head_dim != 64 && head_dim != 128)
        return set_error(SR_ERR_UNSUPPORTED, "history_compress: head_dim must be 64 or 128");
    if (cfg.grid_h < 1 || cfg.grid_w < 1 || cfg.pool_h < 1 || cfg.pool_w < 1 || cfg.pool_h > 8 || cfg.pool_w > 8)
        return set_error(SR_ERR_INVALID_ARG, "history_compress: grid >= 1 and 1 <= pool <= 8 required");
    if (n_batch == 0 || n_frames == 0) return SR_OK;
    if ((k_in == nullptr) != (k_out == nullptr) || (v_in == nullptr) != (v_out == nullptr))
        return set_error(SR_ERR_INVALID_ARG, "history_compress: in/out must be both given or both NULL");
    for (const void *p : {k_in, v_in, static_cast<const void *>(k_out), static_cast<const void *>(v_out)})
        if (p && !aligned16(p)) return set_error(SR_ERR_INVALID_ARG, "history_compress: tensors must be 16-byte aligned");
    for (int64_t s : {in_batch_stride, in_frame_stride, in_token_stride, in_head_stride, out_batch_stride,
                      out_frame_stride, out_token_stride, out_head_stride})
        if (!stride_ok(s)) return set_error(SR_ERR_INVALID_ARG, "history_compress: strides must be multiples of 8");
    if (pos_out && !frame_t) return set_error(SR_ERR_INVALID_ARG, "history_compress: pos_out needs frame_t");
    int rc = rope_out_check("history_compress", rot, head_dim);
    if (rc != SR_OK) return rc;
    if (rot && rot->k_rot && !k_in) return set_error(SR_ERR_INVALID_ARG, "history_compress: rotation needs K");
    PoolLaunch l{k_in, v_in, k_out, v_out, n_batch, n_frames, n_heads, head_dim, cfg,
                 in_batch_stride, in_frame_stride, in_token_stride, in_head_stride,
                 out_batch_stride, out_frame_stride, out_token_stride, out_head_stride,
                 frame_t, pos_out, pos_batch_stride, slot_of_src, static_cast<cudaStream_t>(stream)};
    if (rot && rot->k_rot) {
        l.k_rot = rot->k_rot;
        l.rot_pos = rot->pos;
        l.rot_pos_b = rot->pos_batch_stride;
        l.t_origin = rot->t_origin_dev;
        l.rot_cfg = rot->cfg;
        l.rot_scale = rot->out_scale;
    }
    return launch_history_compress(l);
}

int sr_kv_append(void *k_buf, void *v_buf, float *pos_buf, int32_t n_batch, int32_t n_heads, int32_t head_dim,
                 int32_t buf_tokens, int32_t dst_token, const void *k_src, const void *v_src, const float *pos_src,
                 int32_t n_tokens, const int32_t *n_valid_dev, int64_t src_batch_stride, int64_t src_token_stride,
                 int64_t src_head_stride, int64_t pos_src_batch_stride, const sr_rope_out *rot, void *stream) {
    g_last_error[0] = 0;
    if (n_batch < 0 || n_heads < 1 || n_tokens < 0 || buf_tokens < 0 || dst_token < 0)
        return set_error(SR_ERR_INVALID_ARG, "kv_append: bad sizes");
    if (head_dim != 64 && head_dim != 128) return set_error(SR_ERR_UNSUPPORTED, "kv_append: head_dim must be 64 or 128");
    if (static_cast<int64_t>(dst_token) + n_tokens > buf_tokens)
        return set_error(SR_ERR_INVALID_ARG, "kv_append: slots [%d, %d) exceed the buffer (%d tokens)", dst_token,
                         dst_token + n_tokens, buf_tokens);
    if (n_batch == 0 || n_tokens == 0) return SR_OK;
    const bool rotate = rot && rot->k_rot;
    if ((k_src && !k_buf && !rotate) || (v_src && !v_buf) || (pos_src && !pos_buf))
        return set_error(SR_ERR_INVALID_ARG, "kv_append: source given without its buffer");
    int rc = rope_out_check("kv_append", rot, head_dim);
    if (rc != SR_OK) return rc;
    if (rotate && !k_src) return set_error(SR_ERR_INVALID_ARG, "kv_append: rotation needs k_src");
    for (const void *p : {static_cast<const void *>(k_buf), static_cast<const void *>(v_buf), k_src, v_src})
        if (p && !aligned16(p)) return set_error(SR_ERR_INVALID_ARG, "kv_append: tensors must be 16-byte aligned");
    if (!stride_ok(src_batch_stride) || !stride_ok(src_token_stride) || !stride_ok(src_head_stride))
        return set_error(SR_ERR_INVALID_ARG, "kv_append: strides must be multiples of 8");
    AppendLaunch l{k_buf, v_buf, pos_buf, n_batch, n_heads, head_dim, buf_tokens, dst_token, k_src, v_src, pos_src,
                   n_tokens, n_valid_dev, src_batch_stride, src_token_stride, src_head_stride, pos_src_batch_stride,
                   static_cast<cudaStream_t>(stream)};
    if (rotate) {
        if (n_batch > 65535) return set_error(SR_ERR_INVALID_ARG, "kv_append: too many sessions");
        l.k_rot = rot->k_rot;
        l.rot_pos = rot->pos;
        l.rot_pos_b = rot->pos_batch_stride;
        l.t_origin = rot->t_origin_dev;
        l.rot_cfg = rot->cfg;
        l.rot_scale = rot->out_scale;
    }
    return launch_kv_append(l);
}

int sr_stream_clock_advance(double *clock_dev, double frames, void *stream) {
    g_last_error[0] = 0;
    if (!clock_dev || (reinterpret_cast<uintptr_t>(clock_dev) & 7u))
        return set_error(SR_ERR_INVALID_ARG, "stream_clock_advance: clock must be an 8-byte aligned device double");
    return launch_clock_advance(clock_dev, frames, static_cast<cudaStream_t>(stream));
}

size_t sr_chunk_attention_workspace_bytes(int32_t n_batch, int32_t n_heads, int32_t head_dim, int32_t q_cap) {
    if (n_batch < 1 || n_heads < 1 || q_cap < 1 || (head_dim != 64 && head_dim != 128)) return 0;
    return attention_schedule(n_batch, n_heads, head_dim, q_cap, attention_sm_count()).workspace_bytes;
}

int sr_chunk_attention_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                           const sr_kv_layout *layout, const int32_t *kv_len_dev, const int32_t *q_len_dev,
                           int32_t n_batch, int32_t n_heads, int32_t head_dim, int32_t q_cap, float softmax_scale,
                           void *workspace, size_t workspace_bytes, int32_t *status_dev, void *stream) {
    g_last_error[0] = 0;
    if (!layout) return set_error(SR_ERR_INVALID_ARG, "chunk_attention: layout is NULL");
    if (head_dim != 64 && head_dim != 128)
        return set_error(SR_ERR_UNSUPPORTED, "chunk_attention: head_dim must be 64 or 128");
    if (n_batch < 0 || n_batch > 65535 || n_heads < 1 || n_heads > 65535 || q_cap < 1)
        return set_error(SR_ERR_INVALID_ARG, "chunk_attention: bad sizes (batch %d, heads %d, q_cap %d)", n_batch,
                         n_heads, q_cap);
    if (layout->n_seg < 1 || layout->n_seg > SR_MAX_SEG)
        return set_error(SR_ERR_INVALID_ARG, "chunk_attention: n_seg must be in [1, %d]", SR_MAX_SEG);
    int64_t kv_tokens = 0;
    for (int s = 0; s < layout->n_seg; ++s) {
        if (layout->cap[s] < SR_TILE || layout->cap[s] % SR_TILE)
            return set_error(SR_ERR_INVALID_ARG, "chunk_attention: cap[%d] = %d is not a positive multiple of %d", s,
                             layout->cap[s], SR_TILE);
        kv_tokens += layout->cap[s];
    }
    if (kv_tokens > (int64_t(1) << 31) - 1) return set_error(SR_ERR_INVALID_ARG, "chunk_attention: buffer too long");
    if (!(softmax_scale > 0.f)) return set_error(SR_ERR_INVALID_ARG, "chunk_attention: softmax_scale must be > 0");
    if (n_batch == 0) return SR_OK;
    if (!q || !k || !v || !o || !kv_len_dev || !q_len_dev)
        return set_error(SR_ERR_INVALID_ARG, "chunk_attention: null tensor");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return set_error(SR_ERR_INVALID_ARG, "chunk_attention: q, k, v, o must be 16-byte aligned");
    AttnLaunch a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.lse = lse;
    a.kv_len = kv_len_dev;
    a.q_len = q_len_dev;
    a.status = status_dev;
    for (int s = 0; s < SR_MAX_SEG; ++s) a.cap[s] = s < layout->n_seg ? layout->cap[s] : 0;
    a.n_seg = layout->n_seg;
    a.n_batch = n_batch;
    a.n_heads = n_heads;
    a.head_dim = head_dim;
    a.q_cap = q_cap;
    a.kv_tokens = kv_tokens;
    a.softmax_scale = softmax_scale;
    if (workspace && !aligned16(workspace))
        return set_error(SR_ERR_INVALID_ARG, "chunk_attention: workspace must be 16-byte aligned");
    a.workspace = workspace;
    a.workspace_bytes = workspace ? workspace_bytes : 0;
    a.stream = static_cast<cudaStream_t>(stream);
    a.wait_limit_ns = attention_wait_limit_ns();
    a.withheld_tile = attention_withheld_tile();
    return launch_chunk_attention(a);
}

}  // extern "C"
