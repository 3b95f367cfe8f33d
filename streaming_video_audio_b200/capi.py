"""ctypes binding of libsr.so (include/sr.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of the method itself: it checks dtypes/devices, reads pointers
and strides off torch tensors and passes the caller's current CUDA stream.
All work runs in the library's kernels.  If libsr.so is missing, importing
the library raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsr.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sr.h")

SR_OK, SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_CUDA, SR_ERR_DEVICE_TIMEOUT = 0, 1, 2, 3, 4
SR_MAX_SEG = 8
SR_TILE = 128

_lock = threading.Lock()
_lib = None


class SrError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


class sr_rope_cfg(ctypes.Structure):
    _fields_ = [("base", ctypes.c_float), ("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32),
                ("d_w", ctypes.c_int32)]


class sr_pool_cfg(ctypes.Structure):
    _fields_ = [("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32), ("pool_h", ctypes.c_int32),
                ("pool_w", ctypes.c_int32)]


class sr_kv_layout(ctypes.Structure):
    _fields_ = [("n_seg", ctypes.c_int32), ("cap", ctypes.c_int32 * SR_MAX_SEG)]


class sr_rope_out(ctypes.Structure):
    _fields_ = [("k_rot", ctypes.c_void_p), ("pos", ctypes.c_void_p), ("pos_batch_stride", ctypes.c_int64),
                ("t_origin_dev", ctypes.c_void_p), ("cfg", sr_rope_cfg), ("out_scale", ctypes.c_float)]


class RopeOut:
    """A fused rotation of the K a call writes (sr_rope_out): k_rot is the
    destination (the layout of the call's K output), pos the fp32 (t, h, w)
    of every token ([B, N, 3], token stride 3), t_origin an optional CUDA
    float64 tensor whose first element is added to every t."""

    def __init__(self, k_rot: torch.Tensor, pos: torch.Tensor, split: Sequence[int], base: float = 10000.0,
                 t_origin: Optional[torch.Tensor] = None, out_scale: float = 1.0):
        self.k_rot, self.pos, self.split, self.base = k_rot, pos, split, base
        self.t_origin, self.out_scale = t_origin, out_scale

    def struct(self, n_tokens: int):
        _cuda(self.k_rot, torch.bfloat16, "k_rot")
        _cuda(self.pos, torch.float32, "rot.pos")
        _cuda(self.t_origin, torch.float64, "t_origin")
        B = self.pos.shape[0]
        if tuple(self.pos.shape) != (B, n_tokens, 3) or self.pos.stride(1) != 3 or self.pos.stride(2) != 1:
            raise ValueError(f"rotation positions must be [B, {n_tokens}, 3] with token stride 3")
        cfg = sr_rope_cfg(float(self.base), int(self.split[0]), int(self.split[1]), int(self.split[2]))
        return sr_rope_out(_ptr(self.k_rot), _ptr(self.pos), self.pos.stride(0), _ptr(self.t_origin), cfg,
                           float(self.out_scale))


_vp, _i32, _i64, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float

_SIGS = {
    "sr_version": ([], ctypes.c_int),
    "sr_get_last_error": ([], ctypes.c_char_p),
    "sr_rope3d_apply": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, sr_rope_cfg, _f32,
                         _i64, _i64, _i64, _i64, _i64, _i64, _i64, _vp, _vp], ctypes.c_int),
    "sr_qknorm_rope3d_apply": ([_vp, _vp, _vp, _vp, _f32, _vp, _i32, _i32, _i32, _i32, _vp, sr_rope_cfg, _f32,
                                _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _vp, _vp],
                               ctypes.c_int),
    "sr_gather_tokens": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _i64, _i64, _vp, _vp, _i64, _vp],
                         ctypes.c_int),
    "sr_scatter_tokens": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i64, _i64, _i64, _i64, _vp], ctypes.c_int),
    "sr_gather_rope3d_tokens": ([_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, sr_rope_cfg, _f32,
                                 _i64, _i64, _i64, _i64, _i64, _vp, _vp], ctypes.c_int),
    "sr_history_compress": ([_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, sr_pool_cfg,
                             _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _vp, _vp, _i64, _vp,
                             ctypes.POINTER(sr_rope_out), _vp], ctypes.c_int),
    "sr_kv_append": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp,
                      _i64, _i64, _i64, _i64, ctypes.POINTER(sr_rope_out), _vp], ctypes.c_int),
    "sr_stream_clock_advance": ([_vp, ctypes.c_double, _vp], ctypes.c_int),
    "sr_chunk_attention_fwd": ([_vp, _vp, _vp, _vp, _vp, ctypes.POINTER(sr_kv_layout), _vp, _vp, _i32, _i32,
                                _i32, _i32, _f32, _vp, ctypes.c_size_t, _vp, _vp], ctypes.c_int),
    "sr_chunk_attention_workspace_bytes": ([_i32, _i32, _i32, _i32], ctypes.c_size_t),
    "sr_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_int),
    "sr_set_withheld_kv_tile": ([_i32], ctypes.c_int),
}


def load():
    """Load libsr.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libsr.so not found at {LIB_PATH}; build it with "
                                   "`python -m streaming_video_audio_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGS.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def declared_functions():
    """Names of the functions include/sr.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(sr_\w+)\s*\(", src, flags=re.M)))


def _check(fn: str, rc: int):
    if rc != SR_OK:
        raise SrError(fn, rc, load().sr_get_last_error().decode(errors="replace"))


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _cuda(t: Optional[torch.Tensor], dtype, name: str):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def sr_version() -> int:
    return int(load().sr_version())


def sr_rope3d_apply(x: torch.Tensor, y: torch.Tensor, pos: Optional[torch.Tensor], split: Sequence[int],
                    base: float = 10000.0, out_scale: float = 1.0, n_valid: Optional[torch.Tensor] = None,
                    t_origin: Optional[torch.Tensor] = None, stream=None) -> None:
    """x, y: [B, N, H, D] bf16 views (any strides, D contiguous); pos: [B, N, 3]
    fp32 with token stride 3 (or None); n_valid: int32 [B] or None; t_origin:
    CUDA float64 tensor whose first element is added to every t (or None)."""
    _cuda(t_origin, torch.float64, "t_origin")
    _cuda(x, torch.bfloat16, "x")
    _cuda(y, torch.bfloat16, "y")
    _cuda(pos, torch.float32, "pos")
    _cuda(n_valid, torch.int32, "n_valid")
    B, N, H, D = x.shape
    if tuple(y.shape) != (B, N, H, D) or x.stride(3) != 1 or y.stride(3) != 1:
        raise ValueError("x and y must be [B, N, H, D] with contiguous D")
    pb = 0
    if pos is not None:
        if tuple(pos.shape) != (B, N, 3) or pos.stride(1) != 3 or pos.stride(2) != 1:
            raise ValueError("pos must be [B, N, 3] with token stride 3")
        pb = pos.stride(0)
    cfg = sr_rope_cfg(float(base), int(split[0]), int(split[1]), int(split[2]))
    _check("sr_rope3d_apply", load().sr_rope3d_apply(
        _ptr(x), _ptr(y), _ptr(pos), B, N, H, D, _ptr(n_valid), cfg, float(out_scale),
        x.stride(0), x.stride(1), x.stride(2), y.stride(0), y.stride(1), y.stride(2), pb, _ptr(t_origin),
        _stream(stream)))


def sr_qknorm_rope3d_apply(x: torch.Tensor, y: torch.Tensor, gamma: torch.Tensor, eps: float,
                           pos: Optional[torch.Tensor], split: Sequence[int], base: float = 10000.0,
                           out_scale: float = 1.0, n_valid: Optional[torch.Tensor] = None,
                           y_raw: Optional[torch.Tensor] = None, t_origin: Optional[torch.Tensor] = None,
                           stream=None) -> None:
    """Per-head RMSNorm (gain gamma: fp32 [D], contiguous) then RoPE.  x, y,
    y_raw: [B, N, H, D] bf16 views (D contiguous); pos and t_origin as in
    sr_rope3d_apply."""
    _cuda(t_origin, torch.float64, "t_origin")
    _cuda(x, torch.bfloat16, "x")
    _cuda(y, torch.bfloat16, "y")
    _cuda(y_raw, torch.bfloat16, "y_raw")
    _cuda(gamma, torch.float32, "gamma")
    _cuda(pos, torch.float32, "pos")
    _cuda(n_valid, torch.int32, "n_valid")
    B, N, H, D = x.shape
    if tuple(y.shape) != (B, N, H, D) or x.stride(3) != 1 or y.stride(3) != 1:
        raise ValueError("x and y must be [B, N, H, D] with contiguous D")
    if y_raw is not None and (tuple(y_raw.shape) != (B, N, H, D) or y_raw.stride(3) != 1):
        raise ValueError("y_raw must be [B, N, H, D] with contiguous D")
    if gamma.numel() != D or not gamma.is_contiguous():
        raise ValueError("gamma must be contiguous fp32 [D]")
    pb = 0
    if pos is not None:
        if tuple(pos.shape) != (B, N, 3) or pos.stride(1) != 3 or pos.stride(2) != 1:
            raise ValueError("pos must be [B, N, 3] with token stride 3")
        pb = pos.stride(0)
    rs = y_raw.stride() if y_raw is not None else (0, 0, 0)
    cfg = sr_rope_cfg(float(base), int(split[0]), int(split[1]), int(split[2]))
    _check("sr_qknorm_rope3d_apply", load().sr_qknorm_rope3d_apply(
        _ptr(x), _ptr(y), _ptr(y_raw), _ptr(gamma), float(eps), _ptr(pos), B, N, H, D, _ptr(n_valid), cfg,
        float(out_scale), x.stride(0), x.stride(1), x.stride(2), y.stride(0), y.stride(1), y.stride(2),
        rs[0], rs[1], rs[2], pb, _ptr(t_origin), _stream(stream)))


def sr_gather_tokens(dst: torch.Tensor, src: torch.Tensor, idx: torch.Tensor, src_pos: Optional[torch.Tensor] = None,
                     dst_pos: Optional[torch.Tensor] = None, stream=None) -> None:
    """dst [B, S, H, D] view (D contiguous) <- rows of src [T, H, D] (view, D
    contiguous) picked by idx int32 [B, S] (contiguous; < 0 -> zeros);
    optional positions src_pos [T, 3] -> dst_pos [B, S, 3] (token stride 3)."""
    for t, n in ((dst, "dst"), (src, "src")):
        _cuda(t, torch.bfloat16, n)
    _cuda(idx, torch.int32, "idx")
    B, S, H, D = dst.shape
    if src.dim() != 3 or src.shape[1:] != (H, D) or src.stride(2) != 1 or dst.stride(3) != 1:
        raise ValueError("src must be [T, H, D] and dst [B, S, H, D] with contiguous D")
    if tuple(idx.shape) != (B, S) or not idx.is_contiguous():
        raise ValueError("idx must be contiguous int32 [B, S]")
    pb = 0
    if dst_pos is not None:
        _cuda(dst_pos, torch.float32, "dst_pos")
        _cuda(src_pos, torch.float32, "src_pos")
        if tuple(dst_pos.shape) != (B, S, 3) or dst_pos.stride(1) != 3 or not src_pos.is_contiguous():
            raise ValueError("dst_pos must be [B, S, 3] (token stride 3), src_pos contiguous [T, 3]")
        pb = dst_pos.stride(0)
    _check("sr_gather_tokens", load().sr_gather_tokens(
        _ptr(dst), _ptr(src), _ptr(idx), B, S, H, D, src.stride(0), src.stride(1), dst.stride(0), dst.stride(1),
        dst.stride(2), _ptr(src_pos), _ptr(dst_pos), pb, _stream(stream)))


def sr_gather_rope3d_tokens(dst: torch.Tensor, src: torch.Tensor, idx: torch.Tensor, src_pos: torch.Tensor,
                            split: Sequence[int], base: float = 10000.0, out_scale: float = 1.0,
                            t_origin: Optional[torch.Tensor] = None, stream=None) -> None:
    """As sr_gather_tokens, every copied row rotated by the 3-D RoPE of its
    source token's position src_pos [T, 3] (fp32, contiguous), plus the first
    element of t_origin (CUDA float64, optional) on t."""
    _cuda(t_origin, torch.float64, "t_origin")
    for t, n in ((dst, "dst"), (src, "src")):
        _cuda(t, torch.bfloat16, n)
    _cuda(idx, torch.int32, "idx")
    _cuda(src_pos, torch.float32, "src_pos")
    B, S, H, D = dst.shape
    if src.dim() != 3 or src.shape[1:] != (H, D) or src.stride(2) != 1 or dst.stride(3) != 1:
        raise ValueError("src must be [T, H, D] and dst [B, S, H, D] with contiguous D")
    if tuple(idx.shape) != (B, S) or not idx.is_contiguous():
        raise ValueError("idx must be contiguous int32 [B, S]")
    if src_pos is None or src_pos.shape != (src.shape[0], 3) or not src_pos.is_contiguous():
        raise ValueError("src_pos must be contiguous fp32 [T, 3]")
    cfg = sr_rope_cfg(float(base), int(split[0]), int(split[1]), int(split[2]))
    _check("sr_gather_rope3d_tokens", load().sr_gather_rope3d_tokens(
        _ptr(dst), _ptr(src), _ptr(idx), _ptr(src_pos), B, S, H, D, cfg, float(out_scale), src.stride(0),
        src.stride(1), dst.stride(0), dst.stride(1), dst.stride(2), _ptr(t_origin), _stream(stream)))


def sr_scatter_tokens(dst: torch.Tensor, src: torch.Tensor, idx: torch.Tensor, stream=None) -> None:
    """Rows of src [B, S, H, D] (view, D contiguous) to dst [T, H, D] at
    idx [B, S] (int32, contiguous; < 0 skipped; indices must not repeat)."""
    for t, n in ((dst, "dst"), (src, "src")):
        _cuda(t, torch.bfloat16, n)
    _cuda(idx, torch.int32, "idx")
    B, S, H, D = src.shape
    if dst.dim() != 3 or dst.shape[1:] != (H, D) or dst.stride(2) != 1 or src.stride(3) != 1:
        raise ValueError("dst must be [T, H, D] and src [B, S, H, D] with contiguous D")
    if tuple(idx.shape) != (B, S) or not idx.is_contiguous():
        raise ValueError("idx must be contiguous int32 [B, S]")
    _check("sr_scatter_tokens", load().sr_scatter_tokens(
        _ptr(dst), _ptr(src), _ptr(idx), B, S, H, D, dst.stride(0), dst.stride(1), src.stride(0), src.stride(1),
        src.stride(2), _stream(stream)))


def sr_history_compress(k_in: Optional[torch.Tensor], v_in: Optional[torch.Tensor],
                        k_out: Optional[torch.Tensor], v_out: Optional[torch.Tensor],
                        grid_hw: Sequence[int], pool_hw: Sequence[int],
                        frame_t: Optional[torch.Tensor] = None, pos_out: Optional[torch.Tensor] = None,
                        slot_of_src: Optional[torch.Tensor] = None, rot: Optional[RopeOut] = None,
                        stream=None) -> None:
    """k_in, v_in: [B, F, Gh*Gw, H, D] bf16 views; k_out, v_out: [B, F, cells, H, D]
    views (D contiguous; K and V views share strides); frame_t: fp32 [B, F]
    contiguous; pos_out: [B, F*cells, 3] fp32 (token stride 3); slot_of_src:
    int32 [F*Gh*Gw]; rot: fused rotation of the pooled K (rot.k_rot with
    k_out's strides, rot.pos [B, F*cells, 3])."""
    ref_in = k_in if k_in is not None else v_in
    ref_out = k_out if k_out is not None else v_out
    for t, n in ((k_in, "k_in"), (v_in, "v_in"), (k_out, "k_out"), (v_out, "v_out")):
        _cuda(t, torch.bfloat16, n)
    _cuda(frame_t, torch.float32, "frame_t")
    _cuda(pos_out, torch.float32, "pos_out")
    _cuda(slot_of_src, torch.int32, "slot_of_src")
    if ref_in is None or ref_out is None:
        raise ValueError("need at least one of K or V")
    if k_in is not None and v_in is not None and (k_in.stride() != v_in.stride() or k_out.stride() != v_out.stride()):
        raise ValueError("K and V views must share strides")
    B, F, T, H, D = ref_in.shape
    gh, gw = grid_hw
    ph, pw = pool_hw
    cells = (-(-gh // ph)) * (-(-gw // pw))
    if T != gh * gw or tuple(ref_out.shape) != (B, F, cells, H, D) or ref_in.stride(4) != 1 or ref_out.stride(4) != 1:
        raise ValueError("bad history_compress shapes")
    pb = 0
    if pos_out is not None:
        if frame_t is None or tuple(frame_t.shape) != (B, F) or not frame_t.is_contiguous():
            raise ValueError("pos_out needs frame_t [B, F] contiguous")
        if tuple(pos_out.shape) != (B, F * cells, 3) or pos_out.stride(1) != 3 or pos_out.stride(2) != 1:
            raise ValueError("pos_out must be [B, F*cells, 3] with token stride 3")
        pb = pos_out.stride(0)
    if slot_of_src is not None and (slot_of_src.numel() != F * gh * gw or not slot_of_src.is_contiguous()):
        raise ValueError("slot_of_src must be int32 [F*Gh*Gw] contiguous")
    cfg = sr_pool_cfg(int(gh), int(gw), int(ph), int(pw))
    si, so = ref_in.stride(), ref_out.stride()
    ro = None
    if rot is not None:
        if k_out is None or tuple(rot.k_rot.shape) != tuple(k_out.shape) or rot.k_rot.stride() != k_out.stride():
            raise ValueError("rot.k_rot must have k_out's shape and strides")
        ro = ctypes.byref(rot.struct(F * cells))
    _check("sr_history_compress", load().sr_history_compress(
        _ptr(k_in), _ptr(v_in), _ptr(k_out), _ptr(v_out), B, F, H, D, cfg,
        si[0], si[1], si[2], si[3], so[0], so[1], so[2], so[3],
        _ptr(frame_t), _ptr(pos_out), pb, _ptr(slot_of_src), ro, _stream(stream)))


def sr_kv_append(k_buf: Optional[torch.Tensor], v_buf: Optional[torch.Tensor], pos_buf: Optional[torch.Tensor],
                 dst_token: int, k_src: Optional[torch.Tensor], v_src: Optional[torch.Tensor],
                 pos_src: Optional[torch.Tensor], n_valid: Optional[torch.Tensor] = None,
                 rot: Optional[RopeOut] = None, stream=None) -> None:
    """k_buf, v_buf: [B, H, Cap, D] contiguous bf16; pos_buf: [B, Cap, 3] fp32
    contiguous; k_src, v_src: [B, N, H, D] views (D contiguous, same strides);
    pos_src: [B, N, 3] (token stride 3); rot: K rotated on its way into
    rot.k_rot ([B, H, Cap, D] contiguous) at rot.pos [B, N, 3]; with rot,
    k_buf may be None."""
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf"), (k_src, "k_src"), (v_src, "v_src")):
        _cuda(t, torch.bfloat16, n)
    _cuda(pos_buf, torch.float32, "pos_buf")
    _cuda(pos_src, torch.float32, "pos_src")
    _cuda(n_valid, torch.int32, "n_valid")
    buf = k_buf if k_buf is not None else (v_buf if v_buf is not None else (rot.k_rot if rot is not None else None))
    src = k_src if k_src is not None else v_src
    if buf is None:
        raise ValueError("need a K or V buffer")
    B, H, cap, D = buf.shape
    for t in (k_buf, v_buf, rot.k_rot if rot is not None else None):
        if t is not None and (tuple(t.shape) != (B, H, cap, D) or not t.is_contiguous()):
            raise ValueError("k_buf / v_buf / rot.k_rot must be contiguous [B, H, Cap, D]")
    if pos_buf is not None and (tuple(pos_buf.shape) != (B, cap, 3) or not pos_buf.is_contiguous()):
        raise ValueError("pos_buf must be contiguous [B, Cap, 3]")
    if src is not None:
        N = src.shape[1]
        if tuple(src.shape) != (B, N, H, D) or src.stride(3) != 1:
            raise ValueError("sources must be [B, N, H, D] with contiguous D")
        if k_src is not None and v_src is not None and k_src.stride() != v_src.stride():
            raise ValueError("K and V sources must share strides")
        ss = src.stride()
    else:
        N = pos_src.shape[1]
        ss = (0, 0, 0)
    psb = 0
    if pos_src is not None:
        if tuple(pos_src.shape) != (B, N, 3) or pos_src.stride(1) != 3 or pos_src.stride(2) != 1:
            raise ValueError("pos_src must be [B, N, 3] with token stride 3")
        psb = pos_src.stride(0)
    ro = ctypes.byref(rot.struct(N)) if rot is not None else None
    _check("sr_kv_append", load().sr_kv_append(
        _ptr(k_buf), _ptr(v_buf), _ptr(pos_buf), B, H, D, cap, int(dst_token), _ptr(k_src), _ptr(v_src),
        _ptr(pos_src), N, _ptr(n_valid), ss[0], ss[1], ss[2], psb, ro, _stream(stream)))


def sr_stream_clock_advance(clock: torch.Tensor, frames: float, stream=None) -> None:
    """clock: CUDA float64 tensor; its first element += frames, on the stream."""
    _cuda(clock, torch.float64, "clock")
    _check("sr_stream_clock_advance", load().sr_stream_clock_advance(_ptr(clock), float(frames), _stream(stream)))


def make_layout(caps: Sequence[int]) -> sr_kv_layout:
    if not 1 <= len(caps) <= SR_MAX_SEG:
        raise ValueError("1..8 segments")
    lay = sr_kv_layout()
    lay.n_seg = len(caps)
    for i, c in enumerate(caps):
        lay.cap[i] = int(c)
    return lay


def sr_set_wait_limit_ns(limit_ns: int) -> None:
    """Bound of every pipeline wait in the attention kernels (0: the 1 s default)."""
    _check("sr_set_wait_limit_ns", load().sr_set_wait_limit_ns(int(limit_ns)))


def sr_set_withheld_kv_tile(tile: int) -> None:
    """Test hook of the bounded-wait failure path: withhold the load of one K
    tile in later attention launches (-1: off)."""
    _check("sr_set_withheld_kv_tile", load().sr_set_withheld_kv_tile(int(tile)))


def sr_chunk_attention_workspace_bytes(n_batch: int, n_heads: int, head_dim: int, q_cap: int) -> int:
    return int(load().sr_chunk_attention_workspace_bytes(n_batch, n_heads, head_dim, q_cap))


def sr_chunk_attention_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                           lse: Optional[torch.Tensor], caps: Sequence[int], kv_len: torch.Tensor,
                           q_len: torch.Tensor, softmax_scale: float, status: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """q [B, H, q_cap, D], k, v [B, H, sum(caps), D], o [B, q_cap, H, D] (bf16,
    contiguous); lse fp32 [B, H, q_cap] or None; kv_len int32 [B, n_seg];
    q_len int32 [B]; status int32 [>=1] or None; workspace: a contiguous
    device byte tensor of at least sr_chunk_attention_workspace_bytes(...)
    bytes, or None (no KV split of the last partial wave)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _cuda(t, torch.bfloat16, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _cuda(lse, torch.float32, "lse")
    _cuda(kv_len, torch.int32, "kv_len")
    _cuda(q_len, torch.int32, "q_len")
    _cuda(status, torch.int32, "status")
    B, H, q_cap, D = q.shape
    kv_tokens = int(sum(caps))
    if tuple(k.shape) != (B, H, kv_tokens, D) or tuple(v.shape) != (B, H, kv_tokens, D):
        raise ValueError("k and v must be [B, H, sum(caps), D]")
    if tuple(o.shape) != (B, q_cap, H, D):
        raise ValueError("o must be [B, q_cap, H, D]")
    if lse is not None and (tuple(lse.shape) != (B, H, q_cap) or not lse.is_contiguous()):
        raise ValueError("lse must be contiguous [B, H, q_cap]")
    if tuple(kv_len.shape) != (B, len(caps)) or not kv_len.is_contiguous():
        raise ValueError("kv_len must be contiguous int32 [B, n_seg]")
    if tuple(q_len.shape) != (B,) or not q_len.is_contiguous():
        raise ValueError("q_len must be contiguous int32 [B]")
    ws_bytes = 0
    if workspace is not None:
        if not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        ws_bytes = workspace.numel() * workspace.element_size()
    lay = make_layout(caps)
    _check("sr_chunk_attention_fwd", load().sr_chunk_attention_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(lay), _ptr(kv_len), _ptr(q_len),
        B, H, D, q_cap, float(softmax_scale), _ptr(workspace), ws_bytes, _ptr(status), _stream(stream)))


SR_NOALLOC_SCRATCH_BYTES = 24 * 1024 * 1024


def sr_chunk_attention_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                                   lse: Optional[torch.Tensor], caps: Sequence[int], kv_len: torch.Tensor,
                                   q_len: torch.Tensor, softmax_scale: float, status: Optional[torch.Tensor] = None,
                                   stream=None) -> None:
    """The attention for callers that cannot allocate device memory while they
    run it (a plugin handed only its inputs and outputs, a real-time loop that
    must not call cudaMalloc, an application whose memory belongs to its own
    allocator): same arguments and results as sr_chunk_attention_fwd, with the
    split-KV scratch taken from the library's static 24 MiB device array.  The
    first call on a device resolves that array's address, so make it before
    any stream capture; calls that may overlap on one device must be ordered,
    since they share the array."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _cuda(t, torch.bfloat16, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _cuda(lse, torch.float32, "lse")
    _cuda(kv_len, torch.int32, "kv_len")
    _cuda(q_len, torch.int32, "q_len")
    _cuda(status, torch.int32, "status")
    B, H, q_cap, D = q.shape
    kv_tokens = int(sum(caps))
    if tuple(k.shape) != (B, H, kv_tokens, D) or tuple(v.shape) != (B, H, kv_tokens, D):
        raise ValueError("k and v must be [B, H, sum(caps), D]")
    if tuple(o.shape) != (B, q_cap, H, D):
        raise ValueError("o must be [B, q_cap, H, D]")
    if lse is not None and (tuple(lse.shape) != (B, H, q_cap) or not lse.is_contiguous()):
        raise ValueError("lse must be contiguous [B, H, q_cap]")
    if tuple(kv_len.shape) != (B, len(caps)) or not kv_len.is_contiguous():
        raise ValueError("kv_len must be contiguous int32 [B, n_seg]")
    if tuple(q_len.shape) != (B,) or not q_len.is_contiguous():
        raise ValueError("q_len must be contiguous int32 [B]")
    lib = load()
    fn = lib.sr_chunk_attention_fwd_noalloc
    fn.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.POINTER(sr_kv_layout), _vp, _vp, _i32, _i32, _i32, _i32, _f32,
                   _vp, _vp]
    fn.restype = ctypes.c_int
    lay = make_layout(caps)
    _check("sr_chunk_attention_fwd_noalloc", fn(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(lay), _ptr(kv_len), _ptr(q_len),
        B, H, D, q_cap, float(softmax_scale), _ptr(status), _stream(stream)))
