"""CPU checks of the C-ABI boundary: the library loads without a GPU, exports
every function include/sr.h declares, and rejects bad arguments on the host
before launching anything (no compute calls are made here)."""
import ctypes

import pytest

from streaming_video_audio_b200 import capi

EXPECTED = {"sr_version", "sr_get_last_error", "sr_rope3d_apply", "sr_history_compress", "sr_kv_append",
            "sr_chunk_attention_fwd", "sr_chunk_attention_workspace_bytes", "sr_qknorm_rope3d_apply",
            "sr_gather_tokens", "sr_gather_rope3d_tokens", "sr_scatter_tokens", "sr_chunk_attention_fwd_noalloc",
            "sr_set_wait_limit_ns", "sr_set_withheld_kv_tile", "sr_stream_clock_advance"}


def test_header_declares_the_boundary():
    assert EXPECTED <= set(capi.declared_functions())


def test_library_exports_every_declared_symbol():
    lib = capi.load()
    for name in capi.declared_functions():
        assert hasattr(lib, name), name
    assert capi.sr_version() == 1


def _err(lib):
    return lib.sr_get_last_error().decode()


def test_attention_rejects_bad_arguments_on_host():
    lib = capi.load()
    lay = capi.make_layout([128, 256])
    args = lambda **kw: dict(dict(q=None, k=None, v=None, o=None, lse=None, lay=ctypes.byref(lay), kl=None, ql=None,
                                  B=1, H=1, D=128, qcap=100, scale=0.1), **kw)

    def call(a):
        return lib.sr_chunk_attention_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["lay"], a["kl"], a["ql"],
                                          a["B"], a["H"], a["D"], a["qcap"], a["scale"], None, 0, None, None)

    assert call(args(D=96)) == capi.SR_ERR_UNSUPPORTED and "head_dim" in _err(lib)
    assert call(args(qcap=0)) == capi.SR_ERR_INVALID_ARG
    assert call(args(scale=0.0)) == capi.SR_ERR_INVALID_ARG
    assert call(args()) == capi.SR_ERR_INVALID_ARG and "null" in _err(lib)
    bad = capi.make_layout([100])
    assert call(args(lay=ctypes.byref(bad))) == capi.SR_ERR_INVALID_ARG and "multiple" in _err(lib)
    assert call(args(B=0)) == capi.SR_OK                       # zero work: nothing launched
    for n_seg in (0, capi.SR_MAX_SEG + 1):                       # segment count outside [1, SR_MAX_SEG]
        lay_bad = capi.make_layout([128])
        lay_bad.n_seg = n_seg
        assert call(args(lay=ctypes.byref(lay_bad))) == capi.SR_ERR_INVALID_ARG and "n_seg" in _err(lib)
    assert call(args(q=16, k=32, v=48, o=72, kl=1, ql=1)) == capi.SR_ERR_INVALID_ARG   # misaligned o
    assert "aligned" in _err(lib)


def test_rope_rejects_bad_arguments_on_host():
    lib = capi.load()
    cfg = capi.sr_rope_cfg(10000.0, 32, 48, 48)
    call = lambda D=128, c=cfg, x=16, y=32, xs=(0, 5120, 128), t0=None: lib.sr_rope3d_apply(
        x, y, None, 1, 4, 40, D, None, c, 1.0, xs[0], xs[1], xs[2], 0, 5120, 128, 0, t0, None)
    assert call(D=64) == capi.SR_ERR_INVALID_ARG                          # split does not sum to D
    assert call(c=capi.sr_rope_cfg(10000.0, 30, 50, 48)) == capi.SR_ERR_INVALID_ARG
    assert call(x=8) == capi.SR_ERR_INVALID_ARG                           # misaligned
    assert call(xs=(0, 5120, 100)) == capi.SR_ERR_INVALID_ARG             # stride not a multiple of 8
    assert call(t0=20) == capi.SR_ERR_INVALID_ARG and "t_origin" in _err(lib)   # clock not 8-byte aligned
    assert lib.sr_rope3d_apply(16, 32, None, 1, 0, 40, 128, None, cfg, 1.0, 0, 0, 0, 0, 0, 0, 0, None,
                               None) == capi.SR_OK


def test_append_and_pool_reject_bad_arguments_on_host():
    lib = capi.load()
    rc = lib.sr_kv_append(16, 32, None, 1, 2, 128, 256, 200, 48, 64, None, 100, None, 0, 256, 128, 0, None, None)
    assert rc == capi.SR_ERR_INVALID_ARG and "exceed" in _err(lib)
    # a fused rotation needs positions and sub-blocks that sum to head_dim
    rot = capi.sr_rope_out(80, None, 0, None, capi.sr_rope_cfg(10000.0, 32, 48, 48), 1.0)
    rc = lib.sr_kv_append(None, 32, None, 1, 2, 128, 256, 0, 48, 64, None, 100, None, 0, 256, 128, 0,
                          ctypes.byref(rot), None)
    assert rc == capi.SR_ERR_INVALID_ARG and "positions" in _err(lib)
    rot = capi.sr_rope_out(80, 96, 0, None, capi.sr_rope_cfg(10000.0, 32, 48, 40), 1.0)
    rc = lib.sr_kv_append(None, 32, None, 1, 2, 128, 256, 0, 48, 64, None, 100, None, 0, 256, 128, 0,
                          ctypes.byref(rot), None)
    assert rc == capi.SR_ERR_INVALID_ARG and "sub-blocks" in _err(lib)
    rc = lib.sr_kv_append(None, 32, None, 1, 2, 128, 256, 0, 48, 64, None, 100, None, 0, 256, 128, 0, None, None)
    assert rc == capi.SR_ERR_INVALID_ARG and "without its buffer" in _err(lib)    # K with no buffer, no rotation
    assert lib.sr_stream_clock_advance(None, 3.0, None) == capi.SR_ERR_INVALID_ARG
    cfg = capi.sr_pool_cfg(24, 42, 9, 2)
    rc = lib.sr_history_compress(16, 32, 48, 64, 1, 1, 2, 128, cfg, 0, 0, 256, 128, 0, 0, 256, 128,
                                 None, None, 0, None, None, None)
    assert rc == capi.SR_ERR_INVALID_ARG
    cfg = capi.sr_pool_cfg(24, 42, 2, 2)
    rc = lib.sr_history_compress(16, None, 48, 64, 1, 1, 2, 128, cfg, 0, 0, 256, 128, 0, 0, 256, 128,
                                 None, None, 0, None, None, None)
    assert rc == capi.SR_ERR_INVALID_ARG
    rot = capi.sr_rope_out(88, 96, 0, None, capi.sr_rope_cfg(10000.0, 32, 48, 48), 1.0)   # k_rot misaligned
    rc = lib.sr_history_compress(16, 32, 48, 64, 1, 1, 2, 128, cfg, 0, 0, 256, 128, 0, 0, 256, 128,
                                 None, None, 0, None, ctypes.byref(rot), None)
    assert rc == capi.SR_ERR_INVALID_ARG and "k_rot" in _err(lib)


def test_gather_and_scatter_reject_bad_arguments_on_host():
    lib = capi.load()
    cfg = capi.sr_rope_cfg(10000.0, 32, 48, 48)
    # dst, src, idx, src_pos, B, S, H, D, cfg, scale, src_t, src_h, dst_b, dst_s, dst_h, stream
    def rope(dst=16, src=32, idx=48, pos=64, S=10, D=128, c=cfg, ts=512):
        # dst, src, idx, src_pos, B, S, H, D, cfg, scale, src_t, src_h, dst_b, dst_s, dst_h, stream
        return lib.sr_gather_rope3d_tokens(dst, src, idx, pos, 2, S, 4, D, c, 1.0, ts, 128, 5120, 512, 128, None,
                                           None)

    assert rope(pos=None) == capi.SR_ERR_INVALID_ARG and "src_pos" in _err(lib)
    assert rope(c=capi.sr_rope_cfg(10000.0, 32, 48, 40)) == capi.SR_ERR_INVALID_ARG
    assert rope(D=96) == capi.SR_ERR_UNSUPPORTED
    assert rope(dst=24) == capi.SR_ERR_INVALID_ARG and "aligned" in _err(lib)
    assert rope(ts=500) == capi.SR_ERR_INVALID_ARG                        # stride not a multiple of 8
    assert rope(idx=None) == capi.SR_ERR_INVALID_ARG and "null" in _err(lib)
    assert rope(S=0) == capi.SR_OK                                         # zero work: nothing launched
    # gather: positions must come as a pair; scatter: null source
    assert lib.sr_gather_tokens(16, 32, 48, 2, 10, 4, 128, 512, 128, 5120, 512, 128, 64, None, 0, None) == \
        capi.SR_ERR_INVALID_ARG
    assert lib.sr_scatter_tokens(16, None, 48, 2, 10, 4, 128, 512, 128, 5120, 512, 128, None) == capi.SR_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(capi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(capi, "_lib", None)
    with pytest.raises(RuntimeError, match="libsr.so not found"):
        capi.load()


def test_failure_settings_validate_on_host():
    lib = capi.load()
    assert lib.sr_set_withheld_kv_tile(-2) == capi.SR_ERR_INVALID_ARG
    assert lib.sr_set_withheld_kv_tile(-1) == capi.SR_OK
    assert lib.sr_set_wait_limit_ns(0) == capi.SR_OK       # back to the default


def _device_sms():
    """SMs of CUDA device 0, or the 148 of a B200 the library assumes without one."""
    import torch
    if torch.cuda.is_available():
        return torch.cuda.get_device_properties(0).multi_processor_count
    return 148


@pytest.mark.parametrize("B,H,D,q_cap", [
    (1, 40, 128, 3044),   # streaming chunk: 480 units = 3 waves + 36, split 4 ways
    (1, 40, 128, 2276),   # 360 units = 2 waves + 64, split 2 ways
    (77, 4, 128, 512),    # VAE window layer: 616 units = 4 waves + 24, split 6 ways
    (1, 40, 64, 3044),
    (2, 2, 64, 70),       # 4 units: split 8 ways (the cap)
    (1, 37, 128, 1024),   # 148 units: whole waves, no workspace
    (1, 62, 128, 1024),   # 248 units: a remainder of 100 cannot be split in 2
])
def test_attention_workspace_follows_the_split_schedule(B, H, D, q_cap):
    """The split-KV schedule, restated: units are (session, head, 256-row
    query block); whole waves of one unit per SM run whole; the r units of a
    last partial wave are split into s = min(8, SMs // r) KV parts when s >= 2.
    Every part keeps fp32 O for 256 rows x D and (m, l) for 256 rows."""
    sms = _device_sms()
    units = B * H * -(-q_cap // 256)
    rest = units % sms
    s = min(8, sms // rest) if rest else 0
    parts = rest * s if s >= 2 else 0
    expected = parts * 256 * D * 4 + parts * 4 * 128 * 4
    assert capi.sr_chunk_attention_workspace_bytes(B, H, D, q_cap) == expected
