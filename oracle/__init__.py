"""fp64 CPU oracle for the chunk-streaming joint video+audio attention step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with ``streaming_video_audio_b200`` and never imports it; the only common
import is ``workloads`` (seeded draws, no method arithmetic).

The numeric kernels are plain C in ``sr_oracle.c`` (fp64, OpenMP over rows);
this module loads it through ctypes, builds the window layout and positions
from its own reading of the pages (``oracle.layout``) and strings the steps
together.  Pins that hold it to something other than itself live in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsr_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle in place (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            lp = ctypes.POINTER(ctypes.c_long)
            lib.sro_rope3d.argtypes = [dp, dp, dp, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_double]
            lib.sro_pool.argtypes = [dp, dp, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_long]
            lib.sro_attention.argtypes = [dp, dp, dp, lp, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                          ctypes.c_double, dp, dp]
            lib.sro_rms_norm.argtypes = [dp, dp, dp, ctypes.c_long, ctypes.c_int, ctypes.c_double]
            lib.sro_num_threads.restype = ctypes.c_int
            lib.sro_set_num_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (bf16 inputs convert exactly)
        import torch
        a = a.detach().to(torch.float64).cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def num_threads() -> int:
    return int(_load().sro_num_threads())


def set_num_threads(n: int) -> None:
    _load().sro_set_num_threads(int(n))


def rope3d(x, pos, split: Tuple[int, int, int], base: float = 10000.0) -> np.ndarray:
    """y = R(pos) x per vector.  x: [..., D], pos: [n, 3] broadcast over the
    middle axes of x ([n, D] or [n, H, D])."""
    x = _f64(x)
    pos = _f64(pos)
    D = x.shape[-1]
    assert sum(split) == D and all(d % 2 == 0 for d in split)
    n = x.shape[0]
    per = int(np.prod(x.shape[1:-1])) if x.ndim > 2 else 1
    xf = x.reshape(n * per, D)
    pf = np.ascontiguousarray(np.repeat(pos.reshape(n, 3), per, axis=0))
    y = np.empty_like(xf)
    _load().sro_rope3d(_dp(xf), _dp(y), _dp(pf), xf.shape[0], D, split[0], split[1], split[2], float(base))
    return y.reshape(x.shape)


def rms_norm(x, gamma, eps: float) -> np.ndarray:
    """Per-vector RMSNorm over the last axis with gain gamma [D]."""
    x = _f64(x)
    g = _f64(gamma).reshape(-1)
    D = x.shape[-1]
    assert g.size == D
    xf = np.ascontiguousarray(x.reshape(-1, D))
    y = np.empty_like(xf)
    _load().sro_rms_norm(_dp(xf), _dp(y), _dp(g), xf.shape[0], D, float(eps))
    return y.reshape(x.shape)


def pool(x, ph: int, pw: int) -> np.ndarray:
    """Mean over valid members of each ph x pw cell (ceil mode).
    x: [F, Gh, Gw, C] -> [F, ceil(Gh/ph), ceil(Gw/pw), C]."""
    x = _f64(x)
    F, Gh, Gw = x.shape[:3]
    C = int(np.prod(x.shape[3:])) if x.ndim > 3 else 1
    y = np.empty((F, -(-Gh // ph), -(-Gw // pw)) + x.shape[3:], dtype=np.float64)
    _load().sro_pool(_dp(x), _dp(y), F, Gh, Gw, ph, pw, C)
    return y


def attention(q, k, v, scale: float, rows: Optional[Sequence[int]] = None):
    """Plain softmax attention of one head.  q: [nq, D], k, v: [nk, D].
    Returns (o [len(rows) or nq, D], lse [...])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    D = q.shape[1]
    assert k.shape[1] == D and v.shape[1] == D and k.shape[0] == v.shape[0]
    if rows is None:
        nq, rp = q.shape[0], None
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        assert rows_arr.size == 0 or (rows_arr.min() >= 0 and rows_arr.max() < q.shape[0])
        nq = rows_arr.size
        rp = rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_long))
    o = np.empty((nq, D), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    if nq:
        _load().sro_attention(_dp(q), _dp(k), _dp(v), rp, nq, k.shape[0], D, float(scale), _dp(o), _dp(lse))
    return o, lse


from . import layout  # noqa: E402  (layout needs nothing above but keeps the public surface here)
from .session import (session_reference, session_kv, pooled_tier, prefix_reference, moving_reference,  # noqa: E402,F401
                      slide_window)
