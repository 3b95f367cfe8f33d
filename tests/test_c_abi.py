"""The boundary from plain C: tests/c_abi_attention.c includes only
include/sr.h (and the CUDA runtime for its buffers), links libsr.so, and
checks an attention call against the fp64 oracle's attention.  Compiling and
linking it needs no GPU; running it does."""
import os
import shutil
import subprocess

import pytest

from streaming_video_audio_b200 import build as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(out_dir: str) -> str:
    import oracle
    if shutil.which("gcc") is None or not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")):
        pytest.skip("gcc or the CUDA runtime headers are missing")
    lib = b.build()
    ora = oracle.build()
    exe = os.path.join(out_dir, "c_abi_attention")
    libdirs = [os.path.dirname(lib), os.path.dirname(ora), os.path.join(CUDA, "lib64")]
    cmd = ["gcc", "-std=c11", "-O2", os.path.join(ROOT, "tests", "c_abi_attention.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           lib, ora, "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm", "-o", exe]
    cmd += [f"-Wl,-rpath,{d}" for d in libdirs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_caller_compiles_and_links(tmp_path):
    exe = _compile(str(tmp_path))
    assert os.access(exe, os.X_OK)


@pytest.mark.gpu
def test_c_caller_matches_oracle(tmp_path):
    exe = _compile(str(tmp_path))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    print(r.stdout, r.stderr)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
