"""The library marks its calls and grid launches with NVTX ranges.

A small NVTX tool (tests/nvtx_counter.c, loaded through
NVTX_INJECTION64_PATH) counts the pushes and pops and keeps the names.  The
calls here fail their argument checks on the host, so no GPU is needed:
each still opens and closes its range.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _cuda_include():
    for d in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include")):
        if os.path.exists(os.path.join(d, "nvtx3", "nvToolsExt.h")):
            return d
    pytest.skip("nvtx3 headers not found")


def test_calls_open_and_close_nvtx_ranges(tmp_path):
    sys.path.insert(0, ROOT)
    from compressed_kv_cache_routing_b200 import build
    lib = build.build()
    tool = tmp_path / "libnvtx_counter.so"
    subprocess.check_call(["gcc", "-shared", "-fPIC", "-O1", "-I", _cuda_include(),
                           os.path.join(HERE, "nvtx_counter.c"), "-o", str(tool)])
    out = tmp_path / "ranges.txt"
    code = (
        "import ctypes\n"
        f"lib = ctypes.CDLL({str(lib)!r})\n"
        "f = ctypes.c_float\n"
        "lib.basiskv_decode_attn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, f,\n"
        "                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]\n"
        "lib.basiskv_decode_attn_latent.argtypes = lib.basiskv_decode_attn.argtypes\n"
        "assert lib.basiskv_decode_attn(None, 1, None, 1, f(1.0), None, None, None) != 0\n"
        "assert lib.basiskv_decode_attn_latent(None, 1, None, 1, f(1.0), None, None, None) != 0\n"
    )
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(tool), NVTX_COUNTER_OUT=str(out))
    subprocess.check_call([sys.executable, "-c", code], env=env)
    lines = out.read_text().splitlines()
    pushes = int(lines[0].split()[1])
    pops = int(lines[1].split()[1])
    assert pushes == pops == 2, lines
    assert lines[2:] == ["basiskv_decode_attn", "basiskv_decode_attn_latent"], lines
