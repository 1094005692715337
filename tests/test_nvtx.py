"""Tracing: each call of the C ABI opens an NVTX range named after itself in
the domain "csa" and closes it on every return path, the early rejections
included.

A child process loads the library with a small NVTX injection library
(tests/nvtx_probe.c, built here with gcc) named by NVTX_INJECTION64_PATH,
which records every range push and pop to a file.  The calls made are ones
that argument validation rejects before any device is touched, so the test
needs no GPU.
"""
import os
import re
import shutil
import subprocess
import sys

import pytest

from sparse_compressed_attention_csa_b200 import build as B

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

_CHILD = r"""
import ctypes, sys
lib = ctypes.CDLL(sys.argv[1])
# a null parameter block: rejected with CSA_ERR_INVALID_ARGUMENT
assert lib.csa_compress(None, 0, None, None, 1, 16, None, None, None) != 0
assert lib.csa_sparse_attn(None, 0, None, None, None, None, 16, None, None, None, 0, None,
                           1, 1, None, None, ctypes.c_size_t(0), None) != 0
sz = ctypes.c_size_t(0)
assert lib.csa_workspace_size(None, 0, 1, 1, 16, ctypes.byref(sz)) != 0
# no range: a plain getter
lib.csa_abi_version()
"""


def _cuda_include():
    for d in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include")):
        if os.path.exists(os.path.join(d, "nvtx3", "nvToolsExt.h")):
            return d
    return None


def test_every_call_is_an_nvtx_range(tmp_path):
    inc = _cuda_include()
    gcc = shutil.which("gcc")
    if inc is None or gcc is None:
        pytest.skip("gcc or the NVTX v3 headers are not here")
    so = str(tmp_path / "nvtx_probe.so")
    r = subprocess.run([gcc, "-shared", "-fPIC", "-O1", "-I", inc,
                        os.path.join(HERE, "nvtx_probe.c"), "-o", so, "-ldl"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    lib = B.build()
    log = tmp_path / "ranges.txt"
    env = dict(os.environ, NVTX_INJECTION64_PATH=so, CSA_NVTX_PROBE_LOG=str(log))
    r = subprocess.run([sys.executable, "-c", _CHILD, lib], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = log.read_text().splitlines()
    assert lines[0] == "domain csa"
    assert lines[1:] == [
        "push csa csa_compress", "pop csa",
        "push csa csa_sparse_attn", "pop csa",
        "push csa csa_workspace_size", "pop csa",
    ]


def test_every_launching_call_opens_a_range():
    # the source check behind the runtime one: each entry point that
    # validates, plans or launches starts with its range
    src = open(os.path.join(ROOT, "sparse_compressed_attention_csa_b200", "csrc",
                            "csa_lib.cu")).read()
    bodies = re.findall(r"CSA_API csa_status_t (\w+)\(.*?\) \{\n(.*?)\n", src, flags=re.S)
    assert len(bodies) >= 14
    for name, first in bodies:
        assert first.strip() == f'const CallRange trace("{name}");', name
