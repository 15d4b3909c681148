"""NVTX ranges of the C ABI, recorded by an injection library (host-only, no profiler, no GPU).

Every entry point opens one named range and closes it on every return path, argument errors
included; the stage ranges inside the forward need a device and are not reached here."""

import json
import os
import shutil
import subprocess
import sys

import pytest

from block_sparse_long_meanpool_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CHILD = r"""
import ctypes, json, sys
sys.path.insert(0, sys.argv[1])
from block_sparse_long_meanpool_b200 import moba
lib = moba.load_library()
p = moba.make_params(1, 2048, 4, 4, 64, 256, 3)
bad = moba.make_params(1, 2048, 4, 4, 96, 256, 3)   # unsupported head_dim
N = None
calls = [
    ("moba_attn_fwd", lambda: lib.moba_attn_fwd(ctypes.byref(p), N, N, N, N, N, N, N, 0, N, N, N, N)),
    ("moba_meanpool", lambda: lib.moba_meanpool(ctypes.byref(bad), N, N, N, N)),
    ("moba_minmaxpool", lambda: lib.moba_minmaxpool(ctypes.byref(p), N, N, N, N, N)),
    ("moba_gate_topk", lambda: lib.moba_gate_topk(ctypes.byref(bad), N, N, N, N, N)),
    ("moba_decode_fwd", lambda: lib.moba_decode_fwd(ctypes.byref(p), N, N, N, N, N, N, 0, N, N, N)),
    ("moba_decode_minmax_fwd", lambda: lib.moba_decode_minmax_fwd(ctypes.byref(p), N, N, N, N, N, N, N, 0, N, N, N)),
]
status = [f() for _, f in calls]
rec = ctypes.CDLL(sys.argv[2])
rec.nvtx_recorder_log.restype = ctypes.c_char_p
print(json.dumps({"names": [n for n, _ in calls], "status": status,
                  "log": rec.nvtx_recorder_log().decode().splitlines()}))
"""


@pytest.fixture(scope="module")
def recorder(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    out = str(tmp_path_factory.mktemp("nvtx") / "libnvtx_recorder.so")
    subprocess.run([gcc, "-shared", "-fPIC", "-O1", "-I" + cuda_inc,
                    os.path.join(HERE, "nvtx_recorder.c"), "-o", out], check=True)
    return out


def test_every_entry_point_opens_and_closes_its_range(recorder):
    build.build()
    env = dict(os.environ, NVTX_INJECTION64_PATH=recorder, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", CHILD, ROOT, recorder], env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    got = json.loads(res.stdout.strip().splitlines()[-1])
    assert all(s != 0 for s in got["status"])          # every call took an argument-error return
    want = []
    for name in got["names"]:
        want += ["+" + name, "-"]
    assert got["log"] == want
