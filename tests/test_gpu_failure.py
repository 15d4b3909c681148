"""Failure detection on the GPU without a fault: a bounded device-side wait that nothing can
satisfy must expire, report MOBA_ERR_DEVICE_TIMEOUT through the status word, and leave the
CUDA context usable (a forward afterwards still matches the oracle)."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_meanpool_b200 import moba, workloads as W

from parity import check_out, host

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_reports_timeout():
    assert moba.selftest_timeout(polls=4096) == moba.ERR_DEVICE_TIMEOUT
    # a second run starts from a fresh word and expires again
    assert moba.selftest_timeout(polls=64) == moba.ERR_DEVICE_TIMEOUT


def test_selftest_rejects_bad_arguments():
    lib = moba.load_library()
    assert lib.moba_selftest_timeout(None, 16, None) == moba.ERR_INVALID_ARG
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.moba_selftest_timeout(moba._ptr(word), 0, None) == moba.ERR_INVALID_ARG


def test_context_usable_after_timeout():
    assert moba.selftest_timeout(polls=4096) == moba.ERR_DEVICE_TIMEOUT
    w = W.custom("after_timeout", [700, 300], 4, 2, 64, 128, 3, "k_offsets", 31)
    x = W.make_inputs(w, device="cuda")
    out, lse = moba.attn_fwd(x["q"], x["k"], x["v"], x["cu_seqlens"], w.chunk_size, w.topk)
    torch.cuda.synchronize()
    ref = oracle.moba_forward(host(x["q"]), host(x["k"]), host(x["v"]), np.asarray(w.cu_seqlens),
                              w.chunk_size, w.topk)
    T = w.total_tokens
    check_out(host(out).reshape(T * w.num_q_heads, -1), host(lse).T.reshape(-1),
              ref["out"].reshape(T * w.num_q_heads, -1), ref["lse"].T.reshape(-1))
