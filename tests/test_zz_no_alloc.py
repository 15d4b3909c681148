"""moba_attn_fwd_noalloc: the forward for callers that cannot allocate device memory.

Plugin hosts that own every device allocation, or services that forbid allocation once
running, cannot call cudaMalloc or pass a workspace.  This entry point runs the same forward
from a scratch array in the library's static device memory.  The GPU test calls it twice in
a row through the C ABI and checks both results against moba_attn_fwd (which uses a caller
workspace), within the tolerances the parity tests use.  This file is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

import parity as PT
from block_sparse_long_meanpool_b200 import build, moba
from block_sparse_long_meanpool_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moba.load_library()


def _params(w):
    return moba.make_params(len(w.seqlens), w.total_tokens, w.num_q_heads, w.num_kv_heads,
                            w.head_dim, w.chunk_size, w.topk)


def test_noalloc_rejects_a_problem_larger_than_its_scratch(lib):
    # 1M tokens: the selections alone exceed the static array.  NULL tensors: the size check
    # must answer before any argument is used.
    w = W.WORKLOADS["prefill_1m"]
    p = _params(w)
    rc = lib.moba_attn_fwd_noalloc(ctypes.byref(p), None, None, None, None, None, None, None)
    assert rc == moba.ERR_UNSUPPORTED
    assert b"bytes of scratch" in lib.moba_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("w", [
    W.custom("noalloc_one_wave", [1500, 700], 8, 2, 128, 256, 3, "k_offsets", 71),
    W.custom("noalloc_many_waves", [20000], 16, 4, 128, 512, 4, "k_offsets", 72),
], ids=["one_wave", "many_waves"])
def test_noalloc_matches_the_workspace_forward_twice(lib, w):
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, hq, d = q.shape
    ref_out, ref_lse = moba.attn_fwd(q, k, v, cu, w.chunk_size, w.topk)
    torch.cuda.synchronize()
    p = _params(w)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full((T, hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((hq, T), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.moba_attn_fwd_noalloc(
            ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(cu.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), stream)
        assert rc == moba.OK, lib.moba_last_error()
        torch.cuda.synchronize()
        PT.check_out(PT.host(out).reshape(T * hq, d), PT.host(lse).T.reshape(-1),
                     PT.host(ref_out).reshape(T * hq, d), PT.host(ref_lse).T.reshape(-1))
        assert not np.isnan(PT.host(out)).any()
