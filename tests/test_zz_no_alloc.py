"""moba_attn_fwd_noalloc: the forward for callers that cannot allocate device memory.

Plugin hosts that own every device allocation, or services that forbid allocation once
running, cannot call cudaMalloc or pass a workspace.  This entry point runs the same forward
from a scratch array in the library's static device memory.  The GPU test calls it twice in
a row through the C ABI and checks both results bit for bit against moba_attn_fwd (which uses
a caller workspace) run with the query wave the allocation-free call picks, and one case
against the float64 oracle.  This file is collected last.
"""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import parity as PT
from block_sparse_long_meanpool_b200 import build, moba
from block_sparse_long_meanpool_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moba.load_library()


def _params(w):
    return moba.make_params(len(w.seqlens), w.total_tokens, w.num_q_heads, w.num_kv_heads,
                            w.head_dim, w.chunk_size, w.topk)


def test_binding_knows_the_scratch_size():
    text = open(os.path.join(ROOT, "include", "moba.h")).read()
    m = re.search(r"#define MOBA_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == moba.NOALLOC_SCRATCH_BYTES


def test_noalloc_rejects_a_problem_larger_than_its_scratch(lib):
    # 1M tokens: the selections alone exceed the static array.  NULL tensors: the size check
    # must answer before any argument is used.
    w = W.WORKLOADS["prefill_1m"]
    p = _params(w)
    rc = lib.moba_attn_fwd_noalloc(ctypes.byref(p), None, None, None, None, None, None, None)
    assert rc == moba.ERR_UNSUPPORTED
    assert b"bytes of scratch" in lib.moba_last_error()


def _noalloc_wave(w):
    """The query wave the allocation-free call picks: one wave when the whole workspace fits
    the static array, else the largest multiple of 128 tokens that fits."""
    return moba.choose_wave_tokens(w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                   w.chunk_size, w.topk, len(w.seqlens), moba.NOALLOC_SCRATCH_BYTES)


CASES = [
    W.custom("noalloc_one_wave", [1500, 700], 8, 2, 128, 256, 3, "k_offsets", 71),
    W.custom("noalloc_many_waves", [20000], 16, 4, 128, 512, 4, "k_offsets", 72),
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=["one_wave", "many_waves"])
def test_noalloc_matches_the_workspace_forward_twice(lib, w):
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, hq, d = q.shape
    wave = _noalloc_wave(w)
    assert (wave == 0) == (w.name == "noalloc_one_wave")
    ref_out, ref_lse = moba.attn_fwd(q, k, v, cu, w.chunk_size, w.topk, wave_tokens=wave)
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
        assert lib.moba_device_status_noalloc(stream) == moba.OK, lib.moba_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


@pytest.mark.gpu
def test_noalloc_against_the_oracle(lib):
    """The allocation-free forward of a small ragged GQA case against the float64 oracle on all
    rows (selections that differ from the oracle's must be valid near ties; those rows are
    checked against the oracle over the GPU's selection)."""
    w = W.custom("noalloc_oracle", [900, 1, 333], 4, 2, 64, 128, 3, "qk_offsets", 73)
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, hq, d = q.shape
    p = _params(w)
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((hq, T), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.moba_attn_fwd_noalloc(
        ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(cu.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), stream)
    assert rc == moba.OK, lib.moba_last_error()
    # the selection the forward used: the workspace forward computes the same one
    _, _, sel = moba.attn_fwd(q, k, v, cu, w.chunk_size, w.topk, return_sel=True)
    torch.cuda.synchronize()
    cu_np = np.asarray(w.cu_seqlens)
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    ref = oracle.moba_forward(q_np, k_np, v_np, cu_np, w.chunk_size, w.topk)
    gsel = PT.host(sel, np.int64)
    diff = np.nonzero((gsel != ref["sel"]).any(axis=2))
    rows = [(int(t), int(h)) for h, t in zip(*diff)]
    ties = PT.check_selection(gsel[diff], ref["sel"][diff], rows, q_np, ref["means"], cu_np,
                              w.chunk_size, w.topk, hq // w.num_kv_heads)
    ref_o, ref_l = ref["out"].copy(), ref["lse"].copy()
    if ties:
        tr = [rows[r] for r in sorted(ties)]
        o, l = oracle.attend_rows(q_np, k_np, v_np, cu_np, w.chunk_size,
                                  np.stack([gsel[h, t] for t, h in tr]), tr)
        for i, (t, h) in enumerate(tr):
            ref_o[t, h], ref_l[h, t] = o[i], l[i]
    PT.check_out(PT.host(out).reshape(T * hq, d), PT.host(lse).T.reshape(-1),
                 ref_o.reshape(T * hq, d), ref_l.T.reshape(-1))
