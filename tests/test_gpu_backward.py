"""GPU parity of the backward pass (moba_attn_bwd, through the C ABI) against the float64
oracle's ``moba_backward``.

The backward takes the forward's selection as fixed (the gate has no parameters and routes by
hard top-k, so no gradient flows through it); the GPU forward's own selection is passed to both
sides.  d_out is seeded N(0, 1) bf16, d_lse seeded N(0, 1) fp32 (or absent).

Tolerance, per gradient tensor G against the oracle's R, derived from the arithmetic: P and dS
enter the tensor-core products rounded to bf16 (relative error <= 2^-9 per term, adding up like
a random walk), the result is rounded once more to bf16 (2^-9), and <dO, out> is formed from the
forward's bf16 out (as an attention backward does), which moves every dS of a row by
p_u * <dO, out - out_exact>: up to 2^-9 sum_i |dO_i out_i| per row, so up to a few 1e-3 of the
largest dq or dk element in rows with few attended keys (p close to 1).  Everything else is fp32.
    max |G - R| <= 3e-2 * max |R|    and    mean |G - R| <= 5e-3 * mean |R|.
"""

import numpy as np
import pytest
import torch

import oracle
import oracle_pool as OP
import parity as PT
from block_sparse_long_meanpool_b200 import build, moba
from block_sparse_long_meanpool_b200 import workloads as W

pytestmark = pytest.mark.gpu

GRAD_MAX = 3e-2
GRAD_MEAN = 5e-3


@pytest.fixture(scope="module", autouse=True)
def library():
    build.build()
    moba.load_library()


def check_grad(name, g, r):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    err = np.abs(g - r)
    worst = np.unravel_index(int(err.argmax()), err.shape)
    stats = {"grad": name, "max_abs": float(err.max()), "mean_abs": float(err.mean()),
             "max_ref": float(np.abs(r).max()), "mean_ref": float(np.abs(r).mean()),
             "rms_ref": float(np.sqrt((r ** 2).mean())), "worst_at": [int(x) for x in worst],
             "ref_at_worst": float(r[worst]), "row_max_ref": float(np.abs(r[worst[:-1]]).max())}
    print(stats)
    assert stats["max_abs"] <= GRAD_MAX * stats["max_ref"], stats
    assert stats["mean_abs"] <= GRAD_MEAN * stats["mean_ref"], stats
    return stats


def run_case(w, with_dlse, seed, ex=None, heads=None):
    """heads: check only these query heads (MHA: their KV heads' gradients come from them
    alone), with the oracle on those heads only."""
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, hq, d = q.shape
    hkv = k.shape[1]
    out, lse, sel = moba.attn_fwd(q, k, v, cu, w.chunk_size, w.topk, return_sel=True)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    d_out = torch.randn((T, hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    d_lse = torch.randn((hq, T), generator=gen, device="cuda") if with_dlse else None
    dq, dk, dv = moba.attn_bwd(q, k, v, out, lse, d_out, cu, w.chunk_size, w.topk, sel, d_lse=d_lse)
    torch.cuda.synchronize()
    cu_np = np.asarray(w.cu_seqlens)
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    s_np = PT.host(sel, np.int64)
    do_np = PT.host(d_out)
    dl_np = PT.host(d_lse) if with_dlse else None
    gq, gk, gv = PT.host(dq), PT.host(dk), PT.host(dv)
    if heads is not None:
        assert hq == hkv  # MHA: head h's KV gradients are its own
        q_np, k_np, v_np, do_np = q_np[:, heads], k_np[:, heads], v_np[:, heads], do_np[:, heads]
        s_np = s_np[heads]
        dl_np = dl_np[heads] if dl_np is not None else None
        gq, gk, gv = gq[:, heads], gk[:, heads], gv[:, heads]
    if ex is None:
        rq, rk, rv = oracle.moba_backward(q_np, k_np, v_np, cu_np, w.chunk_size, s_np, do_np, dl_np)
    else:
        rq, rk, rv = OP.backward_by_head(ex, q_np, k_np, v_np, cu_np, w.chunk_size, s_np, do_np, dl_np)
    res, errs = [], []
    for name, g, r in (("dv", gv, rv), ("dk", gk, rk), ("dq", gq, rq)):
        try:
            res.append(check_grad(name, g, r))
        except AssertionError as e:
            errs.append(str(e))
    assert not errs, errs
    return res


SMALL = [
    (W.WORKLOADS["tiny_2k"], True),
    # ragged varlen GQA: empty and 1-token sequences, partial blocks, several key tiles
    (W.custom("bwd_ragged_gqa", [700, 1337, 128, 1, 0, 390], 8, 2, 128, 128, 3, "k_offsets", 81), True),
    (W.custom("bwd_ragged_gqa_no_dlse", [700, 1337, 128, 1, 0, 390], 8, 2, 128, 128, 3, "k_offsets", 81), False),
    # odd GQA group, blocks of 3 key tiles with a partial last block
    (W.custom("bwd_odd_group", [1500, 900], 6, 2, 128, 384, 3, "k_offsets", 82), True),
    # MHA, d = 64, partial blocks
    (W.custom("bwd_mha_d64", [1000, 1700], 3, 3, 64, 384, 3, "qk_offsets", 83), True),
    # many routed blocks per row, 128-token blocks
    (W.custom("bwd_topk8", [3000], 4, 1, 64, 128, 8, "k_offsets", 84), True),
    # every block selected: dense causal attention
    (W.custom("bwd_dense", [1000, 600], 4, 4, 128, 256, 8, "k_offsets", 85), True),
    # one block longer than the sequence
    (W.custom("bwd_single_block", [300, 77], 2, 1, 128, 512, 3, "k_offsets", 86), True),
]


@pytest.mark.parametrize("w,with_dlse", SMALL, ids=[w.name for w, _ in SMALL])
def test_backward_small(w, with_dlse):
    run_case(w, with_dlse, seed=w.seed + 1)


@pytest.fixture(scope="module")
def ex():
    with OP.pool() as e:
        yield e


def test_backward_scaling_8k(ex):
    """All rows and all keys of scaling_8k (2 x 8192 tokens, 16 heads; the oracle split by query
    head)."""
    w = W.ALL_WORKLOADS["scaling_8k"]
    run_case(w, True, seed=w.seed + 2, ex=ex)


def test_backward_long_32k(ex):
    """long_32k (32K tokens, 32 heads MHA, 64 blocks of 512, top-3, needles): every row and every
    key of four heads (one per quarter of the heads); the GPU computes all 32."""
    w = W.ALL_WORKLOADS["long_32k"]
    run_case(w, True, seed=w.seed + 2, ex=ex, heads=[0, 11, 22, 31])


def test_backward_gqa_8k(ex):
    """GQA at 8K tokens: 8 q / 2 kv heads, chunk 512, top-3, all rows and keys."""
    w = W.custom("bwd_gqa_8k", [8192], 8, 2, 128, 512, 3, "k_offsets", 87)
    run_case(w, True, seed=88, ex=ex)


def test_backward_repeats_up_to_summation_order():
    """Two backward calls agree to within the order of their fp32 additions: dK and dV are
    written once per key tile, but the routing lists (and so the order in which a tile's rows
    are added) are filled by atomics, and dq is summed by reductions."""
    w = SMALL[1][0]
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    out, lse, sel = moba.attn_fwd(q, k, v, cu, w.chunk_size, w.topk, return_sel=True)
    d_out = torch.randn(out.shape, device="cuda").to(torch.bfloat16)
    a = moba.attn_bwd(q, k, v, out, lse, d_out, cu, w.chunk_size, w.topk, sel)
    b = moba.attn_bwd(q, k, v, out, lse, d_out, cu, w.chunk_size, w.topk, sel)
    for x_, y_ in zip(a, b):
        diff = (x_.float() - y_.float()).abs().max().item()
        assert diff <= 2 ** -7 * x_.float().abs().max().item(), diff
