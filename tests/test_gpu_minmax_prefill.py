"""GPU parity of the prefill forward with the min/max (Quest-style) gate, through the C ABI,
against the float64 oracle.

The gate scores earlier blocks by s_j = sum_i max(q_i kmin_ji, q_i kmax_ji)
(``oracle.minmax_scores_row`` with ``oracle.block_minmax``), selection rule unchanged.  The
mean gate's 1e-3 relative band does not fit this score (a box over many keys gives scores of
a few hundred that differ by a few units), so the band comes from the kernel's arithmetic
(``parity.minmax_slack``): the products are exact and only the fp32 sum of 2d terms rounds, so
two blocks may swap only when their oracle scores are closer than the sum of their bounds.
Outputs are checked on all rows (small cases) or sampled rows (32K), near-tie rows against the
oracle's attention over the GPU's own selection.
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


@pytest.fixture(scope="module", autouse=True)
def library():
    build.build()
    moba.load_library()


@pytest.fixture(scope="module")
def ex():
    with OP.pool() as e:
        yield e


def _summary(k_np, cu, chunk):
    kmin, kmax = oracle.block_minmax(k_np, cu, chunk)
    return np.stack([kmin, kmax], axis=2)  # [NB, Hkv, 2, d]


CASES = [
    W.WORKLOADS["tiny_2k"],
    W.custom("mm_ragged_gqa", [700, 1337, 128, 1, 0, 390], 8, 2, 128, 128, 3, "k_offsets", 91),
    W.custom("mm_d64_topk5", [3000], 4, 1, 64, 128, 5, "qk_offsets", 92),
    W.custom("mm_topk32", [4500], 2, 1, 128, 128, 32, "k_offsets", 93),
    W.custom("mm_odd_group", [1500, 900], 6, 2, 128, 384, 3, "k_offsets", 94),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_minmax_prefill_all_rows(w):
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu_t = x["q"], x["k"], x["v"], x["cu_seqlens"]
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, gate="minmax",
                                  max_seqlen=w.max_seqlen)
    assert moba.attn_fwd.last_info["gate_path"] == moba.GATE_PATH_TENSOR_CORES
    kmin, kmax = moba.minmaxpool(k, cu_t, chunk)
    sel2 = moba.gate_minmax_topk(q, kmin, kmax, cu_t, chunk, topk)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel2)
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    summ = _summary(k_np, cu, chunk)
    T = q.shape[0]
    rows = [(t, h) for h in range(hq) for t in range(T)]
    osel = oracle.select_blocks_rows(q_np, summ, cu, chunk, topk, rows, score=oracle.minmax_scores_row)
    gsel = PT.host(sel, np.int64)
    g_rows = np.stack([gsel[h, t] for t, h in rows])
    ties = PT.check_selection(g_rows, osel, rows, q_np, summ, cu, chunk, topk, group,
                              score=oracle.minmax_scores_row, slack_fn=PT.minmax_slack)
    ref_o, ref_l = oracle.attend_rows(q_np, k_np, v_np, cu, chunk, g_rows, rows)
    PT.check_out(np.stack([PT.host(out[t, h]) for t, h in rows]), np.array([float(lse[h, t]) for t, h in rows]),
                 ref_o, ref_l)
    assert len(ties) < max(3, 1e-2 * len(rows))


def test_minmax_prefill_long_32k(ex):
    """long_32k (32K tokens, 32 heads, 64 blocks, top-3, needle blocks) with the min/max gate:
    every row's selection against the oracle's, and 2048 sampled rows' outputs."""
    w = W.WORKLOADS["long_32k"]
    x = W.make_inputs(w, device="cuda")
    q, k, v, cu_t = x["q"], x["k"], x["v"], x["cu_seqlens"]
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, gate="minmax",
                                  max_seqlen=w.max_seqlen)
    torch.cuda.synchronize()
    q16, k16, v16 = PT.bf16_bits(q), PT.bf16_bits(k), PT.bf16_bits(v)
    q_np, k_np = PT.from_bits(q16), PT.from_bits(k16)
    summ = _summary(k_np, cu, chunk)
    T = w.total_tokens
    rows = [(t, h) for h in range(hq) for t in range(T)]
    ts = np.array([t for t, _ in rows])
    hs = np.array([h for _, h in rows])
    osel = OP.select_rows_par(ex, rows, q16[ts, hs], summ, cu, chunk, topk, group, minmax=True)
    gsel = PT.host(sel, np.int64)[hs, ts]
    diff = np.nonzero((gsel != osel).any(axis=1))[0]
    ties = PT.check_selection(gsel[diff], osel[diff], [rows[i] for i in diff], q_np, summ, cu, chunk,
                              topk, group, score=oracle.minmax_scores_row, slack_fn=PT.minmax_slack)
    assert len(ties) < 1e-3 * len(rows)
    sample = sorted(set(PT.sample_rows(cu, chunk, hq, topk, 1536, 512, seed=95)) |
                    {rows[diff[i]] for i in ties})
    st = np.array([t for t, _ in sample])
    sh = np.array([h for _, h in sample])
    g_rows = PT.host(sel, np.int64)[sh, st]
    ref_o, ref_l = OP.attend_rows_par(ex, sample, q16[st, sh], k16, v16, cu, chunk, g_rows, group)
    PT.check_out(PT.host(out[st, sh]), PT.host(lse[sh, st]), ref_o, ref_l)


def test_minmax_gate_picks_the_aligned_key_the_mean_misses():
    """One block holds a single key aligned with the query among zeros: the mean dilutes it,
    the min/max box does not.  The constructed rows' routed block differs between the two
    gates, each as its oracle says."""
    T, chunk = 1024, 128
    d = 64
    q = torch.zeros((T, 1, d), dtype=torch.float32)
    k = torch.zeros((T, 1, d), dtype=torch.float32)
    v = torch.randn((T, 1, d), generator=torch.Generator().manual_seed(3))
    k[0:128, 0, 0] = 0.25                  # block 0: every key a little aligned (mean 0.25)
    k[128 + 5, 0, 0] = 4.0                 # block 1: one strongly aligned key (mean 4/128)
    q[:, 0, 0] = 1.0
    q, k, v = (t.to(torch.bfloat16).cuda() for t in (q, k, v))
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    _, _, s_mean = moba.attn_fwd(q, k, v, cu, chunk, 2, return_sel=True)
    _, _, s_mm = moba.attn_fwd(q, k, v, cu, chunk, 2, return_sel=True, gate="minmax", max_seqlen=T)
    torch.cuda.synchronize()
    q_np, k_np = PT.host(q), PT.host(k)
    rows = [(t, 0) for t in range(2 * chunk, T)]
    o_mean = oracle.select_blocks_rows(q_np, oracle.block_means(k_np, [0, T], chunk), [0, T], chunk, 2, rows)
    o_mm = oracle.select_blocks_rows(q_np, _summary(k_np, [0, T], chunk), [0, T], chunk, 2, rows,
                                     score=oracle.minmax_scores_row)
    g_mean = PT.host(s_mean, np.int64)[0, 2 * chunk:]
    g_mm = PT.host(s_mm, np.int64)[0, 2 * chunk:]
    np.testing.assert_array_equal(g_mean, o_mean)
    np.testing.assert_array_equal(g_mm, o_mm)
    assert (g_mean[:, 0] == 0).all() and (g_mm[:, 0] == 1).all()
