"""GPU parity: the CUDA path, called through the C ABI, against the float64 oracle.

Every case feeds the same seeded bf16 inputs to both sides.  Small cases are checked on all
rows; the full-size workloads on all means, all selections (or whole heads at 1M) and
sampled output rows.  Tolerances are in ``parity.py``.
"""

import os

import numpy as np
import pytest
import torch

import oracle
import parity as PT
from block_sparse_long_meanpool_b200 import build, moba
from block_sparse_long_meanpool_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def library():
    build.build()
    moba.load_library()


SMALL = [
    W.WORKLOADS["tiny_2k"],
    # ragged varlen GQA: empty and 1-token sequences, partial tails, several 128-row tiles
    W.custom("ragged_gqa", [700, 1337, 128, 1, 0, 390], 8, 2, 128, 128, 3, "k_offsets", 11),
    W.custom("d64_many_blocks", [3000], 4, 1, 64, 128, 5, "qk_offsets", 12),
    # topk >= number of blocks: dense causal attention
    W.custom("dense_all_blocks", [1000, 600], 4, 4, 128, 256, 8, "k_offsets", 13),
    # topk = 1: the own block only
    W.custom("topk1", [900], 2, 2, 64, 256, 1, "k_offsets", 14),
    # the widest top-k list (31 routed blocks of 35)
    W.custom("topk32", [4500], 2, 1, 128, 128, 32, "k_offsets", 15),
    # one block longer than the sequence
    W.custom("single_block", [300, 77], 2, 1, 128, 512, 3, "k_offsets", 16),
    # odd GQA group (3 query heads per KV head): paired and single heads in current-block work
    W.custom("odd_group", [1500, 900], 6, 2, 128, 384, 3, "k_offsets", 17),
    # MHA with 3 query tiles per block and partial blocks: paired and single query tiles
    W.custom("mha_odd_tiles", [1000, 1700], 3, 3, 64, 384, 3, "qk_offsets", 18),
]


def gpu_inputs(w):
    x = W.make_inputs(w, device="cuda")
    return x["q"], x["k"], x["v"], x["cu_seqlens"]


def full_sel_check(gsel, osel, q_np, om, cu, chunk, topk, group):
    """Compare [Hq, T, topk] selections; returns a boolean [Hq, T] mask of near-tie rows."""
    diff = np.nonzero((gsel != osel).any(axis=2))
    rows = [(int(t), int(h)) for h, t in zip(*diff)]
    ties = PT.check_selection(gsel[diff], osel[diff], rows, q_np, om, cu, chunk, topk, group)
    mask = np.zeros(gsel.shape[:2], dtype=bool)
    for r in ties:
        t, h = rows[r]
        mask[h, t] = True
    return mask


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_all_rows(w):
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, group = w.chunk_size, w.topk, w.num_q_heads // w.num_kv_heads
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    sel_gate = moba.gate_topk(q, means, cu_t, chunk, topk)
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True)
    torch.cuda.synchronize()
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    ref = oracle.moba_forward(q_np, k_np, v_np, cu, chunk, topk)

    PT.check_means(PT.host(means), k_np, cu, chunk, ref["means"])
    gsel = PT.host(sel, np.int64)
    np.testing.assert_array_equal(gsel, PT.host(sel_gate, np.int64))
    ties = full_sel_check(gsel, ref["sel"], q_np, ref["means"], cu, chunk, topk, group)

    T, hq = q.shape[0], q.shape[1]
    rows = [(t, h) for t in range(T) for h in range(hq)]
    keep_skip = [i for i, (t, h) in enumerate(rows) if ties[h, t]]
    out_np, lse_np = PT.host(out), PT.host(lse)
    PT.check_out(out_np.reshape(T * hq, -1), lse_np.T.reshape(-1),
                 ref["out"].reshape(T * hq, -1), ref["lse"].T.reshape(-1), skip=keep_skip)

    # oracle-feed mode: the oracle's selection, no exceptions
    fed = torch.from_numpy(ref["sel"].astype(np.int32)).cuda()
    out2, lse2 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed)
    PT.check_out(PT.host(out2).reshape(T * hq, -1), PT.host(lse2).T.reshape(-1),
                 ref["out"].reshape(T * hq, -1), ref["lse"].T.reshape(-1))


def test_waves_give_bitwise_identical_results():
    w = SMALL[1]
    q, k, v, cu_t = gpu_inputs(w)
    base = moba.attn_fwd(q, k, v, cu_t, w.chunk_size, w.topk, wave_tokens=0)
    for wave in (128, 384, 1024):
        out, lse = moba.attn_fwd(q, k, v, cu_t, w.chunk_size, w.topk, wave_tokens=wave)
        assert moba.attn_fwd.last_info["waves"] == -(-q.shape[0] // wave)
        assert torch.equal(out, base[0]) and torch.equal(lse, base[1])


def test_forced_selections_window_and_sink():
    """Fed selections {c-1, c} (sliding window) and {0, c-1, c} (sink) on a GQA case."""
    w = W.custom("forced", [1500, 640], 4, 2, 128, 128, 3, "k_offsets", 21)
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    T, hq = q.shape[0], q.shape[1]
    for kind in ("swa", "sink"):
        sel = np.full((hq, T, 3), -1, dtype=np.int64)
        for i in range(len(cu) - 1):
            for t in range(cu[i], cu[i + 1]):
                c = (t - cu[i]) // 128
                js = sorted({j for j in ([c - 1, c] if kind == "swa" else [0, c - 1, c]) if j >= 0})
                sel[:, t, :len(js)] = js
        ref_o, ref_l = oracle.attention_masked_dense(q_np, k_np, v_np, cu, 128, sel)
        out, lse = moba.attn_fwd(q, k, v, cu_t, 128, 3, sel=torch.from_numpy(sel.astype(np.int32)).cuda())
        PT.check_out(PT.host(out).reshape(T * hq, -1), PT.host(lse).T.reshape(-1),
                     ref_o.reshape(T * hq, -1), ref_l.T.reshape(-1))


def test_fed_selection_rule_ignores_invalid_entries():
    """Entries >= c, repeats and extra entries are ignored; the own block is always used."""
    w = W.custom("dirty", [1100], 2, 1, 64, 128, 4, "k_offsets", 22)
    q, k, v, cu_t = gpu_inputs(w)
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, 128, 4, return_sel=True)
    s = PT.host(sel, np.int64)
    dirty = s.copy()
    T = q.shape[0]
    for t in range(T):
        c = t // 128
        for h in range(2):
            row = [int(x) for x in s[h, t] if 0 <= x < c]      # routed past blocks, in order
            extra = [c + 1, row[0] if row else c + 2, c, -7]   # future, repeat, own, junk
            new = (row + extra)[:4] if c > 0 else [c, c + 3, -1, 99]
            dirty[h, t] = new
    out2, lse2 = moba.attn_fwd(q, k, v, cu_t, 128, 4,
                               sel=torch.from_numpy(dirty.astype(np.int32)).cuda())
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_empty_input():
    w = W.custom("empty", [0], 2, 2, 64, 128, 3)
    q, k, v, cu_t = gpu_inputs(w)
    out, lse = moba.attn_fwd(q, k, v, cu_t, 128, 3)
    assert out.shape == (0, 2, 64) and lse.shape == (2, 0)


def test_softmax_scale_parameter():
    w = W.custom("scaled", [777], 2, 2, 128, 128, 2, "k_offsets", 23)
    q, k, v, cu_t = gpu_inputs(w)
    out, lse = moba.attn_fwd(q, k, v, cu_t, 128, 2, softmax_scale=0.05)
    cu = np.asarray(w.cu_seqlens)
    ref = oracle.moba_forward(PT.host(q), PT.host(k), PT.host(v), cu, 128, 2, scale=0.05)
    T = q.shape[0]
    PT.check_out(PT.host(out).reshape(T * 2, -1), PT.host(lse).T.reshape(-1),
                 ref["out"].reshape(T * 2, -1), ref["lse"].T.reshape(-1))


FULL = ["scaling_8k", "long_32k", "varlen_gqa", "fine_32k_8_2", "fine_32k_128_32"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    """All means, all selections, sampled output rows; then the oracle-feed mode."""
    w = W.ALL_WORKLOADS[name]
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True)
    torch.cuda.synchronize()
    q_np, k_np, v_np = PT.host(q, np.float32), PT.host(k, np.float32), PT.host(v, np.float32)
    om = oracle.block_means(k_np, cu, chunk)
    PT.check_means(PT.host(means), k_np, cu, chunk, om)
    osel = oracle.select_blocks(q_np, om, cu, chunk, topk)
    gsel = PT.host(sel, np.int64)
    ties = full_sel_check(gsel, osel, q_np, om, cu, chunk, topk, group)
    assert ties.mean() < 1e-3

    rows = PT.sample_rows(cu, chunk, hq, topk, 768, 256, seed=31)
    ref_o, ref_l = oracle.attend_rows(q_np, k_np, v_np, cu, chunk, osel, rows)
    out_np, lse_np = PT.host(out, np.float32), PT.host(lse)
    g_o = np.stack([out_np[t, h] for t, h in rows])
    g_l = np.array([lse_np[h, t] for t, h in rows])
    skip = [i for i, (t, h) in enumerate(rows) if ties[h, t]]
    PT.check_out(g_o, g_l, ref_o, ref_l, skip=skip)

    fed = torch.from_numpy(osel.astype(np.int32)).cuda()
    out2, lse2 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed)
    out2_np, lse2_np = PT.host(out2, np.float32), PT.host(lse2)
    PT.check_out(np.stack([out2_np[t, h] for t, h in rows]),
                 np.array([lse2_np[h, t] for t, h in rows]), ref_o, ref_l)


def test_prefill_1m_sampled():
    """1,048,576 tokens, 32 q / 8 kv heads, chunk 4096, top-12, in the wave configuration the
    bench uses: all block means, whole-head selections for four heads (one per two KV
    heads) plus sampled rows of every head, sampled output rows, and a fed selection."""
    w = W.WORKLOADS["prefill_1m"]
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq, hkv = w.chunk_size, w.topk, w.num_q_heads, w.num_kv_heads
    group = hq // hkv
    n_rows = int(os.environ.get("MOBA_1M_SAMPLED_ROWS_PER_HEAD", "24"))
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True)
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    torch.cuda.synchronize()
    assert moba.attn_fwd.last_info["waves"] >= 1
    k_np, v_np = PT.host(k, np.float32), PT.host(v, np.float32)
    # means, per block through the oracle (blocks are independent)
    om = np.concatenate([oracle.block_means(k_np[b * chunk:(b + 1) * chunk], [0, chunk], chunk)
                         for b in range(nb)])
    PT.check_means(PT.host(means), k_np, cu, chunk, om)
    gsel = PT.host(sel, np.int64)
    heads = [0, 9, 18, 27]
    for h in heads:
        qh = PT.host(q[:, h:h + 1], np.float32)
        osel_h = oracle.select_blocks(qh, om[:, h // group:h // group + 1], cu, chunk, topk)
        full_sel_check(gsel[h:h + 1], osel_h, qh, om[:, h // group:h // group + 1], cu, chunk,
                       topk, 1)
    rows = PT.sample_rows(cu, chunk, hq, topk, n_rows * hq * 3 // 4, n_rows * hq // 4, seed=41)
    q_rows = {}
    for t, h in rows:
        if t not in q_rows:
            q_rows[t] = PT.host(q[t], np.float32)
    ref_sel = np.stack([
        oracle.select_blocks_rows(_QView(q_rows), om, cu, chunk, topk, [(t, h)])[0] for t, h in rows])
    g_rows = np.stack([gsel[h, t] for t, h in rows])
    ties = PT.check_selection(g_rows, ref_sel, rows, _QView(q_rows), om, cu, chunk, topk, group)
    ref_o, ref_l = oracle.attend_rows(_QView(q_rows), k_np, v_np, cu, chunk, ref_sel, rows)
    out_np = {t: PT.host(out[t], np.float32) for t, _ in rows}
    lse_rows = np.array([float(lse[h, t]) for t, h in rows])
    g_o = np.stack([out_np[t][h] for t, h in rows])
    PT.check_out(g_o, lse_rows, ref_o, ref_l, skip=sorted(ties))

    # fed selection defined here: own block, the previous block, block 0 and a
    # pseudo-random far block, all rows; checked on the sampled rows
    T = q.shape[0]
    tt = torch.arange(T, device="cuda", dtype=torch.int64)
    c = tt // chunk
    fed = torch.full((hq, T, topk), -1, dtype=torch.int32, device="cuda")
    hh = torch.arange(hq, device="cuda", dtype=torch.int64)[:, None]
    far = (c[None, :] * 7 + hh * 13) % torch.clamp(c[None, :], min=1)
    cand = torch.stack([torch.zeros_like(far), far, (c - 1).expand_as(far), c.expand_as(far)], dim=2)
    fed[:, :, :4] = cand.to(torch.int32)
    out3, lse3 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed)
    fed_rows = PT.host(fed[:, :, :4], np.int64)
    ref_sel3 = []
    for t, h in rows:
        cc = t // chunk
        ref_sel3.append(sorted({int(j) for j in fed_rows[h, t] if 0 <= j <= cc}))
    ref_sel3 = np.array([r + [-1] * (topk - len(r)) for r in ref_sel3])
    ref_o3, ref_l3 = oracle.attend_rows(_QView(q_rows), k_np, v_np, cu, chunk, ref_sel3, rows)
    g_o3 = np.stack([PT.host(out3[t, h], np.float32) for t, h in rows])
    g_l3 = np.array([float(lse3[h, t]) for t, h in rows])
    PT.check_out(g_o3, g_l3, ref_o3, ref_l3)


class _QView:
    """Row-indexable stand-in for q [T, Hq, d] holding only the sampled tokens."""

    def __init__(self, rows_by_t):
        self.rows = rows_by_t
        first = next(iter(rows_by_t.values()))
        self.shape = (None, first.shape[0], first.shape[1])

    def __getitem__(self, idx):
        t, h = idx
        return self.rows[int(t)][h]


def test_cuda_core_gate_above_257_blocks():
    """More than 257 blocks in one call select the CUDA-core gate (csrc/gate.cu) instead of the
    tensor-core one: its selections against the oracle's, outside the near-tie band."""
    w = W.custom("gate_267_blocks", [20000, 14000], 2, 1, 64, 128, 4, "k_offsets", 25)
    q, k, _, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, group = w.chunk_size, w.topk, w.num_q_heads // w.num_kv_heads
    p = moba.make_params(len(w.seqlens), w.total_tokens, w.num_q_heads, w.num_kv_heads,
                         w.head_dim, chunk, topk)
    assert moba.num_blocks_bound(p) > 257
    means = moba.meanpool(k, cu_t, chunk)
    sel = moba.gate_topk(q, means, cu_t, chunk, topk)
    torch.cuda.synchronize()
    q_np, k_np = PT.host(q), PT.host(k)
    om = oracle.block_means(k_np, cu, chunk)
    osel = oracle.select_blocks(q_np, om, cu, chunk, topk)
    full_sel_check(PT.host(sel, np.int64), osel, q_np, om, cu, chunk, topk, group)
