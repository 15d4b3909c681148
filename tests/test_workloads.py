"""The seeded input generator (host logic, CPU): the recipe the tests and the bench rely on.

Each check restates a property of the value recipe from the data it produced: determinism per
seed, the per-block key offsets, the planted needle blocks and the queries aimed at them, the
query offsets, and the attended-key count the decode roofline uses."""

import numpy as np
import torch

import oracle
from block_sparse_long_meanpool_b200 import workloads as W


def _block_means(x, seqlens, chunk):
    """Mean key row per (block, kv head) from the generated keys, restated here."""
    out, s = [], 0
    for n in seqlens:
        for j in range(0, n, chunk):
            out.append(x[s + j:s + min(j + chunk, n)].mean(dim=0))
        s += n
    return torch.stack(out)


def test_inputs_are_deterministic_per_seed_and_independent_across_seeds():
    w = W.custom("det", [300, 0, 257], 4, 2, 64, 128, 3, "qk_offsets", 5)
    a, b = W.make_inputs(w), W.make_inputs(w)
    c = W.make_inputs(w, seed=w.seed + 7919)
    for key in ("q", "k", "v"):
        assert a[key].dtype == torch.bfloat16 and a[key].is_contiguous()
        assert torch.equal(a[key], b[key])
        assert not torch.equal(a[key], c[key])
    assert a["q"].shape == (557, 4, 64) and a["k"].shape == (557, 2, 64)
    assert a["cu_seqlens"].tolist() == [0, 300, 300, 557] and a["cu_seqlens"].dtype == torch.int32


def test_key_offsets_shift_every_block_by_its_own_vector():
    """k = N(0,1) + a per-(block, kv head) offset ~ 0.5 N(0, I): block means spread with
    variance 0.25 + 1/B across blocks, and rows of one block share the offset."""
    w = W.custom("koff", [128 * 64], 1, 2, 64, 128, 3, "k_offsets", 6)
    x = W.make_inputs(w)
    m = _block_means(x["k"].double(), w.seqlens, 128)               # [64, 2, 64]
    var = m.var().item()
    assert 0.20 < var < 0.32, var
    # the two halves of one block see the same offset: their means agree far better than
    # the means of different blocks do
    k = x["k"].double().view(64, 128, 2, 64)
    half_gap = (k[:, :64].mean(1) - k[:, 64:].mean(1)).var().item()  # ~ 2/64 noise only
    assert half_gap < 0.06 < var
    assert abs(x["q"].double().var().item() - 1.0) < 0.05           # q untouched


def test_query_offsets_reach_about_one_row_in_ten():
    """qk_offsets: a Bernoulli(0.1) subset of query rows gets one block offset added, so the
    query variance grows by 0.1 * 0.25 on average."""
    w = W.custom("qoff", [4096], 8, 8, 64, 256, 3, "qk_offsets", 7)
    q = W.make_inputs(w)["q"].double()
    base = W.make_inputs(W.custom("qoff0", [4096], 8, 8, 64, 256, 3, "k_offsets", 7))["q"].double()
    changed = (q != base).any(dim=-1).double().mean().item()
    assert 0.08 < changed < 0.12, changed


def test_needle_blocks_and_the_queries_aimed_at_them():
    """needles: 8 distinct blocks in 1..nb-2 per sequence carry 2u (|u| = 1) on every key over
    antithetic noise (the block's second half of rows negates the first half's draws), so the
    realised block mean is 2u up to bf16 rounding; about 5% of the rows that have a needle
    strictly before their own block are set to |q| (0.8 u + 0.6 w), w orthogonal to u: cosine
    0.8 with the realised block mean, to within the bf16 rounding of q and k."""
    B, n, d = 256, 256 * 24, 128
    w = W.custom("needle", [n, n], 8, 2, d, B, 3, "needles", 8)
    x = W.make_inputs(w)
    k, q = x["k"].float(), x["q"].float()
    expect = 0.8
    planted = 0
    eligible = 0
    for s in (0, n):
        m = _block_means(k[s:s + n], [n], B)                          # [24, 2, d]
        norms = m.norm(dim=-1)                                       # ~2.1 for needles, ~0.7 else
        needle = (norms > 1.5).all(dim=1)
        idx = torch.nonzero(needle).flatten().tolist()
        assert len(idx) == 8 and min(idx) >= 1 and max(idx) <= 22, idx
        unit = m[idx] / m[idx].norm(dim=-1, keepdim=True)             # [8 needles, 2, d]
        qs = q[s:s + n] / q[s:s + n].norm(dim=-1, keepdim=True)        # [n, 8 heads, d]
        g = torch.arange(8) // 4                                     # kv head of each q head
        cos = torch.einsum("thd,jhd->thj", qs, unit[:, g])           # [n, heads, needles]
        best = cos.max(dim=-1).values
        own = torch.arange(n) // B
        has_before = (torch.tensor(idx)[None, :] < own[:, None]).any(dim=1)
        hit = best > 0.6
        assert not hit[~has_before].any()                            # only after a needle
        assert (best[hit] - expect).abs().max() < 0.01, (expect, best[hit].min(), best[hit].max())
        # the needle blocks' noise cancels: row r and row r + B/2 sum to 4u (bf16 rounding aside)
        for j in idx:
            blk = k[s + j * B:s + (j + 1) * B]
            pair = blk[:B // 2] + blk[B // 2:]
            assert (pair - pair.mean(dim=0, keepdim=True)).abs().max() < 0.05
        planted += hit.sum().item()
        eligible += has_before.sum().item() * 8
    assert 0.035 < planted / eligible < 0.065, planted / eligible


def test_decode_attended_keys_matches_the_attended_key_sets():
    """The decode roofline's key count equals the keys the last row of every sequence attends,
    from the oracle's attended-key sets with every earlier slot filled."""
    for seqlens, chunk, topk in (([700, 1, 0, 390], 128, 3), ([4500], 128, 32), ([1000, 600], 256, 8)):
        cu = np.concatenate([[0], np.cumsum(seqlens)])
        want = 0
        for b, n in enumerate(seqlens):
            if n == 0:
                continue
            t = int(cu[b + 1]) - 1
            c = (n - 1) // chunk
            sel = list(range(max(0, c - (topk - 1)), c + 1))            # any topk-1 earlier blocks
            want += len(oracle.attended_keys(t, sel, cu, chunk))
        assert W.decode_attended_keys(seqlens, chunk, topk) == want
