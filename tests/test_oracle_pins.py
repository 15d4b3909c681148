"""Pins for the float64 oracle: each check compares it with something other than itself.

Library routines it must reduce to (torch's fp64 scaled-dot-product attention
and logsumexp), brute-force enumeration, closed forms worked by hand, the
sparsity figures the analysis page prints, and invariants that hold for any
input.  All CPU, all small.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_meanpool_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(seqlens, hq, hkv, d, seed, offset=0.5, chunk=None):
    """Small float64 inputs with per-block key offsets so the gate has margins."""
    rng = np.random.default_rng(seed)
    T = sum(seqlens)
    q = rng.standard_normal((T, hq, d))
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    if chunk:
        s = 0
        for n in seqlens:
            for a in range(0, n, chunk):
                k[s + a:s + min(a + chunk, n)] += offset * rng.standard_normal((1, hkv, d))
            s += n
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    return q, k, v, cu


def sdpa_reference(q, k, v, cu, mask_fn, scale):
    """torch fp64 SDPA per sequence and head with a boolean mask (True = attend)."""
    T, hq, d = q.shape
    group = hq // k.shape[1]
    out = np.zeros_like(q)
    lse = np.zeros((hq, T))
    for i in range(len(cu) - 1):
        s, e = int(cu[i]), int(cu[i + 1])
        for h in range(hq):
            g = h // group
            qt = torch.from_numpy(q[s:e, h])[None, None]
            kt = torch.from_numpy(k[s:e, g])[None, None]
            vt = torch.from_numpy(v[s:e, g])[None, None]
            m = torch.from_numpy(mask_fn(s, e, h))
            o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
            out[s:e, h] = o[0, 0].numpy()
            z = (qt[0, 0] @ kt[0, 0].T) * scale
            lse[h, s:e] = torch.logsumexp(z.masked_fill(~m, -math.inf), dim=-1).numpy()
    return out, lse


def causal_mask(s, e, h):
    n = e - s
    return np.tril(np.ones((n, n), dtype=bool))


# ----------------------------------------------------------------------------------------
# Attention: reductions to a library routine


@pytest.mark.parametrize("hq,hkv,d,chunk", [(4, 4, 16, 8), (4, 2, 8, 5), (2, 1, 32, 16)])
def test_dense_attention_when_every_block_is_selected(hq, hkv, d, chunk):
    """Course page: with all blocks selected MoBA is exactly dense causal attention."""
    seqlens = [37, 64, 19]
    q, k, v, cu = rand_case(seqlens, hq, hkv, d, seed=1, chunk=chunk)
    nb_max = max((n + chunk - 1) // chunk for n in seqlens)
    res = oracle.moba_forward(q, k, v, cu, chunk, topk=nb_max)
    ref_o, ref_l = sdpa_reference(q, k, v, cu, causal_mask, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(res["out"], ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["lse"], ref_l, rtol=0, atol=1e-12)


def test_topk_larger_than_available_blocks_is_dense():
    q, k, v, cu = rand_case([40], 2, 2, 8, seed=2, chunk=8)
    a = oracle.moba_forward(q, k, v, cu, 8, topk=5)
    b = oracle.moba_forward(q, k, v, cu, 8, topk=50)
    np.testing.assert_array_equal(a["out"], b["out"])


def test_topk1_is_block_local_causal():
    """topk = 1 keeps only the forced current block: block-diagonal causal attention."""
    chunk = 6
    q, k, v, cu = rand_case([29, 13], 3, 3, 8, seed=3, chunk=chunk)

    def mask(s, e, h):
        pos = np.arange(e - s)
        return (pos[:, None] // chunk == pos[None, :] // chunk) & (pos[None, :] <= pos[:, None])

    ref_o, ref_l = sdpa_reference(q, k, v, cu, mask, 0.3)
    res = oracle.moba_forward(q, k, v, cu, chunk, topk=1, scale=0.3)
    np.testing.assert_allclose(res["out"], ref_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(res["lse"], ref_l, atol=1e-12, rtol=0)


def forced_selection(cu, chunk, hq, topk, choose):
    """Selection array where each row's blocks are ``choose(c)`` (sorted, deduplicated)."""
    T = int(cu[-1])
    sel = np.full((hq, T, topk), -1, dtype=np.int64)
    for i in range(len(cu) - 1):
        s, e = int(cu[i]), int(cu[i + 1])
        for t in range(s, e):
            c = (t - s) // chunk
            js = sorted({j for j in choose(c) if 0 <= j <= c})
            sel[:, t, :len(js)] = js
    return sel


@pytest.mark.parametrize("kind", ["swa", "sink"])
def test_forced_selections_reduce_to_window_and_sink(kind):
    """Analysis §2.4: always picking the nearest block is SWA; picking the first and the
    nearest block is attention sink.  Both are masked dense attention."""
    chunk = 4
    q, k, v, cu = rand_case([30, 17], 2, 1, 8, seed=4)
    choose = (lambda c: [c - 1, c]) if kind == "swa" else (lambda c: [0, c - 1, c])
    sel = forced_selection(cu, chunk, 2, 3, choose)

    def mask(s, e, h):
        pos = np.arange(e - s)
        qb, kb = pos[:, None] // chunk, pos[None, :] // chunk
        ok = (kb == qb) | (kb == qb - 1)
        if kind == "sink":
            ok |= kb == 0
        return ok & (pos[None, :] <= pos[:, None])

    res = oracle.moba_forward(q, k, v, cu, chunk, topk=3, sel=sel)
    ref_o, ref_l = sdpa_reference(q, k, v, cu, mask, 1.0 / math.sqrt(8))
    np.testing.assert_allclose(res["out"], ref_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(res["lse"], ref_l, atol=1e-12, rtol=0)


# ----------------------------------------------------------------------------------------
# Selection: brute force, invariants, hand-worked examples


def test_selection_matches_brute_force_subset_enumeration():
    """Top-(k-1) past blocks = the (k-1)-subset of past blocks with the largest score sum."""
    rng = np.random.default_rng(5)
    for trial in range(40):
        chunk = int(rng.integers(1, 4))
        L = int(rng.integers(4, 24))
        topk = int(rng.integers(1, 5))
        hq = 2
        q = rng.standard_normal((L, hq, 3))
        k = rng.standard_normal((L, 1, 3))
        cu = np.array([0, L])
        means = oracle.block_means(k, cu, chunk)
        sel = oracle.select_blocks(q, means, cu, chunk, topk)
        for t in range(L):
            c = t // chunk
            for h in range(hq):
                # block means restated from their definition: average of the block's key rows
                past = [k[j * chunk:(j + 1) * chunk, 0].mean(axis=0) for j in range(c)]
                n = min(topk - 1, c)
                best, best_set = -np.inf, ()
                for subset in itertools.combinations(range(c), n):
                    val = sum(float(q[t, h] @ past[j]) for j in subset)
                    if val > best:
                        best, best_set = val, subset
                expect = sorted(best_set) + [c] + [-1] * (topk - n - 1)
                assert list(sel[h, t]) == expect, (trial, t, h)


def test_selection_invariants():
    """Rule 1: no block after the current one; rule 2: the current block always present;
    |sel| = min(topk, c + 1); ascending, -1 padded (analysis §2.3, course page tests)."""
    chunk, topk = 16, 4
    q, k, v, cu = rand_case([200, 33, 129], 4, 2, 8, seed=6, chunk=chunk)
    sel = oracle.select_blocks(q, oracle.block_means(k, cu, chunk), cu, chunk, topk)
    for i in range(len(cu) - 1):
        s, e = int(cu[i]), int(cu[i + 1])
        for t in range(s, e):
            c = (t - s) // chunk
            for h in range(4):
                row = [int(x) for x in sel[h, t]]
                valid = [x for x in row if x >= 0]
                assert valid == sorted(set(valid))
                assert row[len(valid):] == [-1] * (topk - len(valid))
                assert max(valid) == c and c in valid
                assert len(valid) == min(topk, c + 1)


def test_selection_rows_matches_full_selection():
    chunk, topk = 8, 3
    q, k, v, cu = rand_case([70, 41], 4, 2, 8, seed=7, chunk=chunk)
    means = oracle.block_means(k, cu, chunk)
    full = oracle.select_blocks(q, means, cu, chunk, topk)
    rows = [(t, h) for t in range(0, 111, 3) for h in range(4)]
    part = oracle.select_blocks_rows(q, means, cu, chunk, topk, rows)
    for r, (t, h) in enumerate(rows):
        assert list(part[r]) == list(full[h, t])


def test_hand_worked_example():
    """d = 1, one head, chunk 2, topk 2, scale 1.

    K = [1, 3, 5, 7, 2, 2] gives block means 2, 6, 2.  The query at t = 4 is in block 2.
    q = +1: past scores (2, 6), block 1 wins -> blocks {1, 2}, keys 2, 3, 4 with logits 5, 7, 2.
    q = -1: past scores (-2, -6), block 0 wins -> blocks {0, 2}, keys 0, 1, 4 with logits -1, -3, -2.
    q =  0: both scores 0, a tie -> the lower block 0 wins.
    With V = [10, 20, 30, 40, 50, 60]: out = sum(e^z v) / sum(e^z), lse = log sum(e^z).
    """
    kk = np.array([1, 3, 5, 7, 2, 2], dtype=np.float64).reshape(6, 1, 1)
    vv = np.array([10, 20, 30, 40, 50, 60], dtype=np.float64).reshape(6, 1, 1)
    cu = np.array([0, 6])
    np.testing.assert_array_equal(oracle.block_means(kk, cu, 2)[:, 0, 0], [2.0, 6.0, 2.0])
    for qv, blocks, keys in [(1.0, [1, 2], [2, 3, 4]), (-1.0, [0, 2], [0, 1, 4]), (0.0, [0, 2], [0, 1, 4])]:
        qq = np.zeros((6, 1, 1))
        qq[4, 0, 0] = qv
        res = oracle.moba_forward(qq, kk, vv, cu, 2, topk=2, scale=1.0)
        assert list(res["sel"][0, 4]) == blocks
        z = [qv * kk[u, 0, 0] for u in keys]
        w = [math.exp(x) for x in z]
        expect_out = sum(wi * vv[u, 0, 0] for wi, u in zip(w, keys)) / sum(w)
        assert res["out"][4, 0, 0] == pytest.approx(expect_out, abs=1e-12)
        assert res["lse"][0, 4] == pytest.approx(math.log(sum(w)), abs=1e-12)
    # first block rows attend only their causal prefix: t = 1 sees keys 0, 1
    qq = np.ones((6, 1, 1))
    res = oracle.moba_forward(qq, kk, vv, cu, 2, topk=2, scale=1.0)
    w = [math.exp(1.0), math.exp(3.0)]
    assert res["out"][1, 0, 0] == pytest.approx((10 * w[0] + 20 * w[1]) / sum(w), abs=1e-12)
    assert res["out"][0, 0, 0] == pytest.approx(10.0, abs=1e-12)
    assert res["lse"][0, 0] == pytest.approx(1.0, abs=1e-12)


def test_printed_sparsity_figures_fix_that_topk_counts_the_current_block():
    """The analysis prints 81.25% (8K, 512, top-3), 95.31% (32K, 512, top-3) and
    12 of 256 history blocks (1M, 4096, top-12).  A query in the last block must
    therefore attend exactly topk blocks including its own."""
    with open(os.path.join(GOLDEN, "sparsity.json")) as f:
        cases = json.load(f)["cases"]
    rng = np.random.default_rng(8)
    for case in cases:
        L, chunk, topk = case["seqlen"], case["chunk"], case["topk"]
        nb = L // chunk
        k = rng.standard_normal((L, 1, 1))
        q = rng.standard_normal((L, 1, 1))
        cu = np.array([0, L])
        means = oracle.block_means(k, cu, chunk)
        row = oracle.select_blocks_rows(q, means, cu, chunk, topk, [(L - 1, 0)])[0]
        attended = int((row >= 0).sum())
        assert round(1.0 - attended / nb, 4) == round(case["sparsity"], 4), case


def test_partial_final_block_never_decides_a_selection():
    """The last (partial) block is always the current or a future block, so changing its
    keys leaves every selection as it was."""
    chunk, topk = 10, 3
    q, k, v, cu = rand_case([57, 23], 2, 2, 4, seed=9, chunk=chunk)
    sel_a = oracle.select_blocks(q, oracle.block_means(k, cu, chunk), cu, chunk, topk)
    k2 = k.copy()
    k2[50:57] += 100.0
    k2[80 - 3:80] -= 50.0
    sel_b = oracle.select_blocks(q, oracle.block_means(k2, cu, chunk), cu, chunk, topk)
    np.testing.assert_array_equal(sel_a, sel_b)


# ----------------------------------------------------------------------------------------
# Means: closed forms


def test_means_closed_forms():
    """Constant rows average to the constant; rows 1..n average to (n + 1) / 2; a partial
    final block averages only its valid rows."""
    L, chunk = 23, 8
    k = np.zeros((L, 2, 3))
    k[:, 0, :] = 4.25
    k[:, 1, 0] = np.arange(L)
    k[:, 1, 1] = np.arange(L) ** 2
    means = oracle.block_means(k, np.array([0, L]), chunk)
    assert means.shape == (3, 2, 3)
    np.testing.assert_array_equal(means[:, 0, :], 4.25)
    np.testing.assert_allclose(means[:, 1, 0], [3.5, 11.5, 19.0])  # rows 0-7, 8-15, 16-22
    # sum of squares closed form: (b(b+1)(2b+1) - a(a-1)(2a-1)) / 6 over rows a..b
    sq = lambda a, b: (b * (b + 1) * (2 * b + 1) - (a - 1) * a * (2 * a - 1)) / 6
    np.testing.assert_allclose(means[:, 1, 1], [sq(0, 7) / 8, sq(8, 15) / 8, sq(16, 22) / 7])


# ----------------------------------------------------------------------------------------
# Invariances and structure


def test_key_shift_leaves_selection_and_output_and_shifts_lse():
    chunk, topk, d = 8, 3, 8
    q, k, v, cu = rand_case([64, 30], 2, 2, d, seed=10, chunk=chunk)
    shift = np.random.default_rng(11).standard_normal(d)
    a = oracle.moba_forward(q, k, v, cu, chunk, topk)
    b = oracle.moba_forward(q, k + shift, v, cu, chunk, topk)
    np.testing.assert_array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(a["out"], b["out"], atol=1e-11, rtol=0)
    expect = a["lse"] + (q @ shift).T / math.sqrt(d)
    np.testing.assert_allclose(b["lse"], expect, atol=1e-11, rtol=0)


def test_value_shift_shifts_output():
    chunk, topk = 8, 3
    q, k, v, cu = rand_case([64], 2, 1, 4, seed=12, chunk=chunk)
    shift = np.array([1.5, -2.0, 0.25, 3.0])
    a = oracle.moba_forward(q, k, v, cu, chunk, topk)
    b = oracle.moba_forward(q, k, v + shift, cu, chunk, topk)
    np.testing.assert_allclose(b["out"], a["out"] + shift, atol=1e-12, rtol=0)
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_gqa_equals_mha_with_repeated_kv_heads():
    chunk, topk = 8, 3
    q, k, v, cu = rand_case([50, 21], 4, 2, 8, seed=13, chunk=chunk)
    a = oracle.moba_forward(q, k, v, cu, chunk, topk)
    b = oracle.moba_forward(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1), cu, chunk, topk)
    np.testing.assert_array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(a["out"], b["out"], atol=1e-13, rtol=0)


def test_packed_varlen_equals_separate_sequences():
    chunk, topk = 8, 3
    seqlens = [45, 8, 27]
    q, k, v, cu = rand_case(seqlens, 2, 2, 8, seed=14, chunk=chunk)
    packed = oracle.moba_forward(q, k, v, cu, chunk, topk)
    for i in range(len(seqlens)):
        s, e = int(cu[i]), int(cu[i + 1])
        one = oracle.moba_forward(q[s:e], k[s:e], v[s:e], np.array([0, e - s]), chunk, topk)
        np.testing.assert_array_equal(one["sel"], packed["sel"][:, s:e])
        np.testing.assert_allclose(one["out"], packed["out"][s:e], atol=1e-13, rtol=0)
        np.testing.assert_allclose(one["lse"], packed["lse"][:, s:e], atol=1e-13, rtol=0)


def test_two_formulations_agree():
    """Masked dense (all rows) and per-row gather must give the same numbers."""
    chunk, topk = 8, 3
    q, k, v, cu = rand_case([61, 35], 4, 2, 8, seed=15, chunk=chunk)
    res = oracle.moba_forward(q, k, v, cu, chunk, topk)
    rows = [(t, h) for t in range(96) for h in range(4)]
    o, l = oracle.attend_rows(q, k, v, cu, chunk, res["sel"], rows)
    for r, (t, h) in enumerate(rows):
        np.testing.assert_allclose(o[r], res["out"][t, h], atol=1e-12, rtol=0)
        assert abs(l[r] - res["lse"][h, t]) < 1e-12


def test_softmax_weights_sum_to_one_and_lse_bounds():
    """Output lies in the convex hull of attended values; max logit <= lse <= max + log(n)."""
    chunk, topk = 8, 3
    q, k, v, cu = rand_case([64], 2, 2, 4, seed=16, chunk=chunk)
    v1 = np.ones_like(v)
    res = oracle.moba_forward(q, k, v1, cu, chunk, topk)
    np.testing.assert_allclose(res["out"], 1.0, atol=1e-13)
    for t in range(0, 64, 5):
        for h in range(2):
            u = oracle.attended_keys(t, res["sel"][h, t], cu, chunk)
            z = (k[u, h] @ q[t, h]) / 2.0
            assert z.max() - 1e-12 <= res["lse"][h, t] <= z.max() + math.log(len(u)) + 1e-12


def test_future_block_in_a_fed_selection_is_rejected():
    with pytest.raises(ValueError):
        oracle.attended_keys(1, [0, 1], np.array([0, 8]), 2)


# ----------------------------------------------------------------------------------------
# The measurement formula, against the oracle's attended key sets


@pytest.mark.parametrize("seqlens,chunk,topk", [([37, 64, 19], 8, 3), ([100], 16, 5), ([7], 4, 2)])
def test_selected_block_flops_counts_attended_keys(seqlens, chunk, topk):
    hq, d = 3, 4
    q, k, v, cu = rand_case(seqlens, hq, 1, d, seed=17, chunk=chunk)
    sel = oracle.select_blocks(q, oracle.block_means(k, cu, chunk), cu, chunk, topk)
    n = 0
    for t in range(int(cu[-1])):
        for h in range(hq):
            n += len(oracle.attended_keys(t, sel[h, t], cu, chunk))
    assert W.selected_block_flops(seqlens, hq, d, chunk, topk) == 4 * d * n


# ----------------------------------------------------------------------------------------
# Decode step: the same rule applied to the last row of every cache


def _decode_inputs(seqlens, hq, hkv, d, seed):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    T = int(cu[-1])
    q = rng.standard_normal((T, hq, d))
    k = rng.standard_normal((T, hkv, d)) + 0.5 * rng.standard_normal((1, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    q_new = np.stack([q[cu[b + 1] - 1] if seqlens[b] > 0 else np.zeros((hq, d))
                      for b in range(len(seqlens))])
    return cu, q, k, v, q_new


@pytest.mark.parametrize("seqlens,hq,hkv,chunk,topk", [
    ([700, 0, 600, 1], 4, 2, 128, 3),        # empty and 1-token caches, partial blocks
    ([1024, 385], 2, 2, 128, 4),            # a full last block, MHA
    ([2000], 6, 2, 256, 2),                 # odd GQA group
])
def test_decode_equals_prefill_last_rows(seqlens, hq, hkv, chunk, topk):
    """Decode (row-wise gather) equals the prefill forward's last row of every sequence
    (masked-dense formulation), selections included."""
    cu, q, k, v, q_new = _decode_inputs(seqlens, hq, hkv, 16, 40 + len(seqlens))
    full = oracle.moba_forward(q, k, v, cu, chunk, topk)
    dec = oracle.moba_decode(q_new, k, v, cu, chunk, topk)
    for b, n in enumerate(seqlens):
        if n == 0:
            assert np.all(dec["out"][b] == 0) and np.all(np.isneginf(dec["lse"][:, b]))
            assert np.all(dec["sel"][b] == -1)
            continue
        t = int(cu[b + 1]) - 1
        np.testing.assert_allclose(dec["out"][b], full["out"][t], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dec["lse"][:, b], full["lse"][:, t], rtol=0, atol=1e-12)
        assert np.array_equal(dec["sel"][b], full["sel"][:, t])


def test_decode_with_every_block_selected_is_dense_attention_of_the_last_row():
    """topk >= blocks: the new query attends to its whole cache (torch fp64 SDPA)."""
    seqlens, hq, hkv, d = [900, 333], 4, 2, 16
    cu, q, k, v, q_new = _decode_inputs(seqlens, hq, hkv, d, 7)
    dec = oracle.moba_decode(q_new, k, v, cu, 128, 16)
    scale = 1.0 / math.sqrt(d)
    for b in range(len(seqlens)):
        s, e = int(cu[b]), int(cu[b + 1])
        for h in range(hq):
            g = h // (hq // hkv)
            qt = torch.from_numpy(q_new[b, h])[None, None, None]
            kt = torch.from_numpy(k[s:e, g])[None, None]
            vt = torch.from_numpy(v[s:e, g])[None, None]
            o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
            z = (kt[0, 0] @ qt[0, 0, 0]) * scale
            np.testing.assert_allclose(dec["out"][b, h], o[0, 0, 0].numpy(), rtol=0, atol=1e-12)
            assert abs(dec["lse"][h, b] - torch.logsumexp(z, 0).item()) < 1e-12


# ---- min/max (Quest-style) gate: block_minmax, minmax_scores_row, moba_decode(gate="minmax")

def _corner_max(q_row, lo, hi):
    """max of <q, x> over the box lo <= x <= hi, by enumerating its 2^d corners."""
    best = -np.inf
    for pick in itertools.product((0, 1), repeat=len(q_row)):
        x = np.where(np.array(pick) == 1, hi, lo)
        best = max(best, float(np.dot(q_row, x)))
    return best


def test_minmax_score_is_the_largest_inner_product_over_the_box():
    """The score equals the maximum of <q, x> over the box's corners (a linear function
    peaks at a corner), bounds <q, k> of every key of the block from above, and equals
    <q, k> for a one-token block."""
    rng = np.random.default_rng(11)
    for trial in range(60):
        d = int(rng.integers(1, 6))
        n = int(rng.integers(1, 7))
        keys = rng.standard_normal((n, 1, d))
        q = rng.standard_normal(d)
        q[rng.random(d) < 0.2] = 0.0
        kmin, kmax = oracle.block_minmax(keys, np.array([0, n]), n)
        s = oracle.minmax_scores_row(q, np.stack([kmin[:, 0], kmax[:, 0]], axis=1))[0]
        assert abs(s - _corner_max(q, kmin[0, 0], kmax[0, 0])) < 1e-12, trial
        assert s >= max(float(q @ keys[i, 0]) for i in range(n)) - 1e-12
        if n == 1:
            assert abs(s - float(q @ keys[0, 0])) < 1e-12


def test_block_minmax_closed_forms():
    """Keys linear in the position inside their sequence: each channel's minimum and
    maximum sit at the block's first or last valid row, by the sign of the slope; the
    partial final block and a one-token block included."""
    seqlens, chunk, hkv, d = [23, 1, 16], 8, 2, 3
    cu = np.concatenate([[0], np.cumsum(seqlens)])
    slope = np.array([[1.5, -2.0, 0.0], [-0.25, 3.0, 1.0]])
    off = np.array([[0.5, 1.0, -7.0], [2.0, -1.0, 0.0]])
    k = np.zeros((int(cu[-1]), hkv, d))
    for b, n in enumerate(seqlens):
        for p in range(n):
            k[cu[b] + p] = slope * p + off
    kmin, kmax = oracle.block_minmax(k, cu, chunk)
    blk = 0
    for b, n in enumerate(seqlens):
        for j in range(-(-n // chunk)):
            first, last = j * chunk, min((j + 1) * chunk, n) - 1
            a, z = slope * first + off, slope * last + off
            np.testing.assert_array_equal(kmin[blk], np.minimum(a, z))
            np.testing.assert_array_equal(kmax[blk], np.maximum(a, z))
            blk += 1
    assert blk == kmin.shape[0] == 3 + 1 + 2


def test_minmax_decode_selection_matches_brute_force():
    """Decode with the min/max gate routes the (k-1)-subset of earlier blocks with the
    largest sum of box maxima (block summaries restated from the keys, scores from the
    corners), over varlen caches, GQA and empty caches."""
    rng = np.random.default_rng(12)
    for trial in range(25):
        hq, hkv, d = 4, 2, 3
        chunk = int(rng.integers(1, 5))
        seqlens = [int(x) for x in rng.integers(0, 20, size=3)]
        topk = int(rng.integers(1, 5))
        cu, q, k, v, q_new = _decode_inputs(seqlens, hq, hkv, d, 100 + trial)
        dec = oracle.moba_decode(q_new, k, v, cu, chunk, topk, gate="minmax")
        for b, n in enumerate(seqlens):
            if n == 0:
                assert np.all(dec["sel"][b] == -1)
                continue
            s = int(cu[b])
            c = (n - 1) // chunk
            for h in range(hq):
                g = h // (hq // hkv)
                score = []
                for j in range(c):
                    rows = k[s + j * chunk:s + (j + 1) * chunk, g]
                    score.append(_corner_max(q_new[b, h], rows.min(axis=0), rows.max(axis=0)))
                m = min(topk - 1, c)
                best, best_set = -np.inf, ()
                for subset in itertools.combinations(range(c), m):
                    val = sum(score[j] for j in subset)
                    if val > best:
                        best, best_set = val, subset
                expect = sorted(best_set) + [c] + [-1] * (topk - m - 1)
                assert list(dec["sel"][b, h]) == expect, (trial, b, h)


def test_minmax_gate_finds_the_single_matching_key_the_mean_dilutes():
    """The case the analysis (§5.1 item 6) gives for a stronger summary: block 1 holds one
    key aligned with q among zeros, so its mean (4/16) loses to block 0's uniform 0.5 while
    its box maximum (4) wins.  The output is softmax attention over blocks {1, 3} (torch
    fp64 SDPA)."""
    chunk, d = 16, 2
    k = np.zeros((53, 1, d))
    k[0:16, 0] = [0.5, 0.0]
    k[16 + 7, 0] = [4.0, 0.0]
    k[32:48, 0] = [-1.0, 0.0]
    k[48:53, 0] = [0.0, 1.0]
    v = np.random.default_rng(3).standard_normal((53, 1, d))
    cu = np.array([0, 53])
    q_new = np.array([[[1.0, 0.0]]])
    mean_dec = oracle.moba_decode(q_new, k, v, cu, chunk, 2)
    mm_dec = oracle.moba_decode(q_new, k, v, cu, chunk, 2, gate="minmax")
    assert list(mean_dec["sel"][0, 0]) == [0, 3]
    assert list(mm_dec["sel"][0, 0]) == [1, 3]
    keys = np.r_[16:32, 48:53]
    qt = torch.tensor(q_new[0, 0])[None, None, None]
    kt = torch.from_numpy(k[keys, 0])[None, None]
    vt = torch.from_numpy(v[keys, 0])[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=1 / math.sqrt(d))
    np.testing.assert_allclose(mm_dec["out"][0, 0], o[0, 0, 0].numpy(), rtol=0, atol=1e-12)


def test_minmax_decode_with_every_block_selected_equals_the_mean_gate():
    """topk >= blocks: the gate decides nothing, so both summaries give the same step."""
    cu, q, k, v, q_new = _decode_inputs([300, 77, 0], 4, 1, 8, 9)
    a = oracle.moba_decode(q_new, k, v, cu, 32, 16)
    b = oracle.moba_decode(q_new, k, v, cu, 32, 16, gate="minmax")
    assert np.array_equal(a["sel"], b["sel"])
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_minmax_score_is_the_centre_radius_contraction():
    """For either sign of q_i, max(q_i lo_i, q_i hi_i) = q_i (lo_i + hi_i)/2 + |q_i| (hi_i - lo_i)/2,
    so the min/max score is the length-2d product of [q, |q|] with [centre; radius] (torch fp64
    matmul over all blocks at once)."""
    rng = np.random.default_rng(13)
    k = rng.standard_normal((700, 3, 16)) + rng.standard_normal((1, 3, 16))
    cu = np.array([0, 300, 700])
    kmin, kmax = oracle.block_minmax(k, cu, 64)
    q = rng.standard_normal((5, 16))
    q[:, :3] = 0.0
    for g in range(3):
        centre = torch.from_numpy((kmin[:, g] + kmax[:, g]) / 2)
        radius = torch.from_numpy((kmax[:, g] - kmin[:, g]) / 2)
        lhs = torch.cat([torch.from_numpy(q), torch.from_numpy(np.abs(q))], dim=1)
        rhs = torch.cat([centre, radius], dim=1)
        want = (lhs @ rhs.T).numpy()
        for r in range(q.shape[0]):
            got = oracle.minmax_scores_row(q[r], np.stack([kmin[:, g], kmax[:, g]], axis=1))
            np.testing.assert_allclose(got, want[r], rtol=1e-13, atol=1e-12)


def test_minmax_score_is_the_positive_negative_part_contraction():
    """max(q_i lo_i, q_i hi_i) = max(q_i, 0) hi_i + min(q_i, 0) lo_i (lo_i <= hi_i), so the
    min/max score is the length-2d product of [q+, q-] with [kmax; kmin], whose operands are
    the bf16 inputs themselves (torch fp64 matmul over all blocks at once; zeros included)."""
    rng = np.random.default_rng(14)
    k = rng.standard_normal((600, 2, 16)) * 3 + rng.standard_normal((1, 2, 16))
    cu = np.array([0, 100, 600])
    kmin, kmax = oracle.block_minmax(k, cu, 48)
    q = rng.standard_normal((6, 16))
    q[:, :4] = 0.0
    q[0] = np.abs(q[0])   # all non-negative
    q[1] = -np.abs(q[1])  # all non-positive
    for g in range(2):
        lhs = torch.cat([torch.from_numpy(np.maximum(q, 0)), torch.from_numpy(np.minimum(q, 0))], dim=1)
        rhs = torch.cat([torch.from_numpy(kmax[:, g]), torch.from_numpy(kmin[:, g])], dim=1)
        want = (lhs @ rhs.T).numpy()
        for r in range(q.shape[0]):
            got = oracle.minmax_scores_row(q[r], np.stack([kmin[:, g], kmax[:, g]], axis=1))
            np.testing.assert_allclose(got, want[r], rtol=1e-13, atol=1e-12)


# ---- backward: moba_backward (dq, dk, dv for the forward's selection)

def _bw_case(seqlens, hq, hkv, d, chunk, topk, seed):
    cu, q, k, v, _ = _decode_inputs(seqlens, hq, hkv, d, seed)
    rng = np.random.default_rng(seed + 1000)
    fwd = oracle.moba_forward(q, k, v, cu, chunk, topk)
    d_out = rng.standard_normal(q.shape)
    d_lse = rng.standard_normal((hq, q.shape[0]))
    return cu, q, k, v, fwd, d_out, d_lse


def _autograd_masked(q, k, v, cu, chunk, sel, d_out, d_lse, scale):
    """torch fp64 autograd through the library's masked SDPA and logsumexp, with the mask
    built from the attended key sets (KV heads repeated for GQA; autograd sums them back)."""
    T, hq, d = q.shape
    group = hq // k.shape[1]
    allowed = torch.zeros((hq, T, T), dtype=torch.bool)
    for h in range(hq):
        for t in range(T):
            allowed[h, t, torch.from_numpy(oracle.attended_keys(t, sel[h, t], cu, chunk))] = True
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kr = kt.repeat_interleave(group, dim=1).transpose(0, 1)
    vr = vt.repeat_interleave(group, dim=1).transpose(0, 1)
    qh = qt.transpose(0, 1)
    out = torch.nn.functional.scaled_dot_product_attention(qh, kr, vr, attn_mask=allowed, scale=scale)
    z = (qh @ kr.transpose(1, 2)) * scale
    lse = torch.logsumexp(z.masked_fill(~allowed, float("-inf")), dim=-1)
    loss = (out.transpose(0, 1) * torch.from_numpy(d_out)).sum() + (lse * torch.from_numpy(d_lse)).sum()
    loss.backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("seqlens,hq,hkv,d,chunk,topk", [
    ([37, 0, 50, 1], 4, 2, 8, 8, 3),     # varlen GQA, empty and 1-token sequences, partial blocks
    ([64], 2, 2, 16, 16, 2),             # MHA
    ([45, 30], 6, 2, 4, 5, 4),           # odd group, chunk not a power of two
])
def test_backward_matches_autograd_of_masked_attention(seqlens, hq, hkv, d, chunk, topk):
    cu, q, k, v, fwd, d_out, d_lse = _bw_case(seqlens, hq, hkv, d, chunk, topk, 21 + hq)
    scale = 1.0 / math.sqrt(d)
    got = oracle.moba_backward(q, k, v, cu, chunk, fwd["sel"], d_out, d_lse)
    want = _autograd_masked(q, k, v, cu, chunk, fwd["sel"], d_out, d_lse, scale)
    for g, w_ in zip(got, want):
        np.testing.assert_allclose(g, w_, rtol=1e-10, atol=1e-12)


def test_backward_with_every_block_selected_is_causal_attention_backward():
    """topk >= blocks: the gradients of torch's fp64 causal SDPA (no mask built by the test)."""
    seqlens, hq, d = [70], 2, 8
    cu, q, k, v, fwd, d_out, _ = _bw_case(seqlens, hq, hq, d, 16, 8, 5)
    dq, dk, dv = oracle.moba_backward(q, k, v, cu, 16, fwd["sel"], d_out)
    qt, kt, vt = (torch.tensor(x.transpose(1, 0, 2), requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    (out * torch.from_numpy(d_out.transpose(1, 0, 2))).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy().transpose(1, 0, 2), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy().transpose(1, 0, 2), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy().transpose(1, 0, 2), rtol=1e-10, atol=1e-12)


def test_backward_matches_finite_differences_of_the_forward():
    """Central differences of L = <d_out, out> + <d_lse, lse> through the oracle's own forward
    with the selection held fixed."""
    cu, q, k, v, fwd, d_out, d_lse = _bw_case([23, 17], 4, 2, 4, 4, 3, 8)
    sel = fwd["sel"]
    grads = oracle.moba_backward(q, k, v, cu, 4, sel, d_out, d_lse)

    def loss(qq, kk, vv):
        o, l = oracle.attention_masked_dense(qq, kk, vv, cu, 4, sel)
        return float((o * d_out).sum() + (l * d_lse).sum())

    rng = np.random.default_rng(9)
    eps = 1e-6
    for which, x in enumerate((q, k, v)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grads[which][idx]) < 1e-6 * max(1.0, abs(fd)), (which, idx, fd, grads[which][idx])


def test_backward_closed_form_sums():
    """Softmax weights sum to one, so per KV head the value gradients sum to the sum of d_out
    over the rows that read it, and the key gradients sum to scale * sum of d_lse * q (zero
    without d_lse)."""
    seqlens, hq, hkv, d = [40, 25], 4, 2, 8
    cu, q, k, v, fwd, d_out, d_lse = _bw_case(seqlens, hq, hkv, d, 8, 3, 12)
    scale = 1.0 / math.sqrt(d)
    group = hq // hkv
    _, dk0, dv0 = oracle.moba_backward(q, k, v, cu, 8, fwd["sel"], d_out)
    _, dk1, _ = oracle.moba_backward(q, k, v, cu, 8, fwd["sel"], d_out, d_lse)
    for g in range(hkv):
        hs = list(range(g * group, (g + 1) * group))
        np.testing.assert_allclose(dv0[:, g].sum(axis=0), d_out[:, hs].sum(axis=(0, 1)), atol=1e-11)
        np.testing.assert_allclose(dk0[:, g].sum(axis=0), 0.0, atol=1e-11)
        want = scale * sum((d_lse[h][:, None] * q[:, h]).sum(axis=0) for h in hs)
        np.testing.assert_allclose(dk1[:, g].sum(axis=0), want, atol=1e-11)


def test_backward_gqa_equals_mha_with_repeated_kv_heads():
    cu, q, k, v, fwd, d_out, d_lse = _bw_case([30, 21], 4, 2, 8, 8, 3, 14)
    dq, dk, dv = oracle.moba_backward(q, k, v, cu, 8, fwd["sel"], d_out, d_lse)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    dq2, dk2, dv2 = oracle.moba_backward(q, kr, vr, cu, 8, fwd["sel"], d_out, d_lse)
    np.testing.assert_allclose(dq, dq2, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(dk2.shape[0], 2, 2, -1).sum(axis=2), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(dv2.shape[0], 2, 2, -1).sum(axis=2), atol=1e-13)
