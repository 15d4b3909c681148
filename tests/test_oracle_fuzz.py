"""Property-based checks of the oracle over random shapes (CPU; hypothesis).

The pins in test_oracle_pins.py use chosen shapes; these draw the shapes (ragged and empty
sequences, block sizes that do and do not divide the lengths, GQA groups, topk below and above
the block count) and check the relations that must hold for every one of them: the two
attention formulations agree, the selection rules hold for both gates, the decode step equals
the prefill's last rows, and the backward's closed-form sums."""

import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    batch = draw(st.integers(1, 3))
    seqlens = draw(st.lists(st.integers(0, 40), min_size=batch, max_size=batch))
    if sum(seqlens) == 0:
        seqlens[0] = draw(st.integers(1, 40))
    hkv = draw(st.integers(1, 2))
    hq = hkv * draw(st.integers(1, 3))
    d = draw(st.integers(1, 8))
    chunk = draw(st.integers(1, 9))
    topk = draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    T = int(cu[-1])
    q = rng.standard_normal((T, hq, d))
    k = rng.standard_normal((T, hkv, d)) + rng.standard_normal((1, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    return dict(seqlens=seqlens, cu=cu, q=q, k=k, v=v, chunk=chunk, topk=topk, rng=rng)


def _check_selection(sel_row, c, topk):
    valid = [int(x) for x in sel_row if x >= 0]
    assert valid == sorted(set(valid))
    assert list(sel_row[len(valid):]) == [-1] * (topk - len(valid))
    assert c in valid and max(valid) == c
    assert len(valid) == min(topk, c + 1)


@SETTINGS
@given(problems())
def test_formulations_agree_and_selection_rules_hold(p):
    q, k, v, cu, chunk, topk = p["q"], p["k"], p["v"], p["cu"], p["chunk"], p["topk"]
    res = oracle.moba_forward(q, k, v, cu, chunk, topk)
    hq = q.shape[1]
    rows = [(t, h) for t in range(q.shape[0]) for h in range(hq)]
    o, l = oracle.attend_rows(q, k, v, cu, chunk, res["sel"], rows)
    for r, (t, h) in enumerate(rows):
        np.testing.assert_allclose(o[r], res["out"][t, h], atol=1e-11, rtol=0)
        assert abs(l[r] - res["lse"][h, t]) < 1e-11
        i = int(np.searchsorted(cu, t, side="right") - 1)
        _check_selection(res["sel"][h, t], (t - int(cu[i])) // chunk, topk)
    rs = oracle.select_blocks_rows(q, res["means"], cu, chunk, topk, rows)
    assert np.array_equal(rs, np.stack([res["sel"][h, t] for t, h in rows]))


@SETTINGS
@given(problems())
def test_decode_is_the_prefill_last_row_and_minmax_follows_the_rules(p):
    q, k, v, cu, chunk, topk = p["q"], p["k"], p["v"], p["cu"], p["chunk"], p["topk"]
    seqlens = p["seqlens"]
    q_new = np.stack([q[cu[b + 1] - 1] if n > 0 else np.zeros(q.shape[1:]) for b, n in enumerate(seqlens)])
    full = oracle.moba_forward(q, k, v, cu, chunk, topk)
    dec = oracle.moba_decode(q_new, k, v, cu, chunk, topk)
    mm = oracle.moba_decode(q_new, k, v, cu, chunk, topk, gate="minmax")
    for b, n in enumerate(seqlens):
        if n == 0:
            for r in (dec, mm):
                assert np.all(r["out"][b] == 0) and np.all(np.isneginf(r["lse"][:, b]))
                assert np.all(r["sel"][b] == -1)
            continue
        t = int(cu[b + 1]) - 1
        np.testing.assert_allclose(dec["out"][b], full["out"][t], atol=1e-11, rtol=0)
        np.testing.assert_allclose(dec["lse"][:, b], full["lse"][:, t], atol=1e-11, rtol=0)
        assert np.array_equal(dec["sel"][b], full["sel"][:, t])
        c = (n - 1) // chunk
        for h in range(q.shape[1]):
            _check_selection(mm["sel"][b, h], c, topk)


@SETTINGS
@given(problems())
def test_backward_closed_form_sums(p):
    q, k, v, cu, chunk, topk, rng = p["q"], p["k"], p["v"], p["cu"], p["chunk"], p["topk"], p["rng"]
    T, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    res = oracle.moba_forward(q, k, v, cu, chunk, topk)
    d_out = rng.standard_normal(q.shape)
    d_lse = rng.standard_normal((hq, T))
    scale = 1.0 / math.sqrt(d)
    _, dk, dv = oracle.moba_backward(q, k, v, cu, chunk, res["sel"], d_out, d_lse)
    for g in range(hkv):
        hs = list(range(g * group, (g + 1) * group))
        np.testing.assert_allclose(dv[:, g].sum(axis=0), d_out[:, hs].sum(axis=(0, 1)), atol=1e-9)
        want = scale * sum((d_lse[h][:, None] * q[:, h]).sum(axis=0) for h in hs)
        np.testing.assert_allclose(dk[:, g].sum(axis=0), want, atol=1e-9)
