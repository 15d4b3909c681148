"""CPU checks of the GPU parity helpers themselves (tests/parity.py): the selection rule that
decides which GPU rows count as valid near-tie alternatives must reject every other kind of
difference."""

import numpy as np

import parity as PT


def test_near_tie_rule_rejects_planted_mistakes():
    """The near-tie rule of the selection check, on hand-made rows: a swap inside the band
    passes; a swap outside it, a duplicated block, a missing own block, an unsorted row, a
    future block and bad padding fail."""
    scores = np.array([5.0, 1.0, 3.0, 2.9999, 0.5])   # blocks 0..4 of a row with c = 5
    ref = [0, 2, 5]                                    # topk 3: the best 2 routed + own block
    assert PT.near_tie_alternative([0, 3, 5], ref, scores, 5, 3)   # 3 for 2: within 1e-3
    for bad in ([0, 1, 5],        # 1 for 2: far outside the band
                [2, 2, 5],        # duplicate
                [0, 2, 4],        # own block missing
                [2, 0, 5],        # not ascending
                [0, 6, 5]):       # a future block
        assert not PT.near_tie_alternative(bad, ref, scores, 5, 3), bad
    # c = 2 with topk 4: both past blocks routed, then the own block, then -1
    sc2 = np.array([1.0, 2.0])
    assert PT.near_tie_alternative([0, 1, 2, -1], [0, 1, 2, -1], sc2, 2, 4)
    assert not PT.near_tie_alternative([0, 1, 2, 3], [0, 1, 2, -1], sc2, 2, 4)


def test_well_formed_rows():
    assert PT.well_formed([1, 3, 4], 4, 3)
    assert PT.well_formed([0, -1, -1], 0, 3)           # block 0: own block only
    assert not PT.well_formed([0, 4, -1, -1], 4, 4)    # too few routed blocks for c = 4
    assert not PT.well_formed([1, 3, 4, 4], 4, 3)      # own block repeated


def test_check_selection_counts_ties_and_fails_otherwise():
    """check_selection on two rows of a tiny problem: an equal-score swap is a tie; a swap of
    a clearly better block fails."""
    import pytest
    q = np.zeros((3000, 1, 2))
    q[:, 0, 0] = 1.0
    means = np.zeros((4, 1, 2))
    means[:, 0, 0] = [1.0, 1.0, 0.5, 0.0]              # blocks 0 and 1 tie, 2 is worse
    cu = [0, 3000]
    rows = [(2500, 0)]                                  # c = 3 with chunk 800 (blocks 0, 1, 2 past)
    ref = np.array([[0, 3, -1]])                        # topk 3: one routed block + own
    ties = PT.check_selection(np.array([[1, 3, -1]]), ref, rows, q, means, cu, 800, 2, 1)
    assert ties == {0}
    with pytest.raises(AssertionError):
        PT.check_selection(np.array([[2, 3, -1]]), ref, rows, q, means, cu, 800, 2, 1)


def test_oracle_pool_pieces_equal_the_whole_oracle():
    """The parallel checker only splits the oracle's work: every driver of oracle_pool gives the
    oracle's own result on a small ragged GQA problem (spawned workers, as on the GPU machine)."""
    import oracle
    import oracle_pool as OP

    rng = np.random.default_rng(5)
    T, hq, hkv, d, chunk, topk = 420, 4, 2, 16, 64, 3
    cu = [0, 250, 250, 420]
    to_bf16 = lambda a: PT.from_bits((a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
    q = to_bf16(rng.standard_normal((T, hq, d)))
    k = to_bf16(rng.standard_normal((T, hkv, d)))
    v = to_bf16(rng.standard_normal((T, hkv, d)))
    bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    ref = oracle.moba_forward(q, k, v, cu, chunk, topk)
    rows = [(t, h) for t in range(0, T, 7) for h in range(hq)]
    ts = np.array([t for t, _ in rows])
    hs = np.array([h for _, h in rows])
    sel_rows = ref["sel"][hs, ts]
    do = rng.standard_normal((T, hq, d))
    dl = rng.standard_normal((hq, T))
    with OP.pool() as ex:
        o, l = OP.dense_all_heads(ex, bits(q), bits(k), bits(v), cu, chunk, ref["sel"])
        assert np.abs(o - ref["out"]).max() < 1e-12 and np.abs(l - ref["lse"]).max() < 1e-12
        o2, l2 = OP.attend_rows_par(ex, rows, bits(q)[ts, hs], bits(k), bits(v), cu, chunk, sel_rows, hq // hkv)
        assert np.abs(o2 - ref["out"][ts, hs]).max() < 1e-12
        assert np.abs(l2 - ref["lse"][hs, ts]).max() < 1e-12
        s2 = OP.select_rows_par(ex, rows, bits(q)[ts, hs], ref["means"], cu, chunk, topk, hq // hkv)
        assert (s2 == sel_rows).all()
        full = OP.select_and_compare_heads(ex, lambda h: bits(q)[:, h], ref["means"],
                                           lambda h: ref["sel"][h].astype(np.int16), cu, chunk, topk,
                                           hq // hkv, range(hq))
        assert all((full[h][0] == ref["sel"][h]).all() and len(full[h][1]) == 0 for h in range(hq))
        g = OP.backward_by_head(ex, q, k, v, cu, chunk, ref["sel"], do, dl)
    r = oracle.moba_backward(q, k, v, cu, chunk, ref["sel"], do, dl)
    assert all(np.abs(a - b).max() < 1e-10 for a, b in zip(g, r))


def test_shared_input_drivers_equal_the_whole_oracle():
    """The drivers that read the inputs from shared-memory files give the oracle's result."""
    import oracle
    import oracle_pool as OP

    rng = np.random.default_rng(6)
    T, hq, hkv, d, chunk, topk = 300, 4, 2, 16, 32, 3
    cu = [0, 300]
    bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q16 = bits(rng.standard_normal((T, hq, d)))
    k16 = bits(rng.standard_normal((T, hkv, d)))
    v16 = bits(rng.standard_normal((T, hkv, d)))
    q, k, v = PT.from_bits(q16), PT.from_bits(k16), PT.from_bits(v16)
    ref = oracle.moba_forward(q, k, v, cu, chunk, topk)
    rows = [(t, h) for t in range(0, T, 5) for h in range(hq)]
    ts = np.array([t for t, _ in rows])
    hs = np.array([h for _, h in rows])
    with OP.pool() as ex, OP.Shared(q=q16.transpose(1, 0, 2), k=k16.transpose(1, 0, 2),
                                    v=v16.transpose(1, 0, 2)) as sh:
        o, l, cpu = OP.submit_attend_shared(ex, rows, q16[ts, hs], sh, cu, chunk, ref["sel"][hs, ts],
                                            hq // hkv).result()
        assert np.abs(o - ref["out"][ts, hs]).max() < 1e-12 and np.abs(l - ref["lse"][hs, ts]).max() < 1e-12
        assert cpu > 0
        full = OP.submit_select_compare_shared(ex, sh, ref["means"], lambda h: ref["sel"][h].astype(np.int16),
                                               cu, chunk, topk, hq // hkv, range(hq)).result()
        assert all((full[h][0] == ref["sel"][h]).all() and len(full[h][1]) == 0 for h in range(hq))
