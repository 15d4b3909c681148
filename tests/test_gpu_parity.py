"""GPU parity: the CUDA path, called through the C ABI, against the float64 oracle.

Every case feeds the same seeded bf16 inputs to both sides.  Selections are compared in full
(every row of every head) except on the length sweep, where whole heads and sampled rows are
compared; a row may differ only as a valid near-tie alternative (``parity.check_selection``),
and such a row's output is checked against the oracle's attention over the GPU's own
selection.  Outputs are compared on all rows for the small cases and the scaling, long and
varlen workloads, and on sampled rows (4096 per head at 1M) for the larger ones; then the
oracle's selection is fed back (``sel_in``) and the outputs must match with no exception.
The full-size checks run the oracle on the host cores through ``oracle_pool``.  Tolerances
are in ``parity.py``.
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
    """Compare [Hq, T, topk] selections; returns the (t, h) rows whose GPU selection is a valid
    near-tie alternative to the oracle's (any other difference fails)."""
    diff = np.nonzero((gsel != osel).any(axis=2))
    rows = [(int(t), int(h)) for h, t in zip(*diff)]
    ties = PT.check_selection(gsel[diff], osel[diff], rows, q_np, om, cu, chunk, topk, group)
    return [rows[r] for r in sorted(ties)]


def with_tie_rows(ref_o, ref_l, ties, gsel, q_np, k_np, v_np, cu, chunk, scale=None):
    """Copies of the oracle's out [T, Hq, d] / lse [Hq, T] in which every near-tie row holds the
    oracle's attention over the GPU's selection of that row."""
    ref_o, ref_l = ref_o.copy(), ref_l.copy()
    if ties:
        sel_rows = np.stack([gsel[h, t] for t, h in ties])
        o, l = oracle.attend_rows(q_np, k_np, v_np, cu, chunk, sel_rows, ties, scale)
        for i, (t, h) in enumerate(ties):
            ref_o[t, h] = o[i]
            ref_l[h, t] = l[i]
    return ref_o, ref_l


def check_all_rows(out, lse, ref_o, ref_l):
    T, hq = out.shape[0], out.shape[1]
    return PT.check_out(PT.host(out).reshape(T * hq, -1), PT.host(lse).T.reshape(-1),
                        ref_o.reshape(T * hq, -1), ref_l.T.reshape(-1))


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_all_rows(w):
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, group = w.chunk_size, w.topk, w.num_q_heads // w.num_kv_heads
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    sel_gate = moba.gate_topk(q, means, cu_t, chunk, topk)
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=w.max_seqlen,
                                  check_status=True)
    torch.cuda.synchronize()
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    ref = oracle.moba_forward(q_np, k_np, v_np, cu, chunk, topk)

    PT.check_means(PT.host(means), k_np, cu, chunk, ref["means"])
    gsel = PT.host(sel, np.int64)
    # the gate sized by the batch's block bound and by max_seqlen select the same blocks
    np.testing.assert_array_equal(gsel, PT.host(sel_gate, np.int64))
    ties = full_sel_check(gsel, ref["sel"], q_np, ref["means"], cu, chunk, topk, group)
    ref_o, ref_l = with_tie_rows(ref["out"], ref["lse"], ties, gsel, q_np, k_np, v_np, cu, chunk)
    check_all_rows(out, lse, ref_o, ref_l)

    # oracle-feed mode: the oracle's selection, no exceptions
    fed = torch.from_numpy(ref["sel"].astype(np.int32)).cuda()
    out2, lse2 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed)
    check_all_rows(out2, lse2, ref["out"], ref["lse"])


WIDE = [
    # 256 blocks: 256 score columns, the four warpgroups of a tile merge their lists twice
    W.custom("wide_256_top12", [32768], 4, 1, 128, 128, 12, "k_offsets", 31),
    # topk - 1 > 11: two warpgroups per tile, 128-column slices
    W.custom("wide_256_top17", [32768], 2, 1, 64, 128, 17, "k_offsets", 32),
    W.custom("wide_256_top32", [32768], 2, 1, 128, 128, 32, "k_offsets", 33),
    # 128 blocks: two tile groups of two warpgroups each
    W.custom("wide_128_top8", [16384, 9000], 4, 2, 128, 128, 8, "k_offsets", 34),
]


@pytest.mark.parametrize("w", WIDE, ids=[w.name for w in WIDE])
def test_gate_with_merged_warpgroup_lists(w):
    """The tensor-core gate when several warpgroups rank slices of one tile's scores and merge
    their lists: every selection against the oracle's, then sampled outputs."""
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    p = moba.make_params(len(w.seqlens), w.total_tokens, hq, w.num_kv_heads, w.head_dim, chunk, topk,
                         max_seqlen=w.max_seqlen)
    ws = torch.empty(moba.workspace_size(p), dtype=torch.uint8, device="cuda")
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=w.max_seqlen,
                                  workspace=ws, wave_tokens=0)
    assert moba.attn_fwd.last_info["gate_path"] == moba.GATE_PATH_TENSOR_CORES
    moba.device_status(p, ws)  # no bounded wait gave up
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    om = oracle.block_means(k_np, cu, chunk)
    osel = oracle.select_blocks(q_np, om, cu, chunk, topk)
    gsel = PT.host(sel, np.int64)
    ties = full_sel_check(gsel, osel, q_np, om, cu, chunk, topk, group)
    assert len(ties) < 1e-3 * gsel.shape[0] * gsel.shape[1]
    rows = sorted(set(PT.sample_rows(cu, chunk, hq, topk, 192, 64, seed=35)) | set(ties))
    ref_o, ref_l = oracle.attend_rows(q_np, k_np, v_np, cu, chunk, np.stack([gsel[h, t] for t, h in rows]), rows)
    PT.check_out(np.stack([PT.host(out[t, h]) for t, h in rows]), np.array([float(lse[h, t]) for t, h in rows]),
                 ref_o, ref_l)


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
        check_all_rows(out, lse, ref_o, ref_l)


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
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, 128, 2, softmax_scale=0.05, return_sel=True)
    cu = np.asarray(w.cu_seqlens)
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    ref = oracle.moba_forward(q_np, k_np, v_np, cu, 128, 2, scale=0.05)
    gsel = PT.host(sel, np.int64)
    ties = full_sel_check(gsel, ref["sel"], q_np, ref["means"], cu, 128, 2, 1)
    ref_o, ref_l = with_tie_rows(ref["out"], ref["lse"], ties, gsel, q_np, k_np, v_np, cu, 128, 0.05)
    check_all_rows(out, lse, ref_o, ref_l)


# ---- full-size workloads ------------------------------------------------------------------

@pytest.mark.parametrize("name", ["scaling_8k", "long_32k", "varlen_gqa"])
def test_full_size_all_rows(name, ex):
    """All means, all selections and all output rows (masked-dense oracle over every head),
    then the oracle-feed mode on all rows."""
    w = W.ALL_WORKLOADS[name]
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=w.max_seqlen,
                                  check_status=True)
    torch.cuda.synchronize()
    q16, k16, v16 = PT.bf16_bits(q), PT.bf16_bits(k), PT.bf16_bits(v)
    q_np, k_np, v_np = PT.from_bits(q16), PT.from_bits(k16), PT.from_bits(v16)
    om = oracle.block_means(k_np, cu, chunk)
    PT.check_means(PT.host(means), k_np, cu, chunk, om)
    osel = oracle.select_blocks(q_np, om, cu, chunk, topk)
    gsel = PT.host(sel, np.int64)
    ties = full_sel_check(gsel, osel, q_np, om, cu, chunk, topk, group)
    assert len(ties) < 1e-3 * gsel.shape[0] * gsel.shape[1]

    ref_o, ref_l = OP.dense_all_heads(ex, q16, k16, v16, cu, chunk, osel)
    t_o, t_l = with_tie_rows(ref_o, ref_l, ties, gsel, q_np, k_np, v_np, cu, chunk)
    check_all_rows(out, lse, t_o, t_l)

    fed = torch.from_numpy(osel.astype(np.int32)).cuda()
    out2, lse2 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed)
    check_all_rows(out2, lse2, ref_o, ref_l)


@pytest.mark.parametrize("name", ["fine_32k_8_2", "fine_32k_128_32"])
def test_granularity_sweep_sampled(name, ex):
    """Block granularity at 75% sparsity (8 blocks / top-2 and 128 blocks / top-32 at 32K):
    all means and selections, sampled output rows, and the oracle-feed mode."""
    w = W.ALL_WORKLOADS[name]
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=w.max_seqlen,
                                  check_status=True)
    torch.cuda.synchronize()
    q16, k16, v16 = PT.bf16_bits(q), PT.bf16_bits(k), PT.bf16_bits(v)
    q_np, k_np = PT.from_bits(q16), PT.from_bits(k16)
    om = oracle.block_means(k_np, cu, chunk)
    PT.check_means(PT.host(means), k_np, cu, chunk, om)
    osel = oracle.select_blocks(q_np, om, cu, chunk, topk)
    gsel = PT.host(sel, np.int64)
    ties = full_sel_check(gsel, osel, q_np, om, cu, chunk, topk, group)
    assert len(ties) < 1e-3 * gsel.shape[0] * gsel.shape[1]

    rows = sorted(set(PT.sample_rows(cu, chunk, hq, topk, 768, 256, seed=31)) | set(ties))
    ts = np.array([t for t, _ in rows])
    hs = np.array([h for _, h in rows])
    q_rows = q16[ts, hs]
    g_rows, o_rows = gsel[hs, ts], osel[hs, ts]
    ref_g = OP.attend_rows_par(ex, rows, q_rows, k16, v16, cu, chunk, g_rows, group)
    ref_f = OP.attend_rows_par(ex, rows, q_rows, k16, v16, cu, chunk, o_rows, group)
    PT.check_out(PT.host(out[ts, hs]), PT.host(lse[hs, ts]), *ref_g)

    fed = torch.from_numpy(osel.astype(np.int32)).cuda()
    out2, lse2 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed)
    PT.check_out(PT.host(out2[ts, hs]), PT.host(lse2[hs, ts]), *ref_f)


class _Bf16Rows:
    """[T, Hkv, d] slices of a head-major [Hkv, T, d] array of bf16 bits, widened on access
    (check_means reads the keys block by block)."""

    def __init__(self, u16_head_major):
        self.u16 = u16_head_major

    def __getitem__(self, sl):
        return PT.from_bits(self.u16[:, sl]).transpose(1, 0, 2)


def _block_means_by_block(k16_hm, w):
    """The oracle's block means of a single-sequence workload, one block at a time (blocks
    are independent), so that the keys are never widened all at once."""
    chunk = w.chunk_size
    nb = moba.num_blocks(w.seqlens, chunk)
    return np.concatenate([oracle.block_means(PT.from_bits(k16_hm[:, b * chunk:(b + 1) * chunk]).transpose(1, 0, 2),
                                              [0, min(chunk, w.total_tokens - b * chunk)], chunk)
                           for b in range(nb)])


def _head_major_bits(t):
    """bf16 [T, H, d] on the device -> head-major [H, T, d] uint16 bits on the host."""
    return PT.bf16_bits(t.transpose(0, 1))


def _long_prefill_check(ex, w, sel_heads, n_uniform, n_strat, seed):
    """The checks of a long single-sequence prefill in the bench's wave configuration:
    - all block means;
    - the full selection of every head in ``sel_heads`` against oracle.select_blocks;
    - n_uniform + n_strat sampled rows of every head (plus every near-tie row found): their
      selections against the oracle's and their outputs against oracle.attend_rows over the
      GPU's selection;
    - the oracle-feed mode: the oracle's selections (whole heads where computed, the sampled
      rows elsewhere) fed back, the sampled rows' outputs compared with no exception.
    The keys, values and the fully checked heads' queries go to the workers through shared
    memory (oracle_pool.Shared); the full-head selections run while the rows are attended."""
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq, hkv = w.chunk_size, w.topk, w.num_q_heads, w.num_kv_heads
    group = hq // hkv
    T = w.total_tokens
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=w.max_seqlen,
                                  check_status=True)
    nb = moba.num_blocks(w.seqlens, chunk)
    means = moba.meanpool(k, cu_t, chunk, num_blocks_out=nb)
    torch.cuda.synchronize()
    assert moba.attn_fwd.last_info["waves"] >= 1
    k16, v16 = _head_major_bits(k), _head_major_bits(v)
    om = _block_means_by_block(k16, w)
    PT.check_means(PT.host(means), _Bf16Rows(k16), cu, chunk, om)
    sel_heads = list(sel_heads)
    q16_full = _head_major_bits(q[:, sel_heads])

    rows = PT.sample_rows_per_head(cu, chunk, hq, topk, n_uniform, n_strat, seed)
    with OP.Shared(q=q16_full, k=k16, v=v16) as sh:
        del q16_full
        # the whole heads' selections (position i of the shared q is head sel_heads[i])
        futs = [ex.submit(OP._select_compare_shared, sh.ref("q"), i, np.ascontiguousarray(om[:, h // group]),
                          sel[h].cpu().numpy().astype(np.int16), cu, chunk, topk)
                for i, h in enumerate(sel_heads)]
        # the sampled rows, attended over the GPU's selection while the whole heads are checked
        ts_t = torch.tensor([t for t, _ in rows], device="cuda")
        hs_t = torch.tensor([h for _, h in rows], device="cuda")
        g_rows = sel[hs_t, ts_t].cpu().numpy().astype(np.int64)
        q_rows = PT.bf16_bits(q[ts_t, hs_t])
        att_p = OP.submit_attend_shared(ex, rows, q_rows, sh, cu, chunk, g_rows, group)
        full, bad = {}, []
        for h, f in zip(sel_heads, futs):
            osel_h, tt, b, _ = f.result()
            full[h] = (osel_h, tt)
            bad += [(h,) + x for x in b]
        assert not bad, f"{len(bad)} selection mismatches outside the near-tie band: {bad[:5]}"
        ties = sorted({(int(t), h) for h, (_, tt) in full.items() for t in tt} - set(rows))
        assert len(ties) < 1e-3 * T * len(sel_heads)
        # the near-tie rows of the whole heads that the sample did not draw
        if ties:
            tt_t = torch.tensor([t for t, _ in ties], device="cuda")
            th_t = torch.tensor([h for _, h in ties], device="cuda")
            tie_g = sel[th_t, tt_t].cpu().numpy().astype(np.int64)
            tie_p = OP.submit_attend_shared(ex, ties, PT.bf16_bits(q[tt_t, th_t]), sh, cu, chunk, tie_g, group)

        # the sampled rows' oracle selections: whole heads where computed, else row by row
        ts, hs = ts_t.cpu().numpy(), hs_t.cpu().numpy()
        o_rows = np.zeros_like(g_rows)
        in_full = np.isin(hs, sel_heads)
        for h, (osel_h, _) in full.items():
            m = hs == h
            o_rows[m] = osel_h[ts[m]]
        rest = np.nonzero(~in_full)[0]
        if len(rest):
            o_rows[rest] = OP.select_rows_par(ex, [rows[i] for i in rest], q_rows[rest], om, cu, chunk, topk, group)
            ties_rest = PT.check_selection(g_rows[rest], o_rows[rest], [rows[i] for i in rest],
                                           _RowQ(rows, q_rows), om, cu, chunk, topk, group)
            assert len(ties_rest) < max(3, 1e-2 * len(rest))

        ref_o, ref_l, _ = att_p.result()
        PT.check_out(PT.host(out[ts_t, hs_t]), PT.host(lse[hs_t, ts_t]), ref_o, ref_l)
        if ties:
            t_o, t_l, _ = tie_p.result()
            PT.check_out(PT.host(out[tt_t, th_t]), PT.host(lse[th_t, tt_t]), t_o, t_l)

        # oracle-feed mode (the output buffers are reused)
        fed = sel.clone()
        for h, (osel_h, _) in full.items():
            fed[h] = torch.from_numpy(osel_h.astype(np.int32)).cuda()
        fed[hs_t, ts_t] = torch.from_numpy(o_rows.astype(np.int32)).cuda()
        moba.attn_fwd(q, k, v, cu_t, chunk, topk, sel=fed, out=out, lse=lse, check_status=True)
        diff = np.nonzero((g_rows != o_rows).any(axis=1))[0]
        ref_o, ref_l = ref_o.copy(), ref_l.copy()
        if len(diff):
            o2, l2, _ = OP.submit_attend_shared(ex, [rows[i] for i in diff], q_rows[diff], sh, cu, chunk,
                                                o_rows[diff], group).result()
            ref_o[diff], ref_l[diff] = o2, l2
        PT.check_out(PT.host(out[ts_t, hs_t]), PT.host(lse[hs_t, ts_t]), ref_o, ref_l)


class _RowQ:
    """q[t, h] of the sampled rows only (parity.check_selection reads the rows it checks)."""

    def __init__(self, rows, q_rows16):
        self.idx = {r: i for i, r in enumerate(rows)}
        self.q = q_rows16

    def __getitem__(self, th):
        return PT.from_bits(self.q[self.idx[(int(th[0]), int(th[1]))]])


def test_prefill_1m(ex):
    """1,048,576 tokens, 32 q / 8 kv heads, chunk 4096, top-12: all block means, the full
    selection of all 32 heads, 4096 sampled rows per head (3584 uniform + 512 stratified),
    and the oracle-feed mode with the oracle's whole selection."""
    w = W.WORKLOADS["prefill_1m"]
    _long_prefill_check(ex, w, list(range(w.num_q_heads)), 3584, 512, seed=41)


def test_prefill_2m_length_sweep(ex):
    """Length sweep, 2,097,152 tokens in 256 blocks of 8192, top-12: full selections of two
    heads (of different KV heads), 128 sampled rows per head, the oracle-feed mode."""
    w = W.ALL_WORKLOADS["prefill_2m"]
    _long_prefill_check(ex, w, [0, 17], 96, 32, seed=42)


def test_prefill_10m_length_sweep(ex):
    """Length sweep, 10,485,760 tokens in 256 blocks of 40,960 (the 8 q / 2 kv head-group
    share), top-12: the full selection of one head, 24 sampled rows per head, the oracle-feed
    mode."""
    w = W.ALL_WORKLOADS["prefill_10m"]
    _long_prefill_check(ex, w, [5], 16, 8, seed=43)


def test_cuda_core_gate_above_257_blocks():
    """A sequence of more than 257 blocks selects the CUDA-core gate (csrc/gate.cu) instead of
    the tensor-core one: its selections against the oracle's (valid near ties allowed)."""
    w = W.custom("gate_313_blocks", [40000, 3000], 2, 1, 64, 128, 4, "k_offsets", 25)
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, group = w.chunk_size, w.topk, w.num_q_heads // w.num_kv_heads
    means = moba.meanpool(k, cu_t, chunk)
    sel = moba.gate_topk(q, means, cu_t, chunk, topk, max_seqlen=w.max_seqlen)
    _, _, sel2 = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=w.max_seqlen,
                                  check_status=True)
    assert moba.attn_fwd.last_info["gate_path"] == moba.GATE_PATH_CUDA_CORES
    torch.cuda.synchronize()
    assert torch.equal(sel, sel2)
    q_np, k_np = PT.host(q), PT.host(k)
    om = oracle.block_means(k_np, cu, chunk)
    osel = oracle.select_blocks(q_np, om, cu, chunk, topk)
    full_sel_check(PT.host(sel, np.int64), osel, q_np, om, cu, chunk, topk, group)


def test_packed_batch_uses_the_tensor_core_gate():
    """A packed batch of 40 sequences of 2048 tokens (640 blocks in all, 16 per sequence):
    with max_seqlen the tensor-core gate runs (sized for 16 blocks); without it the batch-wide
    block bound sends the call to the CUDA-core gate.  Both selections match the oracle's,
    and the outputs match on all rows."""
    w = W.custom("packed_40x2k", [2048] * 40, 4, 2, 128, 128, 3, "k_offsets", 26)
    q, k, v, cu_t = gpu_inputs(w)
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, group = w.chunk_size, w.topk, w.num_q_heads // w.num_kv_heads
    out, lse, sel = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True, max_seqlen=2048)
    assert moba.attn_fwd.last_info["gate_path"] == moba.GATE_PATH_TENSOR_CORES
    _, _, sel_cc = moba.attn_fwd(q, k, v, cu_t, chunk, topk, return_sel=True)
    assert moba.attn_fwd.last_info["gate_path"] == moba.GATE_PATH_CUDA_CORES
    torch.cuda.synchronize()
    q_np, k_np, v_np = PT.host(q), PT.host(k), PT.host(v)
    ref = oracle.moba_forward(q_np, k_np, v_np, cu, chunk, topk)
    gsel = PT.host(sel, np.int64)
    ties = full_sel_check(gsel, ref["sel"], q_np, ref["means"], cu, chunk, topk, group)
    full_sel_check(PT.host(sel_cc, np.int64), ref["sel"], q_np, ref["means"], cu, chunk, topk, group)
    ref_o, ref_l = with_tie_rows(ref["out"], ref["lse"], ties, gsel, q_np, k_np, v_np, cu, chunk)
    check_all_rows(out, lse, ref_o, ref_l)


def test_max_seqlen_too_small_is_reported_not_faulted():
    """A max_seqlen shorter than a real sequence: no out-of-bounds access, the status word
    reads MOBA_ERR_INVALID_ARG, and the next call with the right bound is correct again."""
    w = W.custom("short_promise", [3000, 500], 2, 1, 64, 128, 3, "k_offsets", 27)
    q, k, v, cu_t = gpu_inputs(w)
    p = moba.make_params(len(w.seqlens), w.total_tokens, 2, 1, 64, 128, 3, max_seqlen=1750)
    ws = torch.empty(moba.workspace_size(p), dtype=torch.uint8, device="cuda")
    moba.attn_fwd(q, k, v, cu_t, 128, 3, workspace=ws, max_seqlen=1750)
    with pytest.raises(moba.MobaError) as e:
        moba.device_status(p, ws)
    assert e.value.status == moba.ERR_INVALID_ARG
    out, lse = moba.attn_fwd(q, k, v, cu_t, 128, 3, workspace=ws, max_seqlen=3000)
    moba.device_status(p, ws)
    ref_o, ref_l = moba.attn_fwd(q, k, v, cu_t, 128, 3)
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
