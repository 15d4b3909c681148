"""Decode step on the GPU (moba_decode_fwd and moba_decode_minmax_fwd through the C ABI)
against the float64 oracle.

The new query of each sequence sits at its cache's last row, so the reference is the oracle's
row-wise selection and attention of those rows (oracle.moba_decode, pinned against the prefill
forward's last rows on the CPU; with gate="minmax", pinned by box-corner enumeration and
brute-force selection).  Tolerances as for the prefill path; the min/max block summary
(moba_minmaxpool) is exact."""

import numpy as np
import pytest
import torch

import oracle
import parity as PT
from block_sparse_long_meanpool_b200 import moba
from block_sparse_long_meanpool_b200 import workloads as W

pytestmark = pytest.mark.gpu


def decode_inputs(w):
    """Caches from the workload recipe; the new query of sequence b is q at its last row."""
    x = W.make_inputs(w, device="cuda")
    cu = np.asarray(w.cu_seqlens)
    q_full, k, v, cu_t = x["q"], x["k"], x["v"], x["cu_seqlens"]
    last = [int(cu[b + 1]) - 1 if cu[b + 1] > cu[b] else 0 for b in range(len(cu) - 1)]
    q_new = q_full[torch.tensor(last, device="cuda")].contiguous()
    empty = [b for b in range(len(cu) - 1) if cu[b + 1] == cu[b]]
    if empty:
        q_new[torch.tensor(empty, device="cuda")] = 0
    return q_new, q_full, k, v, cu_t


def gpu_decode(w, q_new, k, v, cu_t, return_sel=False, gate="mean"):
    p = moba.make_params(len(w.seqlens), w.total_tokens, w.num_q_heads, w.num_kv_heads,
                         w.head_dim, w.chunk_size, w.topk)
    ws = torch.empty(moba.load_library().moba_decode_workspace_size(p), dtype=torch.uint8,
                     device="cuda")
    if gate == "mean":
        means = moba.meanpool(k, cu_t, w.chunk_size)
        out, lse = moba.decode_fwd(q_new, k, v, cu_t, means, w.chunk_size, w.topk, workspace=ws)
    else:
        k_min, k_max = moba.minmaxpool(k, cu_t, w.chunk_size)
        out, lse = moba.decode_minmax_fwd(q_new, k, v, cu_t, k_min, k_max, w.chunk_size, w.topk,
                                          workspace=ws)
    torch.cuda.synchronize()
    if not return_sel:
        return out, lse
    # white-box: the selection is the workspace's first region, [batch * Hq, topk] int32
    rows = len(w.seqlens) * w.num_q_heads
    sel = ws[: rows * w.topk * 4].view(torch.int32).reshape(len(w.seqlens), w.num_q_heads, w.topk)
    return out, lse, sel.cpu().numpy()


def decode_slack(q_row, summary_rows):
    """Error bound of the decode min/max gate's score of each block: every term
    max(q_i kmin_i, q_i kmax_i) is exact (bf16 x bf16 in fp32), and the kernel sums them in 4
    accumulators of d/8 pair sums and two more adds, so a score is off by at most
    (d/4 + 2) 2^-24 sum_i |t_i|.  (The mean gate's 1e-3 relative band would cover every row
    here: a box over thousands of N(0, 1) keys gives scores of a few hundred that differ by a
    few units.)  ``summary_rows`` is [n, 2, d] (min, max)."""
    q = np.asarray(q_row, dtype=np.float64)
    mm = np.asarray(summary_rows, dtype=np.float64)
    terms = np.maximum(q * mm[:, 0, :], q * mm[:, 1, :])
    return (q.shape[0] / 4 + 2) * 2.0 ** -24 * np.abs(terms).sum(axis=1)


class _NewQuery:
    """q[t, h] for the decode step: the new query of the sequence whose last cache row is t."""

    def __init__(self, q_new, cu):
        self.q = q_new
        self.row_of = {int(cu[b + 1]) - 1: b for b in range(len(cu) - 1) if cu[b + 1] > cu[b]}
        self.shape = (int(cu[-1]),) + tuple(q_new.shape[1:])

    def __getitem__(self, th):
        return self.q[self.row_of[int(th[0])], int(th[1])]


def check_decode(w, q_new_np, k_np, v_np, sel, out, lse, ref, gate):
    """Every (sequence, head) row: the GPU's selection is the oracle's or a valid near-tie
    alternative of it (the band of R9 for the mean gate, the kernel's error bound for the
    min/max gate), and its output matches the oracle's attention over the GPU's selection."""
    cu = np.asarray(w.cu_seqlens)
    chunk, topk, hq = w.chunk_size, w.topk, w.num_q_heads
    group = hq // w.num_kv_heads
    if gate == "mean":
        summary, score, slack = oracle.block_means(k_np, cu, chunk), oracle.gate_scores_row, None
    else:
        kmin, kmax = oracle.block_minmax(k_np, cu, chunk)
        summary, score, slack = np.stack([kmin, kmax], axis=2), oracle.minmax_scores_row, decode_slack
    qv = _NewQuery(q_new_np, cu)
    rows, g_rows, o_rows = [], [], []
    for b in range(len(w.seqlens)):
        n = w.seqlens[b]
        if n == 0:
            continue
        t, c = int(cu[b + 1]) - 1, (n - 1) // chunk
        for h in range(hq):
            # the decode selection lists the own block first and the routed blocks best first;
            # as a prefill row: routed blocks ascending, the own block, -1 padding
            got = [int(x) for x in sel[b, h] if x >= 0]
            assert got[0] == c and len(got) == len(set(got)), (b, h, got)
            g_rows.append(sorted(got[1:]) + [c] + [-1] * (topk - len(got)))
            o_rows.append([int(x) for x in ref["sel"][b, h]])
            rows.append((t, h))
    # the oracle's decode selection is already in that form (select_blocks_rows)
    g_rows, o_rows = np.array(g_rows), np.array(o_rows)
    ties = PT.check_selection(g_rows, o_rows, rows, qv, summary, cu, chunk, topk, group, score=score,
                              slack_fn=slack)
    ref_o, ref_l = oracle.attend_rows(qv, k_np, v_np, cu, chunk, g_rows, rows)
    batch_of = {t: qv.row_of[t] for t, _ in rows}
    og = np.stack([out[batch_of[t], h] for t, h in rows])
    lg = np.array([lse[h, batch_of[t]] for t, h in rows])
    PT.check_out(og, lg, ref_o, ref_l)
    return ties


SMALL = [
    W.custom("dec_ragged_gqa", [700, 1337, 128, 1, 0, 390], 8, 2, 128, 128, 3, "k_offsets", 61),
    W.custom("dec_d64_mha", [3000, 1500], 4, 4, 64, 128, 5, "qk_offsets", 62),
    W.custom("dec_odd_group", [2000, 999], 6, 2, 128, 256, 4, "k_offsets", 63),
    W.custom("dec_topk1", [900, 257], 2, 2, 64, 128, 1, "k_offsets", 64),
    W.custom("dec_topk32", [4500], 2, 1, 128, 128, 32, "k_offsets", 65),
    W.custom("dec_dense", [1000, 600], 4, 4, 128, 256, 8, "k_offsets", 66),
]


@pytest.mark.parametrize("gate", ["mean", "minmax"])
@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_decode_small(w, gate):
    q_new, _, k, v, cu_t = decode_inputs(w)
    out, lse, sel = gpu_decode(w, q_new, k, v, cu_t, return_sel=True, gate=gate)
    qn, kn, vn = PT.host(q_new), PT.host(k), PT.host(v)
    ref = oracle.moba_decode(qn, kn, vn, np.asarray(w.cu_seqlens), w.chunk_size, w.topk, gate=gate)
    o, l = PT.host(out), PT.host(lse)
    for b in [b for b in range(len(w.seqlens)) if w.seqlens[b] == 0]:
        assert np.all(o[b] == 0) and np.all(np.isneginf(l[:, b]))
    check_decode(w, qn, kn, vn, sel, o, l, ref, gate)


def test_decode_matches_prefill_last_rows_on_gpu():
    """The decode step and the prefill forward agree on every sequence's last row."""
    w = W.custom("dec_vs_prefill", [3000, 1024, 777], 8, 2, 128, 256, 3, "k_offsets", 67)
    q_new, q_full, k, v, cu_t = decode_inputs(w)
    out, lse = gpu_decode(w, q_new, k, v, cu_t)
    pout, plse = moba.attn_fwd(q_full, k, v, cu_t, w.chunk_size, w.topk)
    torch.cuda.synchronize()
    cu = np.asarray(w.cu_seqlens)
    last = [int(cu[b + 1]) - 1 for b in range(len(w.seqlens))]
    a = PT.host(out)
    b_ = PT.host(pout)[last]
    assert np.abs(a - b_).max() <= PT.OUT_MAX_ABS
    assert np.abs(PT.host(lse) - PT.host(plse)[:, last]).max() <= PT.LSE_ABS


@pytest.mark.parametrize("gate", ["mean", "minmax"])
def test_decode_long_cache(gate):
    """A 256K-token cache with the 1M workload's block size and top-k (64 blocks of 4096)."""
    w = W.custom("dec_256k", [1 << 18], 8, 2, 128, 4096, 12, "k_offsets", 68)
    q_new, _, k, v, cu_t = decode_inputs(w)
    out, lse, sel = gpu_decode(w, q_new, k, v, cu_t, return_sel=True, gate=gate)
    qn, kn, vn = PT.host(q_new), PT.host(k), PT.host(v)
    ref = oracle.moba_decode(qn, kn, vn, np.asarray(w.cu_seqlens), w.chunk_size, w.topk, gate=gate)
    check_decode(w, qn, kn, vn, sel, PT.host(out), PT.host(lse), ref, gate)


@pytest.mark.parametrize("w", [SMALL[0], SMALL[1], W.custom("mm_long", [1 << 17, 5000], 8, 8, 128, 4096, 4,
                                                            "k_offsets", 69)],
                         ids=["dec_ragged_gqa", "dec_d64_mha", "mm_long"])
def test_minmaxpool_is_exact(w):
    """The bf16 min/max summary equals the oracle's extrema bit for bit (extrema of bf16
    values are bf16 values), partial blocks included."""
    _, _, k, _, cu_t = decode_inputs(w)
    nb = moba.num_blocks(w.seqlens, w.chunk_size)
    k_min, k_max = moba.minmaxpool(k, cu_t, w.chunk_size, num_blocks_out=nb)
    torch.cuda.synchronize()
    rmin, rmax = oracle.block_minmax(PT.host(k), np.asarray(w.cu_seqlens), w.chunk_size)
    assert k_min.shape == rmin.shape and k_max.shape == rmax.shape
    np.testing.assert_array_equal(PT.host(k_min), rmin)
    np.testing.assert_array_equal(PT.host(k_max), rmax)


def test_minmax_gate_routes_the_single_matching_key_on_gpu():
    """Block 1 holds one key aligned with q among zeros: its mean (4/128) loses to block 0's
    uniform 0.5, its box maximum (4) wins.  The mean path routes block 0, the min/max path
    block 1; both outputs match the oracle."""
    d, chunk, L = 64, 128, 3 * 128 + 40
    k = torch.zeros((L, 1, d), dtype=torch.float32)
    k[0:128, 0, 0] = 0.5
    k[128 + 77, 0, 0] = 4.0
    k[256:384, 0, 0] = -1.0
    k[384:, 0, 1] = 1.0
    g = torch.Generator().manual_seed(70)
    v = torch.randn((L, 1, d), generator=g)
    q_new = torch.zeros((1, 1, d))
    q_new[0, 0, 0] = 1.0
    k, v, q_new = (t.to(torch.bfloat16).cuda().contiguous() for t in (k, v, q_new))
    cu_t = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    w = W.custom("mm_spike", [L], 1, 1, d, chunk, 2, "k_offsets", 70)
    qn, kn, vn = PT.host(q_new), PT.host(k), PT.host(v)
    for gate, routed in (("mean", 0), ("minmax", 1)):
        out, lse, sel = gpu_decode(w, q_new, k, v, cu_t, return_sel=True, gate=gate)
        assert sorted(int(x) for x in sel[0, 0]) == sorted([routed, 3]), (gate, sel[0, 0])
        ref = oracle.moba_decode(qn, kn, vn, np.array([0, L]), chunk, 2, gate=gate)
        assert sorted(ref["sel"][0, 0]) == sorted([routed, 3])
        PT.check_out(PT.host(out)[0], PT.host(lse)[:, 0], ref["out"][0], ref["lse"][:, 0])
