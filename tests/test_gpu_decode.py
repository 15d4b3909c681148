"""Decode step on the GPU (moba_decode_fwd through the C ABI) against the float64 oracle.

The new query of each sequence sits at its cache's last row, so the reference is the oracle's
row-wise selection and attention of those rows (oracle.moba_decode, pinned against the prefill
forward's last rows on the CPU).  Tolerances as for the prefill path."""

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


def gpu_decode(w, q_new, k, v, cu_t, return_sel=False):
    means = moba.meanpool(k, cu_t, w.chunk_size)
    p = moba.make_params(len(w.seqlens), w.total_tokens, w.num_q_heads, w.num_kv_heads,
                         w.head_dim, w.chunk_size, w.topk)
    ws = torch.empty(moba.load_library().moba_decode_workspace_size(p), dtype=torch.uint8,
                     device="cuda")
    out, lse = moba.decode_fwd(q_new, k, v, cu_t, means, w.chunk_size, w.topk, workspace=ws)
    torch.cuda.synchronize()
    if not return_sel:
        return out, lse
    # white-box: the selection is the workspace's first region, [batch * Hq, topk] int32
    rows = len(w.seqlens) * w.num_q_heads
    sel = ws[: rows * w.topk * 4].view(torch.int32).reshape(len(w.seqlens), w.num_q_heads, w.topk)
    return out, lse, sel.cpu().numpy()


def near_tie_rows(w, q_new_np, k_np, ref):
    """(b, h) rows whose last routed and first excluded past scores are within the band."""
    cu = np.asarray(w.cu_seqlens)
    means = oracle.block_means(k_np, cu, w.chunk_size)
    tab = oracle.block_table(cu, w.chunk_size)
    group = w.num_q_heads // w.num_kv_heads
    ties = set()
    for b in range(len(w.seqlens)):
        n = w.seqlens[b]
        if n == 0:
            continue
        c = (n - 1) // w.chunk_size
        b0 = int(tab["cu_blocks"][b])
        for h in range(w.num_q_heads):
            if PT._near_tie(q_new_np[b, h], means[b0:b0 + c, h // group], min(w.topk - 1, c)):
                ties.add((b, h))
    return ties


SMALL = [
    W.custom("dec_ragged_gqa", [700, 1337, 128, 1, 0, 390], 8, 2, 128, 128, 3, "k_offsets", 61),
    W.custom("dec_d64_mha", [3000, 1500], 4, 4, 64, 128, 5, "qk_offsets", 62),
    W.custom("dec_odd_group", [2000, 999], 6, 2, 128, 256, 4, "k_offsets", 63),
    W.custom("dec_topk1", [900, 257], 2, 2, 64, 128, 1, "k_offsets", 64),
    W.custom("dec_topk32", [4500], 2, 1, 128, 128, 32, "k_offsets", 65),
    W.custom("dec_dense", [1000, 600], 4, 4, 128, 256, 8, "k_offsets", 66),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_decode_small(w):
    q_new, _, k, v, cu_t = decode_inputs(w)
    out, lse, sel = gpu_decode(w, q_new, k, v, cu_t, return_sel=True)
    qn, kn, vn = PT.host(q_new), PT.host(k), PT.host(v)
    ref = oracle.moba_decode(qn, kn, vn, np.asarray(w.cu_seqlens), w.chunk_size, w.topk)
    ties = near_tie_rows(w, qn, kn, ref)
    B, hq = len(w.seqlens), w.num_q_heads
    keep = np.ones((B, hq), dtype=bool)
    for b in range(B):
        for h in range(hq):
            got = sorted(int(x) for x in sel[b, h] if x >= 0)
            want = sorted(int(x) for x in ref["sel"][b, h] if x >= 0)
            if got != want:
                assert (b, h) in ties, (b, h, got, want)
                keep[b, h] = False
    o, l = PT.host(out), PT.host(lse)
    empty = [b for b in range(B) if w.seqlens[b] == 0]
    for b in empty:
        assert np.all(o[b] == 0) and np.all(np.isneginf(l[:, b]))
    rows = [(b, h) for b in range(B) for h in range(hq) if keep[b, h] and w.seqlens[b] > 0]
    og = np.stack([o[b, h] for b, h in rows])
    orf = np.stack([ref["out"][b, h] for b, h in rows])
    lg = np.array([l[h, b] for b, h in rows])
    lr = np.array([ref["lse"][h, b] for b, h in rows])
    PT.check_out(og, lg, orf, lr)


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


def test_decode_long_cache():
    """A 256K-token cache with the 1M workload's block size and top-k (64 blocks of 4096)."""
    w = W.custom("dec_256k", [1 << 18], 8, 2, 128, 4096, 12, "k_offsets", 68)
    q_new, _, k, v, cu_t = decode_inputs(w)
    out, lse = gpu_decode(w, q_new, k, v, cu_t)
    qn, kn, vn = PT.host(q_new), PT.host(k), PT.host(v)
    ref = oracle.moba_decode(qn, kn, vn, np.asarray(w.cu_seqlens), w.chunk_size, w.topk)
    ties = near_tie_rows(w, qn, kn, ref)
    rows = [(0, h) for h in range(w.num_q_heads) if (0, h) not in ties]
    o, l = PT.host(out), PT.host(lse)
    PT.check_out(np.stack([o[b, h] for b, h in rows]), np.array([l[h, b] for b, h in rows]),
                 np.stack([ref["out"][b, h] for b, h in rows]), np.array([ref["lse"][h, b] for b, h in rows]))
