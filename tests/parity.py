"""Comparison helpers for the GPU parity tests (CUDA path through the C ABI vs the oracle).

Tolerances (bf16 inputs, fp32 accumulation):
  * block means: the fp32 recursive-summation bound, |err| <= (n_seq + 12) u sum|k| / n,
    u = 2^-24, n_seq = the longest per-thread chain (ceil(n / 8));
  * selections: identical, except rows whose last routed and first excluded past-block
    scores differ by less than 1e-3 relative (near-ties); feeding the oracle's selection
    removes that exception;
  * out: max-abs 2e-2 and mean-abs 2e-3; lse: abs 1e-3.
"""

import numpy as np
import torch

import oracle

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
TIE_REL = 1e-3


def host(t, dtype=np.float64):
    """bf16/fp32/int device tensor -> numpy (exact widening)."""
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy().astype(dtype, copy=False)


def check_means(gpu_means, k_np, cu, chunk, oracle_means):
    """Means within the fp32 summation bound of the float64 oracle."""
    tab = oracle.block_table(cu, chunk)
    g = np.asarray(gpu_means, dtype=np.float64)
    assert g.shape == oracle_means.shape
    worst = 0.0
    for b in range(len(tab["start"])):
        rows = k_np[tab["start"][b]:tab["end"][b]]
        n = rows.shape[0]
        bound = ((n + 7) // 8 + 12) * 2.0 ** -24 * np.abs(rows).sum(axis=0) / n
        bound = bound + 2.0 ** -24 * np.abs(oracle_means[b])
        err = np.abs(g[b] - oracle_means[b])
        assert np.all(err <= bound), (b, float(err.max()), float(bound.min()))
        worst = max(worst, float(err.max()))
    return worst


def _near_tie(q_row, seq_means_past, n_route):
    """True when the n_route-th and (n_route+1)-th best past scores are within the band."""
    sc = np.sort(oracle.gate_scores_row(q_row, seq_means_past))[::-1]
    if len(sc) <= n_route or n_route == 0:
        return False
    a, b = sc[n_route - 1], sc[n_route]
    return abs(a - b) < TIE_REL * max(abs(a), abs(b))


def check_selection(gpu_sel, ref_sel, rows, q_np, oracle_means, cu, chunk, topk, group):
    """gpu_sel / ref_sel: [n, topk] for the listed (t, h) rows.  Returns the set of row
    indices that differ but lie in the near-tie band; any other difference fails."""
    gpu_sel = np.asarray(gpu_sel)
    ref_sel = np.asarray(ref_sel)
    tab = oracle.block_table(cu, chunk)
    cu = np.asarray(cu)
    ties = set()
    bad = []
    diff = np.nonzero((gpu_sel != ref_sel).any(axis=1))[0]
    for r in diff:
        t, h = rows[r]
        i = int(np.searchsorted(cu, t, side="right") - 1)
        c = (t - int(cu[i])) // chunk
        b0 = int(tab["cu_blocks"][i])
        n_route = min(topk - 1, c)
        if _near_tie(q_np[t, h], oracle_means[b0:b0 + c, h // group], n_route):
            ties.add(int(r))
        else:
            bad.append((t, h, list(gpu_sel[r]), list(ref_sel[r])))
    assert not bad, f"{len(bad)} selection mismatches outside the near-tie band: {bad[:5]}"
    return ties


def check_out(out_gpu, lse_gpu, out_ref, lse_ref, skip=()):
    """out [n, d] and lse [n] of the same rows; rows in ``skip`` are excluded."""
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    out_ref = np.asarray(out_ref, dtype=np.float64)
    keep = np.ones(out_gpu.shape[0], dtype=bool)
    keep[list(skip)] = False
    err = np.abs(out_gpu[keep] - out_ref[keep])
    lerr = np.abs(np.asarray(lse_gpu, dtype=np.float64)[keep] - np.asarray(lse_ref)[keep])
    stats = {"out_max_abs": float(err.max()), "out_mean_abs": float(err.mean()),
             "lse_max_abs": float(lerr.max()), "rows": int(keep.sum())}
    assert stats["out_max_abs"] <= OUT_MAX_ABS, stats
    assert stats["out_mean_abs"] <= OUT_MEAN_ABS, stats
    assert stats["lse_max_abs"] <= LSE_ABS, stats
    return stats


def sample_rows(cu, chunk, hq, topk, n_uniform, n_strat, seed):
    """Uniform rows plus stratified ones: first/last token of blocks and rows with c < topk."""
    rng = np.random.default_rng(seed)
    cu = np.asarray(cu)
    T = int(cu[-1])
    rows = set()
    for t in rng.integers(0, T, n_uniform):
        rows.add((int(t), int(rng.integers(0, hq))))
    tab = oracle.block_table(cu, chunk)
    starts, ends, local = tab["start"], tab["end"], tab["local"]
    cand = []
    for b in range(len(starts)):
        cand += [int(starts[b]), int(ends[b]) - 1]
        if local[b] < topk:
            cand.append(int(rng.integers(starts[b], ends[b])))
    for t in rng.choice(cand, size=min(n_strat, len(cand)), replace=False):
        rows.add((int(t), int(rng.integers(0, hq))))
    return sorted(rows)
