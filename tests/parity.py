"""Comparison helpers for the GPU parity tests (CUDA path through the C ABI vs the oracle).

Tolerances (bf16 inputs, fp32 accumulation):
  * block means: the fp32 recursive-summation bound, |err| <= (n_seq + 12) u sum|k| / n,
    u = 2^-24, n_seq = the longest per-thread chain (ceil(n / 8));
  * selections: every GPU row is well formed (routed past blocks ascending and distinct, then
    the own block, then -1) and routes the oracle's blocks, except that a block may be
    swapped for another whose oracle gate score lies within 1e-3 relative of it (a near tie at
    the top-k cut); feeding the oracle's selection removes that exception;
  * out: max-abs 2e-2 and mean-abs 2e-3; lse: abs 1e-3.  A row whose GPU selection is a valid
    near-tie alternative is checked against the oracle's attention over the GPU's selection,
    so no row is left out of the output check.
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


def bf16_bits(t):
    """bf16 tensor -> numpy uint16 of its bit patterns (half the bytes of a float32 copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(u16):
    """uint16 bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(u16).astype(np.uint32) << 16).view(np.float32)


# every bf16 bit pattern's value as float64 (exact): one table lookup widens bf16 bits to
# float64 in a single pass over the data
with np.errstate(invalid="ignore"):  # the NaN patterns widen to NaN, as they should
    BF16_TO_F64 = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def from_bits64(u16):
    """uint16 bf16 bit patterns -> float64 (exact), through BF16_TO_F64."""
    return BF16_TO_F64[np.asarray(u16)]


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


def row_block(cu, chunk, t):
    """(sequence start, first global block of the sequence, own block c) of token t."""
    cu = np.asarray(cu)
    i = int(np.searchsorted(cu, t, side="right") - 1)
    nb = (np.diff(cu[:i + 1]) + chunk - 1) // chunk
    return int(cu[i]), int(nb.sum()), (t - int(cu[i])) // chunk


def well_formed(sel_row, c, topk):
    """A selection row as the library writes it: min(topk - 1, c) distinct routed past blocks
    in ascending order, then the own block c, then -1 padding."""
    n = min(topk - 1, c)
    r = [int(x) for x in sel_row]
    routed = r[:n]
    return (all(0 <= j < c for j in routed) and routed == sorted(set(routed))
            and r[n] == c and all(x == -1 for x in r[n + 1:]))


def near_tie_alternative(gpu_row, ref_row, scores, c, topk, tie_rel=TIE_REL, slack=None):
    """True when gpu_row is a well-formed selection that routes the oracle's blocks except for
    swaps at the top-k cut: every oracle block it drops and every block it routes instead have
    oracle scores within tie_rel (relative) of each other, or, when ``slack`` (an absolute error
    bound of the GPU's score per block) is given, within the sum of their two bounds.
    ``scores`` are the oracle's gate scores of blocks 0..c-1 of the row."""
    if not well_formed(gpu_row, c, topk):
        return False
    n = min(topk - 1, c)
    g = {int(x) for x in gpu_row[:n]}
    o = {int(x) for x in ref_row[:n]}
    for i in o - g:
        for j in g - o:
            a, b = float(scores[i]), float(scores[j])
            band = tie_rel * max(abs(a), abs(b)) if slack is None else float(slack[i] + slack[j])
            if a - b > band:
                return False
    return True


def minmax_slack(q_row, summary_rows):
    """Absolute error bound of the GPU's min/max gate score of each block: the score is the fp32
    sum of the 2d exact products q+_i kmax_i and q-_i kmin_i (q+ = max(q, 0), q- = min(q, 0)),
    added in an order the tensor core chooses, so it is off by at most
    (2d - 1) 2^-24 sum_i (|q+_i kmax_i| + |q-_i kmin_i|).  ``summary_rows`` is [n, 2, d]
    (index 0 = min, 1 = max)."""
    q = np.asarray(q_row, dtype=np.float64)
    mm = np.asarray(summary_rows, dtype=np.float64)
    qp, qn = np.maximum(q, 0.0), np.minimum(q, 0.0)
    mag = np.abs(mm[:, 1, :] * qp).sum(axis=1) + np.abs(mm[:, 0, :] * qn).sum(axis=1)
    return (2 * q.shape[0] - 1) * 2.0 ** -24 * mag


def check_selection(gpu_sel, ref_sel, rows, q, summary, cu, chunk, topk, group,
                    score=oracle.gate_scores_row, tie_rel=TIE_REL, slack_fn=None):
    """gpu_sel / ref_sel: [n, topk] for the listed (t, h) rows.  Returns the set of row
    indices whose GPU selection differs from the oracle's as a valid near-tie alternative
    (``near_tie_alternative``; with ``slack_fn(q_row, summary_rows)`` the band is the GPU's
    error bound per block instead of the relative band); any other difference, or a malformed
    row, fails."""
    gpu_sel = np.asarray(gpu_sel)
    ref_sel = np.asarray(ref_sel)
    ties = set()
    bad = []
    diff = np.nonzero((gpu_sel != ref_sel).any(axis=1))[0]
    for r in diff:
        t, h = rows[r]
        _, b0, c = row_block(cu, chunk, t)
        q_row = np.asarray(q[t, h], dtype=np.float64)
        summ = np.asarray(summary[b0:b0 + c, h // group], dtype=np.float64)
        sc = score(q_row, summ)
        slack = slack_fn(q_row, summ) if slack_fn is not None else None
        if near_tie_alternative(gpu_sel[r], ref_sel[r], sc, c, topk, tie_rel, slack):
            ties.add(int(r))
        else:
            bad.append((t, h, list(gpu_sel[r]), list(ref_sel[r])))
    assert not bad, f"{len(bad)} selection mismatches outside the near-tie band: {bad[:5]}"
    return ties


def check_out(out_gpu, lse_gpu, out_ref, lse_ref):
    """out [n, d] and lse [n] of the same rows, every row checked."""
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    out_ref = np.asarray(out_ref, dtype=np.float64)
    err = np.abs(out_gpu - out_ref)
    lerr = np.abs(np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_ref, dtype=np.float64))
    stats = {"out_max_abs": float(err.max()), "out_mean_abs": float(err.mean()),
             "lse_max_abs": float(lerr.max()), "rows": int(out_gpu.shape[0])}
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


def sample_rows_per_head(cu, chunk, hq, topk, n_uniform, n_strat, seed):
    """For every head: n_uniform uniformly drawn tokens plus n_strat stratified ones (first and
    last token of blocks, and tokens of blocks 0..topk-1, where c < topk), distinct per head."""
    rng = np.random.default_rng(seed)
    cu = np.asarray(cu)
    T = int(cu[-1])
    tab = oracle.block_table(cu, chunk)
    cand = []
    for b in range(len(tab["start"])):
        s, e = int(tab["start"][b]), int(tab["end"][b])
        cand += [s, e - 1]
        if tab["local"][b] < topk:
            cand += [int(x) for x in rng.integers(s, e, 4)]
    cand = np.unique(np.asarray(cand))
    rows = []
    for h in range(hq):
        ts = set(int(t) for t in rng.choice(cand, size=min(n_strat, len(cand)), replace=False))
        while len(ts) < min(T, n_uniform + n_strat):
            ts.update(int(t) for t in rng.integers(0, T, n_uniform + n_strat - len(ts)))
        rows += [(t, h) for t in sorted(ts)]
    return rows
