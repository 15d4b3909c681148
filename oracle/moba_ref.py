"""Plain float64 definition of the MoBA causal prefill forward (CPU, NumPy), with its decode
step, the min/max (Quest-style) gate variant and the backward pass.

TEST INFRASTRUCTURE ONLY: see ``oracle/__init__.py``.  Slow on purpose; every
step is written the way the pages define it so that it can be checked by eye.

Sources (cited by page title and section):

* "《MoBA: Mixture of Block Attention for Long-Context LLMs》深度解读报告"
  (called *the analysis* below):
  §2.1 block partitioning, §2.2 mean-pooled gate and hard top-k routing,
  §2.3 the two causality rules (future blocks masked, current block forced and
  causally masked), §3.2 the separate causal current block and the final
  online-softmax merge.
* "Paper: MoBA (Moonshot)" course module F26 (called *the course page*):
  with every block selected the method is exactly dense attention; routing is
  per query head.

Readings taken where the pages are silent (each is listed with its reason in
the design notes):

* ``topk`` counts the forced current block: a row routes ``topk - 1`` past
  blocks plus its own block.  This is what makes the analysis's printed
  sparsities come out (81.25% = 1 - 3/16 at 8K with 512-token blocks and
  top-3; 12/256 history blocks at 1M with 4096-token blocks and top-12).
* ``topk`` larger than the number of available blocks selects all of them.
* The gate score is the plain dot product, no scaling (ranking is invariant
  to any positive scale).
* Ties between equal gate scores go to the lower block index.
* A final partial block is allowed; its mean is over its valid tokens.
* The attention softmax uses ``scale`` (default ``1/sqrt(d)``); ``lse`` is the
  natural-log log-sum-exp of the scaled logits.
* GQA: query head ``h`` reads KV head ``h // (Hq // Hkv)``.

Array conventions: ``q`` is ``[T, Hq, d]``, ``k`` and ``v`` are
``[T, Hkv, d]`` (packed varlen, row ``t`` of every sequence back to back),
``cu_seqlens`` is ``[batch + 1]`` with ``cu_seqlens[0] == 0``.  All floating
point arrays are float64 (the bf16 inputs are exact in float64).
Selections ``sel`` are ``[Hq, T, topk]`` of block indices local to the row's
sequence, ascending, padded with ``-1``.
"""

import math

import numpy as np


def block_table(cu_seqlens, chunk):
    """Cut every sequence into blocks of ``chunk`` tokens.

    The analysis, §2.1: a context of length N is split into n = N/B blocks and
    block i (1-indexed) covers positions (i-1)B+1 .. iB.  With 0-indexed
    positions relative to the sequence start ``s`` this is block ``j`` =
    ``[s + j*B, s + (j+1)*B)``.  Blocks never cross a sequence boundary; a
    final partial block ends at the sequence end (reading: the pages leave the
    non-divisible case open).

    Returns a dict of int64 arrays: ``cu_blocks`` ``[batch+1]`` (block prefix
    per sequence) and, per global block, ``start``, ``end``, ``seq``,
    ``local`` (index within its sequence).
    """
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    if cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must start at 0 and be non-decreasing")
    start, end, seq, local, cu_blocks = [], [], [], [], [0]
    for i in range(len(cu) - 1):
        s, e = cu[i], cu[i + 1]
        n = (e - s + chunk - 1) // chunk
        for j in range(n):
            start.append(s + j * chunk)
            end.append(min(s + (j + 1) * chunk, e))
            seq.append(i)
            local.append(j)
        cu_blocks.append(cu_blocks[-1] + n)
    as64 = lambda x: np.asarray(x, dtype=np.int64)
    return {"cu_blocks": as64(cu_blocks), "start": as64(start), "end": as64(end),
            "seq": as64(seq), "local": as64(local)}


def block_means(k, cu_seqlens, chunk):
    """Mean-pooled key of every block, per KV head: ``[NB, Hkv, d]`` float64.

    The analysis, §2.2: the block's representation in the gate is
    meanpool(K[I_i]), the average of the block's keys.  For a partial final
    block the average is over its valid tokens.
    """
    k = np.asarray(k, dtype=np.float64)
    tab = block_table(cu_seqlens, chunk)
    nb = len(tab["start"])
    means = np.zeros((nb, k.shape[1], k.shape[2]), dtype=np.float64)
    for b in range(nb):
        rows = k[tab["start"][b]:tab["end"][b]]
        means[b] = rows.sum(axis=0) / rows.shape[0]
    return means


def block_minmax(k, cu_seqlens, chunk):
    """Per-channel minimum and maximum key of every block, per KV head.

    The analysis (§1.3 and its list of limitations, §5.1 item 6) names Quest as the MoBA
    variant with min/max pooling in place of the mean and calls it the stronger block
    summary (§6.3 lists it as the gate's next step), without writing the summary out.  Reading: Quest's published one (Tang et al.,
    2024, "Quest: Query-Aware Sparsity for Efficient Long-Context LLM Inference"), the
    element-wise minimum and maximum of the block's keys, over its valid tokens.

    Returns ``(kmin, kmax)``, each ``[NB, Hkv, d]`` float64.
    """
    k = np.asarray(k, dtype=np.float64)
    tab = block_table(cu_seqlens, chunk)
    nb = len(tab["start"])
    kmin = np.zeros((nb, k.shape[1], k.shape[2]), dtype=np.float64)
    kmax = np.zeros_like(kmin)
    for b in range(nb):
        rows = k[tab["start"][b]:tab["end"][b]]
        kmin[b] = rows.min(axis=0)
        kmax[b] = rows.max(axis=0)
    return kmin, kmax


def minmax_scores_row(q_row, minmax_rows):
    """Min/max gate affinities of one query row against a list of block summaries.

    Quest's block score (the reading of :func:`block_minmax`): per channel i the larger of
    ``q_i * kmax_i`` and ``q_i * kmin_i``, summed over the channels.  It is the largest value
    ``<q, x>`` takes over the box ``kmin <= x <= kmax``, so an upper bound of ``<q, k>`` over
    every key of the block.  ``minmax_rows`` is ``[n, 2, d]`` (index 0 = min, 1 = max);
    returns ``[n]``.
    """
    q_row = np.asarray(q_row, dtype=np.float64)
    mm = np.asarray(minmax_rows, dtype=np.float64)
    return np.maximum(mm[:, 0, :] * q_row, mm[:, 1, :] * q_row).sum(axis=1)


def gate_scores_row(q_row, means_rows):
    """Gate affinities of one query row against a list of block means.

    The analysis, §2.2: s_i = <q, meanpool(K[I_i])>, a plain inner product
    (no router parameters, no scaling).  ``q_row`` is ``[d]``,
    ``means_rows`` is ``[n, d]``; returns ``[n]``.
    """
    return np.asarray(means_rows, dtype=np.float64) @ np.asarray(q_row, dtype=np.float64)


def _route_past(scores_past, n_route):
    """Indices of the ``n_route`` largest past-block scores, ties to the lower index.

    ``scores_past`` is ``[rows, c]`` (blocks ``0..c-1`` of the sequence; every
    later block is either the forced current block or a masked future block).
    A stable sort of the negated scores keeps equal scores in ascending block
    order.  Returns ``[rows, n_route]`` ascending.
    """
    order = np.argsort(-scores_past, axis=1, kind="stable")[:, :n_route]
    return np.sort(order, axis=1)


def select_blocks(q, means, cu_seqlens, chunk, topk):
    """Top-k block selection of every query row: ``[Hq, T, topk]`` int64.

    The analysis, §2.2-§2.3, per query token and per query head (the course
    page: per-head routing):

    1. score every block of the row's sequence by ``<q, mean_j>``;
    2. rule 1: a future block (one ending after the query) gets score -inf;
    3. rule 2: the query's own block ``c = (t - s) // B`` is always selected
       (gate 1) and so does not compete;
    4. hard top-k: the ``topk - 1`` best past blocks ``j < c`` are routed
       (all of them when fewer exist).

    Blocks ``j >= c`` are therefore never candidates, which is why only the
    scores of ``j < c`` are formed.  Output rows are ascending, ``-1`` padded.
    """
    q = np.asarray(q, dtype=np.float64)
    means = np.asarray(means, dtype=np.float64)
    T, Hq, _ = q.shape
    Hkv = means.shape[1]
    if topk < 1 or Hq % Hkv:
        raise ValueError("topk >= 1 and Hq % Hkv == 0 required")
    group = Hq // Hkv
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    tab = block_table(cu, chunk)
    sel = np.full((Hq, T, topk), -1, dtype=np.int64)
    for i in range(len(cu) - 1):
        s, e = int(cu[i]), int(cu[i + 1])
        b0, b1 = int(tab["cu_blocks"][i]), int(tab["cu_blocks"][i + 1])
        for h in range(Hq):
            seq_means = means[b0:b1, h // group, :]
            for c in range(b1 - b0):
                t0, t1 = s + c * chunk, min(s + (c + 1) * chunk, e)
                n_route = min(topk - 1, c)
                if n_route > 0:
                    scores_past = q[t0:t1, h, :] @ seq_means[:c].T
                    sel[h, t0:t1, :n_route] = _route_past(scores_past, n_route)
                sel[h, t0:t1, n_route] = c
    return sel


def select_blocks_rows(q, means, cu_seqlens, chunk, topk, rows, score=gate_scores_row):
    """Selection for a list of ``(t, h)`` rows, one row at a time.

    Same definition as :func:`select_blocks` (the analysis, §2.2-§2.3), for
    sampled rows of inputs too large to select in full.  ``means`` is the block
    summary indexed ``[block, kv_head, ...]`` and ``score(q_row, summaries)``
    the gate affinity: the mean gate by default, or the stacked
    ``[NB, Hkv, 2, d]`` min/max summary with :func:`minmax_scores_row`.
    Returns ``[len(rows), topk]`` int64.
    """
    means = np.asarray(means)
    Hq, Hkv = q.shape[1], means.shape[1]
    group = Hq // Hkv
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    tab = block_table(cu, chunk)
    out = np.full((len(rows), topk), -1, dtype=np.int64)
    for r, (t, h) in enumerate(rows):
        i = int(np.searchsorted(cu, t, side="right") - 1)
        s = int(cu[i])
        c = (t - s) // chunk
        b0 = int(tab["cu_blocks"][i])
        n_route = min(topk - 1, c)
        if n_route > 0:
            sc = score(q[t, h].astype(np.float64), means[b0:b0 + c, h // group].astype(np.float64))
            out[r, :n_route] = _route_past(sc[None, :], n_route)[0]
        out[r, n_route] = c
    return out


def attended_keys(t, sel_row, cu_seqlens, chunk):
    """Key positions a query at token ``t`` attends, given its selected blocks.

    The analysis, §2.2: attention runs over the union I of the selected
    blocks.  §2.3 rule 2: inside the current block a causal mask applies, so
    only keys ``u <= t`` of block ``c`` are kept.  A past block lies wholly
    before ``t``.  A selected block after ``c`` is an error (rule 1).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    i = int(np.searchsorted(cu, t, side="right") - 1)
    s, e = int(cu[i]), int(cu[i + 1])
    c = (t - s) // chunk
    keys = []
    for j in sel_row:
        j = int(j)
        if j < 0:
            continue
        if j > c:
            raise ValueError("a future block was selected")
        a = s + j * chunk
        b = t + 1 if j == c else min(a + chunk, e)
        keys.append(np.arange(a, b, dtype=np.int64))
    return np.concatenate(keys) if keys else np.zeros(0, dtype=np.int64)


def attend_rows(q, k, v, cu_seqlens, chunk, sel, rows, scale=None):
    """Softmax attention of sampled rows over their selected blocks.

    The analysis, §2.2: out = Softmax(q^T K[I]) V[I] with I the union of the
    selected blocks, here with the logits scaled by ``scale`` (default
    ``1/sqrt(d)``), and lse = log(sum(exp(logits))).  ``sel`` is the full
    ``[Hq, T, topk]`` selection or a ``[len(rows), topk]`` one aligned with
    ``rows``.  Returns ``out [n, d]`` and ``lse [n]`` float64.
    """
    d = q.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    group = q.shape[1] // k.shape[1]
    out = np.zeros((len(rows), d), dtype=np.float64)
    lse = np.zeros(len(rows), dtype=np.float64)
    per_row = np.asarray(sel).ndim == 2
    for r, (t, h) in enumerate(rows):
        sel_row = sel[r] if per_row else sel[h, t]
        u = attended_keys(t, sel_row, cu_seqlens, chunk)
        g = h // group
        kk = np.asarray(k[u, g], dtype=np.float64)
        vv = np.asarray(v[u, g], dtype=np.float64)
        z = scale * (kk @ np.asarray(q[t, h], dtype=np.float64))
        zmax = z.max()
        p = np.exp(z - zmax)
        denom = p.sum()
        out[r] = (p @ vv) / denom
        lse[r] = zmax + math.log(denom)
    return out, lse


def attention_masked_dense(q, k, v, cu_seqlens, chunk, sel, scale=None):
    """All rows at once as masked dense causal attention.

    Second formulation of the same definition, used to cross-check
    :func:`attend_rows`: for each sequence, head and query block, the logits
    against every earlier key are formed and every key outside the row's
    selected blocks, or after the row, is set to -inf before the softmax
    (the analysis, §2.2-§2.3).  Returns ``out [T, Hq, d]``, ``lse [Hq, T]``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    group = Hq // k.shape[1]
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    out = np.zeros((T, Hq, d), dtype=np.float64)
    lse = np.zeros((Hq, T), dtype=np.float64)
    for i in range(len(cu) - 1):
        s, e = int(cu[i]), int(cu[i + 1])
        nb = (e - s + chunk - 1) // chunk
        for h in range(Hq):
            g = h // group
            for c in range(nb):
                t0, t1 = s + c * chunk, min(s + (c + 1) * chunk, e)
                key_pos = np.arange(s, t1)
                key_blk = (key_pos - s) // chunk
                qpos = np.arange(t0, t1)
                allowed = np.zeros((t1 - t0, t1 - s), dtype=bool)
                for r, t in enumerate(qpos):
                    chosen = [int(j) for j in sel[h, t] if j >= 0]
                    allowed[r] = np.isin(key_blk, chosen) & (key_pos <= t)
                z = scale * (q[t0:t1, h] @ k[s:t1, g].T)
                z = np.where(allowed, z, -np.inf)
                zmax = z.max(axis=1, keepdims=True)
                p = np.exp(z - zmax)
                denom = p.sum(axis=1, keepdims=True)
                out[t0:t1, h] = (p @ v[s:t1, g]) / denom
                lse[h, t0:t1] = zmax[:, 0] + np.log(denom[:, 0])
    return out, lse


def moba_forward(q, k, v, cu_seqlens, chunk, topk, scale=None, sel=None):
    """The whole forward: means, selection (unless given), attention.

    The five steps of the analysis's Algorithm 1 commentary (§3.2) compose to
    this plain definition: block means (§2.2), gate scores with the future
    mask and the forced current block and hard top-k (§2.2-§2.3), then
    softmax attention over the union of the selected blocks, causal inside
    the current block.  Dispatch and the online-softmax merge of §3.2 are an
    evaluation order of the same sum and so do not appear here.

    Returns a dict with ``out [T, Hq, d]``, ``lse [Hq, T]``, ``sel`` and
    ``means``, all computed in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    means = block_means(k, cu_seqlens, chunk)
    if sel is None:
        sel = select_blocks(q, means, cu_seqlens, chunk, topk)
    out, lse = attention_masked_dense(q, k, v, cu_seqlens, chunk, sel, scale)
    return {"out": out, "lse": lse, "sel": sel, "means": means}


def moba_backward(q, k, v, cu_seqlens, chunk, sel, d_out, d_lse=None, scale=None):
    """Gradients of the forward's ``out`` and ``lse`` with respect to ``q``, ``k`` and ``v``.

    Reading: the gate has no parameters (the analysis, §2.5) and routes by hard top-k (§2.2),
    so the selection is piecewise constant in ``q`` and ``k``: its derivative is zero wherever
    it exists, and the gradient reaches q, k and v only through the softmax attention over the
    selected union (§2.2-§2.3).  ``sel`` is the selection the forward used.

    Per row ``(t, h)`` with attended keys U (:func:`attended_keys`), logits
    ``z_u = scale * <q, k_u>``, ``p = softmax(z)``, ``out = sum_u p_u v_u`` and
    ``lse = log sum_u exp(z_u)``, the chain rule gives, with ``dp_u = <d_out, v_u>``:

    * ``dv_u += p_u * d_out``
    * ``dz_u = p_u * (dp_u - <d_out, out>) + p_u * d_lse``  (d lse / d z_u = p_u)
    * ``dq = scale * sum_u dz_u k_u`` and ``dk_u += scale * dz_u * q``

    A KV head collects the contributions of every query head that reads it (GQA).
    ``d_out`` is ``[T, Hq, d]``, ``d_lse`` ``[Hq, T]`` or None (zero).  Returns
    ``dq [T, Hq, d]``, ``dk`` and ``dv [T, Hkv, d]``, float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    T, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    group = Hq // k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for t in range(T):
        for h in range(Hq):
            u = attended_keys(t, sel[h, t], cu_seqlens, chunk)
            g = h // group
            z = scale * (k[u, g] @ q[t, h])
            p = np.exp(z - z.max())
            p /= p.sum()
            o = p @ v[u, g]
            dp = v[u, g] @ d_out[t, h]
            dz = p * (dp - d_out[t, h] @ o)
            if d_lse is not None:
                dz += p * float(d_lse[h, t])
            dq[t, h] = scale * (dz @ k[u, g])
            dk[u, g] += scale * np.outer(dz, q[t, h])
            dv[u, g] += np.outer(p, d_out[t, h])
    return dq, dk, dv


class _LastRowQueries:
    """``q[t, h]`` view for the decode step: the new query of the sequence whose last row is
    ``t``.  Only those rows exist (the per-row functions read nothing else)."""

    def __init__(self, q_new, cu_seqlens):
        self.q_new = np.asarray(q_new, dtype=np.float64)
        cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
        self.row_of = {int(cu[b + 1]) - 1: b for b in range(len(cu) - 1) if cu[b + 1] > cu[b]}
        self.shape = (int(cu[-1]),) + self.q_new.shape[1:]

    def __getitem__(self, th):
        t, h = th
        return self.q_new[self.row_of[int(t)], h]


def moba_decode(q_new, k, v, cu_seqlens, chunk, topk, scale=None, gate="mean"):
    """Decode step: one new query per sequence against its KV cache.

    The cache of sequence b is rows ``cu[b] .. cu[b+1]-1`` of ``k`` / ``v``; its last row is
    the new token's key and value, so the new query sits at position ``t = cu[b+1] - 1`` and
    the rule of the analysis (§2.2-§2.3) applies to it unchanged: its own block
    ``c = (t - cu[b]) // chunk`` is forced (all cached tokens of that block precede or equal t),
    the ``topk - 1`` best earlier blocks by ``q . mean_j`` are routed, and the softmax runs over
    the union.  This is exactly the prefill forward's row t, computed row by row.

    ``gate="minmax"`` scores the earlier blocks with the min/max summary instead
    (:func:`block_minmax`, :func:`minmax_scores_row`); everything else is unchanged.

    ``q_new`` is ``[batch, Hq, d]``.  Returns ``out [batch, Hq, d]``, ``lse [Hq, batch]`` and
    ``sel [batch, Hq, topk]`` (float64 / int64); an empty sequence has no query: zeros, -inf
    and an all ``-1`` selection.
    """
    q_new = np.asarray(q_new, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    batch, Hq, d = q_new.shape
    out = np.zeros((batch, Hq, d), dtype=np.float64)
    lse = np.full((Hq, batch), -np.inf, dtype=np.float64)
    sel = np.full((batch, Hq, topk), -1, dtype=np.int64)
    rows = [(int(cu[b + 1]) - 1, h) for b in range(batch) if cu[b + 1] > cu[b] for h in range(Hq)]
    if not rows:
        return {"out": out, "lse": lse, "sel": sel}
    qv = _LastRowQueries(q_new, cu)
    if gate == "mean":
        s_rows = select_blocks_rows(qv, block_means(k, cu, chunk), cu, chunk, topk, rows)
    elif gate == "minmax":
        kmin, kmax = block_minmax(k, cu, chunk)
        s_rows = select_blocks_rows(qv, np.stack([kmin, kmax], axis=2), cu, chunk, topk, rows,
                                    score=minmax_scores_row)
    else:
        raise ValueError("gate must be 'mean' or 'minmax'")
    o_rows, l_rows = attend_rows(qv, k, v, cu, chunk, s_rows, rows, scale)
    for r, (t, h) in enumerate(rows):
        b = qv.row_of[t]
        out[b, h] = o_rows[r]
        lse[h, b] = l_rows[r]
        sel[b, h] = s_rows[r]
    return {"out": out, "lse": lse, "sel": sel}
