"""The float64 oracle on many host cores, for the full-size GPU parity tests.

Test infrastructure only.  Nothing here computes any part of the method: every function
below calls an ``oracle`` function unchanged on an independent piece of the problem (one
query head, or one group of sampled rows of one KV head) and the pieces are spread over
worker processes.  Rows of different heads are independent in the definition (the analysis
page of the MoBA paper, §2.2-§2.3: the gate and the attention are per query row and per
query head), so the pieces together are exactly the oracle's result.

The pool is started with the ``spawn`` method: the test process has already initialised CUDA,
and a child forked from it can hang.  Inputs travel as bf16 bit patterns (uint16) and are
widened exactly inside the worker.  Each worker runs one BLAS thread.
"""

import math
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

import oracle
import parity as PT


def n_workers():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return max(1, min(n, int(os.environ.get("MOBA_ORACLE_WORKERS", "32"))))


def _init_worker():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass


def pool():
    """A spawn-started process pool (use as a context manager)."""
    return ProcessPoolExecutor(n_workers(), mp_context=mp.get_context("spawn"),
                               initializer=_init_worker)


class Shared:
    """Large read-only inputs shared with the workers through .npy files in shared memory
    (/dev/shm when it has room, else the temporary directory), which each worker memory-maps
    once, instead of pickling them into every task.  Use as a context manager; ``ref(name)``
    is what a task receives."""

    def __init__(self, **arrays):
        import shutil
        import tempfile
        need = sum(a.nbytes for a in arrays.values()) + (1 << 30)
        base = "/dev/shm" if os.path.isdir("/dev/shm") and shutil.disk_usage("/dev/shm").free > need else None
        self.dir = tempfile.mkdtemp(prefix="moba_oracle_", dir=base)
        self.paths = {}
        for name, a in arrays.items():
            path = os.path.join(self.dir, name + ".npy")
            np.save(path, np.ascontiguousarray(a))
            self.paths[name] = path

    def ref(self, name):
        return self.paths[name]

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        import shutil
        shutil.rmtree(self.dir, ignore_errors=True)


_maps = {}


def _mapped(path):
    """The memory-mapped array at path (opened once per worker process)."""
    if path not in _maps:
        _maps[path] = np.load(path, mmap_mode="r")
    return _maps[path]


# ---- worker tasks (top level, so that they pickle) ------------------------------------------

def _dense_head(q16, k16, v16, cu, chunk, sel_h, scale):
    """oracle.attention_masked_dense for one query head: q16 [T, d], k16 / v16 [T, d] of its
    KV head, sel_h [T, topk].  Returns out [T, d], lse [T]."""
    q = PT.from_bits(q16)[:, None, :]
    k = PT.from_bits(k16)[:, None, :]
    v = PT.from_bits(v16)[:, None, :]
    out, lse = oracle.attention_masked_dense(q, k, v, cu, chunk, sel_h[None], scale)
    return out[:, 0, :], lse[0]


def _select_head(q16, means_g, cu, chunk, topk):
    """oracle.select_blocks for one query head against its KV head's block summary.
    Returns [T, topk] int16."""
    q = PT.from_bits(q16)[:, None, :]
    sel = oracle.select_blocks(q, means_g[:, None, :], cu, chunk, topk)
    return sel[0].astype(np.int16)


def _compare_head(gsel_h, osel_h, q16, means_g, cu, chunk, topk):
    """Rows of one head whose GPU selection differs from the oracle's: returns (tokens of the
    rows that are valid near-tie alternatives, list of the other rows)."""
    diff = np.nonzero((gsel_h != osel_h).any(axis=1))[0]
    ties, bad = [], []
    for t in diff:
        t = int(t)
        _, b0, c = PT.row_block(cu, chunk, t)
        sc = oracle.gate_scores_row(PT.from_bits(q16[t]).astype(np.float64), means_g[b0:b0 + c])
        if PT.near_tie_alternative(gsel_h[t], osel_h[t], sc, c, topk):
            ties.append(t)
        else:
            bad.append((t, [int(x) for x in gsel_h[t]], [int(x) for x in osel_h[t]]))
    return np.asarray(ties, dtype=np.int64), bad


def _select_rows(q_rows16, ts, summary_g, cu, chunk, topk, minmax):
    """oracle.select_blocks_rows for sampled tokens of one query head: the mean gate against
    summary_g [NB, d], or the min/max gate against summary_g [NB, 2, d] (min, max)."""
    score = oracle.minmax_scores_row if minmax else oracle.gate_scores_row
    return oracle.select_blocks_rows(_RowsView(q_rows16, ts), summary_g[:, None], cu, chunk, topk,
                                     [(int(t), i) for i, t in enumerate(ts)], score=score)


def _attend(q_rows16, ts, k16, v16, cu, chunk, sel_rows, scale):
    """oracle.attend_rows for sampled tokens of query heads of one KV head: q_rows16 [n, d]
    (each row's own query), ts [n], k16 / v16 [T, d], sel_rows [n, topk]."""
    k = PT.from_bits(k16)[:, None, :]
    v = PT.from_bits(v16)[:, None, :]
    return oracle.attend_rows(_RowsView(q_rows16, ts), k, v, cu, chunk, sel_rows,
                              [(int(t), i) for i, t in enumerate(ts)], scale)


def _attend_shared(q_rows16, ts, kpath, vpath, g, cu, chunk, sel_rows, scale):
    """As _attend, with KV head g of the shared head-major keys and values, read row by row
    from the memory map.  Returns (out, lse, CPU seconds of the task)."""
    import time
    c0 = time.process_time()
    o, l = oracle.attend_rows(_RowsView(q_rows16, ts), _HeadRows(kpath, g), _HeadRows(vpath, g), cu, chunk,
                              sel_rows, [(int(t), i) for i, t in enumerate(ts)], scale)
    return o, l, time.process_time() - c0


class _HeadRows:
    """k[u, 0] stand-in for oracle.attend_rows over one head of a shared head-major bf16-bits
    file: the rows u are read from the memory map and widened exactly when asked for."""

    def __init__(self, path, g):
        self.rows = _mapped(path)[g]
        self.shape = (self.rows.shape[0], 1, self.rows.shape[1])

    def __getitem__(self, idx):
        u, g = idx
        assert g == 0
        return PT.from_bits64(self.rows[np.asarray(u)])


def _select_compare_shared(qpath, h, means_g, gsel_h, cu, chunk, topk):
    """oracle.select_blocks for query head h of the shared head-major q, then the comparison
    with the GPU's selection of that head (as _compare_head).  Returns (oracle selection int16,
    near-tie tokens, other differing rows, CPU seconds)."""
    import time
    c0 = time.process_time()
    q16 = np.asarray(_mapped(qpath)[h])
    osel = _select_head(q16, means_g, cu, chunk, topk)
    ties, bad = (np.zeros(0, dtype=np.int64), []) if gsel_h is None else \
        _compare_head(gsel_h, osel, q16, means_g, cu, chunk, topk)
    return osel, ties, bad, time.process_time() - c0


def _backward_head(q_h, k_g, v_g, cu, chunk, sel_h, dout_h, dlse_h, scale):
    """oracle.moba_backward for one query head against its KV head: returns that head's dq and
    its contribution to the KV head's dk and dv."""
    dq, dk, dv = oracle.moba_backward(q_h[:, None], k_g[:, None], v_g[:, None], cu, chunk, sel_h[None],
                                      dout_h[:, None], None if dlse_h is None else dlse_h[None], scale)
    return dq[:, 0], dk[:, 0], dv[:, 0]


class _RowsView:
    """q stand-in for oracle.attend_rows / select_blocks_rows over n sampled rows that all read
    one KV head: row (t, i) is the i-th sampled row's query.  With n "heads" against one KV
    head, the oracle's GQA mapping sends every row to that KV head."""

    def __init__(self, q_rows16, ts):
        self.q = q_rows16
        self.ts = np.asarray(ts)
        self.shape = (None, len(ts), q_rows16.shape[1])

    def __getitem__(self, idx):
        t, i = idx
        assert int(self.ts[i]) == int(t)
        return PT.from_bits(self.q[i])


# ---- drivers used by the tests -----------------------------------------------------------------

def dense_all_heads(ex, q16, k16, v16, cu, chunk, sel, scale=None):
    """oracle.attention_masked_dense over all heads: q16 [T, Hq, d], k16 / v16 [T, Hkv, d]
    (bf16 bits), sel [Hq, T, topk].  Returns out [T, Hq, d], lse [Hq, T] (float64)."""
    T, hq, d = q16.shape
    group = hq // k16.shape[1]
    futs = [ex.submit(_dense_head, np.ascontiguousarray(q16[:, h]), np.ascontiguousarray(k16[:, h // group]),
                      np.ascontiguousarray(v16[:, h // group]), cu, chunk, np.ascontiguousarray(sel[h]), scale)
            for h in range(hq)]
    out = np.zeros((T, hq, d))
    lse = np.zeros((hq, T))
    for h, f in enumerate(futs):
        out[:, h], lse[h] = f.result()
    return out, lse


def select_and_compare_heads(ex, q_head16, means, gsel, cu, chunk, topk, group, heads):
    """oracle.select_blocks per listed head, compared with the GPU's selection of that head.
    q_head16(h) returns that head's q bits [T, d]; gsel(h) its GPU selection [T, topk].
    Returns {h: (oracle selection [T, topk] int16, tie tokens)}; fails on any row that is not
    a valid near-tie alternative."""
    sel_f = {h: ex.submit(_select_head, q_head16(h), np.ascontiguousarray(means[:, h // group]), cu,
                          chunk, topk) for h in heads}
    res, cmp_f = {}, {}
    for h in heads:
        osel = sel_f[h].result()
        g = gsel(h)
        res[h] = osel
        cmp_f[h] = ex.submit(_compare_head, g, osel, q_head16(h), np.ascontiguousarray(means[:, h // group]),
                             cu, chunk, topk)
    out = {}
    bad = []
    for h in heads:
        ties, b = cmp_f[h].result()
        bad += [(h,) + x for x in b]
        out[h] = (res[h], ties)
    assert not bad, f"{len(bad)} selection mismatches outside the near-tie band: {bad[:5]}"
    return out


def attend_rows_par(ex, rows, q_row16, k16, v16, cu, chunk, sel_rows, group, scale=None):
    """oracle.attend_rows for sampled (t, h) rows, grouped by KV head.  q_row16 [n, d] holds
    each row's query bits, sel_rows [n, topk] its selection, k16 / v16 [T, Hkv, d] the keys
    and values (bf16 bits).  Returns out [n, d], lse [n] in the order of ``rows``.  About one
    task per worker, so that each KV head's keys and values travel to few workers."""
    n = len(rows)
    rows_per_task = max(256, math.ceil(n / n_workers()))
    g_of = np.array([h // group for _, h in rows])
    ts = np.array([t for t, _ in rows])
    futs = []
    for g in np.unique(g_of):
        idx = np.nonzero(g_of == g)[0]
        kg = np.ascontiguousarray(k16[:, g])
        vg = np.ascontiguousarray(v16[:, g])
        n_tasks = max(1, math.ceil(len(idx) / rows_per_task))
        for part in np.array_split(idx, n_tasks):
            futs.append((part, ex.submit(_attend, q_row16[part], ts[part], kg, vg, cu, chunk,
                                         sel_rows[part], scale)))
    out = np.zeros((n, q_row16.shape[1]))
    lse = np.zeros(n)
    for part, f in futs:
        out[part], lse[part] = f.result()
    return out, lse


def select_rows_par(ex, rows, q_row16, means, cu, chunk, topk, group, minmax=False):
    """oracle.select_blocks_rows for sampled (t, h) rows, split by head into about one task
    per worker.  ``means`` is [NB, Hkv, d], or [NB, Hkv, 2, d] (min, max) with minmax=True."""
    hs = np.array([h for _, h in rows])
    ts = np.array([t for t, _ in rows])
    res = np.zeros((len(rows), topk), dtype=np.int64)
    futs = []
    per_task = max(64, math.ceil(len(rows) / n_workers()))
    for h in np.unique(hs):
        idx_h = np.nonzero(hs == h)[0]
        for idx in np.array_split(idx_h, max(1, math.ceil(len(idx_h) / per_task))):
            futs.append((idx, ex.submit(_select_rows, q_row16[idx], ts[idx],
                                        np.ascontiguousarray(means[:, h // group]), cu, chunk, topk, minmax)))
    for idx, f in futs:
        res[idx] = f.result()
    return res


def backward_by_head(ex, q, k, v, cu, chunk, sel, d_out, d_lse=None, scale=None):
    """oracle.moba_backward split by query head: dq of each head is that head's; dk and dv of a
    KV head are the sums of its query heads' contributions (the oracle's GQA rule)."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    futs = [ex.submit(_backward_head, np.ascontiguousarray(q[:, h]), np.ascontiguousarray(k[:, h // group]),
                      np.ascontiguousarray(v[:, h // group]), cu, chunk, np.ascontiguousarray(sel[h]),
                      np.ascontiguousarray(d_out[:, h]), None if d_lse is None else np.ascontiguousarray(d_lse[h]),
                      scale) for h in range(hq)]
    dq = np.zeros((T, hq, d))
    dk = np.zeros((T, hkv, d))
    dv = np.zeros((T, hkv, d))
    for h, f in enumerate(futs):
        a, b, c = f.result()
        dq[:, h] = a
        dk[:, h // group] += b
        dv[:, h // group] += c
    return dq, dk, dv


class Pending:
    """Futures submitted to the pool and the function that assembles their results."""

    def __init__(self, futs, finish):
        self.futs, self.finish = futs, finish

    def result(self):
        return self.finish([f.result() for f in self.futs])


def submit_attend_shared(ex, rows, q_row16, shared, cu, chunk, sel_rows, group, scale=None):
    """oracle.attend_rows over the (t, h) rows with the keys and values of ``shared`` ("k",
    "v": head-major [Hkv, T, d] bf16 bits), in tasks of one KV head, about four per worker.
    ``.result()`` gives (out [n, d], lse [n], CPU seconds of all tasks)."""
    n = len(rows)
    per_task = max(32, math.ceil(n / (4 * n_workers())))
    g_of = np.array([h // group for _, h in rows], dtype=np.int64)
    ts = np.array([t for t, _ in rows], dtype=np.int64)
    parts, futs = [], []
    for g in np.unique(g_of):
        idx = np.nonzero(g_of == g)[0]
        for part in np.array_split(idx, max(1, math.ceil(len(idx) / per_task))):
            parts.append(part)
            futs.append(ex.submit(_attend_shared, q_row16[part], ts[part], shared.ref("k"), shared.ref("v"),
                                  int(g), cu, chunk, sel_rows[part], scale))

    def finish(res):
        out = np.zeros((n, q_row16.shape[1]))
        lse = np.zeros(n)
        cpu = 0.0
        for part, (o, l, c) in zip(parts, res):
            out[part], lse[part] = o, l
            cpu += c
        return out, lse, cpu

    return Pending(futs, finish)


def submit_select_compare_shared(ex, shared, means, gsel, cu, chunk, topk, group, heads):
    """oracle.select_blocks for each listed query head of ``shared`` ("q": head-major
    [Hq, T, d] bf16 bits) against its KV head's summary, compared with gsel(h) (the GPU's
    selection of the head, or None to skip the comparison).  ``.result()`` gives
    {h: (oracle selection int16 [T, topk], near-tie tokens)} and fails on any row that is not a
    valid near-tie alternative."""
    heads = list(heads)
    futs = [ex.submit(_select_compare_shared, shared.ref("q"), int(h), np.ascontiguousarray(means[:, h // group]),
                      gsel(h), cu, chunk, topk) for h in heads]

    def finish(res):
        out, bad = {}, []
        for h, (osel, ties, b, _) in zip(heads, res):
            bad += [(h,) + x for x in b]
            out[h] = (osel, ties)
        assert not bad, f"{len(bad)} selection mismatches outside the near-tie band: {bad[:5]}"
        return out

    return Pending(futs, finish)


def timed(name, *args):
    """Runs the task ``name`` of this module in the worker and returns (its result, the CPU
    seconds it took)."""
    import time
    c0 = time.process_time()
    r = globals()[name](*args)
    return r, time.process_time() - c0
