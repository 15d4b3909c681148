"""The selection method of the tensor-core gate, restated on the host and checked against the
definition of the hard top-k (the analysis page of the MoBA paper, §2.2-§2.3: the topk - 1 best
past blocks, ties to the lower block index).

The kernel (csrc/gate_tc.cu) never sorts (score, index) pairs.  Per row it
  1. keeps the k largest scores as values only, inserting the scores two at a time by a min/max
     merge network: val'[i] = max(val[i], min(val[i-1], a), min(val[i-2], b)) for a pair a >= b
     (val[-1] = val[-2] = +inf);
  2. marks the blocks whose score is at least v_k, the smallest kept value;
  3. when equal scores at v_k mark more than k blocks, drops the highest of them.
This file checks, on random rows with many exact ties, that these steps give the same block set
as sorting by (score descending, index ascending).  It tests the method, not the kernel: the GPU
parity tests compare the kernel's selections with the oracle's.
"""

import numpy as np
import pytest


def network_topk(scores, k, kmax):
    """Steps 1-3 above in float32, with a list of kmax >= k positions as the kernel keeps."""
    s = np.asarray(scores, dtype=np.float32)
    val = [np.float32(-np.inf)] * kmax
    x = list(s) + ([np.float32(-np.inf)] if len(s) % 2 else [])
    for e in range(0, len(x), 2):
        a, b = max(x[e], x[e + 1]), min(x[e], x[e + 1])
        old = list(val)
        for i in range(kmax - 1, 1, -1):
            val[i] = max(old[i], min(old[i - 1], a), min(old[i - 2], b))
        if kmax >= 2:
            val[1] = max(old[1], min(old[0], a), b)
        val[0] = max(old[0], a)
    vk = min(val[:k])
    marked = [j for j in range(len(s)) if s[j] >= vk]
    excess = len(marked) - k
    for j in reversed(list(marked)):
        if excess <= 0:
            break
        if s[j] == vk:
            marked.remove(j)
            excess -= 1
    return sorted(marked)


def definition_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda j: (-float(scores[j]), j))
    return sorted(order[:k])


@pytest.mark.parametrize("kmax", [2, 4, 8, 11, 16, 32])
def test_network_selection_equals_the_sorted_top_k(kmax):
    rng = np.random.default_rng(kmax)
    for trial in range(300):
        k = int(rng.integers(1, kmax + 1))
        c = int(rng.integers(k + 1, 257))
        kind = trial % 3
        if kind == 0:
            s = rng.standard_normal(c).astype(np.float32)
        elif kind == 1:
            s = rng.integers(-3, 4, c).astype(np.float32)  # many exact ties
        else:
            s = np.full(c, np.float32(rng.standard_normal()), np.float32)
            s[rng.integers(0, c, 5)] += 1  # a few distinct scores above a plateau of ties
        assert network_topk(s, k, kmax) == definition_topk(s, k), (k, kmax, c)


def test_all_equal_scores_keep_the_lowest_blocks():
    s = np.zeros(40, np.float32)
    assert network_topk(s, 11, 11) == list(range(11))
