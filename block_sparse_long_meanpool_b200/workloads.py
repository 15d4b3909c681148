"""Seeded synthetic workloads for the MoBA prefill forward.

This module only makes inputs: shapes, seeds and the value structure of the
five workloads (block-offset keys, planted needle blocks, packed varlen
sequences).  It holds none of the method's arithmetic (no block means, gate
scores, selection or attention), so both the CUDA path and the float64 oracle
can be fed from it.  It also holds the algorithmic FLOP count used to report
throughput, which is a measurement formula, not part of the forward.

Every tensor is drawn from a ``torch.Generator`` seeded per workload, in
float32, then rounded to bf16 (round to nearest even).  The same call on the
same device gives the same bits.
"""

from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    seqlens: List[int]
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    chunk_size: int
    topk: int
    structure: str  # "qk_offsets" | "k_offsets" | "needles"
    seed: int
    description: str = ""

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def cu_seqlens(self) -> List[int]:
        cu = [0]
        for n in self.seqlens:
            cu.append(cu[-1] + int(n))
        return cu

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens)) if self.seqlens else 0


# The five workloads.  Shapes follow the analysis page's training/eval
# settings (8K/512/top-3, 32K/512/top-3, 1M/4096/top-12) and a varlen GQA mix.
WORKLOADS = {
    "tiny_2k": Workload(
        "tiny_2k", [2048], 4, 4, 64, 256, 3, "qk_offsets", 1001,
        "1 x 2048 tokens, 4 heads MHA, d=64, chunk 256 (8 blocks), top-3"),
    "scaling_8k": Workload(
        "scaling_8k", [8192, 8192], 16, 16, 128, 512, 3, "k_offsets", 1002,
        "2 x 8192 tokens, 16 heads MHA, d=128, chunk 512 (16 blocks), top-3"),
    "long_32k": Workload(
        "long_32k", [32768], 32, 32, 128, 512, 3, "needles", 1003,
        "1 x 32768 tokens, 32 heads MHA, d=128, chunk 512 (64 blocks), top-3, 8 needle blocks"),
    "varlen_gqa": Workload(
        "varlen_gqa", [1000, 5000, 17000, 40000], 32, 8, 128, 1024, 4, "k_offsets", 1004,
        "4 packed sequences {1000,5000,17000,40000}, 32 q / 8 kv heads, d=128, chunk 1024, top-4"),
    "prefill_1m": Workload(
        "prefill_1m", [1048576], 32, 8, 128, 4096, 12, "k_offsets", 1005,
        "1 x 1,048,576 tokens, 32 q / 8 kv heads, d=128, chunk 4096 (256 blocks), top-12"),
}

# Sweeps on the same kernels.
# Block granularity at fixed 75% sparsity on 32K tokens: n blocks, n/4 selected (the analysis,
# §4.2, Figure 4: 8 choose 2 ... 128 choose 32).
GRANULARITY_32K = {
    f"fine_32k_{n}_{n // 4}": Workload(
        f"fine_32k_{n}_{n // 4}", [32768], 32, 8, 128, 32768 // n, n // 4, "k_offsets", 1100 + n,
        f"1 x 32768 tokens, 32 q / 8 kv heads, d=128, {n} blocks of {32768 // n}, top-{n // 4}")
    for n in (8, 16, 32, 64, 128)
}
# Context length with block count and top-k fixed and the block size growing with the
# length (the analysis, §4.5: how the 10M-token measurement was set up), Llama-3.1-8B shape.
LENGTH_SWEEP = {
    f"prefill_{m}m": Workload(
        f"prefill_{m}m", [m << 20], 32, 8, 128, (m << 20) // 256, 12, "k_offsets", 1200 + m,
        f"1 x {m << 20} tokens, 32 q / 8 kv heads, d=128, 256 blocks of {(m << 20) // 256}, top-12")
    for m in (2, 4)
}
# The 1M workload's block shape (4096-token blocks, top-12, 32 q / 8 kv heads) on 128K tokens:
# small enough for a full profiler capture of one attention launch.
LENGTH_SWEEP["prefill_128k"] = Workload(
    "prefill_128k", [1 << 17], 32, 8, 128, 4096, 12, "k_offsets", 1230,
    "1 x 131072 tokens, 32 q / 8 kv heads, d=128, 32 blocks of 4096, top-12")
# 10M tokens with the same 256 blocks and top-12 (blocks of 40,960 tokens).  A 32 q / 8 kv-head
# layer does not fit one GPU at this length (q and out alone are 168 GB), so this is one GPU's
# share of it when the layer is split four ways by KV-head group: 8 q / 2 kv heads.
LENGTH_SWEEP["prefill_10m"] = Workload(
    "prefill_10m", [10 << 20], 8, 2, 128, (10 << 20) // 256, 12, "k_offsets", 1210,
    "1 x 10485760 tokens, 8 q / 2 kv heads (a quarter of a 32/8-head layer), d=128, "
    "256 blocks of 40960, top-12")
# A packed training batch of many short sequences: 64 x 8192 tokens, 1024 blocks of 512 in all
# but 16 per sequence (the gate is sized by the longest sequence, given as max_seqlen).
PACKED = {
    "packed_64x8k": Workload(
        "packed_64x8k", [8192] * 64, 32, 8, 128, 512, 3, "k_offsets", 1400,
        "64 packed sequences of 8192 tokens, 32 q / 8 kv heads, d=128, chunk 512 (16 blocks each, "
        "1024 in all), top-3"),
}
ALL_WORKLOADS = {**WORKLOADS, **GRANULARITY_32K, **LENGTH_SWEEP, **PACKED}

# Decode step: caches of these shapes, one new query per sequence (its last row).
DECODE_WORKLOADS = {
    "decode_32k_b64": Workload(
        "decode_32k_b64", [32768] * 64, 32, 8, 128, 512, 3, "k_offsets", 1301,
        "64 caches of 32768 tokens, 32 q / 8 kv heads, d=128, chunk 512 (64 blocks), top-3"),
    "decode_128k_b16": Workload(
        "decode_128k_b16", [131072] * 16, 32, 8, 128, 2048, 8, "k_offsets", 1302,
        "16 caches of 131072 tokens, 32 q / 8 kv heads, d=128, chunk 2048 (64 blocks), top-8"),
    "decode_1m_b1": Workload(
        "decode_1m_b1", [1 << 20], 32, 8, 128, 4096, 12, "k_offsets", 1303,
        "1 cache of 1,048,576 tokens, 32 q / 8 kv heads, d=128, chunk 4096 (256 blocks), top-12"),
}


def decode_attended_keys(seqlens, chunk, topk):
    """Keys one new query attends to, summed over the sequences: its own block up to the new
    token plus min(topk - 1, c) whole earlier blocks.  A measurement formula."""
    keys = 0
    for n in seqlens:
        if n <= 0:
            continue
        c = (n - 1) // chunk
        keys += (n - c * chunk) + chunk * min(topk - 1, c)
    return keys


def custom(name, seqlens, hq, hkv, d, chunk, topk, structure="k_offsets", seed=7):
    """A workload of any shape with the same value recipe (for tests and sweeps)."""
    return Workload(name, [int(x) for x in seqlens], hq, hkv, d, chunk, topk, structure, seed)


def _block_layout(seqlens, chunk):
    """Token -> (sequence, block start offsets) bookkeeping for planting structure."""
    blocks = []  # (seq, start, end)
    for i, (s, n) in enumerate(zip(_cum(seqlens), seqlens)):
        for j in range((n + chunk - 1) // chunk):
            blocks.append((i, s + j * chunk, min(s + (j + 1) * chunk, s + n)))
    return blocks


def _cum(seqlens):
    out, acc = [], 0
    for n in seqlens:
        out.append(acc)
        acc += n
    return out


def _token_block_ids(seqlens, chunk, device):
    lens = [e - s for (_, s, e) in _block_layout(seqlens, chunk)]
    ids = torch.arange(len(lens), device=device)
    return torch.repeat_interleave(ids, torch.tensor(lens, device=device))


def _randn(gen, shape, device, chunk_rows=1 << 16):
    """N(0,1) float32, drawn in row chunks so that huge inputs stay bounded."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(r0 + chunk_rows, shape[0])
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """Seeded bf16 ``q [T,Hq,d]``, ``k``/``v [T,Hkv,d]`` and int32 ``cu_seqlens``.

    Value recipe per structure:

    * ``k_offsets``: q, k, v ~ N(0,1); every (block, kv head) draws an offset
      vector ~ 0.5 N(0, I_d) that is added to each key row of that block.
    * ``qk_offsets``: as ``k_offsets``; in addition a Bernoulli(0.1) subset of
      query rows (t, h) gets the offset of a block chosen uniformly among the
      blocks of its sequence that start at or before t.
    * ``needles``: q, k, v ~ N(0,1); 8 distinct needle blocks per sequence
      (uniform in 1..nb-2) each get a random unit direction u per kv head; their
      key noise is antithetic (the second half of the block's rows are the first
      half's draws negated) and 2.0 u is added to each key row, so the block's
      mean key is 2u up to the bf16 rounding.  A Bernoulli(0.05) subset of
      query rows that have a needle block strictly before their own block is
      replaced by |q| (0.8 u + 0.6 w), w a random unit vector orthogonal to
      u, for one such needle chosen uniformly: cosine 0.8 with the block's
      mean key.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    T, hq, hkv, d, B = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_size
    q = _randn(gen, (T, hq, d), device)
    k = _randn(gen, (T, hkv, d), device)
    v = _randn(gen, (T, hkv, d), device)
    blocks = _block_layout(w.seqlens, B)
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=device)
    if T == 0:
        return {"q": q, "k": k, "v": v, "cu_seqlens": cu}

    if w.structure in ("k_offsets", "qk_offsets"):
        off = 0.5 * torch.randn((len(blocks), hkv, d), generator=gen, device=device)
        bid = _token_block_ids(w.seqlens, B, device)
        for r0 in range(0, T, 1 << 16):
            r1 = min(r0 + (1 << 16), T)
            k[r0:r1] = (k[r0:r1].float() + off[bid[r0:r1]]).to(torch.bfloat16)
        if w.structure == "qk_offsets":
            pick = torch.rand((T, hq), generator=gen, device=device) < 0.1
            u = torch.rand((T, hq), generator=gen, device=device)
            starts = torch.tensor([b[1] for b in blocks], device=device)
            seq_first = torch.tensor(_first_block_of_seq(blocks, len(w.seqlens)), device=device)
            seq_of_tok = torch.repeat_interleave(
                torch.arange(len(w.seqlens), device=device),
                torch.tensor(w.seqlens, device=device))
            t = torch.arange(T, device=device)
            first = seq_first[seq_of_tok]                                  # first block of t's sequence
            n_avail = torch.searchsorted(starts, t, right=True) - first   # blocks starting <= t
            pos = torch.minimum((u * n_avail[:, None]).long(), (n_avail - 1)[:, None])
            j = first[:, None] + pos
            grp = hq // hkv
            heads = torch.arange(hq, device=device) // grp
            add = off[j, heads[None, :]]                                   # [T, hq, d]
            qf = q.float()
            qf = torch.where(pick[..., None], qf + add, qf)
            q = qf.to(torch.bfloat16)
    elif w.structure == "needles":
        grp = hq // hkv
        qf = q.float()
        kf = k.float()
        for i, (s, n) in enumerate(zip(_cum(w.seqlens), w.seqlens)):
            nb = (n + B - 1) // B
            if nb < 4:
                continue
            cand = torch.randperm(nb - 2, generator=gen, device=device)[:8] + 1
            needles, _ = torch.sort(cand)
            dirs = torch.randn((len(needles), hkv, d), generator=gen, device=device)
            dirs = dirs / dirs.norm(dim=-1, keepdim=True)
            for a, j in enumerate(needles.tolist()):
                r0, r1 = s + j * B, min(s + (j + 1) * B, s + n)
                # antithetic noise: the block's second half repeats the first half's draws
                # negated, so the noise sums to zero and the block mean is exactly 2u before
                # the final bf16 rounding (needle blocks are never a sequence's partial last
                # block, and B is even)
                hb = (r1 - r0) // 2
                kf[r0 + hb:r0 + 2 * hb] = -kf[r0:r0 + hb]
                kf[r0:r1] += 2.0 * dirs[a][None]
            pick = torch.rand((n, hq), generator=gen, device=device) < 0.05
            u = torch.rand((n, hq), generator=gen, device=device)
            wv = torch.randn((n, hq, d), generator=gen, device=device)
            own = torch.arange(n, device=device) // B                       # own block, local
            n_before = (needles[None, :] < own[:, None]).sum(dim=1)          # needles strictly before
            which = torch.minimum((u * n_before[:, None]).long(), (n_before - 1).clamp(min=0)[:, None])
            ok = pick & (n_before[:, None] > 0)
            heads = torch.arange(hq, device=device) // grp
            ud = dirs[which, heads[None, :]]                                 # [n, hq, d]
            wv = wv - (wv * ud).sum(-1, keepdim=True) * ud
            wv = wv / wv.norm(dim=-1, keepdim=True)
            qs = qf[s:s + n]
            newq = qs.norm(dim=-1, keepdim=True) * (0.8 * ud + 0.6 * wv)
            qf[s:s + n] = torch.where(ok[..., None], newq, qs)
        q = qf.to(torch.bfloat16)
        k = kf.to(torch.bfloat16)
    else:
        raise ValueError(f"unknown structure {w.structure}")
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(), "cu_seqlens": cu}


def _first_block_of_seq(blocks, nseq):
    first = [0] * nseq
    seen = set()
    for idx, (i, _, _) in enumerate(blocks):
        if i not in seen:
            first[i] = idx
            seen.add(i)
    return first


def selected_block_flops(seqlens, num_q_heads, head_dim, chunk, topk):
    """Algorithmic FLOPs of the attention over the selected blocks.

    4 * d * Hq * sum_t [ (t - s - c*B + 1) + B * min(topk - 1, c) ]: QK^T and
    PV (2 FLOPs per multiply-add each) over the causal prefix of the row's own
    block plus ``topk - 1`` whole past blocks (fewer for the first blocks).
    Past candidate blocks are always full, so the count does not depend on
    which blocks were chosen.
    """
    total = 0
    for n in seqlens:
        nb = (n + chunk - 1) // chunk
        for c in range(nb):
            rows = min(chunk, n - c * chunk)
            causal = rows * (rows + 1) // 2
            past = rows * chunk * min(topk - 1, c)
            total += causal + past
    return 4 * head_dim * num_q_heads * total
