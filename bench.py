"""MoBA causal prefill forward benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole forward (block table, mean-pool, gate + top-k, routing, block attention,
merge: every query wave) over one batch of synthetic inputs already resident in HBM.
Timing: CUDA events on the launching stream between a barrier + synchronize on both sides,
max over ranks.  Inputs (q, k, v >= 2.7 GB at the default 1M-token workload) exceed the
126 MB L2, so no flush is needed between steps.  Multi-GPU runs are weak scaling: every
rank runs its own independently seeded problem; there is no collective on the data path.

``--impl reference`` times the float64 CPU oracle instead (rank 0 only) on a bounded
sample of rows of the same workload and reports the same metric.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "prefill_1m"
METRIC = "MoBA prefill tokens/s (causal forward, all heads of one attention layer)"


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id):
        self.device_id = device_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        load = [s for s, p in zip(sm, pw) if p is not None and p > 250.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows),
                "samples_under_load": len(load), "power_w_max": max(pw) if pw else None}


def dist_setup():
    """One process per GPU: NCCL process group when WORLD_SIZE > 1 (gloo without CUDA)."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x, world):
    """Max of a host float over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist

    if world == 1:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    import torch.distributed as dist

    if world > 1:
        dist.barrier()


def rank_seed(w, rank):
    """Weak scaling: every rank draws its own independent problem."""
    return w.seed + 7919 * rank


def job_value(tokens_per_rank, world, ms_max):
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def cpu_oracle_sample(w, budget_s, seed=0, inputs=None):
    """Times the float64 oracle on sampled query rows of workload w (bounded CPU work).

    Per sampled row (t, h): gate selection (against the block means) and attention over its
    selected blocks.  The block means of the whole input are computed once and charged to
    the sample in proportion (rows sampled / all rows).  Returns (tokens/s, detail).
    """
    import numpy as np
    import torch

    import oracle
    from block_sparse_long_meanpool_b200 import workloads as W

    x = inputs if inputs is not None else W.make_inputs(w, device="cpu")
    k = x["k"].float().numpy()
    v = x["v"].float().numpy()
    qt = x["q"]
    cu = np.asarray(w.cu_seqlens)
    T, hq = w.total_tokens, w.num_q_heads
    t0 = time.perf_counter()
    means = oracle.block_means(k, cu, w.chunk_size)
    t_means = time.perf_counter() - t0
    rng = np.random.default_rng(seed)

    class QRows:
        shape = (T, hq, w.head_dim)

        def __getitem__(self, idx):
            t, h = idx
            return qt[int(t), int(h)].float().numpy()

    qv = QRows()
    done, t_rows = 0, 0.0
    while t_rows < budget_s:
        rows = [(int(rng.integers(0, T)), int(rng.integers(0, hq))) for _ in range(8)]
        a = time.perf_counter()
        sel = oracle.select_blocks_rows(qv, means, cu, w.chunk_size, w.topk, rows)
        oracle.attend_rows(qv, k, v, cu, w.chunk_size, sel, rows)
        t_rows += time.perf_counter() - a
        done += len(rows)
    frac = done / float(T * hq)
    seconds = t_rows + t_means * frac
    tokens = done / hq
    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        threads = 1
    del torch
    detail = {"rows": done, "row_seconds": t_rows, "means_seconds_full": t_means,
              "cores": threads,
              "sample": (f"{done} uniformly sampled (token, head) rows of {w.name} "
                         f"({T} tokens x {hq} heads): per-row gate + top-k + attention, plus "
                         f"the full-input block means charged at {frac:.2e} of their "
                         f"{t_means:.1f} s")}
    return tokens / seconds, detail


def run_reference(args, w, world, rank):
    """--impl reference: the float64 CPU oracle on a bounded sample, rank 0 only."""
    if rank != 0:
        return
    from block_sparse_long_meanpool_b200 import workloads as W

    inputs = W.make_inputs(w, device="cpu") if w.total_tokens <= (1 << 17) else None
    if inputs is None:
        import torch
        if torch.cuda.is_available():
            g = W.make_inputs(w, device="cuda")
            inputs = {kk: vv.cpu() for kk, vv in g.items()}
            del g
            torch.cuda.empty_cache()
        else:
            inputs = W.make_inputs(w, device="cpu")
    per_step = float(os.environ.get("MOBA_REF_STEP_SECONDS", "8"))
    vals, details = [], []
    for i in range(args.warmup + args.steps):
        val, det = cpu_oracle_sample(w, per_step, seed=100 + i, inputs=inputs)
        if i >= args.warmup:
            vals.append(val)
            details.append(det)
    value = statistics.median(vals)
    ms = 1000.0 * w.total_tokens / value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "description": w.description,
                   "global_batch": len(w.seqlens) * args.gpus, "seq_len": w.max_seqlen,
                   "parallelism": f"dp{args.gpus}", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": details[-1]["cores"],
                         "kind": "oracle", "sample": details[-1]["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w, world, rank, local):
    import torch

    from block_sparse_long_meanpool_b200 import build as _build
    from block_sparse_long_meanpool_b200 import moba
    from block_sparse_long_meanpool_b200 import workloads as W

    if rank == 0:
        _build.build()
    barrier(world)
    lib = moba.load_library()
    del lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, hq, d = q.shape
    hkv = k.shape[1]
    chunk, topk = w.chunk_size, w.topk
    budget = None
    if args.workspace_gb:
        budget = int(args.workspace_gb * (1 << 30))
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((hq, T), dtype=torch.float32, device=dev)
    # first call fixes the wave size and the workspace
    moba.attn_fwd(q, k, v, cu, chunk, topk, out=out, lse=lse, workspace_budget=budget,
                  wave_tokens=args.wave_tokens)
    info0 = dict(moba.attn_fwd.last_info)
    wave_tokens = info0["wave_tokens"]
    ws = torch.empty(info0["workspace_bytes"], dtype=torch.uint8, device=dev)
    waves = info0["waves"]
    n_ev = moba.EV_WAVE0 + 4 * waves

    def step(events=None):
        moba.attn_fwd(q, k, v, cu, chunk, topk, out=out, lse=lse, workspace=ws,
                      wave_tokens=wave_tokens, events=events)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    sampler = ClockSampler(_gpu_id(dev))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(args.steps):
        step(events[i])
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms_local = start.elapsed_time(end) / args.steps
    ms = max_over_ranks(ms_local, world)
    launches = moba.attn_fwd.last_info["launches"]

    # per-stage device times (ms per step, mean over steps)
    def span(i, a, b):
        return events[i][a].elapsed_time(events[i][b])
    st = {"meanpool": 0.0, "gate": 0.0, "route": 0.0, "attention": 0.0, "merge": 0.0}
    for i in range(args.steps):
        st["meanpool"] += span(i, moba.EV_BEGIN, moba.EV_MEANS_DONE)
        st["gate"] += span(i, moba.EV_MEANS_DONE, moba.EV_GATE_DONE)
        for wv in range(waves):
            b = moba.EV_WAVE0 + 4 * wv
            st["route"] += span(i, b, b + 1)
            st["attention"] += span(i, b + 1, b + 2)
            st["merge"] += span(i, b + 2, b + 3)
    st = {kk: vv / args.steps for kk, vv in st.items()}

    peaks = read_peaks()
    f_sel = W.selected_block_flops(w.seqlens, hq, d, chunk, topk)
    attn_ms = st["attention"]
    achieved = f_sel / (attn_ms * 1e-3) / 1e12
    long_step = ms > 200.0
    peak = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    traffic = _read_traffic(w.name)
    value = job_value(T, world, ms)

    # end to end through the public API: pinned host inputs -> H2D -> forward -> D2H
    e2e = None
    if not args.no_e2e:
        qh = q.cpu().pin_memory()
        kh = k.cpu().pin_memory()
        vh = v.cpu().pin_memory()
        cuh = cu.cpu().pin_memory()
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lseh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        h2d = qh.numel() * 2 + kh.numel() * 2 + vh.numel() * 2 + cuh.numel() * 4
        d2h = outh.numel() * 2 + lseh.numel() * 4
        n_e2e = max(1, min(args.steps, 3))

        def e2e_step():
            q.copy_(qh, non_blocking=True)
            k.copy_(kh, non_blocking=True)
            v.copy_(vh, non_blocking=True)
            cu.copy_(cuh, non_blocking=True)
            step()
            outh.copy_(out, non_blocking=True)
            lseh.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n_e2e):
            e2e_step()
        b.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world)
        e2e = {"value": job_value(T, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x_cpu = {kk: vv.cpu() for kk, vv in x.items()}
        val, det = cpu_oracle_sample(w, args.cpu_seconds, seed=7, inputs=x_cpu)
        cpu = {"value": val, "unit": "tokens/s", "cores": det["cores"], "kind": "oracle",
               "sample": det["sample"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, generated on device)",
            "config": {"workload": w.name, "description": w.description,
                       "global_batch": len(w.seqlens) * world, "seq_len": w.max_seqlen,
                       "tokens_per_gpu": T, "q_heads": hq, "kv_heads": hkv, "head_dim": d,
                       "chunk_size": chunk, "topk": topk, "parallelism": f"dp{world}",
                       "wave_tokens": wave_tokens or T, "waves": waves,
                       "l2": "inputs larger than L2 (no flush)"},
            "selected_block_tflops": achieved,
            "selected_block_tflops_over_step": f_sel / (ms * 1e-3) / 1e12,
            "frac_of_bf16_peak": achieved / peak,
            "stage_ms": st,
            "roofline": {"bound": "tensor", "kernel": "attention (block attention, all waves)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "peak_kind": ("bf16 sustained" if long_step else "bf16 burst")
                                      + f" ({peaks['source']})",
                         "traffic": traffic},
            "hbm_stages": _hbm_stage_rates(w, st, peaks),
            "clocks": clocks,
            "gpu_launches": launches * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def run_decode(args, w, world, rank, local):
    """Decode step: one moba_decode_fwd per step over caches of the workload's shape."""
    import torch

    import oracle
    from block_sparse_long_meanpool_b200 import build as _build
    from block_sparse_long_meanpool_b200 import moba
    from block_sparse_long_meanpool_b200 import workloads as W

    if rank == 0:
        _build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    k, v, cu = x["k"], x["v"], x["cu_seqlens"]
    B, hq, hkv, d = len(w.seqlens), w.num_q_heads, w.num_kv_heads, w.head_dim
    chunk, topk = w.chunk_size, w.topk
    last = torch.tensor([c - 1 for c in w.cu_seqlens[1:]], device=dev)
    q_new = x["q"][last].contiguous()
    # cache state, kept outside the timed step: the block means or the min/max summary
    if args.gate == "minmax":
        k_min, k_max = moba.minmaxpool(k, cu, chunk)
    else:
        means = moba.meanpool(k, cu, chunk)
    p = moba.make_params(B, w.total_tokens, hq, hkv, d, chunk, topk)
    ws = torch.empty(moba.load_library().moba_decode_workspace_size(p), dtype=torch.uint8, device=dev)
    out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((hq, B), dtype=torch.float32, device=dev)

    def step():
        if args.gate == "minmax":
            moba.decode_minmax_fwd(q_new, k, v, cu, k_min, k_max, chunk, topk, workspace=ws, out=out, lse=lse)
        else:
            moba.decode_fwd(q_new, k, v, cu, means, chunk, topk, workspace=ws, out=out, lse=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(_gpu_id(dev))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        step()
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, world)

    peaks = read_peaks()
    keys = W.decode_attended_keys(w.seqlens, chunk, topk)
    algo_bytes = keys * hq * d * 2 * 2 + B * hq * d * 2 + B * hq * (d * 2 + 4)
    gbs = algo_bytes / (ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        qh = q_new.cpu().pin_memory()
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lseh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

        def e2e_step():
            q_new.copy_(qh, non_blocking=True)
            step()
            outh.copy_(out, non_blocking=True)
            lseh.copy_(lse, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        e2e = {"value": B * world / (e_ms * 1e-3), "unit": "sequences/s",
               "h2d_bytes_per_step": qh.numel() * 2,
               "d2h_bytes_per_step": outh.numel() * 2 + lseh.numel() * 4, "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on the first sequence's cache (means included), as it stands
        n0 = w.seqlens[0]
        kh = k[:n0].double().cpu().numpy()
        vh = v[:n0].double().cpu().numpy()
        qh1 = q_new[:1].double().cpu().numpy()
        t0 = time.time()
        oracle.moba_decode(qh1, kh, vh, [0, n0], chunk, topk, gate=args.gate)
        dt = time.time() - t0
        cpu = {"value": 1.0 / dt, "unit": "sequences/s", "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"1 of {B} sequences (its whole {n0}-token cache: block summary, gate, attention)"}

    if rank == 0:
        line = {
            "metric": "MoBA decode sequences/s (one new token per sequence, all heads of one attention layer)",
            "value": B * world / (ms * 1e-3),
            "unit": "sequences/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded, generated on device)",
            "config": {"workload": w.name, "description": w.description, "sequences": B,
                       "cache_tokens": w.total_tokens, "q_heads": hq, "kv_heads": hkv,
                       "head_dim": d, "chunk_size": chunk, "topk": topk,
                       "gate": args.gate,
                       "block_summary": ("cached bf16 block min/max (moba_minmaxpool once, outside the step)"
                                         if args.gate == "minmax" else
                                         "cached block means (moba_meanpool once, outside the step)"),
                       "l2": "caches larger than L2 (no flush)", "parallelism": f"dp{world}"},
            "roofline": {"bound": "hbm", "kernel": "decode step (gate, block attention, merge)",
                         "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "peak_kind": "HBM copy (measured)",
                         "traffic": None,
                         "bytes_per_step": algo_bytes,
                         "note": "selected blocks' K and V per query head; query heads of one KV head that pick the same block share it through L2"},
            "clocks": clocks,
            "gpu_launches": 3 * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def run_decode_reference(args, w, world, rank):
    """The float64 oracle's decode step on the host cores, one sequence's cache per step."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from block_sparse_long_meanpool_b200 import workloads as W

    n0 = w.seqlens[0]
    one = W.custom(w.name + "_seq0", [n0], w.num_q_heads, w.num_kv_heads, w.head_dim,
                   w.chunk_size, w.topk, w.structure, w.seed)
    x = W.make_inputs(one, device="cpu")
    k = x["k"].double().numpy()
    v = x["v"].double().numpy()
    q1 = x["q"][n0 - 1:n0].double().numpy()
    oracle.moba_decode(q1, k, v, [0, n0], w.chunk_size, w.topk, gate=args.gate)  # warm-up
    t0 = time.time()
    for _ in range(args.steps):
        oracle.moba_decode(q1, k, v, [0, n0], w.chunk_size, w.topk, gate=args.gate)
    dt = (time.time() - t0) / args.steps
    value = 1.0 / dt
    print(json.dumps({
        "impl": "reference",
        "metric": "MoBA decode sequences/s (one new token per sequence, all heads of one attention layer)",
        "value": value, "unit": "sequences/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "description": w.description, "gate": args.gate},
        "cpu_baseline": {"value": value, "unit": "sequences/s", "cores": os.cpu_count(),
                         "kind": "oracle", "sample": f"1 of {len(w.seqlens)} sequences per step"},
        "e2e": {"value": value, "unit": "sequences/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def _hbm_stage_rates(w, st, peaks):
    """Achieved GB/s of the HBM-bound stages from their algorithmic bytes."""
    T, hq, hkv, d = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim
    nb = sum((n + w.chunk_size - 1) // w.chunk_size for n in w.seqlens)
    mean_bytes = T * hkv * d * 2 + nb * hkv * d * 4
    gate_bytes = T * hq * d * 2 + T * hq * w.topk * 4 + nb * hkv * d * 4
    # merge: every row reads its min(topk, c + 1) partials (c = the row's block in its
    # sequence) as bf16 o + fp32 lse and its slot count, and writes bf16 o + fp32 lse
    slots = 0
    for n in w.seqlens:
        for c in range((n + w.chunk_size - 1) // w.chunk_size):
            rows = min(w.chunk_size, n - c * w.chunk_size)
            slots += rows * min(w.topk, c + 1)
    merge_bytes = hq * (slots * (d * 2 + 4) + T * (1 + d * 2 + 4))
    res = {}
    for name, by in (("meanpool", mean_bytes), ("gate", gate_bytes)):
        ms = st[name]
        gbs = by / (ms * 1e-3) / 1e9 if ms > 0 else None
        res[name] = {"bytes": by, "GB/s": gbs,
                     "frac": (gbs / peaks["hbm_gbs"]) if gbs else None}
    ms = st["merge"]
    gbs = merge_bytes / (ms * 1e-3) / 1e9 if ms > 0 else None
    res["merge"] = {"bytes": merge_bytes, "GB/s": gbs,
                    "frac": (gbs / peaks["hbm_gbs"]) if gbs else None}
    return res


def _attention_source_hash():
    """sha256 over the attention kernel's sources (the kernel the traffic figure belongs to)."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_long_meanpool_b200", "csrc")
    for f in ("attn_tc.cu", "ptx.cuh", "moba_internal.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _read_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary
    (profiles/attention_<workload>.json), or None when it was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", f"attention_{workload}.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_source_sha256") != _attention_source_hash():
        return None
    return rec.get("traffic_bytes_per_launch")


def _gpu_id(dev):
    import torch

    try:
        props = torch.cuda.get_device_properties(dev)
        uuid = str(props.uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev.index] if vis else dev.index


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--wave-tokens", type=int, default=None)
    ap.add_argument("--workspace-gb", type=float, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--decode", action="store_true",
                    help="time the decode step (workloads.DECODE_WORKLOADS) instead of the prefill")
    ap.add_argument("--gate", choices=["mean", "minmax"], default="mean",
                    help="decode gate: block means, or the min/max (Quest-style) block summary")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gate != "mean" and not args.decode:
        ap.error("--gate applies to the decode step (--decode); the prefill gate is the mean gate")
    from block_sparse_long_meanpool_b200 import workloads as W

    if args.decode:
        name = args.workload if args.workload in W.DECODE_WORKLOADS else "decode_32k_b64"
        w = W.DECODE_WORKLOADS[name]
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if args.impl == "reference":
            run_decode_reference(args, w, world, rank)
            return
        world, rank, local = dist_setup()
        try:
            run_decode(args, w, world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    w = W.ALL_WORKLOADS[args.workload]
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
