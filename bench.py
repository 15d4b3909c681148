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


def _cpu_facts():
    """Host cores this process may use and the CPU model (for the baseline records)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_count": os.cpu_count(), "cores_usable": cores, "cpu_model": model}


def cpu_oracle_baseline(w, budget_s, seed=0, inputs=None, dense=False):
    """Times the float64 oracle, as it stands, on the host cores, on a bounded sample of
    workload w, and extrapolates the whole forward's time on those cores.

    Three measured parts, on a spawn pool of one process per usable core (the oracle's own
    functions on independent pieces, tests/oracle_pool.py):
      * the block means of the whole input (one process, measured in full);
      * the gate selection of one whole query head (oracle.select_blocks), times Hq;
      * sampled (token, head) rows' gate selection and attention (oracle.select_blocks_rows and
        oracle.attend_rows), for about budget_s of wall time, scaled to all T * Hq rows.
    The estimate is means + (gate + rows CPU-seconds) / cores.  With dense=True the dense
    causal fp64 attention of the same shape (the oracle with every block selected) is timed on
    one head and reported beside it.  Returns (tokens/s, detail)."""
    import numpy as np
    import torch

    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle_pool as OP
    import parity as PT
    from block_sparse_long_meanpool_b200 import workloads as W

    x = inputs if inputs is not None else W.make_inputs(w, device="cpu")
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    q16, k16, v16 = bits(x["q"]), bits(x["k"]), bits(x["v"])
    cu = np.asarray(w.cu_seqlens)
    T, hq, hkv = w.total_tokens, w.num_q_heads, w.num_kv_heads
    group = hq // hkv
    chunk, topk = w.chunk_size, w.topk
    facts = _cpu_facts()
    workers = OP.n_workers()
    t0 = time.perf_counter()
    means = np.concatenate([oracle.block_means(PT.from_bits(k16[cu[i]:cu[i + 1]]), [0, cu[i + 1] - cu[i]], chunk)
                            for i in range(len(cu) - 1)])
    t_means = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    with OP.pool() as ex, OP.Shared(k=k16.transpose(1, 0, 2), v=v16.transpose(1, 0, 2)) as sh:
        # start the workers (process start, imports) outside the measured parts
        list(ex.map(int, range(workers)))
        h = int(rng.integers(0, hq))
        _, t_gate_head = ex.submit(OP.timed, "_select_head", np.ascontiguousarray(q16[:, h]),
                                   np.ascontiguousarray(means[:, h // group]), cu, chunk, topk).result()
        done, cpu_rows = 0, 0.0
        wall0 = time.perf_counter()
        while time.perf_counter() - wall0 < budget_s:
            rows = sorted({(int(rng.integers(0, T)), int(rng.integers(0, hq))) for _ in range(8 * workers)})
            ts = np.array([t for t, _ in rows])
            hs = np.array([hh for _, hh in rows])
            q_rows = np.ascontiguousarray(q16[ts, hs])
            sel_futs = [ex.submit(OP.timed, "_select_rows", q_rows[part], ts[part],
                                  np.ascontiguousarray(means[:, int(hs[part[0]]) // group]), cu, chunk, topk, False)
                        for part in [np.nonzero(hs == hh)[0] for hh in np.unique(hs)]]
            sel = np.zeros((len(rows), topk), dtype=np.int64)
            for part, f in zip([np.nonzero(hs == hh)[0] for hh in np.unique(hs)], sel_futs):
                r, c = f.result()
                sel[part] = r
                cpu_rows += c
            _, _, c = OP.submit_attend_shared(ex, rows, q_rows, sh, cu, chunk, sel, group).result()
            cpu_rows += c
            done += len(rows)
        dense_s = None
        if dense:
            # every block selected: dense causal attention, one query head
            nbs = [(cu[i + 1] - cu[i] + chunk - 1) // chunk for i in range(len(cu) - 1)]
            all_sel = np.full((1, T, max(nbs)), -1, dtype=np.int64)
            for i in range(len(cu) - 1):
                for t in range(cu[i], cu[i + 1]):
                    c = (t - cu[i]) // chunk
                    all_sel[0, t, :c + 1] = np.arange(c + 1)
            _, c = ex.submit(OP.timed, "_dense_head", np.ascontiguousarray(q16[:, 0]),
                             np.ascontiguousarray(k16[:, 0]), np.ascontiguousarray(v16[:, 0]), cu, chunk,
                             all_sel[0], None).result()
            dense_s = c * hq
    rows_all = float(T * hq)
    cpu_total = t_gate_head * hq + cpu_rows * rows_all / max(done, 1)
    seconds = t_means + cpu_total / workers
    detail = dict(facts)
    detail.update({
        "cores": workers, "rows": done, "row_cpu_seconds": cpu_rows, "means_seconds": t_means,
        "gate_seconds_per_head": t_gate_head,
        "extrapolated": True,
        "sample": (f"{w.name} ({T} tokens x {hq} heads) on {workers} host processes: block means of the "
                   f"whole input ({t_means:.1f} s), the full gate selection of one head ({t_gate_head:.1f} "
                   f"CPU-s, x {hq} heads), {done} uniformly sampled rows' gate + attention ({cpu_rows:.1f} "
                   f"CPU-s, measured in the workers), extrapolated to all rows as means + CPU-seconds / "
                   f"processes")})
    if dense_s is not None:
        detail["dense_causal_fp64_tokens_per_s"] = T / (dense_s / workers)
        detail["dense_causal_fp64_note"] = ("the oracle with every block selected (dense causal attention), "
                                            "one head timed, x heads / processes")
    return T / seconds, detail


def dense_reference_rates(names=("tiny_2k", "scaling_8k", "long_32k")):
    """The dense causal fp64 reference (the oracle with every block selected) on the small
    configurations, timed on the host cores: one query head per workload in a worker process,
    extrapolated to all heads on all processes.  Returns {workload: tokens/s} and the note."""
    import numpy as np
    import torch

    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle_pool as OP
    from block_sparse_long_meanpool_b200 import workloads as W

    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    rates = {}
    workers = OP.n_workers()
    with OP.pool() as ex:
        list(ex.map(int, range(workers)))
        for name in names:
            w = W.ALL_WORKLOADS[name]
            x = W.make_inputs(w, device="cpu")
            q16, k16, v16 = bits(x["q"]), bits(x["k"]), bits(x["v"])
            cu = np.asarray(w.cu_seqlens)
            T, chunk = w.total_tokens, w.chunk_size
            nb = max((int(cu[i + 1] - cu[i]) + chunk - 1) // chunk for i in range(len(cu) - 1))
            all_sel = np.full((T, nb), -1, dtype=np.int64)
            for i in range(len(cu) - 1):
                c = (np.arange(cu[i], cu[i + 1]) - cu[i]) // chunk
                all_sel[cu[i]:cu[i + 1]] = np.where(np.arange(nb)[None, :] <= c[:, None], np.arange(nb)[None, :], -1)
            _, c = ex.submit(OP.timed, "_dense_head", np.ascontiguousarray(q16[:, 0]),
                             np.ascontiguousarray(k16[:, 0]), np.ascontiguousarray(v16[:, 0]), cu, chunk,
                             all_sel, None).result()
            rates[name] = T / (c * w.num_q_heads / workers)
    note = ("dense causal attention in float64 (the oracle with every block selected) on the small "
            "configurations: one query head timed in a worker, x heads / processes")
    return rates, note


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
        val, det = cpu_oracle_baseline(w, per_step, seed=100 + i, inputs=inputs)
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
                         "kind": "oracle", "sample": details[-1]["sample"],
                         "cpu_model": details[-1]["cpu_model"], "cpu_count": details[-1]["cpu_count"],
                         "extrapolated": details[-1]["extrapolated"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _time_forward(moba, w, x, steps, warmup, gate="mean", budget=None, wave_tokens=None,
                  max_seqlen=None):
    """CUDA-event timing of the whole forward (one moba_attn_fwd per step, inputs resident) with
    the library's per-stage events.  Returns a dict with ms per step, the stage split, the wave
    plan, launches and gate path, and the output buffers."""
    import torch

    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, hq, d = q.shape
    chunk, topk = w.chunk_size, w.topk
    dev = q.device
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((hq, T), dtype=torch.float32, device=dev)
    # first call fixes the wave size and the workspace
    moba.attn_fwd(q, k, v, cu, chunk, topk, out=out, lse=lse, workspace_budget=budget,
                  wave_tokens=wave_tokens, gate=gate, max_seqlen=max_seqlen)
    info0 = dict(moba.attn_fwd.last_info)
    wt = info0["wave_tokens"]
    ws = torch.empty(info0["workspace_bytes"], dtype=torch.uint8, device=dev)
    waves = info0["waves"]
    n_ev = moba.EV_WAVE0 + 4 * waves

    def step(events=None):
        moba.attn_fwd(q, k, v, cu, chunk, topk, out=out, lse=lse, workspace=ws, wave_tokens=wt,
                      events=events, gate=gate, max_seqlen=max_seqlen)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    return {"step": step, "events": events, "waves": waves, "wave_tokens": wt or T, "ws": ws,
            "out": out, "lse": lse, "info": info0}


def _stage_split(moba, events, waves, steps):
    def span(i, a, b):
        return events[i][a].elapsed_time(events[i][b])
    st = {"meanpool": 0.0, "gate": 0.0, "route": 0.0, "attention": 0.0, "merge": 0.0}
    for i in range(steps):
        st["meanpool"] += span(i, moba.EV_BEGIN, moba.EV_MEANS_DONE)
        st["gate"] += span(i, moba.EV_MEANS_DONE, moba.EV_GATE_DONE)
        for wv in range(waves):
            b = moba.EV_WAVE0 + 4 * wv
            st["route"] += span(i, b, b + 1)
            st["attention"] += span(i, b + 1, b + 2)
            st["merge"] += span(i, b + 2, b + 3)
    return {kk: vv / steps for kk, vv in st.items()}


def _run_timed(fwd, steps):
    """Runs the prepared forward `steps` times between two events; returns ms per step."""
    import torch

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        fwd["step"](fwd["events"][i])
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps


def _sub_forward(moba, W, w, dev, steps, warmup, peaks, gate="mean", max_seqlen=None, seed=None):
    """A forward sub-record on workload w (inputs larger than L2): ms per step, the stage
    split, attention TF/s against the burst peak (steps well under a second) and the gate's
    and merge's HBM rates."""
    import torch

    x = W.make_inputs(w, device=dev, seed=seed)
    fwd = _time_forward(moba, w, x, steps, warmup, gate=gate, max_seqlen=max_seqlen)
    ms = _run_timed(fwd, steps)
    st = _stage_split(moba, fwd["events"], fwd["waves"], steps)
    f_sel = W.selected_block_flops(w.seqlens, w.num_q_heads, w.head_dim, w.chunk_size, w.topk)
    peak = peaks["bf16_tflops_sustained"] if ms > 200.0 else peaks["bf16_tflops"]
    att = f_sel / (st["attention"] * 1e-3) / 1e12
    rec = {"workload": w.name, "gate": gate, "max_seqlen": max_seqlen, "steps": steps,
           "ms_per_step": ms, "tokens_per_s": w.total_tokens / (ms * 1e-3), "stage_ms": st,
           "attention_tflops": att, "attention_frac": att / peak,
           "peak_kind": "bf16 sustained" if ms > 200.0 else "bf16 burst",
           "gate_path": {1: "tensor cores", 2: "cuda cores"}.get(fwd["info"]["gate_path"], "none"),
           "hbm_stages": _hbm_stage_rates(w, st, peaks, gate)}
    del x, fwd
    torch.cuda.empty_cache()
    return rec


def _sub_decode(moba, W, w, dev, peaks, gate="mean", steps=50, warmup=5):
    """A decode-step sub-record on decode workload w (caches larger than L2): one moba_decode_fwd
    (or moba_decode_minmax_fwd) per step, the cache summary built outside the timing, as
    `bench.py --decode` times it; sequences/s and the HBM rate of the attended K/V bytes."""
    import torch

    x = W.make_inputs(w, device=dev)
    k, v, cu = x["k"], x["v"], x["cu_seqlens"]
    B, hq, hkv, d = len(w.seqlens), w.num_q_heads, w.num_kv_heads, w.head_dim
    chunk, topk = w.chunk_size, w.topk
    last = torch.tensor([c - 1 for c in w.cu_seqlens[1:]], device=dev)
    q_new = x["q"][last].contiguous()
    del x
    if gate == "minmax":
        k_min, k_max = moba.minmaxpool(k, cu, chunk)
    else:
        means = moba.meanpool(k, cu, chunk)
    p = moba.make_params(B, w.total_tokens, hq, hkv, d, chunk, topk)
    ws = torch.empty(moba.load_library().moba_decode_workspace_size(p), dtype=torch.uint8, device=dev)
    out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((hq, B), dtype=torch.float32, device=dev)

    def step():
        if gate == "minmax":
            moba.decode_minmax_fwd(q_new, k, v, cu, k_min, k_max, chunk, topk, workspace=ws, out=out, lse=lse)
        else:
            moba.decode_fwd(q_new, k, v, cu, means, chunk, topk, workspace=ws, out=out, lse=lse)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    keys = W.decode_attended_keys(w.seqlens, chunk, topk)
    algo_bytes = keys * hq * d * 2 * 2 + B * hq * d * 2 + B * hq * (d * 2 + 4)
    gbs = algo_bytes / (ms * 1e-3) / 1e9
    rec = {"workload": w.name, "gate": gate, "steps": steps, "ms_per_step": ms,
           "sequences_per_s": B / (ms * 1e-3), "algorithmic_bytes": algo_bytes, "GB/s": gbs,
           "hbm_frac": gbs / peaks["hbm_gbs"]}
    del k, v, ws, out, lse
    torch.cuda.empty_cache()
    return rec


def _sub_backward(moba, W, w, x, dev, peaks, steps=3, warmup=3):
    """A backward sub-record on workload w: the forward runs once (outside the timing) for
    out, lse and its selection; then moba_attn_bwd is timed.  TF/s counts the algorithmic
    backward work as 2.5 x the forward's selected-block FLOPs (QK^T, dP, dV, dK, dQ); the
    kernels execute 3.5 x (S and dP are recomputed for dQ)."""
    import torch

    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    out, lse, sel = moba.attn_fwd(q, k, v, cu, w.chunk_size, w.topk, return_sel=True,
                                  max_seqlen=w.max_seqlen)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 77)
    d_out = torch.randn(out.shape, generator=g, device=dev).to(torch.bfloat16)
    d_lse = torch.randn(lse.shape, generator=g, device=dev)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    moba.attn_bwd(q, k, v, out, lse, d_out, cu, w.chunk_size, w.topk, sel, d_lse=d_lse,
                  dq=dq, dk=dk, dv=dv)
    wsb = torch.empty(moba.attn_bwd.last_info["workspace_bytes"], dtype=torch.uint8, device=dev)

    def step():
        moba.attn_bwd(q, k, v, out, lse, d_out, cu, w.chunk_size, w.topk, sel, d_lse=d_lse,
                      workspace=wsb, dq=dq, dk=dk, dv=dv)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    f_sel = W.selected_block_flops(w.seqlens, w.num_q_heads, w.head_dim, w.chunk_size, w.topk)
    peak = peaks["bf16_tflops_sustained"] if ms > 200.0 else peaks["bf16_tflops"]
    alg = 2.5 * f_sel / (ms * 1e-3) / 1e12
    rec = {"workload": w.name, "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "tokens_per_s": w.total_tokens / (ms * 1e-3),
           "algorithmic_tflops": alg, "frac": alg / peak,
           "executed_tflops": 3.5 * f_sel / (ms * 1e-3) / 1e12,
           "peak_kind": "bf16 sustained" if ms > 200.0 else "bf16 burst",
           "note": "dq, dk, dv for the forward's selection; algorithmic work 2.5 x the forward's "
                   "selected-block FLOPs, executed 3.5 x"}
    del out, lse, sel, d_out, d_lse, dq, dk, dv, wsb
    torch.cuda.empty_cache()
    return rec


def _e2e_pipelined(moba, w, x, fwd, steps, world):
    """End to end through the public API with pinned host buffers: every step copies its inputs
    host -> device, runs moba_attn_fwd and reads out and lse back.  Steps are pipelined over two
    device buffer sets and two streams for the copies: step i+1's upload and step i-1's
    download run while step i computes.  Every copy of every timed step is inside the timed
    region (events on the compute stream after waiting for the copy streams)."""
    import torch

    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    out, lse, ws = fwd["out"], fwd["lse"], fwd["ws"]
    chunk, topk, wt = w.chunk_size, w.topk, fwd["info"]["wave_tokens"]
    host = {n: t.cpu().pin_memory() for n, t in (("q", q), ("k", k), ("v", v), ("cu", cu))}
    outh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    lseh = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    dev_in = [{"q": q, "k": k, "v": v, "cu": cu},
              {n: torch.empty_like(t) for n, t in (("q", q), ("k", k), ("v", v), ("cu", cu))}]
    dev_out = [(out, lse), (torch.empty_like(out), torch.empty_like(lse))]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]
    computed = [ev(), ev()]
    out_read = [ev(), ev()]

    def run(n):
        for i in range(n):
            bsel = i % 2
            s_in.wait_event(computed[bsel]) if i >= 2 else None
            with torch.cuda.stream(s_in):
                for name in ("q", "k", "v", "cu"):
                    dev_in[bsel][name].copy_(host[name], non_blocking=True)
                in_ready[bsel].record(s_in)
            main.wait_event(in_ready[bsel])
            if i >= 2:
                main.wait_event(out_read[bsel])
            di = dev_in[bsel]
            o, l = dev_out[bsel]
            moba.attn_fwd(di["q"], di["k"], di["v"], di["cu"], chunk, topk, out=o, lse=l,
                          workspace=ws, wave_tokens=wt)
            computed[bsel].record(main)
            s_out.wait_event(computed[bsel])
            with torch.cuda.stream(s_out):
                outh[bsel].copy_(o, non_blocking=True)
                lseh[bsel].copy_(l, non_blocking=True)
                out_read[bsel].record(s_out)
        main.wait_event(out_read[(n - 1) % 2])
        if n >= 2:
            main.wait_event(out_read[(n - 2) % 2])

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(main)
    run(steps)
    b.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    del dev_in[1], dev_out[1]
    torch.cuda.empty_cache()
    return {"value": job_value(w.total_tokens, world, e2e_ms), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "steps": steps,
            "pipelining": "two device buffer sets; uploads and downloads on their own streams "
                          "overlap the neighbouring steps' compute; the first upload and the last "
                          "download are inside the timed steps"}


def run_backward(args, w, world, rank, local):
    """--backward: one moba_attn_bwd per step (the forward runs once, outside the timing, for
    out, lse and its selection), weak scaling like the forward."""
    import torch

    from block_sparse_long_meanpool_b200 import build as _build
    from block_sparse_long_meanpool_b200 import moba
    from block_sparse_long_meanpool_b200 import workloads as W

    if rank == 0:
        _build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    peaks = read_peaks()
    sampler = ClockSampler(_gpu_id(dev))
    barrier(world)
    sampler.start()
    rec = _sub_backward(moba, W, w, x, dev, peaks, steps=args.steps, warmup=args.warmup)
    clocks = sampler.stop()
    ms = max_over_ranks(rec["ms_per_step"], world)
    if rank == 0:
        f_sel = W.selected_block_flops(w.seqlens, w.num_q_heads, w.head_dim, w.chunk_size, w.topk)
        alg = 2.5 * f_sel / (ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"] if ms > 200.0 else peaks["bf16_tflops"]
        print(json.dumps({
            "metric": "MoBA backward tokens/s (dq, dk, dv of one attention layer, all heads)",
            "value": job_value(w.total_tokens, world, ms), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, generated on device)",
            "config": {"workload": w.name, "description": w.description, "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": {"bound": "tensor", "kernel": "backward (dK/dV and dQ kernels)",
                         "achieved": alg, "peak": peak, "unit": "TFLOP/s", "frac": alg / peak,
                         "peak_kind": ("bf16 sustained" if ms > 200.0 else "bf16 burst") + f" ({peaks['source']})",
                         "traffic": None,
                         "note": rec["note"]},
            "executed_tflops": rec["executed_tflops"],
            "clocks": clocks,
            "gpu_launches": 9 * args.steps,  # block table, 4 routing kernels, 4 backward kernels
            "e2e": None,
            "cpu_baseline": None,
        }), flush=True)


def run_ours(args, w, world, rank, local):
    import torch

    from block_sparse_long_meanpool_b200 import build as _build
    from block_sparse_long_meanpool_b200 import moba
    from block_sparse_long_meanpool_b200 import workloads as W

    if rank == 0:
        _build.build()
    barrier(world)
    moba.load_library()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = W.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    q, k = x["q"], x["k"]
    T, hq, d = q.shape
    hkv = k.shape[1]
    chunk, topk = w.chunk_size, w.topk
    budget = int(args.workspace_gb * (1 << 30)) if args.workspace_gb else None
    max_seqlen = w.max_seqlen
    fwd = _time_forward(moba, w, x, args.steps, args.warmup, gate=args.gate, budget=budget,
                        wave_tokens=args.wave_tokens, max_seqlen=max_seqlen)
    waves, wave_tokens = fwd["waves"], fwd["wave_tokens"]
    sampler = ClockSampler(_gpu_id(dev))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ms_local = _run_timed(fwd, args.steps)
    clocks = sampler.stop()
    barrier(world)
    ms = max_over_ranks(ms_local, world)
    launches = moba.attn_fwd.last_info["launches"]
    st = _stage_split(moba, fwd["events"], waves, args.steps)

    peaks = read_peaks()
    f_sel = W.selected_block_flops(w.seqlens, hq, d, chunk, topk)
    attn_ms = st["attention"]
    achieved = f_sel / (attn_ms * 1e-3) / 1e12
    long_step = ms > 200.0
    peak = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    traffic = _read_traffic(w.name)
    value = job_value(T, world, ms)

    e2e = None
    if not args.no_e2e:
        # up to 8 pipelined steps: the first upload and the last download (the pipeline's fill
        # and drain) are inside the timed region and are shared by the steps
        e2e = _e2e_pipelined(moba, w, x, fwd, max(1, min(args.steps, 8)), world)

    # sub-records, measured in this same run (rank 0 of a one-GPU run only)
    subs = {}
    if rank == 0 and world == 1 and not args.no_sub_records:
        del fwd
        torch.cuda.empty_cache()
        if w.name != "long_32k":
            subs["long_32k"] = _sub_forward(moba, W, W.WORKLOADS["long_32k"], dev, 20, 5, peaks,
                                            max_seqlen=W.WORKLOADS["long_32k"].max_seqlen)
        subs["packed_64x8k"] = _sub_forward(moba, W, W.ALL_WORKLOADS["packed_64x8k"], dev, 10, 3, peaks,
                                            max_seqlen=8192)
        if args.gate == "mean":
            subs["minmax_gate"] = _sub_forward(moba, W, w, dev, 3, 3, peaks, gate="minmax",
                                               max_seqlen=max_seqlen, seed=rank_seed(w, rank))
        subs["backward"] = _sub_backward(moba, W, w, x, dev, peaks)
        # the paper's block-granularity sweep at 32K (fixed sparsity, blocks of 4096 down to 256)
        sweep = {}
        for gw in W.GRANULARITY_32K.values():
            r = _sub_forward(moba, W, gw, dev, 10, 3, peaks, max_seqlen=gw.max_seqlen)
            sweep[gw.name] = {"tokens_per_s": r["tokens_per_s"], "ms_per_step": r["ms_per_step"],
                              "attention_tflops": r["attention_tflops"],
                              "attention_frac": r["attention_frac"], "stage_ms": r["stage_ms"]}
        subs["granularity_32k"] = sweep
        dw = W.DECODE_WORKLOADS["decode_32k_b64"]
        subs["decode_32k_b64"] = _sub_decode(moba, W, dw, dev, peaks)
        subs["decode_32k_b64_minmax"] = _sub_decode(moba, W, dw, dev, peaks, gate="minmax")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x_cpu = {kk: vv.cpu() for kk, vv in x.items()}
        del x
        torch.cuda.empty_cache()
        val, det = cpu_oracle_baseline(w, args.cpu_seconds, seed=7, inputs=x_cpu,
                                       dense=w.total_tokens <= (1 << 16))
        cpu = {"value": val, "unit": "tokens/s", "cores": det["cores"], "kind": "oracle",
               "sample": det["sample"], "cpu_model": det["cpu_model"], "cpu_count": det["cpu_count"],
               "extrapolated": det["extrapolated"], "gate_seconds_per_head": det["gate_seconds_per_head"],
               "means_seconds": det["means_seconds"], "rows_sampled": det["rows"]}
        if "dense_causal_fp64_tokens_per_s" in det:
            cpu["dense_causal_fp64_tokens_per_s"] = det["dense_causal_fp64_tokens_per_s"]
            cpu["dense_causal_fp64_note"] = det["dense_causal_fp64_note"]
        else:
            rates, note = dense_reference_rates()
            cpu["dense_causal_fp64_small_configs_tokens_per_s"] = rates
            cpu["dense_causal_fp64_note"] = note

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, generated on device)",
            "config": {"workload": w.name, "description": w.description,
                       "global_batch": len(w.seqlens) * world, "seq_len": w.max_seqlen,
                       "tokens_per_gpu": T, "q_heads": hq, "kv_heads": hkv, "head_dim": d,
                       "chunk_size": chunk, "topk": topk, "gate": args.gate,
                       "parallelism": f"dp{world}", "wave_tokens": wave_tokens, "waves": waves,
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
            "hbm_stages": _hbm_stage_rates(w, st, peaks, args.gate),
            "clocks": clocks,
            "gpu_launches": launches * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        line.update(subs)
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


def _hbm_stage_rates(w, st, peaks, gate="mean"):
    """Achieved GB/s of the HBM-bound stages from their algorithmic bytes (the block summary:
    fp32 means, or the bf16 min and max, the same bytes)."""
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
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (moba_attn_bwd) instead of the forward")
    ap.add_argument("--decode", action="store_true",
                    help="time the decode step (workloads.DECODE_WORKLOADS) instead of the prefill")
    ap.add_argument("--gate", choices=["mean", "minmax"], default="mean",
                    help="gate: block means, or the min/max (Quest-style) block summary")
    ap.add_argument("--no-sub-records", action="store_true",
                    help="skip the long_32k, packed-batch, min/max-gate and backward sub-records")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
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
    if args.backward:
        if args.impl == "reference":
            ap.error("--backward has no reference arm")
        world, rank, local = dist_setup()
        try:
            run_backward(args, w, world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
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
