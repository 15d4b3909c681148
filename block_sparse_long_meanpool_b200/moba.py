"""Thin ctypes binding of libmoba.so (include/moba.h).

Argument marshalling and shape checks only: every step of the forward and of the decode step
runs in the library's CUDA kernels.
PyTorch provides device memory, the current stream and events.  There is no fallback: if
the library is missing or the tensors are not on a CUDA device, the calls raise.
"""

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoba.so")

# Every symbol the C ABI exports (checked by the CPU test suite).
EXPORTS = (
    "moba_num_blocks_bound",
    "moba_workspace_size",
    "moba_meanpool",
    "moba_minmaxpool",
    "moba_gate_topk",
    "moba_gate_minmax_topk",
    "moba_attn_fwd",
    "moba_attn_fwd_noalloc",
    "moba_bwd_workspace_size",
    "moba_attn_bwd",
    "moba_decode_workspace_size",
    "moba_decode_fwd",
    "moba_decode_minmax_fwd",
    "moba_device_status",
    "moba_device_status_noalloc",
    "moba_selftest_timeout",
    "moba_status_string",
    "moba_last_error",
)

# moba_status codes
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(6)

# moba_run_info event slots
EV_BEGIN, EV_MEANS_DONE, EV_GATE_DONE, EV_WAVE0 = 0, 1, 2, 3
# moba_run_info.gate_path
GATE_PATH_NONE, GATE_PATH_TENSOR_CORES, GATE_PATH_CUDA_CORES = 0, 1, 2


class MobaParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("total_tokens", ctypes.c_int),
        ("max_seqlen", ctypes.c_int),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("chunk_size", ctypes.c_int),
        ("topk", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
        ("wave_tokens", ctypes.c_int),
        ("gate", ctypes.c_int),
    ]


class MobaRunInfo(ctypes.Structure):
    _fields_ = [
        ("events", ctypes.POINTER(ctypes.c_void_p)),
        ("n_events", ctypes.c_int),
        ("launches", ctypes.c_int),
        ("waves", ctypes.c_int),
        ("gate_path", ctypes.c_int),
    ]


class MobaError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(message)
        self.status = status


_lib = None


def load_library(path=LIB_PATH):
    """Loads libmoba.so and declares its signatures.  Raises if it has not been built."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m block_sparse_long_meanpool_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(MobaParams)
    vp = ctypes.c_void_p
    lib.moba_num_blocks_bound.argtypes = [P]
    lib.moba_num_blocks_bound.restype = ctypes.c_int
    lib.moba_workspace_size.argtypes = [P]
    lib.moba_workspace_size.restype = ctypes.c_size_t
    lib.moba_meanpool.argtypes = [P, vp, vp, vp, vp]
    lib.moba_meanpool.restype = ctypes.c_int
    lib.moba_minmaxpool.argtypes = [P, vp, vp, vp, vp, vp]
    lib.moba_minmaxpool.restype = ctypes.c_int
    lib.moba_gate_topk.argtypes = [P, vp, vp, vp, vp, vp]
    lib.moba_gate_topk.restype = ctypes.c_int
    lib.moba_gate_minmax_topk.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.moba_gate_minmax_topk.restype = ctypes.c_int
    lib.moba_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp,
                                  ctypes.POINTER(MobaRunInfo), vp]
    lib.moba_attn_fwd.restype = ctypes.c_int
    lib.moba_attn_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
    lib.moba_attn_fwd_noalloc.restype = ctypes.c_int
    lib.moba_bwd_workspace_size.argtypes = [P]
    lib.moba_bwd_workspace_size.restype = ctypes.c_size_t
    lib.moba_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp, vp, vp]
    lib.moba_attn_bwd.restype = ctypes.c_int
    lib.moba_decode_workspace_size.argtypes = [P]
    lib.moba_decode_workspace_size.restype = ctypes.c_size_t
    lib.moba_decode_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp, vp]
    lib.moba_decode_fwd.restype = ctypes.c_int
    lib.moba_decode_minmax_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp, vp]
    lib.moba_decode_minmax_fwd.restype = ctypes.c_int
    lib.moba_device_status.argtypes = [P, vp, vp]
    lib.moba_device_status.restype = ctypes.c_int
    lib.moba_device_status_noalloc.argtypes = [vp]
    lib.moba_device_status_noalloc.restype = ctypes.c_int
    lib.moba_selftest_timeout.argtypes = [vp, ctypes.c_uint, vp]
    lib.moba_selftest_timeout.restype = ctypes.c_int
    lib.moba_status_string.argtypes = [ctypes.c_int]
    lib.moba_status_string.restype = ctypes.c_char_p
    lib.moba_last_error.argtypes = []
    lib.moba_last_error.restype = ctypes.c_char_p
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status):
    if status != OK:
        lib = load_library()
        name = lib.moba_status_string(status).decode()
        msg = lib.moba_last_error().decode()
        raise MobaError(status, f"{name}: {msg}")


GATES = {"mean": 0, "minmax": 1}  # moba_params.gate (MOBA_GATE_MEAN, MOBA_GATE_MINMAX)


def make_params(batch, total_tokens, num_q_heads, num_kv_heads, head_dim, chunk_size, topk,
                softmax_scale=None, wave_tokens=0, max_seqlen=0, gate="mean"):
    return MobaParams(int(batch), int(total_tokens), int(max_seqlen or 0), int(num_q_heads),
                      int(num_kv_heads), int(head_dim), int(chunk_size), int(topk),
                      float(softmax_scale) if softmax_scale else 0.0, int(wave_tokens),
                      GATES[gate] if isinstance(gate, str) else int(gate))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require(cond, msg):
    if not cond:
        raise ValueError(msg)


def _check_qkv(q, k, v=None):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            continue
        _require(t.is_cuda, f"{name} must be a CUDA tensor")
        _require(t.dtype == torch.bfloat16, f"{name} must be bf16")
        _require(t.dim() == 3 and t.is_contiguous(), f"{name} must be contiguous [T, H, d]")


def _require_buffer(t, name, shape, dtype, device):
    """A caller-supplied buffer the kernels read or write whole: exact shape, dtype, layout and
    device (a wrong shape would be an out-of-bounds access on the device, not an error)."""
    _require(tuple(t.shape) == tuple(shape), f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    _require(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    _require(t.is_contiguous(), f"{name} must be contiguous")
    _require(t.device == device, f"{name} must be on {device}, got {t.device}")


def _rows_backed(t):
    """Rows of t[0]'s size that the memory behind t.data_ptr() holds (a view such as
    ``meanpool(..., num_blocks_out=n)`` keeps the block-count bound's rows behind it)."""
    row = t.shape[1] * t.shape[2] * t.element_size()
    avail = t.untyped_storage().nbytes() - t.storage_offset() * t.element_size()
    return avail // row if row else 0


def _require_summary(t, name, dtype, nb_bound, hkv, d, device):
    """A per-block summary indexed by global block id [NB, Hkv, d].  The kernels index it by
    block without knowing how many rows the caller has, so the memory behind it must hold the
    block-count bound's rows (moba_num_blocks_bound; ``meanpool`` and ``minmaxpool`` always
    allocate that many)."""
    _require(t.dim() == 3 and tuple(t.shape[1:]) == (hkv, d),
             f"{name} must be [NB, {hkv}, {d}], got {tuple(t.shape)}")
    _require(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    _require(t.is_contiguous(), f"{name} must be contiguous")
    _require(t.device == device, f"{name} must be on {device}, got {t.device}")
    _require(_rows_backed(t) >= nb_bound,
             f"{name} must be backed by >= {nb_bound} block rows (moba_num_blocks_bound), has {_rows_backed(t)}")


def _validate_decode(q, k, v, cu_seqlens, summary, out, lse, chunk_size, topk):
    """Shapes, dtypes and devices of a decode call (host-only; no CUDA needed).  ``summary`` is
    a list of (name, tensor, dtype) block summaries."""
    batch, hq, d = q.shape
    T, hkv, dk = k.shape
    _require(dk == d, f"k head_dim {dk} differs from q head_dim {d}")
    _require(tuple(v.shape) == tuple(k.shape), "v must have k's shape [T, Hkv, d]")
    _require(v.device == q.device and k.device == q.device, "q, k and v must be on one device")
    _require(cu_seqlens.dtype == torch.int32 and cu_seqlens.numel() == batch + 1,
             "cu_seqlens must be an int32 tensor of batch + 1 entries")
    bound = num_blocks_bound(make_params(batch, T, hq, hkv, d, chunk_size, topk))
    for name, t, dtype in summary:
        _require_summary(t, name, dtype, bound, hkv, d, q.device)
    if out is not None:
        _require_buffer(out, "out", (batch, hq, d), torch.bfloat16, q.device)
    if lse is not None:
        _require_buffer(lse, "lse", (hq, batch), torch.float32, q.device)


def num_blocks(seqlens, chunk_size):
    """Exact block count sum(ceil(L_i / chunk)) from host-side sequence lengths."""
    return int(sum((int(n) + chunk_size - 1) // chunk_size for n in seqlens))


def num_blocks_bound(params):
    n = load_library().moba_num_blocks_bound(ctypes.byref(params))
    if n < 0:
        raise MobaError(ERR_INVALID_ARG, load_library().moba_last_error().decode())
    return n


def workspace_size(params):
    n = load_library().moba_workspace_size(ctypes.byref(params))
    if n == 0 and params.total_tokens > 0:
        raise MobaError(ERR_INVALID_ARG, load_library().moba_last_error().decode())
    return n


def meanpool(k, cu_seqlens, chunk_size, num_blocks_out=None):
    """Block means fp32 [NB, Hkv, d] of k bf16 [T, Hkv, d] (moba_meanpool)."""
    _check_qkv(None, k)
    batch = cu_seqlens.numel() - 1
    T, hkv, d = k.shape
    p = make_params(batch, T, hkv, hkv, d, chunk_size, 1)
    bound = max(load_library().moba_num_blocks_bound(ctypes.byref(p)), 0)
    nb = bound if num_blocks_out is None else min(int(num_blocks_out), bound)
    # the kernel writes every real block, so the buffer always has the bound's rows
    out = torch.empty((max(bound, 1), hkv, d), dtype=torch.float32, device=k.device)
    _check(load_library().moba_meanpool(ctypes.byref(p), _ptr(k), _ptr(cu_seqlens), _ptr(out),
                                        _stream(k.device)))
    return out[:nb]


def minmaxpool(k, cu_seqlens, chunk_size, num_blocks_out=None):
    """Min/max block summary (moba_minmaxpool): (k_min, k_max), bf16 [NB, Hkv, d] each."""
    _check_qkv(None, k)
    batch = cu_seqlens.numel() - 1
    T, hkv, d = k.shape
    p = make_params(batch, T, hkv, hkv, d, chunk_size, 1)
    bound = max(load_library().moba_num_blocks_bound(ctypes.byref(p)), 0)
    nb = bound if num_blocks_out is None else min(int(num_blocks_out), bound)
    # the kernel writes every real block, so the buffers always have the bound's rows
    k_min = torch.empty((max(bound, 1), hkv, d), dtype=torch.bfloat16, device=k.device)
    k_max = torch.empty_like(k_min)
    _check(load_library().moba_minmaxpool(ctypes.byref(p), _ptr(k), _ptr(cu_seqlens), _ptr(k_min),
                                          _ptr(k_max), _stream(k.device)))
    return k_min[:nb], k_max[:nb]


def gate_topk(q, k_mean, cu_seqlens, chunk_size, topk, num_kv_heads=None, max_seqlen=None):
    """Selections int32 [Hq, T, topk] (moba_gate_topk).  ``max_seqlen``: the longest sequence,
    when known (sizes the gate per sequence rather than by the whole call's block count)."""
    _check_qkv(q, None)
    _require(k_mean.dtype == torch.float32 and k_mean.is_contiguous(), "k_mean must be fp32")
    batch = cu_seqlens.numel() - 1
    T, hq, d = q.shape
    hkv = num_kv_heads or k_mean.shape[1]
    p = make_params(batch, T, hq, hkv, d, chunk_size, topk, max_seqlen=max_seqlen)
    _require_summary(k_mean, "k_mean", torch.float32, num_blocks_bound(p), hkv, d, q.device)
    sel = torch.empty((hq, T, topk), dtype=torch.int32, device=q.device)
    _check(load_library().moba_gate_topk(ctypes.byref(p), _ptr(q), _ptr(k_mean), _ptr(cu_seqlens),
                                         _ptr(sel), _stream(q.device)))
    return sel


def gate_minmax_topk(q, k_min, k_max, cu_seqlens, chunk_size, topk, max_seqlen=None):
    """Selections int32 [Hq, T, topk] with the min/max block summary (moba_gate_minmax_topk):
    k_min, k_max bf16 [NB, Hkv, d] from ``minmaxpool``."""
    _check_qkv(q, None)
    batch = cu_seqlens.numel() - 1
    T, hq, d = q.shape
    hkv = k_min.shape[1]
    p = make_params(batch, T, hq, hkv, d, chunk_size, topk, max_seqlen=max_seqlen)
    bound = num_blocks_bound(p)
    _require_summary(k_min, "k_min", torch.bfloat16, bound, hkv, d, q.device)
    _require_summary(k_max, "k_max", torch.bfloat16, bound, hkv, d, q.device)
    sel = torch.empty((hq, T, topk), dtype=torch.int32, device=q.device)
    _check(load_library().moba_gate_minmax_topk(ctypes.byref(p), _ptr(q), _ptr(k_min), _ptr(k_max),
                                                _ptr(cu_seqlens), _ptr(sel), _stream(q.device)))
    return sel


def _decode(fn, summary, q, k, v, cu_seqlens, chunk_size, topk, softmax_scale, workspace, out, lse):
    _check_qkv(q, k, v)
    _require(cu_seqlens.is_cuda, "cu_seqlens must be a CUDA tensor")
    _validate_decode(q, k, v, cu_seqlens, summary, out, lse, chunk_size, topk)
    batch, hq, d = q.shape
    T, hkv, _ = k.shape
    p = make_params(batch, T, hq, hkv, d, chunk_size, topk, softmax_scale)
    lib = load_library()
    n = lib.moba_decode_workspace_size(ctypes.byref(p))
    if n == 0:
        raise MobaError(ERR_INVALID_ARG, lib.moba_last_error().decode())
    if workspace is None:
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((batch, hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((hq, batch), dtype=torch.float32, device=q.device)
    _check(getattr(lib, fn)(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                            *[_ptr(t) for _, t, _ in summary], _ptr(workspace),
                            ctypes.c_size_t(workspace.numel()), _ptr(out), _ptr(lse), _stream(q.device)))
    return out, lse


def decode_fwd(q, k, v, cu_seqlens, k_mean, chunk_size, topk, softmax_scale=None,
               workspace=None, out=None, lse=None):
    """Decode step (moba_decode_fwd): one new query per sequence against its KV cache.

    q bf16 [batch, Hq, d] (the new token's query of each sequence); k, v bf16 [T, Hkv, d]
    packed caches whose last row per sequence is the new token; cu_seqlens int32 [batch + 1];
    k_mean fp32 block means of these caches (``meanpool``).  Returns (out bf16 [batch, Hq, d],
    lse fp32 [Hq, batch]).
    """
    return _decode("moba_decode_fwd", [("k_mean", k_mean, torch.float32)], q, k, v, cu_seqlens, chunk_size, topk,
                   softmax_scale, workspace, out, lse)


def decode_minmax_fwd(q, k, v, cu_seqlens, k_min, k_max, chunk_size, topk, softmax_scale=None,
                      workspace=None, out=None, lse=None):
    """Decode step with the min/max gate (moba_decode_minmax_fwd): as ``decode_fwd``, with the
    bf16 block summary (k_min, k_max) of ``minmaxpool`` in place of the means."""
    return _decode("moba_decode_minmax_fwd", [("k_min", k_min, torch.bfloat16), ("k_max", k_max, torch.bfloat16)],
                   q, k, v, cu_seqlens, chunk_size, topk,
                   softmax_scale, workspace, out, lse)


def device_status(params, workspace):
    """moba_device_status: raises MobaError when the status word a previous moba_attn_fwd left
    in ``workspace`` is not MOBA_OK (waits for the current stream)."""
    _check(load_library().moba_device_status(ctypes.byref(params), _ptr(workspace),
                                             _stream(workspace.device)))


def device_status_noalloc(device=None):
    """moba_device_status_noalloc: raises MobaError when the most recent allocation-free forward
    on ``device`` left an error in its status word (waits for the current stream)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(load_library().moba_device_status_noalloc(_stream(dev)))


NOALLOC_SCRATCH_BYTES = 64 << 20  # MOBA_NOALLOC_SCRATCH_BYTES of include/moba.h


def selftest_timeout(device=None, polls=4096):
    """moba_selftest_timeout: runs the bounded-wait self-test on `device` and returns the status
    word it left (MOBA_ERR_DEVICE_TIMEOUT when the wait expired as it must)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(load_library().moba_selftest_timeout(_ptr(word), int(polls), _stream(dev)))
    return int(word.item())


def choose_wave_tokens(T, hq, hkv, d, chunk_size, topk, batch, budget_bytes):
    """Query tokens per wave: 0 (one wave over all T tokens) when that workspace fits in
    budget_bytes, else the largest multiple of 128 whose workspace fits, or 128 when even
    that does not.  A wave also keeps wave * hq * topk below 2^31 (int32 partial indices).
    The workspace size never decreases as the wave grows, so a bisection over multiples of
    128 against moba_workspace_size finds the exact largest fit."""
    lib = load_library()

    def size(w):
        return lib.moba_workspace_size(ctypes.byref(make_params(batch, T, hq, hkv, d, chunk_size, topk, None, w)))

    if T * hq * topk < 2 ** 31 and size(0) <= budget_bytes:
        return 0
    hi = min((T - 1) // 128, (2 ** 31 - 1) // (hq * topk * 128))  # tiles of a wave shorter than T
    if hi < 1:
        return 0 if T <= 128 else 128
    lo = 1
    if size(128) > budget_bytes:
        return 128
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if size(128 * mid) <= budget_bytes:
            lo = mid
        else:
            hi = mid - 1
    return 128 * lo


def attn_fwd(q, k, v, cu_seqlens, chunk_size, topk, softmax_scale=None, sel=None,
             return_sel=False, wave_tokens=None, workspace=None, events=None,
             workspace_budget=None, out=None, lse=None, max_seqlen=None, gate="mean",
             check_status=False):
    """MoBA causal prefill forward (moba_attn_fwd).

    q bf16 [T, Hq, d], k/v bf16 [T, Hkv, d], cu_seqlens int32 [batch + 1] on the device.
    sel: optional int32 [Hq, T, topk] selection to use instead of the gate.
    max_seqlen: the longest sequence's length when known on the host (0 / None: unknown).
    gate: "mean" (the paper's mean-pooled block summary) or "minmax" (the min/max summary).
    check_status: wait for the call and raise MobaError if its device status word is not OK (a
    bounded device wait gave up, or max_seqlen was shorter than a sequence).
    Returns (out bf16 [T, Hq, d], lse fp32 [Hq, T]) and, with return_sel, the gate's
    selection.  ``events`` may be a list of torch.cuda.Event recorded at the library's stage
    boundaries; the call's moba_run_info is returned in ``attn_fwd.last_info``.
    """
    _check_qkv(q, k, v)
    T, hq, d = q.shape
    hkv = k.shape[1]
    _require(k.shape == v.shape and k.shape[0] == T and k.shape[2] == d, "k/v shape mismatch")
    _require(cu_seqlens.dtype == torch.int32 and cu_seqlens.is_cuda, "cu_seqlens int32 CUDA")
    batch = cu_seqlens.numel() - 1
    dev = q.device
    if wave_tokens is None:
        if workspace_budget is None:
            free, _ = torch.cuda.mem_get_info(dev)
            workspace_budget = min(int(free * 0.45), 48 << 30)
        wave_tokens = choose_wave_tokens(T, hq, hkv, d, chunk_size, topk, batch, workspace_budget)
    p = make_params(batch, T, hq, hkv, d, chunk_size, topk, softmax_scale, wave_tokens, max_seqlen, gate)
    need = workspace_size(p)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
    else:
        _require_buffer(out, "out", (T, hq, d), torch.bfloat16, dev)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=dev)
    else:
        _require_buffer(lse, "lse", (hq, T), torch.float32, dev)
    sel_out = None
    if sel is not None:
        _require_buffer(sel, "sel", (hq, T, topk), torch.int32, dev)
    elif return_sel:
        sel_out = torch.empty((hq, T, topk), dtype=torch.int32, device=dev)
    info = MobaRunInfo()
    ev_arr = None
    if events:
        stream = torch.cuda.current_stream(dev)
        for e in events:
            if not e.cuda_event:
                e.record(stream)
        ev_arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        info.events = ctypes.cast(ev_arr, ctypes.POINTER(ctypes.c_void_p))
        info.n_events = len(events)
    status = load_library().moba_attn_fwd(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(sel), _ptr(sel_out),
        _ptr(workspace), ctypes.c_size_t(workspace.numel()), _ptr(out), _ptr(lse),
        ctypes.byref(info), _stream(dev))
    _check(status)
    attn_fwd.last_info = {"launches": info.launches, "waves": info.waves,
                          "gate_path": info.gate_path, "wave_tokens": wave_tokens,
                          "workspace_bytes": need}
    if check_status:
        device_status(p, workspace)
    if return_sel and sel is None:
        return out, lse, sel_out
    return out, lse


attn_fwd.last_info = None


def attn_bwd(q, k, v, out, lse, d_out, cu_seqlens, chunk_size, topk, sel, d_lse=None,
             softmax_scale=None, workspace=None, dq=None, dk=None, dv=None, max_seqlen=None):
    """Backward of the MoBA forward (moba_attn_bwd): gradients of out and lse with respect to
    q, k and v, with the forward's selection ``sel`` held fixed.

    q bf16 [T, Hq, d], k/v bf16 [T, Hkv, d], out bf16 [T, Hq, d] and lse fp32 [Hq, T] (the
    forward's outputs), d_out bf16 [T, Hq, d], d_lse fp32 [Hq, T] or None, sel int32
    [Hq, T, topk].  Returns (dq bf16 [T, Hq, d], dk, dv bf16 [T, Hkv, d]); the call's
    workspace size and launches are in ``attn_bwd.last_info``.
    """
    _check_qkv(q, k, v)
    T, hq, d = q.shape
    hkv = k.shape[1]
    dev = q.device
    _require(k.shape == v.shape and k.shape[0] == T and k.shape[2] == d, "k/v shape mismatch")
    _require(cu_seqlens.dtype == torch.int32 and cu_seqlens.is_cuda, "cu_seqlens int32 CUDA")
    _require_buffer(out, "out", (T, hq, d), torch.bfloat16, dev)
    _require_buffer(lse, "lse", (hq, T), torch.float32, dev)
    _require_buffer(d_out, "d_out", (T, hq, d), torch.bfloat16, dev)
    if d_lse is not None:
        _require_buffer(d_lse, "d_lse", (hq, T), torch.float32, dev)
    _require_buffer(sel, "sel", (hq, T, topk), torch.int32, dev)
    batch = cu_seqlens.numel() - 1
    p = make_params(batch, T, hq, hkv, d, chunk_size, topk, softmax_scale, 0, max_seqlen)
    lib = load_library()
    need = lib.moba_bwd_workspace_size(ctypes.byref(p))
    if need == 0 and T > 0:
        raise MobaError(ERR_INVALID_ARG, lib.moba_last_error().decode())
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if dq is None:
        dq = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
    else:
        _require_buffer(dq, "dq", (T, hq, d), torch.bfloat16, dev)
    if dk is None:
        dk = torch.empty((T, hkv, d), dtype=torch.bfloat16, device=dev)
    else:
        _require_buffer(dk, "dk", (T, hkv, d), torch.bfloat16, dev)
    if dv is None:
        dv = torch.empty((T, hkv, d), dtype=torch.bfloat16, device=dev)
    else:
        _require_buffer(dv, "dv", (T, hkv, d), torch.bfloat16, dev)
    _check(lib.moba_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                             _ptr(d_out), _ptr(d_lse), _ptr(cu_seqlens), _ptr(sel), _ptr(workspace),
                             ctypes.c_size_t(workspace.numel()), _ptr(dq), _ptr(dk), _ptr(dv),
                             _stream(dev)))
    attn_bwd.last_info = {"workspace_bytes": need}
    return dq, dk, dv


attn_bwd.last_info = None
