"""Host-only checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments with the documented status before touching the GPU."""

import ctypes
import os
import re

import pytest
import torch

from block_sparse_long_meanpool_b200 import build, moba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moba.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moba.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moba_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(moba.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def params(**kw):
    base = dict(batch=1, total_tokens=2048, num_q_heads=4, num_kv_heads=4, head_dim=64,
                chunk_size=256, topk=3, softmax_scale=None, wave_tokens=0, max_seqlen=0)
    base.update(kw)
    return moba.make_params(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), moba.ERR_INVALID_ARG),
    (dict(total_tokens=-1), moba.ERR_INVALID_ARG),
    (dict(num_kv_heads=3), moba.ERR_INVALID_ARG),
    (dict(topk=0), moba.ERR_INVALID_ARG),
    (dict(chunk_size=0), moba.ERR_INVALID_ARG),
    (dict(wave_tokens=-128), moba.ERR_INVALID_ARG),
    (dict(head_dim=96), moba.ERR_UNSUPPORTED),
    (dict(chunk_size=100), moba.ERR_UNSUPPORTED),
    (dict(topk=33), moba.ERR_UNSUPPORTED),
    (dict(wave_tokens=100), moba.ERR_UNSUPPORTED),
    (dict(max_seqlen=-1), moba.ERR_INVALID_ARG),
    (dict(max_seqlen=4096), moba.ERR_INVALID_ARG),             # longer than all tokens
    (dict(batch=2, max_seqlen=1000), moba.ERR_INVALID_ARG),    # 2 x 1000 < 2048 tokens
])
def test_invalid_params_are_rejected(lib, kw, status):
    p = params(**kw)
    assert lib.moba_workspace_size(ctypes.byref(p)) == 0
    assert lib.moba_num_blocks_bound(ctypes.byref(p)) == -1
    rc = lib.moba_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, 0, None,
                           None, None, None)
    assert rc == status, lib.moba_last_error()
    assert lib.moba_last_error()
    assert lib.moba_meanpool(ctypes.byref(p), None, None, None, None) == status
    assert lib.moba_gate_topk(ctypes.byref(p), None, None, None, None, None) == status


def test_null_params_and_null_pointers(lib):
    assert lib.moba_attn_fwd(None, None, None, None, None, None, None, None, 0, None, None,
                             None, None) == moba.ERR_INVALID_ARG
    p = params()
    assert lib.moba_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, 0, None,
                             None, None, None) == moba.ERR_INVALID_ARG
    assert b"NULL" in lib.moba_last_error()
    assert lib.moba_device_status(ctypes.byref(p), None, None) == moba.ERR_WORKSPACE


def test_empty_input_is_a_no_op(lib):
    p = params(total_tokens=0)
    assert lib.moba_workspace_size(ctypes.byref(p)) > 0
    assert lib.moba_num_blocks_bound(ctypes.byref(p)) == 0
    info = moba.MobaRunInfo()
    rc = lib.moba_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, 0, None,
                           None, ctypes.byref(info), None)
    assert rc == moba.OK and info.launches == 0
    assert lib.moba_meanpool(ctypes.byref(p), None, None, None, None) == moba.OK


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="hands fake device addresses to the library: host-only check")
def test_workspace_and_alignment_checks_precede_any_launch(lib):
    p = params()
    fake = ctypes.c_void_p(1 << 20)
    need = lib.moba_workspace_size(ctypes.byref(p))
    rc = lib.moba_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, None, None, fake, need - 1,
                           fake, fake, None, None)
    assert rc == moba.ERR_WORKSPACE
    assert str(need).encode() in lib.moba_last_error()
    rc = lib.moba_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, None, None, None, need,
                           fake, fake, None, None)
    assert rc == moba.ERR_WORKSPACE
    odd = ctypes.c_void_p((1 << 20) + 8)
    rc = lib.moba_attn_fwd(ctypes.byref(p), odd, fake, fake, fake, None, None, fake, need,
                           fake, fake, None, None)
    assert rc == moba.ERR_INVALID_ARG
    rc = lib.moba_attn_fwd(ctypes.byref(p), fake, fake, fake, fake, None, None,
                           ctypes.c_void_p((1 << 20) + 128), need, fake, fake, None, None)
    assert rc == moba.ERR_WORKSPACE
    # 32-bit partial-output indices: one wave of 1M tokens x 64 heads x top-32 is refused
    big = params(total_tokens=1 << 20, num_q_heads=64, num_kv_heads=8, head_dim=128,
                 chunk_size=4096, topk=32, wave_tokens=0)
    need_big = lib.moba_workspace_size(ctypes.byref(big))
    assert need_big > 0
    rc = lib.moba_attn_fwd(ctypes.byref(big), fake, fake, fake, fake, None, None, fake,
                           need_big, fake, fake, None, None)
    assert rc == moba.ERR_UNSUPPORTED


def test_max_seqlen_is_accepted_when_consistent(lib):
    for kw in (dict(max_seqlen=2048), dict(batch=2, max_seqlen=1024), dict(batch=3, max_seqlen=1500)):
        assert lib.moba_workspace_size(ctypes.byref(params(**kw))) > 0, kw


def test_noalloc_status_read_without_a_forward(lib):
    """With no allocation-free forward run in this process there is nothing to read: OK, or a
    CUDA error when no device can be queried (this host has none); never a device access."""
    rc = lib.moba_device_status_noalloc(None)
    assert rc in (moba.OK, moba.ERR_CUDA), rc
    if rc == moba.ERR_CUDA:
        assert lib.moba_last_error()


def test_status_strings(lib):
    for code in range(6):
        assert lib.moba_status_string(code).startswith(b"MOBA_")
    assert lib.moba_status_string(99) == b"MOBA_ERR_UNKNOWN"


def test_workspace_grows_with_the_wave_and_block_bound(lib):
    sizes = [lib.moba_workspace_size(ctypes.byref(params(total_tokens=8192, wave_tokens=w)))
             for w in (128, 1024, 4096, 0)]
    assert sizes == sorted(sizes) and sizes[0] < sizes[-1]
    p = params(batch=3, total_tokens=1000, chunk_size=256)
    assert lib.moba_num_blocks_bound(ctypes.byref(p)) == 4 + 2


WAVE_CASES = [  # T, Hq, Hkv, d, chunk, topk, batch
    (1 << 20, 32, 8, 128, 4096, 12, 1), (1 << 22, 32, 8, 128, 16384, 12, 1),
    (10 << 20, 8, 2, 128, 40960, 12, 1), (63000, 32, 8, 128, 1024, 4, 4),
    (32768, 32, 32, 128, 512, 3, 1), (32768, 32, 8, 128, 256, 32, 1), (2048, 4, 4, 64, 256, 3, 1),
    (200000, 16, 16, 64, 128, 8, 50), (100, 4, 4, 64, 128, 3, 1),
]


def test_workspace_size_never_decreases_with_the_wave(lib):
    for T, hq, hkv, d, chunk, topk, batch in WAVE_CASES:
        waves = [128 * k for k in (1, 2, 3, 5, 8, 13, 100, 1000, 4000) if 128 * k < T] + [0]  # 0: one wave
        sizes = [lib.moba_workspace_size(ctypes.byref(moba.make_params(batch, T, hq, hkv, d, chunk, topk, None, w)))
                 for w in waves]
        assert all(x > 0 for x in sizes) and sizes == sorted(sizes), (T, sizes)


def test_wave_choice_is_the_largest_that_fits(lib):
    """Every budget gets one wave when it fits, else the largest multiple of 128 whose
    workspace fits (the next one does not), or 128 when nothing fits."""
    for T, hq, hkv, d, chunk, topk, batch in WAVE_CASES:
        def size(w):
            return lib.moba_workspace_size(ctypes.byref(moba.make_params(batch, T, hq, hkv, d, chunk, topk, None, w)))
        full = size(0)
        for frac in (0.01, 0.05, 0.1, 0.3, 0.6, 0.9, 1.0, 1.1):
            budget = int(full * frac)
            w = moba.choose_wave_tokens(T, hq, hkv, d, chunk, topk, batch, budget)
            if w == 0:
                assert full <= budget or T <= 128
                continue
            assert w % 128 == 0 and 0 < w < T and w * hq * topk < 2 ** 31
            if size(w) > budget:
                assert w == 128, (T, frac, w)
                continue
            nxt = w + 128
            assert nxt >= T or nxt * hq * topk >= 2 ** 31 or size(nxt) > budget, (T, frac, w)


def test_wave_choice_respects_budget(lib):
    w = moba.choose_wave_tokens(1 << 20, 32, 8, 128, 4096, 12, 1, 8 << 30)
    assert w > 0 and w % 128 == 0
    p = moba.make_params(1, 1 << 20, 32, 8, 128, 4096, 12, None, w)
    assert lib.moba_workspace_size(ctypes.byref(p)) <= 8 << 30
    assert moba.choose_wave_tokens(2048, 4, 4, 64, 256, 3, 1, 1 << 30) == 0


def test_decode_workspace_size_and_argument_checks(lib):
    p = params()
    need = lib.moba_decode_workspace_size(ctypes.byref(p))
    assert need > 0
    bad = params(head_dim=96)
    assert lib.moba_decode_workspace_size(ctypes.byref(bad)) == 0
    assert lib.moba_decode_fwd(None, None, None, None, None, None, None, 0, None, None, None) == moba.ERR_INVALID_ARG
    assert lib.moba_decode_fwd(ctypes.byref(p), None, None, None, None, None, None, need,
                               None, None, None) == moba.ERR_INVALID_ARG
    big = params(batch=70000)
    assert lib.moba_decode_workspace_size(ctypes.byref(big)) > 0


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="hands fake device addresses to the library: host-only check")
def test_decode_checks_precede_any_launch(lib):
    p = params()
    fake = ctypes.c_void_p(1 << 20)
    need = lib.moba_decode_workspace_size(ctypes.byref(p))
    rc = lib.moba_decode_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, need - 1,
                             fake, fake, None)
    assert rc == moba.ERR_WORKSPACE
    odd = ctypes.c_void_p((1 << 20) + 8)
    rc = lib.moba_decode_fwd(ctypes.byref(p), odd, fake, fake, fake, fake, fake, need,
                             fake, fake, None)
    assert rc == moba.ERR_INVALID_ARG
    big = params(batch=70000)
    rc = lib.moba_decode_fwd(ctypes.byref(big), fake, fake, fake, fake, fake, fake,
                             lib.moba_decode_workspace_size(ctypes.byref(big)), fake, fake, None)
    assert rc == moba.ERR_UNSUPPORTED


def test_minmax_argument_checks(lib):
    p = params()
    assert lib.moba_minmaxpool(None, None, None, None, None, None) == moba.ERR_INVALID_ARG
    assert lib.moba_minmaxpool(ctypes.byref(p), None, None, None, None, None) == moba.ERR_INVALID_ARG
    need = lib.moba_decode_workspace_size(ctypes.byref(p))
    assert lib.moba_decode_minmax_fwd(None, None, None, None, None, None, None, None, 0, None, None,
                                      None) == moba.ERR_INVALID_ARG
    assert lib.moba_decode_minmax_fwd(ctypes.byref(p), None, None, None, None, None, None, None, need,
                                      None, None, None) == moba.ERR_INVALID_ARG
    bad = params(head_dim=96)
    assert lib.moba_minmaxpool(ctypes.byref(bad), None, None, None, None, None) == moba.ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="hands fake device addresses to the library: host-only check")
def test_minmax_checks_precede_any_launch(lib):
    p = params()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    # k_max misaligned, k_min missing
    assert lib.moba_minmaxpool(ctypes.byref(p), fake, fake, fake, odd, None) == moba.ERR_INVALID_ARG
    assert lib.moba_minmaxpool(ctypes.byref(p), fake, fake, None, fake, None) == moba.ERR_INVALID_ARG
    need = lib.moba_decode_workspace_size(ctypes.byref(p))
    # only one half of the summary given
    rc = lib.moba_decode_minmax_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, need,
                                    fake, fake, None)
    assert rc == moba.ERR_INVALID_ARG
    rc = lib.moba_decode_minmax_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, odd, fake, need,
                                    fake, fake, None)
    assert rc == moba.ERR_INVALID_ARG
    rc = lib.moba_decode_minmax_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, need - 1,
                                    fake, fake, None)
    assert rc == moba.ERR_WORKSPACE


def test_selftest_argument_checks(lib):
    assert lib.moba_selftest_timeout(None, 16, None) == moba.ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    assert lib.moba_selftest_timeout(fake, 0, None) == moba.ERR_INVALID_ARG
    assert lib.moba_selftest_timeout(fake, (1 << 20) + 1, None) == moba.ERR_INVALID_ARG


def _meta(*shape, dtype=torch.bfloat16):
    return torch.empty(shape, dtype=dtype, device="meta")


def test_decode_binding_rejects_mismatched_buffers(lib):
    """The binding checks every caller-supplied tensor's shape, dtype and backing memory before
    any launch (host-only: meta tensors, no device memory)."""
    B, T, hq, hkv, d, chunk, topk = 3, 1000, 4, 2, 64, 128, 3
    bound = moba.num_blocks_bound(moba.make_params(B, T, hq, hkv, d, chunk, topk))
    q, k, v = _meta(B, hq, d), _meta(T, hkv, d), _meta(T, hkv, d)
    cu = _meta(B + 1, dtype=torch.int32)
    means = _meta(bound, hkv, d, dtype=torch.float32)
    kmin, kmax = _meta(bound, hkv, d), _meta(bound, hkv, d)
    out, lse = _meta(B, hq, d), _meta(hq, B, dtype=torch.float32)
    ok_mean = [("k_mean", means, torch.float32)]
    ok_mm = [("k_min", kmin, torch.bfloat16), ("k_max", kmax, torch.bfloat16)]
    moba._validate_decode(q, k, v, cu, ok_mean, out, lse, chunk, topk)
    moba._validate_decode(q, k, v, cu, ok_mm, None, None, chunk, topk)
    # a view of fewer rows is fine while its memory holds the bound's rows (as meanpool returns)
    moba._validate_decode(q, k, v, cu, [("k_mean", means[:bound - 2], torch.float32)], out, lse, chunk, topk)
    bad = [
        (q, _meta(T, hkv, 128), _meta(T, hkv, 128), cu, ok_mean, out, lse),          # head_dim
        (q, k, _meta(T - 1, hkv, d), cu, ok_mean, out, lse),                         # v shape
        (q, k, v, _meta(B, dtype=torch.int32), ok_mean, out, lse),                   # cu entries
        (q, k, v, cu, [("k_mean", _meta(bound - 1, hkv, d, dtype=torch.float32), torch.float32)], out, lse),
        (q, k, v, cu, [("k_mean", means[1:], torch.float32)], out, lse),             # offset view
        (q, k, v, cu, [("k_mean", _meta(bound, hkv, d), torch.float32)], out, lse),  # dtype
        (q, k, v, cu, [("k_min", _meta(bound, 1, d), torch.bfloat16)], out, lse),    # kv heads
        (q, k, v, cu, ok_mm, _meta(B, hq, d + 1), lse),                              # out shape
        (q, k, v, cu, ok_mm, out.float(), lse),                                      # out dtype
        (q, k, v, cu, ok_mm, out, _meta(B, hq, dtype=torch.float32)),                # lse layout
    ]
    for i, args in enumerate(bad):
        with pytest.raises(ValueError):
            moba._validate_decode(*args, chunk, topk)
            pytest.fail(f"case {i} accepted")


def test_decode_workspace_follows_the_split_rule(lib):
    """The decode workspace: selections and slot counts per (sequence, head) row, and fp32
    partials for topk * splits key ranges per row.  splits doubles from 1 while the grid has
    fewer than 1184 (row, block, range) tasks (8 per SM), every row's partials still fit one
    warp's merge (topk * splits <= 64) and a range keeps at least 128 keys."""
    def align(x):
        return (x + 255) // 256 * 256

    for batch, hq, d, chunk, topk in [(64, 32, 128, 512, 3), (16, 32, 128, 2048, 8), (1, 32, 128, 4096, 12),
                                      (1, 4, 64, 128, 32), (3, 8, 64, 256, 1), (5000, 32, 128, 512, 3),
                                      (2, 6, 128, 1024, 4)]:
        s = 1
        while batch * hq * topk * s < 1184 and topk * s * 2 <= 64 and chunk // (s * 2) >= 128:
            s *= 2
        rows, parts = batch * hq, topk * s
        want = align(4 * rows * topk) + align(4 * rows) + align(4 * rows * parts * d) + align(4 * rows * parts)
        p = moba.make_params(batch, 1 << 20, hq, hq // 2 if hq % 2 == 0 else hq, d, chunk, topk)
        assert lib.moba_decode_workspace_size(ctypes.byref(p)) == want, (batch, hq, chunk, topk, s)


def test_product_package_never_touches_the_oracle():
    """The oracle is test infrastructure: nothing under the package imports or names it."""
    pkg = os.path.join(ROOT, "block_sparse_long_meanpool_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "oracle." not in text, f


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="build"):
        moba.load_library(str(tmp_path / "libmoba.so"))


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "moba.h"

/* A C99 client: every entry point linked, the host-side ones called, the compute ones on
   their argument-error paths (nothing reaches a device). */
int main(void) {
    moba_params p;
    memset(&p, 0, sizeof p);
    p.batch = 1; p.total_tokens = 2048; p.num_q_heads = 4; p.num_kv_heads = 4;
    p.head_dim = 64; p.chunk_size = 256; p.topk = 3;
    printf("%d %zu %zu\n", moba_num_blocks_bound(&p), moba_workspace_size(&p), moba_decode_workspace_size(&p));
    printf("%d %d %d %d %d %d %d %d %d %d\n",
           (int)moba_meanpool(NULL, NULL, NULL, NULL, NULL),
           (int)moba_minmaxpool(&p, NULL, NULL, NULL, NULL, NULL),
           (int)moba_gate_topk(&p, NULL, NULL, NULL, NULL, NULL),
           (int)moba_attn_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL, NULL),
           (int)moba_device_status(&p, NULL, NULL),
           (int)moba_decode_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL),
           (int)moba_decode_minmax_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL),
           (int)moba_selftest_timeout(NULL, 16, NULL),
           (int)moba_attn_fwd_noalloc(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL),
           (int)MOBA_OK);
    printf("%d\n", (int)moba_device_status_noalloc(NULL));
    printf("%s|%s\n", moba_status_string(MOBA_ERR_WORKSPACE), moba_last_error());
    return 0;
}
"""


def test_header_is_plain_c_and_every_entry_point_links(lib, tmp_path):
    """include/moba.h compiles as C99 with warnings as errors, and a C program links and runs
    against libmoba.so (C linkage of every declared entry point)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(moba.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmoba", "-Wl,-rpath," + libdir],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES="")).stdout.splitlines()
    nb, ws, dws = (int(x) for x in out[0].split())
    assert nb == 8 and ws > 0 and dws > 0
    codes = [int(x) for x in out[1].split()]
    I, W = moba.ERR_INVALID_ARG, moba.ERR_WORKSPACE  # device_status with no workspace: WORKSPACE
    assert codes == [I, I, I, I, W, I, I, I, I, moba.OK], codes
    assert int(out[2]) in (moba.OK, moba.ERR_CUDA)
    name, _ = out[3].split("|", 1)
    assert name == lib.moba_status_string(moba.ERR_WORKSPACE).decode()
