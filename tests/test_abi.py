"""The C-ABI library loads without a GPU and exports every declared entry point;
host-side argument checks answer before any CUDA call."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_361_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(pa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(B.LIB_PATH)
    declared = _declared()
    assert len(declared) >= 20
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) <= set(B.exported_symbols())


def test_status_strings_and_version():
    lib = B._lib()
    assert lib.pa_version() == 1
    for code in range(9):
        assert lib.pa_status_string(code)
    assert lib.pa_status_string(99) == b"unknown status"


def _cache(**kw):
    c = dict(k=16, v=32, num_blocks=8, num_kv_heads=2, block_size=16, head_dim=128, dtype=B.PA_BF16)
    c.update(kw)
    return B.pa_cache(**c)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), B.PA_ERR_INVALID_ARG),
    (dict(k=17), B.PA_ERR_INVALID_ARG),
    (dict(num_blocks=0), B.PA_ERR_INVALID_ARG),
    (dict(head_dim=96), B.PA_ERR_UNSUPPORTED),
    (dict(block_size=3), B.PA_ERR_UNSUPPORTED),
    (dict(block_size=64), B.PA_ERR_UNSUPPORTED),
    (dict(dtype=7), B.PA_ERR_UNSUPPORTED),
    (dict(dtype=B.PA_FP8_E4M3), B.PA_ERR_INVALID_ARG),                                  # scales 0
    (dict(dtype=B.PA_FP8_E4M3, k_scale=1.0, v_scale=float("nan")), B.PA_ERR_INVALID_ARG),
    (dict(dtype=B.PA_FP8_E4M3, k_scale=-1.0, v_scale=1.0), B.PA_ERR_INVALID_ARG),
    (dict(dtype=B.PA_FP8_E4M3, k_scale=float("inf"), v_scale=1.0), B.PA_ERR_INVALID_ARG),
    (dict(dtype=B.PA_INT8), B.PA_ERR_INVALID_ARG),                                      # scales 0
    (dict(dtype=B.PA_INT8, k_scale=1.0, v_scale=-2.0), B.PA_ERR_INVALID_ARG),
])
def test_host_checks_before_launch(kw, status):
    lib = B._lib()
    c = _cache(**kw)
    assert lib.pa_reshape_and_cache(16, 16, 16, 1, ctypes.byref(c), None) == status
    assert lib.pa_copy_blocks(ctypes.byref(c), 16, 1, None) == status


@pytest.mark.parametrize("dt", ["float8_e4m3fn", "int8"])
def test_8bit_cache_needs_its_scales(dt):
    import torch
    kc = torch.zeros(4, 1, 16, 64, dtype=getattr(torch, dt))
    vc = torch.zeros_like(kc)
    with pytest.raises(ValueError, match="scales"):
        B.make_cache(kc, vc)
    with pytest.raises(TypeError):
        B.set_kv_scales(kc.float(), vc.float(), 1.0, 1.0)
    assert B.input_dtype(kc.dtype) == torch.bfloat16
    assert B.input_dtype(torch.float32) == torch.float32


def test_8bit_scales_need_matching_caches():
    """K and V of one 8-bit cache share a format: mixed e4m3 / int8 pools or a
    16-bit pool are refused before anything reaches the library."""
    import torch
    k8 = torch.zeros(4, 1, 16, 64, dtype=torch.int8)
    kf = torch.zeros(4, 1, 16, 64, dtype=torch.float8_e4m3fn)
    with pytest.raises(TypeError):
        B.set_kv_scales(k8, kf, 1.0, 1.0)
    with pytest.raises(TypeError):
        B.set_kv_scales(k8.bfloat16(), k8.bfloat16(), 1.0, 1.0)
    with pytest.raises(ValueError, match="match"):
        B.make_cache(k8, kf)


def test_decode_argument_checks():
    lib = B._lib()
    c = _cache()
    args = dict(q=16, B=2, hq=4, tables=16, maxb=4, lens=16, maxctx=64, scale=0.1, out=16, P=-1, ws=0, wsb=0)

    def call(**kw):
        a = dict(args, **kw)
        return lib.pa_decode(a["q"], a["B"], a["hq"], ctypes.byref(c), a["tables"], a["maxb"], a["lens"], a["maxctx"],
                             a["scale"], a["out"], a["P"], a["ws"] or None, a["wsb"], None)
    assert call(hq=3) == B.PA_ERR_INVALID_ARG                  # not a multiple of kv heads
    assert call(hq=32) == B.PA_ERR_UNSUPPORTED                 # group of 16
    assert call(maxctx=65) == B.PA_ERR_INVALID_ARG             # above max_blocks * block_size
    assert call(P=8) == B.PA_ERR_INVALID_ARG                   # not a multiple of block_size
    assert call(scale=float("nan")) == B.PA_ERR_INVALID_ARG
    assert call(q=0) == B.PA_ERR_INVALID_ARG
    assert call(out=8) == B.PA_ERR_INVALID_ARG                 # misaligned
    assert call(B=0) == B.PA_OK                                # nothing to do, nothing launched
    assert call(P=16, maxctx=64) == B.PA_ERR_INVALID_ARG        # split needs a workspace


def test_workspace_sizes():
    # counters (1 + num_seqs * hkv) x 4 B rounded to 256; split adds (m, l) rows rounded to 256 + D floats per row
    cnt = lambda b, hkv: ((1 + b * hkv) * 4 + 255) // 256 * 256
    assert B.pa_decode_workspace_bytes(4, 8, 8, 128, 600, 16, 0) == cnt(4, 8)
    assert B.pa_decode_workspace_bytes(4, 8, 8, 128, 512, 16, 512) == cnt(4, 8)
    rows = 4 * 8 * 2
    assert B.pa_decode_workspace_bytes(4, 8, 8, 128, 600, 16, 512) == \
        cnt(4, 8) + (rows * 8 + 255) // 256 * 256 + rows * 128 * 4
    P = B.pa_decode_partition_tokens(64, 32, 32, 2049, 16)
    assert P == 0 or P % 16 == 0
    # with a dispatch order: never more partitions than without, and no split for many moderate units
    for args in ((256, 32, 8, 4097, 16), (4, 64, 8, 131073, 32), (64, 32, 8, 1513, 16), (64, 32, 32, 2049, 16),
                 (300, 8, 8, 9000, 16), (16, 8, 8, 5000, 8)):
        po, pu = B.pa_decode_ordered_partition_tokens(*args), B.pa_decode_partition_tokens(*args)
        parts = lambda p: 1 if p == 0 else -(-args[3] // p)
        assert parts(po) <= parts(pu)
    assert B.pa_decode_ordered_partition_tokens(256, 32, 8, 4097, 16) == 0
    assert B.pa_decode_partition_tokens(256, 32, 8, 4097, 16) == 1024
    assert B.pa_decode_ordered_partition_tokens(4, 64, 8, 131073, 32) > 0


def test_step_timing_and_copy_swap_host_checks():
    lib = B._lib()
    assert lib.pa_step_host_last_timing(None) == B.PA_ERR_INVALID_ARG
    t = B.pa_step_host_last_timing()
    assert t["total_us"] == 0.0            # no pa_step_host call on this thread
    c = _cache()
    pairs = (ctypes.c_int32 * 2)(0, 1)
    assert lib.pa_swap_blocks_copy(ctypes.byref(c), 16, 16, 4, pairs, -1, 1, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_swap_blocks_copy(ctypes.byref(c), 16, 16, 0, pairs, 1, 1, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_swap_blocks_copy(ctypes.byref(c), 16, 16, 4, pairs, 0, 1, None) == B.PA_OK
    assert lib.pa_swap_blocks_copy(ctypes.byref(c), None, 16, 4, pairs, 1, 1, None) == B.PA_ERR_INVALID_ARG
