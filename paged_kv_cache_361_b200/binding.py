"""ctypes binding of libpagedattn (include/pagedattn.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and passed as raw pointers with the current CUDA stream; every step
of the computation runs in the library's kernels. There is no fallback: if the
shared library is missing, importing a device entry point raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_NO_FREE_BLOCKS, PA_ERR_UNKNOWN_SEQ, PA_ERR_SEQ_EXISTS, \
    PA_ERR_CUDA, PA_ERR_DEVICE_BOUNDS, PA_ERR_DEVICE_TIMEOUT = range(9)
PA_F32, PA_BF16, PA_FP8_E4M3, PA_INT8 = 0, 1, 2, 3
_DTYPE = {torch.float32: PA_F32, torch.bfloat16: PA_BF16, torch.float8_e4m3fn: PA_FP8_E4M3, torch.int8: PA_INT8}
CODED_DTYPES = (torch.float8_e4m3fn, torch.int8)   # 8-bit caches: codes times a per-tensor scale


def input_dtype(cache_dtype):
    """dtype of q and of the new K/V rows for a cache of cache_dtype."""
    return torch.bfloat16 if cache_dtype in CODED_DTYPES else cache_dtype


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib().pa_status_string(status).decode()} (status {status})")


class pa_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("num_blocks", ctypes.c_int64),
                ("num_kv_heads", ctypes.c_int32), ("block_size", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


_L = None
_VP, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_P32, _P64 = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
_PCACHE = ctypes.POINTER(pa_cache)

_SIGS = {
    "pa_status_string": (ctypes.c_char_p, [_I32]),
    "pa_version": (_I32, []),
    "pa_reshape_and_cache": (_I32, [_VP, _VP, _VP, _I32, _PCACHE, _VP]),
    "pa_copy_blocks": (_I32, [_PCACHE, _VP, _I32, _VP]),
    "pa_decode": (_I32, [_VP, _I32, _I32, _PCACHE, _VP, _I32, _VP, _I32, _F, _VP, _I32, _VP, _SZ, _VP]),
    "pa_decode_ordered": (_I32, [_VP, _I32, _I32, _PCACHE, _VP, _I32, _VP, _I32, _VP, _F, _VP, _I32, _VP, _SZ, _VP]),
    "pa_decode_append": (_I32, [_VP, _VP, _VP, _VP, _I32, _I32, _PCACHE, _VP, _I32, _VP, _I32, _VP, _F, _VP, _I32, _VP,
                                _SZ, _VP]),
    "pa_decode_partition_tokens": (_I32, [_I32, _I32, _I32, _I32, _I32]),
    "pa_decode_ordered_partition_tokens": (_I32, [_I32, _I32, _I32, _I32, _I32]),
    "pa_decode_cascade": (_I32, [_VP, _I32, _I32, _PCACHE, _VP, _I32, _VP, _I32, _I32, _VP, _VP, _VP, _VP, _I32, _I32,
                                 _VP, _F, _VP, _VP, _SZ, _VP]),
    "pa_decode_cascade_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "pa_prefill": (_I32, [_VP, _I32, _VP, _I32, _I32, _PCACHE, _VP, _I32, _VP, _I32, _F, _VP, _VP]),
    "pa_decode_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "pa_get_device_error": (_I32, [_VP, _P64]),
    "pa_selftest_wait_timeout": (_I32, [_I64, _VP]),
    "pa_step_host": (_I32, [_VP, _PCACHE, _I32, _VP, _I32, _VP, _VP, _VP, _F, _VP, _I32, _VP, _SZ, _VP, _SZ, _VP]),
    "pa_step_staging_bytes": (_I32, [_I32, _I32, _PCACHE, _I32, _I32, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]),
    "pa_decode_static_workspace": (_I32, [_VP, _I32, _I32, _PCACHE, _VP, _I32, _VP, _I32, _F, _VP, _I32, _VP]),
    "pa_bm_create": (_I32, [_I64, _I32, _VP, ctypes.POINTER(_VP)]),
    "pa_bm_destroy": (None, [_VP]),
    "pa_bm_add_seq": (_I32, [_VP, _I64, _I32, _VP]),
    "pa_bm_fork": (_I32, [_VP, _I64, _I64]),
    "pa_bm_add_seq_cached": (_I32, [_VP, _I64, _VP, _I32, _VP, _P32]),
    "pa_bm_set_host_blocks": (_I32, [_VP, _I64]),
    "pa_bm_swap_out": (_I32, [_VP, _I64, _VP, _I32, _P32]),
    "pa_bm_swap_in": (_I32, [_VP, _I64, _VP, _I32, _P32]),
    "pa_swap_blocks": (_I32, [_PCACHE, _VP, _VP, _I64, _VP, _I32, _I32, _VP]),
    "pa_swap_blocks_copy": (_I32, [_PCACHE, _VP, _VP, _I64, _VP, _I32, _I32, _VP]),
    "pa_step_host_last_timing": (_I32, [_VP]),
    "pa_bm_prefix_groups": (_I32, [_VP, _I32, _VP, _I32, _I32, _VP, _VP, _VP, _VP, _P32, _P32]),
    "pa_bm_longest_first": (_I32, [_VP, _I32, _VP, _VP, _VP]),
    "pa_bm_prefix_stats": (_I32, [_VP, _P64, _P64, _P64]),
    "pa_bm_append_slot": (_I32, [_VP, _I64, _P64, _P32]),
    "pa_bm_append_slots": (_I32, [_VP, _I32, _VP, _VP, _VP, _P32]),
    "pa_bm_free_seq": (_I32, [_VP, _I64]),
    "pa_bm_block_table": (_I32, [_VP, _I64, _VP, _I32, _P32, _P64]),
    "pa_bm_block_tables": (_I32, [_VP, _I32, _VP, _VP, _I32, _I32, _VP]),
    "pa_bm_refcount": (_I32, [_VP, _I32, _P32]),
    "pa_bm_stats": (_I32, [_VP, _P64, _P64, _P64]),
    "pa_bm_free_list": (_I32, [_VP, _VP, _I64, _P64]),
}


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libpagedattn.so is not built ({LIB_PATH}); run python -m paged_kv_cache_361_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _L = lib
    return _L


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _check(status: int, what: str):
    if status != PA_OK:
        raise PagedAttnError(status, what)


def _stream(t: torch.Tensor, stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


# An 8-bit cache (e4m3 or int8) carries its per-tensor scales on the two cache
# tensor objects (set with set_kv_scales); make_cache refuses one without them.
def set_kv_scales(k_cache, v_cache, k_scale: float, v_scale: float):
    if k_cache.dtype not in CODED_DTYPES or v_cache.dtype != k_cache.dtype:
        raise TypeError("scales belong to a float8_e4m3fn or int8 cache")
    k_cache._pa_kv_scale = float(k_scale)
    v_cache._pa_kv_scale = float(v_scale)


def make_cache(k_cache: torch.Tensor, v_cache: torch.Tensor) -> pa_cache:
    """pa_cache view of two [num_blocks][num_kv_heads][block_size][head_dim] tensors."""
    if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache and v_cache must match")
    if k_cache.dtype not in _DTYPE:
        raise TypeError(f"unsupported cache dtype {k_cache.dtype}")
    nb, hkv, bs, d = k_cache.shape
    ks = vs = 1.0
    if k_cache.dtype in CODED_DTYPES:
        ks, vs = getattr(k_cache, "_pa_kv_scale", None), getattr(v_cache, "_pa_kv_scale", None)
        if ks is None or vs is None:
            raise ValueError("8-bit cache without scales: call set_kv_scales(k_cache, v_cache, k_scale, v_scale)")
    return pa_cache(_dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4), nb, hkv, bs, d,
                    _DTYPE[k_cache.dtype], ks, vs)


# --- device operations ---------------------------------------------------------

def pa_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, stream=None):
    c = make_cache(k_cache, v_cache)
    n = int(k.shape[0])
    _dev(k, "k", input_dtype(k_cache.dtype), 3), _dev(v, "v", input_dtype(k_cache.dtype), 3)
    if tuple(k.shape) != (n, c.num_kv_heads, c.head_dim) or k.shape != v.shape:
        raise ValueError("k, v must be [num_tokens][num_kv_heads][head_dim]")
    if slot_mapping.shape != (n,):
        raise ValueError("slot_mapping must be [num_tokens]")
    _check(_lib().pa_reshape_and_cache(k.data_ptr(), v.data_ptr(), _dev(slot_mapping, "slot_mapping", torch.int64),
                                       n, ctypes.byref(c), _stream(k_cache, stream)), "pa_reshape_and_cache")


def pa_copy_blocks(k_cache, v_cache, src_dst_pairs, stream=None):
    c = make_cache(k_cache, v_cache)
    n = int(src_dst_pairs.shape[0])
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [n][2]")
    _check(_lib().pa_copy_blocks(ctypes.byref(c), _dev(src_dst_pairs, "src_dst_pairs", torch.int32), n,
                                 _stream(k_cache, stream)), "pa_copy_blocks")


def pa_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, max_context_len, block_size) -> int:
    return int(_lib().pa_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, max_context_len, block_size))


def pa_decode_ordered_partition_tokens(num_seqs, num_q_heads, num_kv_heads, max_context_len, block_size) -> int:
    """The partition size pa_decode_ordered / pa_decode_append choose for -1 when given a seq_order."""
    return int(_lib().pa_decode_ordered_partition_tokens(num_seqs, num_q_heads, num_kv_heads, max_context_len,
                                                         block_size))


def pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size,
                              partition_tokens=-1) -> int:
    return int(_lib().pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                                block_size, partition_tokens))


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, max_context_len,
              partition_tokens=-1, workspace=None, stream=None, seq_order=None):
    """pa_decode, or pa_decode_ordered when seq_order (device int32, one entry
    per sequence: the dispatch order) is given."""
    c = make_cache(k_cache, v_cache)
    B, hq, d = q.shape
    _dev(q, "q", input_dtype(k_cache.dtype), 3)
    _dev(out, "out", torch.float32, 3)
    if d != c.head_dim or tuple(out.shape) != (B, hq, d):
        raise ValueError("q/out shape mismatch")
    _dev(block_tables, "block_tables", torch.int32, 2)
    _dev(context_lens, "context_lens", torch.int32, 1)
    if block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("block_tables / context_lens must have num_seqs rows")
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_dev(workspace, "workspace"),
                                                            workspace.numel() * workspace.element_size())
    if seq_order is not None:
        _dev(seq_order, "seq_order", torch.int32, 1)
        if seq_order.shape[0] != B:
            raise ValueError("seq_order must have one entry per sequence")
        _check(_lib().pa_decode_ordered(q.data_ptr(), B, hq, ctypes.byref(c), block_tables.data_ptr(),
                                        int(block_tables.shape[1]), context_lens.data_ptr(), int(max_context_len),
                                        seq_order.data_ptr(), float(scale), out.data_ptr(), int(partition_tokens),
                                        ws_ptr, ws_bytes, _stream(q, stream)), "pa_decode_ordered")
        return
    _check(_lib().pa_decode(q.data_ptr(), B, hq, ctypes.byref(c), block_tables.data_ptr(),
                            int(block_tables.shape[1]), context_lens.data_ptr(), int(max_context_len), float(scale),
                            out.data_ptr(), int(partition_tokens), ws_ptr, ws_bytes, _stream(q, stream)), "pa_decode")


def pa_decode_append(q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables, context_lens, scale, out,
                     max_context_len, partition_tokens=-1, workspace=None, stream=None, seq_order=None):
    """One decode step in one launch: the new K/V rows written at their slots
    (as pa_reshape_and_cache) by the decode CTAs, then the decode
    (pa_decode_ordered)."""
    c = make_cache(k_cache, v_cache)
    B, hq, d = q.shape
    _dev(q, "q", input_dtype(k_cache.dtype), 3)
    _dev(k_new, "k_new", input_dtype(k_cache.dtype), 3)
    _dev(v_new, "v_new", input_dtype(k_cache.dtype), 3)
    if tuple(k_new.shape) != (B, c.num_kv_heads, d) or tuple(v_new.shape) != (B, c.num_kv_heads, d):
        raise ValueError("k_new / v_new must be [num_seqs][num_kv_heads][head_dim]")
    _dev(slot_mapping, "slot_mapping", torch.int64, 1)
    _dev(out, "out", torch.float32, 3)
    if d != c.head_dim or tuple(out.shape) != (B, hq, d):
        raise ValueError("q/out shape mismatch")
    _dev(block_tables, "block_tables", torch.int32, 2)
    _dev(context_lens, "context_lens", torch.int32, 1)
    if block_tables.shape[0] != B or context_lens.shape[0] != B or slot_mapping.shape[0] != B:
        raise ValueError("block_tables / context_lens / slot_mapping must have num_seqs rows")
    if seq_order is not None:
        _dev(seq_order, "seq_order", torch.int32, 1)
        if seq_order.shape[0] != B:
            raise ValueError("seq_order must have one entry per sequence")
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_dev(workspace, "workspace"),
                                                            workspace.numel() * workspace.element_size())
    _check(_lib().pa_decode_append(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(), B, hq,
                                   ctypes.byref(c), block_tables.data_ptr(), int(block_tables.shape[1]),
                                   context_lens.data_ptr(), int(max_context_len),
                                   seq_order.data_ptr() if seq_order is not None else None, float(scale),
                                   out.data_ptr(), int(partition_tokens), ws_ptr, ws_bytes, _stream(q, stream)),
           "pa_decode_append")


def pa_prefill(q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, scale, out, max_q_len, max_context_len,
               stream=None):
    """Causal attention of the new tokens q [T][Hq][D] (sequence s owns rows
    cu_q_lens[s]..cu_q_lens[s+1]-1) over the paged cache; out fp32 [T][Hq][D]."""
    c = make_cache(k_cache, v_cache)
    T, hq, d = q.shape
    _dev(q, "q", input_dtype(k_cache.dtype), 3)
    _dev(out, "out", torch.float32, 3)
    if d != c.head_dim or tuple(out.shape) != (T, hq, d):
        raise ValueError("q/out shape mismatch")
    _dev(cu_q_lens, "cu_q_lens", torch.int32, 1)
    _dev(block_tables, "block_tables", torch.int32, 2)
    _dev(context_lens, "context_lens", torch.int32, 1)
    B = int(context_lens.shape[0])
    if cu_q_lens.shape[0] != B + 1 or block_tables.shape[0] != B:
        raise ValueError("cu_q_lens must have num_seqs + 1 entries, block_tables num_seqs rows")
    _check(_lib().pa_prefill(q.data_ptr(), B, cu_q_lens.data_ptr(), int(max_q_len), hq, ctypes.byref(c),
                             block_tables.data_ptr(), int(block_tables.shape[1]), context_lens.data_ptr(),
                             int(max_context_len), float(scale), out.data_ptr(), _stream(q, stream)), "pa_prefill")


def pa_decode_cascade_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size,
                                      max_prefix_tokens) -> int:
    return int(_lib().pa_decode_cascade_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                        max_context_len, block_size, max_prefix_tokens))


def pa_decode_cascade(q, k_cache, v_cache, block_tables, context_lens, scale, out, max_context_len, group_offsets,
                      group_members, group_prefix_tokens, seq_prefix_tokens, max_group_size, max_prefix_tokens,
                      workspace, stream=None, seq_order=None):
    """pa_decode with shared prefixes read once per group (see pagedattn.h);
    seq_order: optional device int32 dispatch order of the suffix CTAs."""
    c = make_cache(k_cache, v_cache)
    B, hq, d = q.shape
    _dev(q, "q", input_dtype(k_cache.dtype), 3)
    _dev(out, "out", torch.float32, 3)
    if d != c.head_dim or tuple(out.shape) != (B, hq, d):
        raise ValueError("q/out shape mismatch")
    _dev(block_tables, "block_tables", torch.int32, 2)
    _dev(context_lens, "context_lens", torch.int32, 1)
    _dev(seq_prefix_tokens, "seq_prefix_tokens", torch.int32, 1)
    if seq_order is not None:
        _dev(seq_order, "seq_order", torch.int32, 1)
        if seq_order.shape[0] != B:
            raise ValueError("seq_order must have one entry per sequence")
    ng = int(group_offsets.shape[0]) - 1
    if ng > 0:
        _dev(group_offsets, "group_offsets", torch.int32, 1)
        _dev(group_members, "group_members", torch.int32, 1)
        _dev(group_prefix_tokens, "group_prefix_tokens", torch.int32, 1)
    _check(_lib().pa_decode_cascade(q.data_ptr(), B, hq, ctypes.byref(c), block_tables.data_ptr(),
                                    int(block_tables.shape[1]), context_lens.data_ptr(), int(max_context_len), ng,
                                    group_offsets.data_ptr() if ng else None,
                                    group_members.data_ptr() if ng else None,
                                    group_prefix_tokens.data_ptr() if ng else None, seq_prefix_tokens.data_ptr(),
                                    int(max_group_size), int(max_prefix_tokens),
                                    seq_order.data_ptr() if seq_order is not None else None, float(scale),
                                    out.data_ptr(),
                                    _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                    _stream(q, stream)), "pa_decode_cascade")


def pa_get_device_error(stream=None):
    """(status, info) of the current device's error word; waits for the stream."""
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    info = ctypes.c_int64(0)
    st = _lib().pa_get_device_error(handle, ctypes.byref(info))
    return int(st), int(info.value)


def pa_decode_static_workspace(q, k_cache, v_cache, block_tables, context_lens, scale, out, max_context_len,
                               partition_tokens=-1, stream=None):
    """pa_decode with the library's fixed device workspace (no allocation)."""
    c = make_cache(k_cache, v_cache)
    B, hq, d = q.shape
    _dev(q, "q", input_dtype(k_cache.dtype), 3)
    _dev(out, "out", torch.float32, 3)
    if d != c.head_dim or tuple(out.shape) != (B, hq, d):
        raise ValueError("q/out shape mismatch")
    _dev(block_tables, "block_tables", torch.int32, 2)
    _dev(context_lens, "context_lens", torch.int32, 1)
    if block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("block_tables / context_lens must have num_seqs rows")
    _check(_lib().pa_decode_static_workspace(q.data_ptr(), B, hq, ctypes.byref(c), block_tables.data_ptr(),
                                             int(block_tables.shape[1]), context_lens.data_ptr(),
                                             int(max_context_len), float(scale), out.data_ptr(),
                                             int(partition_tokens), _stream(q, stream)),
           "pa_decode_static_workspace")


def pa_step_staging_bytes(num_seqs, num_q_heads, k_cache, v_cache, max_context_len, partition_tokens=-1):
    """(device bytes, pinned host bytes) that pa_step_host needs."""
    c = make_cache(k_cache, v_cache)
    db, hb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib().pa_step_staging_bytes(num_seqs, num_q_heads, ctypes.byref(c), max_context_len, partition_tokens,
                                        ctypes.byref(db), ctypes.byref(hb)), "pa_step_staging_bytes")
    return int(db.value), int(hb.value)


def _host(t, name, dtype, shape):
    if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) \
            or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host {dtype} tensor of shape {tuple(shape)}")
    return t.data_ptr()


def pa_step_host(bm: "BlockManager", k_cache, v_cache, seq_ids, q_host, k_host, v_host, scale, out_host,
                 dev_staging, host_staging, partition_tokens=-1, stream=None):
    """One decode step from host buffers (see pagedattn.h); returns after the stream drained."""
    c = make_cache(k_cache, v_cache)
    ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
    n, hq, d = q_host.shape
    _host(q_host, "q_host", input_dtype(k_cache.dtype), (len(ids), hq, c.head_dim))
    _host(k_host, "k_host", input_dtype(k_cache.dtype), (len(ids), c.num_kv_heads, c.head_dim))
    _host(v_host, "v_host", input_dtype(k_cache.dtype), (len(ids), c.num_kv_heads, c.head_dim))
    _host(out_host, "out_host", torch.float32, (len(ids), hq, c.head_dim))
    _dev(dev_staging, "dev_staging")
    if host_staging.is_cuda or not host_staging.is_contiguous():
        raise ValueError("host_staging must be contiguous host memory")
    _check(_lib().pa_step_host(bm._h, ctypes.byref(c), len(ids), _i64p(ids), hq, q_host.data_ptr(), k_host.data_ptr(),
                               v_host.data_ptr(), float(scale), out_host.data_ptr(), int(partition_tokens),
                               dev_staging.data_ptr(), dev_staging.numel() * dev_staging.element_size(),
                               host_staging.data_ptr(), host_staging.numel() * host_staging.element_size(),
                               _stream(k_cache, stream)), "pa_step_host")


def pa_swap_blocks(k_cache, v_cache, host_k, host_v, pairs, to_host: bool, stream=None):
    """Move whole blocks between the device pool and a pinned host pool."""
    c = make_cache(k_cache, v_cache)
    if host_k.is_cuda or host_v.is_cuda or host_k.shape != host_v.shape or host_k.shape[1:] != k_cache.shape[1:] \
            or host_k.dtype != k_cache.dtype or not host_k.is_contiguous() or not host_v.is_contiguous():
        raise ValueError("host pools must be contiguous host tensors shaped like the cache (pinned)")
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n][2]")
    _check(_lib().pa_swap_blocks(ctypes.byref(c), host_k.data_ptr(), host_v.data_ptr(), int(host_k.shape[0]),
                                 _dev(pairs, "pairs", torch.int32), int(pairs.shape[0]), 1 if to_host else 0,
                                 _stream(k_cache, stream)), "pa_swap_blocks")


def pa_swap_blocks_copy(k_cache, v_cache, host_k, host_v, pairs: np.ndarray, to_host: bool, stream=None):
    """pa_swap_blocks on the copy engines: pairs in host memory, one
    cudaMemcpyAsync per tensor per run of consecutive ids."""
    c = make_cache(k_cache, v_cache)
    if host_k.is_cuda or host_v.is_cuda or host_k.shape != host_v.shape or host_k.shape[1:] != k_cache.shape[1:] \
            or host_k.dtype != k_cache.dtype or not host_k.is_contiguous() or not host_v.is_contiguous():
        raise ValueError("host pools must be contiguous host tensors shaped like the cache (pinned)")
    pr = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    _check(_lib().pa_swap_blocks_copy(ctypes.byref(c), host_k.data_ptr(), host_v.data_ptr(), int(host_k.shape[0]),
                                      _i64p(pr), int(pr.shape[0]), 1 if to_host else 0, _stream(k_cache, stream)),
           "pa_swap_blocks_copy")


class pa_step_timing(ctypes.Structure):
    _fields_ = [("block_manager_us", ctypes.c_double), ("metadata_enqueue_us", ctypes.c_double),
                ("chains_enqueue_us", ctypes.c_double), ("wait_us", ctypes.c_double), ("total_us", ctypes.c_double),
                ("chunks", ctypes.c_int32)]


def pa_step_host_last_timing() -> dict:
    """Host phases (microseconds) of this thread's last pa_step_host call."""
    t = pa_step_timing()
    _check(_lib().pa_step_host_last_timing(ctypes.byref(t)), "pa_step_host_last_timing")
    return {name: (int if name == "chunks" else float)(getattr(t, name)) for name, _ in pa_step_timing._fields_}


def pa_selftest_wait_timeout(timeout_ns: int, stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    _check(_lib().pa_selftest_wait_timeout(int(timeout_ns), stream.cuda_stream), "pa_selftest_wait_timeout")


# --- host block manager --------------------------------------------------------

def _i64p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class BlockManager:
    """The C++ block manager behind pa_bm_* (one handle)."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(free_order, dtype=np.int32)
            if self._order.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
            order = _i64p(self._order)
        _check(_lib().pa_bm_create(num_blocks, block_size, order, ctypes.byref(h)), "pa_bm_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            _lib().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int, num_tokens: int) -> np.ndarray:
        slots = np.empty(max(num_tokens, 0), dtype=np.int64)
        _check(_lib().pa_bm_add_seq(self._h, seq_id, num_tokens, _i64p(slots)), "pa_bm_add_seq")
        return slots

    def fork(self, parent: int, child: int):
        _check(_lib().pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def add_seq_cached(self, seq_id: int, tokens):
        """Prefill with prefix reuse: (slots with -1 for cached tokens, n_cached)."""
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(len(tok), dtype=np.int64)
        nc = ctypes.c_int32(0)
        _check(_lib().pa_bm_add_seq_cached(self._h, seq_id, _i64p(tok), len(tok), _i64p(slots), ctypes.byref(nc)),
               "pa_bm_add_seq_cached")
        return slots, int(nc.value)

    def set_host_blocks(self, n: int):
        _check(_lib().pa_bm_set_host_blocks(self._h, n), "pa_bm_set_host_blocks")

    def _swap(self, fn, seq_id):
        cap = max(1, self.num_blocks)
        n = ctypes.c_int32(0)
        out = np.empty((cap, 2), dtype=np.int32)
        _check(fn(self._h, seq_id, _i64p(out), cap, ctypes.byref(n)), fn.__name__)
        return out[:n.value].copy()

    def swap_out(self, seq_id: int) -> np.ndarray:
        """{device, host} pairs of the sequence's blocks."""
        return self._swap(_lib().pa_bm_swap_out, seq_id)

    def swap_in(self, seq_id: int) -> np.ndarray:
        """{host, device} pairs of the sequence's blocks."""
        return self._swap(_lib().pa_bm_swap_in, seq_id)

    def prefix_stats(self) -> dict:
        c, e, h = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib().pa_bm_prefix_stats(self._h, ctypes.byref(c), ctypes.byref(e), ctypes.byref(h)),
               "pa_bm_prefix_stats")
        return dict(cached_blocks=c.value, evictable_blocks=e.value, hit_tokens=h.value)

    def append_slot(self, seq_id: int):
        slot = ctypes.c_int64()
        pair = (ctypes.c_int32 * 2)()
        _check(_lib().pa_bm_append_slot(self._h, seq_id, ctypes.byref(slot), pair), "pa_bm_append_slot")
        return int(slot.value), (None if pair[0] < 0 else (int(pair[0]), int(pair[1])))

    def append_slots(self, seq_ids):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        slots = np.empty(len(ids), dtype=np.int64)
        pairs = np.empty((len(ids), 2), dtype=np.int32)
        n = ctypes.c_int32(0)
        _check(_lib().pa_bm_append_slots(self._h, len(ids), _i64p(ids), _i64p(slots), _i64p(pairs), ctypes.byref(n)),
               "pa_bm_append_slots")
        return slots, pairs[:n.value].copy()

    def free_seq(self, seq_id: int):
        _check(_lib().pa_bm_free_seq(self._h, seq_id), "pa_bm_free_seq")

    def block_table(self, seq_id: int):
        n = ctypes.c_int32()
        L = ctypes.c_int64()
        _check(_lib().pa_bm_block_table(self._h, seq_id, None, 0, ctypes.byref(n), ctypes.byref(L)), "pa_bm_block_table")
        out = np.empty(n.value, dtype=np.int32)
        _check(_lib().pa_bm_block_table(self._h, seq_id, _i64p(out), n.value, ctypes.byref(n), ctypes.byref(L)),
               "pa_bm_block_table")
        return out, int(L.value)

    def block_tables(self, seq_ids, cap: int, pad: int = -1, out=None, lens_out=None):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        if out is None:
            out = np.empty((len(ids), cap), dtype=np.int32)
        if lens_out is None:
            lens_out = np.empty(len(ids), dtype=np.int32)
        _check(_lib().pa_bm_block_tables(self._h, len(ids), _i64p(ids), _i64p(out), cap, pad, _i64p(lens_out)),
               "pa_bm_block_tables")
        return out, lens_out

    def prefix_groups(self, seq_ids, max_group_size: int, align_tokens: int = 64):
        """Shared-prefix groups of a batch (pa_bm_prefix_groups): (offsets,
        members, prefix_tokens, seq_prefix_tokens, max_prefix) as numpy arrays
        and an int."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        offs = np.zeros(n // 2 + 1, dtype=np.int32)
        members = np.zeros(max(n, 1), dtype=np.int32)
        prefix = np.zeros(max(n // 2, 1), dtype=np.int32)
        seq_prefix = np.zeros(max(n, 1), dtype=np.int32)
        ng, mp = ctypes.c_int32(0), ctypes.c_int32(0)
        _check(_lib().pa_bm_prefix_groups(self._h, n, _i64p(ids), int(max_group_size), int(align_tokens), _i64p(offs),
                                          _i64p(members), _i64p(prefix), _i64p(seq_prefix), ctypes.byref(ng),
                                          ctypes.byref(mp)), "pa_bm_prefix_groups")
        g = ng.value
        return offs[:g + 1].copy(), members[:offs[g]].copy(), prefix[:g].copy(), seq_prefix[:n].copy(), int(mp.value)

    def longest_first(self, seq_ids, skip_tokens=None) -> np.ndarray:
        """Row indices of the batch by decreasing (tokens - skip_tokens[row]),
        ties in batch order (pa_bm_longest_first)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        order = np.zeros(max(n, 1), dtype=np.int32)
        skip = None if skip_tokens is None else np.ascontiguousarray(skip_tokens, dtype=np.int32)
        if skip is not None and len(skip) != n:
            raise ValueError("skip_tokens must have one entry per sequence")
        _check(_lib().pa_bm_longest_first(self._h, n, _i64p(ids), _i64p(skip) if skip is not None else None,
                                          _i64p(order)), "pa_bm_longest_first")
        return order[:n].copy()

    def refcount(self, block: int) -> int:
        r = ctypes.c_int32()
        _check(_lib().pa_bm_refcount(self._h, block, ctypes.byref(r)), "pa_bm_refcount")
        return int(r.value)

    def stats(self) -> dict:
        f, u, a = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib().pa_bm_stats(self._h, ctypes.byref(f), ctypes.byref(u), ctypes.byref(a)), "pa_bm_stats")
        return dict(free_blocks=f.value, used_slots=u.value, allocated_slots=a.value,
                    internal_waste=a.value - u.value)

    def free_list(self) -> np.ndarray:
        n = ctypes.c_int64()
        _check(_lib().pa_bm_free_list(self._h, None, 0, ctypes.byref(n)), "pa_bm_free_list")
        out = np.empty(n.value, dtype=np.int32)
        _check(_lib().pa_bm_free_list(self._h, _i64p(out), n.value, ctypes.byref(n)), "pa_bm_free_list")
        return out
