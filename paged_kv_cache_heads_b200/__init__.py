"""paged_kv_cache_heads_b200: Python binding of libpa, the B200 paged KV-cache hot path.

The functions here carry the C entry points' names and only marshal
arguments: device tensors become pointers, the current torch CUDA stream
becomes the ``stream`` argument, and a non-OK status raises ``PAError`` with
the library's message. Every step of the computation runs in libpa's CUDA
kernels; nothing here computes on the host. If ``libpa.so`` has not been
built, the first call raises ``RuntimeError``; there is no fallback.

Build it with ``python -m paged_kv_cache_heads_b200.build``.
"""

from __future__ import annotations

import ctypes as C
import os
import threading

__all__ = [
    "PAError", "PA_FP32", "PA_BF16", "PA_FLAG_SLOT_RANGE", "PA_FLAG_BLOCK_RANGE",
    "PA_FLAG_CONTEXT_RANGE", "PA_FLAG_PAIR_RANGE", "PA_FLAG_WAIT_TIMEOUT", "CacheDesc",
    "library_path", "load_library", "exported_symbols", "pa_store_kv", "pa_copy_blocks",
    "pa_attention", "pa_attention_workspace_size", "pa_attention_static_workspace", "pa_read_device_flags", "pa_get_debug_status", "pa_set_wait_limit_ns", "pa_last_error",
    "pa_version", "BlockManager",
]

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_OUT_OF_BLOCKS, PA_ERR_INDEX = range(6)
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_CUDA",
                4: "PA_ERR_OUT_OF_BLOCKS", 5: "PA_ERR_INDEX"}
PA_FP32, PA_BF16 = 0, 1
PA_FLAG_SLOT_RANGE = 0x1
PA_FLAG_BLOCK_RANGE = 0x2
PA_FLAG_CONTEXT_RANGE = 0x4
PA_FLAG_PAIR_RANGE = 0x8
PA_FLAG_WAIT_TIMEOUT = 0x10
PA_STATIC_WORKSPACE_BYTES = 16 << 20

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.environ.get("PA_LIBRARY", os.path.join(_HERE, "libpa.so"))


class PAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), message))
        self.status = status


class CacheDesc(C.Structure):
    """``pa_cache_desc``: geometry of the K and V caches."""
    _fields_ = [("num_blocks", C.c_int32), ("block_size", C.c_int32), ("num_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("dtype", C.c_int32)]


_P = C.c_void_p
_I32 = C.c_int32
_I64 = C.c_int64
_PI32 = C.POINTER(C.c_int32)
_PI64 = C.POINTER(C.c_int64)

_SIGNATURES = {
    "pa_store_kv": (C.c_int, [_P, _P, _P, _I32, _P, _P, C.POINTER(CacheDesc), _P]),
    "pa_copy_blocks": (C.c_int, [_P, _I32, _P, _P, C.POINTER(CacheDesc), _P]),
    "pa_attention_workspace_size": (C.c_size_t, [_I32, _I32, _I32, _I32, C.POINTER(CacheDesc)]),
    "pa_attention": (C.c_int, [_P, _P, _P, _P, _I32, _P, _P, _I32, _I32, _I32, _I32, _I32, C.c_float,
                               C.POINTER(CacheDesc), _P, _P, C.c_size_t, _P]),
    "pa_attention_static_workspace": (C.c_int, [_P, _P, _P, _P, _I32, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                                 C.c_float, C.POINTER(CacheDesc), _P, _P]),
    "pa_read_device_flags": (C.c_int, [C.POINTER(C.c_uint32), _I32]),
    "pa_get_debug_status": (C.c_int, [_P, C.POINTER(C.c_int32)]),
    "pa_set_wait_limit_ns": (C.c_uint64, [C.c_uint64]),
    "pa_last_error": (C.c_char_p, []),
    "pa_version": (C.c_char_p, []),
    "pa_bm_create": (C.c_int, [_I32, _I32, _PI32, C.POINTER(_P)]),
    "pa_bm_destroy": (None, [_P]),
    "pa_bm_add_seq": (C.c_int, [_P, _I64, _I32, _PI32]),
    "pa_bm_fork": (C.c_int, [_P, _I64, _I64, _I32]),
    "pa_bm_append_tokens": (C.c_int, [_P, _I64, _I32, _PI32, _PI32, _PI32]),
    "pa_bm_free_seq": (C.c_int, [_P, _I64]),
    "pa_bm_slot_mapping": (C.c_int, [_P, _I64, _I32, _I32, _PI32]),
    "pa_bm_block_table": (C.c_int, [_P, _PI64, _I32, _I32, _PI32, _PI32]),
    "pa_bm_num_free": (_I32, [_P]),
    "pa_bm_num_blocks": (_I32, [_P]),
    "pa_bm_refcount": (_I32, [_P, _I32]),
    "pa_bm_seq_len": (_I32, [_P, _I64]),
    "pa_bm_free_list": (_I32, [_P, _PI32, _I32]),
    "pa_bm_get_stats": (C.c_int, [_P, C.c_double, C.c_void_p]),
    "pa_bm_compact": (C.c_int, [_P, _PI32, _I32, _PI32]),
    "pa_bm_cascade_groups": (C.c_int, [_P, _PI64, _I32, _I32, _PI32, _PI32, _PI32]),
    "pa_attention_cascade_workspace_size": (C.c_size_t, [_I32, _I32, _I32, _I32, C.POINTER(CacheDesc)]),
    "pa_attention_cascade": (C.c_int, [_P, _P, _P, _P, _I32, _P, _P, _I32, _I32, _I32, _P, _P, _I32, _I32, _I32,
                                       C.c_float, C.POINTER(CacheDesc), _P, _P, C.c_size_t, _P]),
}


class BlockManagerStats(C.Structure):
    """Mirror of ``pa_bm_stats``."""
    _fields_ = [("num_blocks", C.c_int32), ("free_blocks", C.c_int32), ("held_blocks", C.c_int32),
                ("num_seqs", C.c_int32), ("logical_blocks", C.c_int64), ("tokens", C.c_int64),
                ("used_slots", C.c_int64), ("block_utilisation", C.c_double),
                ("internal_fragmentation", C.c_double), ("sharing_saving", C.c_double),
                ("table_bytes", C.c_double), ("table_overhead", C.c_double), ("alloc_p50_us", C.c_double),
                ("alloc_p99_us", C.c_double), ("alloc_samples", C.c_int64)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}

_lib = None
_lock = threading.Lock()


def load_library():
    """Load libpa.so once; raises RuntimeError if it is missing or incomplete."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError("libpa.so not found at %s; build it with "
                                   "`python -m paged_kv_cache_heads_b200.build`" % path)
            lib = C.CDLL(path)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)  # AttributeError if an entry point is missing
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def exported_symbols():
    """Names of the C entry points this binding expects libpa to export."""
    return sorted(_SIGNATURES)


def _check(status: int):
    if status != PA_OK:
        raise PAError(status, load_library().pa_last_error().decode(errors="replace"))


# --------------------------------------------------------------------------
# argument marshalling
# --------------------------------------------------------------------------

def _ptr(x):
    """Device or host pointer of a torch tensor, or an int address, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream, *tensors):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    for t in tensors:
        if t is not None and not isinstance(t, int) and t.is_cuda:
            return torch.cuda.current_stream(t.device).cuda_stream
    return None


def _desc(cache) -> CacheDesc:
    if isinstance(cache, CacheDesc):
        return cache
    return CacheDesc(*cache)


def pa_version() -> str:
    return load_library().pa_version().decode()


def pa_last_error() -> str:
    return load_library().pa_last_error().decode(errors="replace")


def pa_store_kv(k, v, slot_mapping, num_tokens, k_cache, v_cache, cache, stream=None):
    """Scatter token rows of k/v into cache slots ``slot_mapping`` (see include/pa.h)."""
    d = _desc(cache)
    _check(load_library().pa_store_kv(_ptr(k), _ptr(v), _ptr(slot_mapping), int(num_tokens),
                                      _ptr(k_cache), _ptr(v_cache), C.byref(d),
                                      _stream(stream, k_cache)))


def pa_copy_blocks(src_dst_pairs, num_pairs, k_cache, v_cache, cache, stream=None):
    """Copy block src to block dst in both caches for each pair (see include/pa.h)."""
    d = _desc(cache)
    _check(load_library().pa_copy_blocks(_ptr(src_dst_pairs), int(num_pairs), _ptr(k_cache), _ptr(v_cache),
                                         C.byref(d), _stream(stream, k_cache)))


def pa_attention_workspace_size(num_seqs, num_q_heads, max_query_len, max_context_len, cache) -> int:
    d = _desc(cache)
    return int(load_library().pa_attention_workspace_size(int(num_seqs), int(num_q_heads), int(max_query_len),
                                                          int(max_context_len), C.byref(d)))


def pa_attention(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, query_start_loc,
                 num_seqs, num_q_tokens, num_q_heads, max_query_len, max_context_len, scale, cache, out,
                 workspace=None, workspace_bytes=None, stream=None):
    """Attention of every query row over its paged keys (see include/pa.h)."""
    d = _desc(cache)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None or isinstance(workspace, int) else \
            workspace.numel() * workspace.element_size()
    _check(load_library().pa_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), int(max_blocks_per_seq),
        _ptr(context_lens), _ptr(query_start_loc), int(num_seqs), int(num_q_tokens), int(num_q_heads),
        int(max_query_len), int(max_context_len), float(scale), C.byref(d), _ptr(out), _ptr(workspace),
        int(workspace_bytes), _stream(stream, q, out)))


def pa_attention_static_workspace(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                  query_start_loc, num_seqs, num_q_tokens, num_q_heads, max_query_len,
                                  max_context_len, scale, cache, out, stream=None):
    """pa_attention without a caller workspace: the split-K scratch is a fixed
    array inside libpa (PA_STATIC_WORKSPACE_BYTES), for callers that cannot
    allocate device memory. Calls that overlap on one GPU race on that array."""
    d = _desc(cache)
    _check(load_library().pa_attention_static_workspace(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), int(max_blocks_per_seq),
        _ptr(context_lens), _ptr(query_start_loc), int(num_seqs), int(num_q_tokens), int(num_q_heads),
        int(max_query_len), int(max_context_len), float(scale), C.byref(d), _ptr(out),
        _stream(stream, q, out)))


def pa_attention_cascade_workspace_size(num_seqs, num_q_heads, max_context_len, max_shared_blocks, cache) -> int:
    d = _desc(cache)
    return int(load_library().pa_attention_cascade_workspace_size(int(num_seqs), int(num_q_heads),
                                                                  int(max_context_len), int(max_shared_blocks),
                                                                  C.byref(d)))


def pa_attention_cascade(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, query_start_loc,
                         num_seqs, num_q_heads, max_context_len, shared_blocks, groups, num_groups, max_group_size,
                         max_shared_blocks, scale, cache, out, workspace, workspace_bytes=None, stream=None):
    """Decode attention reading each group's shared prefix blocks once (see include/pa.h)."""
    d = _desc(cache)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None or isinstance(workspace, int) else \
            workspace.numel() * workspace.element_size()
    _check(load_library().pa_attention_cascade(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), int(max_blocks_per_seq), _ptr(context_lens),
        _ptr(query_start_loc), int(num_seqs), int(num_q_heads), int(max_context_len), _ptr(shared_blocks),
        _ptr(groups), int(num_groups), int(max_group_size), int(max_shared_blocks), float(scale), C.byref(d),
        _ptr(out), _ptr(workspace), int(workspace_bytes), _stream(stream, q, out)))


def pa_read_device_flags(clear: bool = True) -> int:
    """OR of PA_FLAG_* raised on the current device since the last clear (synchronises)."""
    v = C.c_uint32(0)
    _check(load_library().pa_read_device_flags(C.byref(v), 1 if clear else 0))
    return int(v.value)


def pa_set_wait_limit_ns(limit_ns: int) -> int:
    """Bound of the kernels' device-side waits from now on; returns the previous one."""
    return int(load_library().pa_set_wait_limit_ns(int(limit_ns)))


def pa_get_debug_status(stream=None) -> int:
    """OR of PA_FLAG_* raised since the last clear, read (and cleared) in the
    order of ``stream`` (default: the current torch stream); waits for that
    stream only."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    elif not isinstance(stream, int):
        stream = stream.cuda_stream
    v = C.c_int32(0)
    _check(load_library().pa_get_debug_status(stream, C.byref(v)))
    return int(v.value)


# --------------------------------------------------------------------------
# block manager
# --------------------------------------------------------------------------

def _i32_buf(n):
    return (C.c_int32 * max(int(n), 1))()


class BlockManager:
    """Host block manager (free list, tables, refcounts, copy-on-write) in libpa.

    Method names follow the ``pa_bm_*`` entry points; results come back as
    Python lists / NumPy arrays of int32.
    """

    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        lib = load_library()
        self._lib = lib
        self.block_size = int(block_size)
        h = C.c_void_p()
        order = None
        if initial_free_order is not None:
            import numpy as np
            self._order = np.ascontiguousarray(initial_free_order, dtype=np.int32)
            if self._order.size != num_blocks:
                raise ValueError("initial_free_order must have num_blocks entries")
            order = self._order.ctypes.data_as(_PI32)
        _check(lib.pa_bm_create(int(num_blocks), int(block_size), order, C.byref(h)))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int, num_tokens: int):
        out = _i32_buf(num_tokens)
        _check(self._lib.pa_bm_add_seq(self._h, int(seq_id), int(num_tokens), out))
        return list(out[:num_tokens])

    def fork(self, parent: int, child: int, num_tokens: int = -1):
        _check(self._lib.pa_bm_fork(self._h, int(parent), int(child), int(num_tokens)))

    def append_tokens(self, seq_id: int, n: int):
        out = _i32_buf(n)
        pair = (C.c_int32 * 2)()
        ncow = C.c_int32(0)
        _check(self._lib.pa_bm_append_tokens(self._h, int(seq_id), int(n), out, pair, C.byref(ncow)))
        return list(out[:n]), ([(pair[0], pair[1])] if ncow.value else [])

    def free_seq(self, seq_id: int):
        _check(self._lib.pa_bm_free_seq(self._h, int(seq_id)))

    def slot_mapping(self, seq_id: int, start: int, n: int):
        out = _i32_buf(n)
        _check(self._lib.pa_bm_slot_mapping(self._h, int(seq_id), int(start), int(n), out))
        return list(out[:n])

    def block_table(self, seq_ids, max_blocks: int):
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        table = np.empty((len(ids), max_blocks), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        _check(self._lib.pa_bm_block_table(self._h, ids.ctypes.data_as(_PI64), len(ids), int(max_blocks),
                                           table.ctypes.data_as(_PI32), lens.ctypes.data_as(_PI32)))
        return table, lens

    def num_free(self) -> int:
        return int(self._lib.pa_bm_num_free(self._h))

    def num_blocks(self) -> int:
        return int(self._lib.pa_bm_num_blocks(self._h))

    def refcount(self, block: int) -> int:
        return int(self._lib.pa_bm_refcount(self._h, int(block)))

    def seq_len(self, seq_id: int) -> int:
        return int(self._lib.pa_bm_seq_len(self._h, int(seq_id)))

    def compact(self):
        """``pa_bm_compact``: remap held blocks to [0, held); returns the (src, dst) moves."""
        import numpy as np
        n = C.c_int32(0)
        status = self._lib.pa_bm_compact(self._h, None, 0, C.byref(n))  # size query; no moves -> done
        if n.value == 0:
            _check(status)
            return []
        pairs = np.empty((n.value, 2), dtype=np.int32)
        _check(self._lib.pa_bm_compact(self._h, pairs.ctypes.data_as(_PI32), n.value, C.byref(n)))
        return [(int(a), int(b)) for a, b in pairs]

    def cascade_groups(self, seq_ids, min_shared_blocks: int = 1):
        """``pa_bm_cascade_groups``: (shared_blocks [n] int32, groups [g, 2] int32) for pa_attention_cascade."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        shared = np.zeros(max(n, 1), dtype=np.int32)
        groups = np.zeros((max(n // 2, 1), 2), dtype=np.int32)
        ng = C.c_int32(0)
        _check(self._lib.pa_bm_cascade_groups(self._h, ids.ctypes.data_as(_PI64), n, int(min_shared_blocks),
                                              shared.ctypes.data_as(_PI32), groups.ctypes.data_as(_PI32),
                                              C.byref(ng)))
        return shared[:n], groups[: ng.value]

    def stats(self, kv_bytes_per_block: float = 0.0) -> dict:
        """``pa_bm_get_stats`` as a dict (monitoring figures of the pool)."""
        st = BlockManagerStats()
        _check(self._lib.pa_bm_get_stats(self._h, float(kv_bytes_per_block), C.byref(st)))
        return st.as_dict()

    def free_list(self):
        n = self.num_blocks()
        out = _i32_buf(n)
        got = self._lib.pa_bm_free_list(self._h, out, n)
        return list(out[:got])
