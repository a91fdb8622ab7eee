"""ctypes binding of libspa (include/spa.h): argument marshalling only.

Every function keeps the C name and argument order.  Tensor arguments may be
torch tensors (their ``data_ptr()`` is passed), plain integers (raw device
addresses) or None (NULL).  ``stream`` may be a ``torch.cuda.Stream``, a raw
``cudaStream_t`` integer, or None for torch's current stream.  A non-zero
status raises :class:`SpaError` carrying ``spa_last_error()``.

The library must have been built (``python -m head_partitioned_sparse_b200.build``);
there is no fallback: if ``libspa.so`` is missing or cannot be loaded, this
module raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspa.so")

SPA_OK = 0
SPA_ERR_INVALID_ARG = -1
SPA_ERR_UNSUPPORTED = -2
SPA_ERR_WORKSPACE = -3
SPA_ERR_CUDA = -4
SPA_ERR_DEVICE_TIMEOUT = -5
SPA_ERR_DEVICE_RANGE = -6
SPA_BF16 = 0
SPA_F32 = 1

SPA_K_INDEX_APPEND, SPA_K_SELECT, SPA_K_ATTEND, SPA_K_COMBINE, SPA_K_KV_APPEND, SPA_K_PREFILL, SPA_K_CP_SELECT = range(7)
SPA_K_COUNT = 7
SPA_CP_STATS, SPA_CP_MASS, SPA_CP_ROUND2, SPA_CP_ROUND3, SPA_CP_ATTEND = range(5)
SPA_CP_NBUF = 6


class SpaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"spa status {status}: {msg}")
        self.status = status


class spa_config(ctypes.Structure):
    _fields_ = [
        ("max_batch", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("idx_dim", ctypes.c_int),
        ("kv_dtype", ctypes.c_int),
        ("max_ctx", ctypes.c_int64),
        ("rope_theta", ctypes.c_double),
        ("idx_scale", ctypes.c_float),
        ("split_rows", ctypes.c_int),
        ("P_q", ctypes.c_void_p),
        ("P_k", ctypes.c_void_p),
    ]


class spa_cp_args(ctypes.Structure):
    _fields_ = [
        ("q_pre", ctypes.c_void_p),
        ("k_cache", ctypes.c_void_p),
        ("v_cache", ctypes.c_void_p),
        ("idx_cache", ctypes.c_void_p),
        ("head_mask", ctypes.POINTER(ctypes.c_uint8)),
        ("seq_lens", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("p", ctypes.c_float),
        ("n_sink", ctypes.c_int),
        ("window", ctypes.c_int),
        ("n_ranks", ctypes.c_int),
        ("rank", ctypes.c_int),
        ("pos0", ctypes.c_int64),
        ("max_seq_len", ctypes.c_int64),
        ("stats", ctypes.c_void_p),
        ("hist1", ctypes.c_void_p),
        ("hist2", ctypes.c_void_p),
        ("hist3", ctypes.c_void_p),
        ("out_all", ctypes.c_void_p),
        ("lse_all", ctypes.c_void_p),
        ("sel_count_opt", ctypes.c_void_p),
        ("list_opt", ctypes.c_void_p),
    ]


_vp, _i, _i64, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
_SIGS = {
    "spa_create": (_i, [ctypes.POINTER(_vp), ctypes.POINTER(spa_config)]),
    "spa_destroy": (_i, [_vp]),
    "spa_workspace_size": (_i, [ctypes.POINTER(spa_config), ctypes.POINTER(ctypes.c_size_t)]),
    "spa_last_error": (ctypes.c_char_p, []),
    "spa_index_append": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp]),
    "spa_select": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp, _vp]),
    "spa_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp, _vp]),
    "spa_select_topk": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i64, _i64, _i, _i, _vp, _vp, _vp]),
    "spa_decode_topk": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i64, _i64, _i, _i, _vp, _vp, _vp]),
    "spa_select_blocks": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp, _vp]),
    "spa_decode_blocks": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp, _vp]),
    "spa_kv_append_compact": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "spa_index_append_compact": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp, _vp]),
    "spa_select_compact": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp, _vp]),
    "spa_decode_compact": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp, _vp]),
    "spa_head_ranks_workspace_size": (_i, [_i, _i, ctypes.POINTER(ctypes.c_size_t)]),
    "spa_head_effective_ranks": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp]),
    "spa_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    "spa_select_compact_sel": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i64, _i, _f, _i64, _i, _i, _vp, _vp, _vp]),
    "spa_decode_compact_sel": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i64, _i, _f, _i64, _i, _i,
                                    _vp, _vp, _vp]),
    "spa_cp_exchange_sizes": (_i, [_vp, _i, _i, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_size_t)]),
    "spa_cp_phase": (_i, [_vp, _i, ctypes.POINTER(spa_cp_args), _vp]),
    "spa_cp_combine": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp]),
    "spa_device_status": (_i, [_vp, _vp]),
    "spa_debug_drop_publish": (_i, [_vp, _i]),
    "spa_set_profiling": (_i, [_vp, ctypes.c_uint]),
    "spa_profile_read": (_i, [_vp, _i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
    "spa_kernel_name": (ctypes.c_char_p, [_i]),
    "spa_launch_count": (_i, [_vp, ctypes.POINTER(ctypes.c_int64)]),
    "spa_select_noalloc": (_i, [_vp, _i, _i, _i, _f, _i64, _vp, _vp, _vp, _vp, _i, _i64, _f, _i, _i, _vp, _vp,
                                _vp]),
}
EXPORTED = tuple(_SIGS)

_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libspa.so (once) and declare every exported signature."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m head_partitioned_sparse_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    raise TypeError(f"expected a tensor, an int address or None, got {type(x)!r}")


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _host_u8(mask) -> ctypes.Array:
    vals = [int(v) for v in (mask.tolist() if hasattr(mask, "tolist") else mask)]
    return (ctypes.c_uint8 * len(vals))(*vals)


def _check(status: int) -> None:
    if status != SPA_OK:
        raise SpaError(status, load().spa_last_error().decode())


def spa_last_error() -> str:
    return load().spa_last_error().decode()


def spa_workspace_size(cfg: spa_config) -> int:
    n = ctypes.c_size_t(0)
    _check(load().spa_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def spa_create(cfg: spa_config) -> int:
    h = ctypes.c_void_p(None)
    _check(load().spa_create(ctypes.byref(h), ctypes.byref(cfg)))
    return h.value


def spa_destroy(h) -> None:
    _check(load().spa_destroy(h))


def spa_index_append(h, k_pre, start_pos, B: int, T: int, idx_cache, stream=None) -> None:
    _check(load().spa_index_append(h, _ptr(k_pre), _ptr(start_pos), B, T, _ptr(idx_cache), _stream(stream)))


def spa_select(h, q_pre, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int, p: float, n_sink: int,
               window: int, sel_idx, sel_count, stream=None) -> None:
    _check(load().spa_select(h, _ptr(q_pre), _ptr(idx_cache), _host_u8(head_mask), _ptr(seq_lens), B,
                             max_seq_len, p, n_sink, window, _ptr(sel_idx), _ptr(sel_count), _stream(stream)))


def spa_decode(h, q_pre, k_cache, v_cache, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int, p: float,
               n_sink: int, window: int, out, sel_count_opt=None, stream=None) -> None:
    _check(load().spa_decode(h, _ptr(q_pre), _ptr(k_cache), _ptr(v_cache), _ptr(idx_cache), _host_u8(head_mask),
                             _ptr(seq_lens), B, max_seq_len, p, n_sink, window, _ptr(out), _ptr(sel_count_opt),
                             _stream(stream)))


def spa_select_topk(h, q_pre, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int, k: int, n_sink: int,
                    window: int, sel_idx, sel_count, stream=None) -> None:
    _check(load().spa_select_topk(h, _ptr(q_pre), _ptr(idx_cache), _host_u8(head_mask), _ptr(seq_lens), B,
                                  max_seq_len, int(k), n_sink, window, _ptr(sel_idx), _ptr(sel_count),
                                  _stream(stream)))


def spa_decode_topk(h, q_pre, k_cache, v_cache, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int, k: int,
                    n_sink: int, window: int, out, sel_count_opt=None, stream=None) -> None:
    _check(load().spa_decode_topk(h, _ptr(q_pre), _ptr(k_cache), _ptr(v_cache), _ptr(idx_cache),
                                  _host_u8(head_mask), _ptr(seq_lens), B, max_seq_len, int(k), n_sink, window,
                                  _ptr(out), _ptr(sel_count_opt), _stream(stream)))


def spa_select_blocks(h, q_pre, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int, p: float, n_sink: int,
                      window: int, sel_idx, sel_count, stream=None) -> None:
    _check(load().spa_select_blocks(h, _ptr(q_pre), _ptr(idx_cache), _host_u8(head_mask), _ptr(seq_lens), B,
                                    max_seq_len, p, n_sink, window, _ptr(sel_idx), _ptr(sel_count),
                                    _stream(stream)))


def spa_decode_blocks(h, q_pre, k_cache, v_cache, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int,
                      p: float, n_sink: int, window: int, out, sel_count_opt=None, stream=None) -> None:
    _check(load().spa_decode_blocks(h, _ptr(q_pre), _ptr(k_cache), _ptr(v_cache), _ptr(idx_cache),
                                    _host_u8(head_mask), _ptr(seq_lens), B, max_seq_len, p, n_sink, window,
                                    _ptr(out), _ptr(sel_count_opt), _stream(stream)))


def spa_kv_append_compact(h, k_new, v_new, start_pos, B: int, T: int, head_mask, n_sink: int, window: int,
                          k_ret, v_ret, k_ring, v_ring, stream=None) -> None:
    _check(load().spa_kv_append_compact(h, _ptr(k_new), _ptr(v_new), _ptr(start_pos), B, T, _host_u8(head_mask),
                                        n_sink, window, _ptr(k_ret), _ptr(v_ret), _ptr(k_ring), _ptr(v_ring),
                                        _stream(stream)))


def spa_index_append_compact(h, k_pre, start_pos, B: int, T: int, head_mask, idx_ret, stream=None) -> None:
    _check(load().spa_index_append_compact(h, _ptr(k_pre), _ptr(start_pos), B, T, _host_u8(head_mask),
                                           _ptr(idx_ret), _stream(stream)))


def spa_select_compact(h, q_pre, idx_ret, head_mask, seq_lens, B: int, max_seq_len: int, p: float, n_sink: int,
                       window: int, sel_idx, sel_count, stream=None) -> None:
    _check(load().spa_select_compact(h, _ptr(q_pre), _ptr(idx_ret), _host_u8(head_mask), _ptr(seq_lens), B,
                                     max_seq_len, p, n_sink, window, _ptr(sel_idx), _ptr(sel_count),
                                     _stream(stream)))


def spa_decode_compact(h, q_pre, k_ret, v_ret, k_ring, v_ring, idx_ret, head_mask, seq_lens, B: int,
                       max_seq_len: int, p: float, n_sink: int, window: int, out, sel_count_opt=None,
                       stream=None) -> None:
    _check(load().spa_decode_compact(h, _ptr(q_pre), _ptr(k_ret), _ptr(v_ret), _ptr(k_ring), _ptr(v_ring),
                                     _ptr(idx_ret), _host_u8(head_mask), _ptr(seq_lens), B, max_seq_len, p, n_sink,
                                     window, _ptr(out), _ptr(sel_count_opt), _stream(stream)))


def spa_head_ranks_workspace_size(n_q_heads: int, n_kv_heads: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().spa_head_ranks_workspace_size(n_q_heads, n_kv_heads, ctypes.byref(n)))
    return n.value


def spa_head_effective_ranks(W_Q, W_K, n_q_heads: int, n_kv_heads: int, d_model: int, n_retrieval: int,
                             workspace, workspace_bytes: int, er_q, er_kv, head_mask, sigma_opt=None,
                             stream=None) -> None:
    _check(load().spa_head_effective_ranks(_ptr(W_Q), _ptr(W_K), n_q_heads, n_kv_heads, d_model, n_retrieval,
                                           _ptr(workspace), workspace_bytes, _ptr(er_q), _ptr(er_kv),
                                           _ptr(head_mask), _ptr(sigma_opt), _stream(stream)))


def spa_prefill(h, q_chunk, k_cache, v_cache, head_mask, start_pos, B: int, T: int, n_sink: int, window: int, out,
                stream=None) -> None:
    _check(load().spa_prefill(h, _ptr(q_chunk), _ptr(k_cache), _ptr(v_cache), _host_u8(head_mask), _ptr(start_pos),
                              B, T, n_sink, window, _ptr(out), _stream(stream)))


def spa_debug_drop_publish(h, enable: bool) -> None:
    _check(load().spa_debug_drop_publish(h, 1 if enable else 0))


SPA_SELECT_TOP_P, SPA_SELECT_TOP_K, SPA_SELECT_BLOCKS = 0, 1, 2


def spa_select_compact_sel(h, q_pre, idx_ret, head_mask, seq_lens, B: int, max_seq_len: int, selector: int,
                           p: float, k: int, n_sink: int, window: int, sel_idx, sel_count, stream=None) -> None:
    _check(load().spa_select_compact_sel(h, _ptr(q_pre), _ptr(idx_ret), _host_u8(head_mask), _ptr(seq_lens), B,
                                         max_seq_len, selector, p, int(k), n_sink, window, _ptr(sel_idx),
                                         _ptr(sel_count), _stream(stream)))


def spa_decode_compact_sel(h, q_pre, k_ret, v_ret, k_ring, v_ring, idx_ret, head_mask, seq_lens, B: int,
                           max_seq_len: int, selector: int, p: float, k: int, n_sink: int, window: int, out,
                           sel_count_opt=None, stream=None) -> None:
    _check(load().spa_decode_compact_sel(h, _ptr(q_pre), _ptr(k_ret), _ptr(v_ret), _ptr(k_ring), _ptr(v_ring),
                                         _ptr(idx_ret), _host_u8(head_mask), _ptr(seq_lens), B, max_seq_len, selector,
                                         p, int(k), n_sink, window, _ptr(out), _ptr(sel_count_opt), _stream(stream)))


def spa_cp_exchange_sizes(h, B: int, n_ranks: int, head_mask) -> Tuple[int, ...]:
    """Byte sizes of the exchange buffers (stats, hist1, hist2, hist3, out_all, lse_all)
    for the host head mask ``head_mask`` [Hkv] (the statistics and histograms hold its
    retrieval slices only)."""
    arr = (ctypes.c_size_t * SPA_CP_NBUF)()
    mask = _host_u8(head_mask)
    _check(load().spa_cp_exchange_sizes(h, B, n_ranks, ctypes.cast(mask, ctypes.POINTER(ctypes.c_uint8)), arr))
    return tuple(int(v) for v in arr)


def make_cp_args(*, q_pre, k_cache, v_cache, idx_cache, head_mask, seq_lens, B: int, p: float, n_sink: int,
                 window: int, n_ranks: int, rank: int, pos0: int, max_seq_len: int, stats, hist1, hist2, hist3,
                 out_all, lse_all, sel_count_opt=None, list_opt=None) -> spa_cp_args:
    """The argument block of spa_cp_phase (it keeps the host head mask alive)."""
    mask = _host_u8(head_mask)
    a = spa_cp_args(_ptr(q_pre), _ptr(k_cache), _ptr(v_cache), _ptr(idx_cache),
                    ctypes.cast(mask, ctypes.POINTER(ctypes.c_uint8)), _ptr(seq_lens), B, p, n_sink, window, n_ranks,
                    rank, int(pos0), int(max_seq_len), _ptr(stats), _ptr(hist1), _ptr(hist2), _ptr(hist3),
                    _ptr(out_all), _ptr(lse_all), _ptr(sel_count_opt), _ptr(list_opt))
    a._mask = mask
    return a


def spa_cp_phase(h, phase: int, args: spa_cp_args, stream=None) -> None:
    _check(load().spa_cp_phase(h, phase, ctypes.byref(args), _stream(stream)))


def spa_cp_combine(h, out_all, lse_all, n_ranks: int, B: int, out, stream=None) -> None:
    _check(load().spa_cp_combine(h, _ptr(out_all), _ptr(lse_all), n_ranks, B, _ptr(out), _stream(stream)))


def spa_device_status(h, stream=None) -> None:
    _check(load().spa_device_status(h, _stream(stream)))


def spa_set_profiling(h, kernel_mask: int) -> None:
    """kernel_mask: bit (1 << SPA_K_...) per kernel to time with CUDA events; 0 = off."""
    _check(load().spa_set_profiling(h, int(kernel_mask)))


def spa_profile_read(h, kernel_id: int) -> Tuple[float, int]:
    ms, n = ctypes.c_double(0.0), ctypes.c_int64(0)
    _check(load().spa_profile_read(h, kernel_id, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def spa_kernel_name(kernel_id: int) -> str:
    return load().spa_kernel_name(kernel_id).decode()


def spa_launch_count(h) -> int:
    n = ctypes.c_int64(0)
    _check(load().spa_launch_count(h, ctypes.byref(n)))
    return n.value


def make_config(*, max_batch: int, n_q_heads: int, n_kv_heads: int, max_ctx: int, kv_dtype: int,
                P_q, P_k, rope_theta: float = 500000.0, idx_scale: float = 0.25, split_rows: int = 0,
                head_dim: int = 128, idx_dim: int = 16) -> spa_config:
    """Fill a spa_config; P_q / P_k are device float32 tensors (or addresses)."""
    return spa_config(max_batch=max_batch, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, head_dim=head_dim,
                      idx_dim=idx_dim, kv_dtype=kv_dtype, max_ctx=max_ctx, rope_theta=rope_theta,
                      idx_scale=idx_scale, split_rows=split_rows, P_q=_ptr(P_q), P_k=_ptr(P_k))


def spa_select_noalloc(P_q, n_q_heads: int, n_kv_heads: int, kv_dtype: int, idx_scale: float, max_ctx: int,
                       q_pre, idx_cache, head_mask, seq_lens, B: int, max_seq_len: int, p: float, n_sink: int,
                       window: int, sel_idx, sel_count, stream=None) -> None:
    """spa_select with no handle and no allocation (static scratch; see include/spa.h)."""
    _check(load().spa_select_noalloc(_ptr(P_q), n_q_heads, n_kv_heads, kv_dtype, idx_scale, max_ctx, _ptr(q_pre),
                                     _ptr(idx_cache), _host_u8(head_mask), _ptr(seq_lens), B, max_seq_len, p,
                                     n_sink, window, _ptr(sel_idx), _ptr(sel_count), _stream(stream)))
