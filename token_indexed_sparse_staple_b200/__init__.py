"""Python binding of libstaple (include/staple.h): the STAPLE embedding-
augmented SwiGLU FFN layer on B200 (sm_100a).

Each function has the name of the C entry point it calls and only marshals
arguments: tensors become device (or host) addresses, streams become
cudaStream_t handles (default: torch's current stream), and a non-zero status
raises StapleError.  There is no fallback: the library must be built
(`python -m token_indexed_sparse_staple_b200.build`) and a B200 must be present
for any compute call.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import _lib
from ._lib import staple_adamw, staple_embed

STAPLE_OK = 0
STAPLE_EINVAL, STAPLE_EIDRANGE, STAPLE_ECUDA, STAPLE_ENOMEM = -1, -2, -3, -4
STAPLE_ETIMEOUT, STAPLE_EUNSUPPORTED, STAPLE_ENODEV = -5, -6, -7
STAPLE_BF16, STAPLE_F32 = 0, 1
STAPLE_EMBED_NONE, STAPLE_EMBED_TABLE, STAPLE_EMBED_ROWS = 0, 1, 2
STAPLE_TABLE_DEVICE, STAPLE_TABLE_HOST_PINNED, STAPLE_TABLE_HOST_REGISTER = 1, 2, 4
STAPLE_EMBED_REPLACE_UP = 1

__all__ = [n for n in _lib.SIGNATURES] + [
    "StapleError", "staple_embed", "staple_adamw", "make_embed", "lib",
]


class StapleError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().staple_status_string(status).decode()
        super().__init__(f"{where}: {msg} ({status})")


def lib():
    return _lib.load()


def _p(x) -> int | None:
    """Address of a tensor / array / raw int (None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _ok(status: int, where: str) -> None:
    if status != STAPLE_OK:
        raise StapleError(status, where)


def make_embed(mode: int, base=None, row_pitch: int = 0, index=None, n_rows: int = 0,
               flags: int = 0) -> staple_embed:
    """flags = STAPLE_EMBED_REPLACE_UP: the STEM layer (the row replaces the
    up-projection)."""
    return staple_embed(mode, flags, _p(base), row_pitch, _p(index), n_rows)


# ------------------------------------------------------------------ context

def staple_abi_version() -> int:
    return lib().staple_abi_version()


def staple_status_string(s: int) -> str:
    return lib().staple_status_string(s).decode()


def staple_context_create(device: int = 0) -> int:
    h = C.c_void_p()
    _ok(lib().staple_context_create(device, C.byref(h)), "staple_context_create")
    return h.value


def staple_context_destroy(ctx: int) -> None:
    _ok(lib().staple_context_destroy(ctx), "staple_context_destroy")


def staple_get_error(ctx: int, stream=None) -> int:
    e = C.c_int32()
    _ok(lib().staple_get_error(ctx, _stream(stream), C.byref(e)), "staple_get_error")
    return e.value


def staple_set_wait_limit(ctx: int, limit_ns: int) -> None:
    """Bound of every kernel wait of later launches, in ns (see include/staple.h)."""
    _ok(lib().staple_set_wait_limit(ctx, int(limit_ns)), "staple_set_wait_limit")


def staple_set_sm_reserve(ctx: int, sms: int) -> None:
    """SMs the tiled GEMMs leave free for work on other streams (see include/staple.h)."""
    _ok(lib().staple_set_sm_reserve(ctx, int(sms)), "staple_set_sm_reserve")


def staple_trace_enable(ctx: int, enable: bool = True) -> None:
    _ok(lib().staple_trace_enable(ctx, int(bool(enable))), "staple_trace_enable")


def staple_trace_read(ctx: int, capacity: int = 1 << 16) -> list[tuple[str, float]]:
    """[(kernel name, device ms)] for the launches since the last read."""
    recs = (_lib.staple_trace_record * capacity)()
    n = C.c_int32()
    _ok(lib().staple_trace_read(ctx, recs, capacity, C.byref(n)), "staple_trace_read")
    return [(recs[i].kernel.decode(), float(recs[i].ms)) for i in range(n.value)]


# ------------------------------------------------------------------- tables

def staple_table_register(ctx: int, base, nbytes: int, V: int, F: int, groups: int, dtype: int,
                          flags: int) -> int:
    h = C.c_void_p()
    _ok(lib().staple_table_register(ctx, _p(base), nbytes, V, F, groups, dtype, flags,
                                    C.byref(h)), "staple_table_register")
    return h.value


def staple_table_unregister(table: int) -> None:
    _ok(lib().staple_table_unregister(table), "staple_table_unregister")


# -------------------------------------------------------------------- cache

def staple_cache_build(ctx: int, table: int, freq: np.ndarray, frac: float, stream=None) -> int:
    freq = np.ascontiguousarray(freq, dtype=np.int64)
    h = C.c_void_p()
    _ok(lib().staple_cache_build(ctx, table, freq.ctypes.data, float(frac), _stream(stream),
                                 C.byref(h)), "staple_cache_build")
    return h.value


def staple_cache_info(cache: int) -> tuple[int, int]:
    k, cap = C.c_int32(), C.c_int32()
    _ok(lib().staple_cache_info(cache, C.byref(k), C.byref(cap)), "staple_cache_info")
    return k.value, cap.value


def staple_cache_hot_ids(cache: int) -> np.ndarray:
    K, _ = staple_cache_info(cache)
    out = np.zeros(K, dtype=np.int32)
    _ok(lib().staple_cache_hot_ids(cache, out.ctypes.data if K else None), "staple_cache_hot_ids")
    return out


def staple_cache_rows(cache: int) -> int:
    p = C.c_void_p()
    _ok(lib().staple_cache_rows(cache, C.byref(p)), "staple_cache_rows")
    return p.value


def staple_cache_free(cache: int) -> None:
    _ok(lib().staple_cache_free(cache), "staple_cache_free")


def staple_workspace_bytes(T: int, D: int, F: int, flags: int = 0) -> int:
    return int(lib().staple_workspace_bytes(T, D, F, flags))


# ---------------------------------------------------------------- retrieval

def staple_dedup(ctx, ids, T, V, unique, inverse, seg_off, sorted_pos, U_dev, stream=None):
    _ok(lib().staple_dedup(ctx, _p(ids), T, V, _p(unique), _p(inverse), _p(seg_off),
                           _p(sorted_pos), _p(U_dev), _stream(stream)), "staple_dedup")


def staple_gather_unique_rows(ctx, cache, table, unique, U_dev, T, slot, miss_list, miss_count,
                              rows, stream=None, side=None):
    st = _stream(stream)
    _ok(lib().staple_gather_unique_rows(ctx, cache, table, _p(unique), _p(U_dev), T, _p(slot),
                                        _p(miss_list), _p(miss_count), _p(rows), st,
                                        st if side is None else _stream(side)),
        "staple_gather_unique_rows")


def staple_gather_rows(ctx, cache, table, ids, T, unique, inverse, seg_off, sorted_pos, U_dev,
                       slot, miss_list, miss_count, rows, stream=None, side=None):
    st = _stream(stream)
    _ok(lib().staple_gather_rows(ctx, cache, table, _p(ids), T, _p(unique), _p(inverse),
                                 _p(seg_off), _p(sorted_pos), _p(U_dev), _p(slot), _p(miss_list),
                                 _p(miss_count), _p(rows), st,
                                 st if side is None else _stream(side)), "staple_gather_rows")


# ---------------------------------------------------------------------- FFN

def staple_ffn_fwd(ctx, dtype, T, D, F, x, embed, w_gate, w_up, w_down, z, y, g_save=None,
                   h_save=None, workspace=None, workspace_bytes=0, stream=None):
    e = C.byref(embed) if embed is not None else None
    _ok(lib().staple_ffn_fwd(ctx, dtype, T, D, F, _p(x), e, _p(w_gate), _p(w_up), _p(w_down),
                             _p(z), _p(y), _p(g_save), _p(h_save), _p(workspace),
                             workspace_bytes, _stream(stream)), "staple_ffn_fwd")


def staple_embed_bwd(ctx, dtype, T, D, F, dy, g_save, h_save, w_down, sorted_pos, inverse,
                     seg_off, U_dev, dgh, dE, workspace=None, workspace_bytes=0, stream=None):
    _ok(lib().staple_embed_bwd(ctx, dtype, T, D, F, _p(dy), _p(g_save), _p(h_save), _p(w_down),
                               _p(sorted_pos), _p(inverse), _p(seg_off), _p(U_dev), _p(dgh),
                               _p(dE), _p(workspace), workspace_bytes, _stream(stream)),
        "staple_embed_bwd")


def staple_embed_grad(ctx, dtype, T, D, F, dh, ld, sorted_pos, inverse, seg_off, U_dev, dE,
                      workspace, workspace_bytes, stream=None):
    """The table-gradient reduction alone (see include/staple.h)."""
    _ok(lib().staple_embed_grad(ctx, dtype, T, D, F, _p(dh), ld, _p(sorted_pos), _p(inverse),
                                _p(seg_off), _p(U_dev), _p(dE), _p(workspace), workspace_bytes,
                                _stream(stream)), "staple_embed_grad")


def staple_embed_grad_to_host(ctx, F, capacity, dE, unique, U_dev, host_dE, host_unique, host_U,
                              stream=None):
    """Rows [0, U) of dE and the U ids to page-locked, mapped host buffers
    (U read on the device; see include/staple.h)."""
    _ok(lib().staple_embed_grad_to_host(ctx, F, capacity, _p(dE), _p(unique), _p(U_dev),
                                        _p(host_dE), _p(host_unique), _p(host_U),
                                        _stream(stream)), "staple_embed_grad_to_host")


def staple_ffn_bwd(ctx, dtype, T, D, F, dy, x, z, dgh, w_gate, w_up, dx, dw_gate, dw_up, dw_down,
                   workspace=None, workspace_bytes=0, stream=None):
    _ok(lib().staple_ffn_bwd(ctx, dtype, T, D, F, _p(dy), _p(x), _p(z), _p(dgh), _p(w_gate),
                             _p(w_up), _p(dx), _p(dw_gate), _p(dw_up), _p(dw_down),
                             _p(workspace), workspace_bytes, _stream(stream)), "staple_ffn_bwd")


def staple_embed_grad_static(dtype, T, F, dh, ld, sorted_pos, inverse, seg_off, dE, stream=None):
    """Table gradient from dh with the library's built-in scratch: no device
    allocation by the caller or the library (see include/staple.h)."""
    _ok(lib().staple_embed_grad_static(dtype, T, F, _p(dh), ld, _p(sorted_pos), _p(inverse),
                                       _p(seg_off), _p(dE), _stream(stream)),
        "staple_embed_grad_static")


def staple_cache_refresh(ctx, cache, table, unique, slot, U_dev, stream=None):
    """Re-read the cached copies of the listed distinct ids from the table
    (after a host-side update; see include/staple.h)."""
    _ok(lib().staple_cache_refresh(ctx, cache, table, _p(unique), _p(slot), _p(U_dev),
                                   _stream(stream)), "staple_cache_refresh")


def staple_adamw_rows(table, table_pitch, dtype, F, ids, U, grad, grad_pitch, m, v, moment_pitch,
                      lr, beta1, beta2, eps, weight_decay, step, threads=0):
    """Host AdamW on the U table rows listed in ids (all host buffers: numpy
    arrays, pinned tensors or raw addresses; see include/staple.h)."""
    hp = staple_adamw(lr, beta1, beta2, eps, weight_decay, step)
    _ok(lib().staple_adamw_rows(_p(table), table_pitch, dtype, F, _p(ids), U, _p(grad), grad_pitch,
                                _p(m), _p(v), moment_pitch, C.byref(hp), threads),
        "staple_adamw_rows")


def staple_gather_unique_rows_bulk(ctx, cache, table, unique, U_dev, T, slot, miss_list,
                                   miss_count, rows, staging_host, staging_dev, list_host,
                                   chunk_rows=256, threads=0, stream=None):
    """Rows of the batch's distinct ids with the misses packed on the host and
    copied in bulk (the prefill path; see include/staple.h).  Blocks the
    calling thread until the probe is done and the rows are packed."""
    _ok(lib().staple_gather_unique_rows_bulk(ctx, cache, table, _p(unique), _p(U_dev), T, _p(slot),
                                             _p(miss_list), _p(miss_count), _p(rows),
                                             _p(staging_host), _p(staging_dev), _p(list_host),
                                             chunk_rows, threads, _stream(stream)),
        "staple_gather_unique_rows_bulk")
