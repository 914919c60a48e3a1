"""The C-ABI library loads and exports every entry point include/staple.h
declares; host-only calls behave without a GPU."""
import os
import re
import subprocess

import pytest

import token_indexed_sparse_staple_b200 as stp
from token_indexed_sparse_staple_b200 import _lib

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def header_functions():
    src = open(os.path.join(ROOT, "include", "staple.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(staple_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from token_indexed_sparse_staple_b200 import build
    build.build()
    return _lib.load()


def test_every_declared_function_is_exported(lib):
    names = header_functions()
    assert len(names) >= 18
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (staple_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)


def test_binding_covers_the_header():
    assert sorted(_lib.SIGNATURES) == header_functions()
    for n in header_functions():
        assert callable(getattr(stp, n)), n


def test_host_only_calls(lib):
    assert stp.staple_abi_version() == 1
    assert stp.staple_status_string(0) == "STAPLE_OK"
    assert "EIDRANGE" in stp.staple_status_string(-2)
    assert stp.staple_status_string(12345) == "STAPLE_UNKNOWN"
    ws = stp.staple_workspace_bytes(16384, 2048, 8192)
    assert ws % 256 == 0 and ws >= 256 * 2 * 8192 * 4
    assert stp.staple_workspace_bytes(-1, 1, 1) == 0


def test_no_device_is_reported_not_faked(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(stp.StapleError) as e:
        stp.staple_context_create(0)
    assert e.value.status == stp.STAPLE_ENODEV


def test_null_arguments_are_rejected_before_any_launch(lib):
    import ctypes as C
    h = C.c_void_p()
    assert lib.staple_context_create(0, None) == stp.STAPLE_EINVAL
    assert lib.staple_table_register(None, None, 0, 1, 1, 1, 0, 1, C.byref(h)) == stp.STAPLE_EINVAL
    assert lib.staple_ffn_fwd(None, 0, 1, 64, 64, None, None, None, None, None, None, None,
                              None, None, None, 0, None) == stp.STAPLE_EINVAL
    assert lib.staple_dedup(None, None, 0, 10, None, None, None, None, None, None) == stp.STAPLE_EINVAL


def test_null_arguments_of_the_later_calls_are_rejected(lib):
    """The calls added after the layer calls validate their arguments before
    touching a device or host buffer: NULL handles and pointers return
    STAPLE_EINVAL (no GPU is needed to check that)."""
    E = stp.STAPLE_EINVAL
    bf = stp.STAPLE_BF16
    assert lib.staple_gather_unique_rows(None, None, None, None, None, 4, None, None, None, None,
                                         None, None) == E
    assert lib.staple_gather_unique_rows_bulk(None, None, None, None, None, 4, None, None, None,
                                              None, None, None, None, 256, 0, None) == E
    assert lib.staple_cache_refresh(None, None, None, None, None, None, None) == E
    assert lib.staple_embed_bwd(None, bf, 4, 64, 64, None, None, None, None, None, None, None,
                                None, None, None, None, 0, None) == E
    assert lib.staple_ffn_bwd(None, bf, 4, 64, 64, None, None, None, None, None, None, None, None,
                              None, None, None, 0, None) == E
    assert lib.staple_embed_grad(None, bf, 4, 64, 64, None, 128, None, None, None, None, None,
                                 None, 0, None) == E
    assert lib.staple_embed_grad_to_host(None, 64, 4, None, None, None, None, None, None,
                                         None) == E
    assert lib.staple_embed_grad_static(bf, 4, 64, None, 64, None, None, None, None, None) == E
    hp = stp.staple_adamw(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    import ctypes as C
    assert lib.staple_adamw_rows(None, 4, stp.STAPLE_F32, 4, None, 1, None, 4, None, None, 4,
                                 C.byref(hp), 1) == E


def test_static_scratch_refuses_sizes_beyond_it(lib):
    """staple_embed_grad_static checks its sizes before anything else, so the
    refusal needs no GPU.  All pointers are NULL: without the size guard the
    call would stop at the NULL check with STAPLE_EINVAL instead, so only the
    guard can give STAPLE_EUNSUPPORTED (and no launch can follow)."""
    U = stp.STAPLE_EUNSUPPORTED
    bf = stp.STAPLE_BF16

    def call(T, F):
        return lib.staple_embed_grad_static(bf, T, F, None, F, None, None, None, None, None)

    # 2 * ceil(T / 64) * F * 4 bytes against the 16 MiB array
    assert call(16385, 8192) == U
    assert call(16448, 8192) == U
    assert call(8193, 16384) == U
    # longer than one dedup (32768 tokens), though small F fits the array
    assert call(32769, 8) == U
    # at the limits the size passes and the NULL pointers are what is refused
    assert call(16384, 8192) == stp.STAPLE_EINVAL
    assert call(32768, 8) == stp.STAPLE_EINVAL
