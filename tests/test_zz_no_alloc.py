"""The allocation-free table-gradient entry point (staple_embed_grad_static)
against the workspace one (staple_embed_bwd).

It serves callers that cannot allocate device memory (their device memory is
owned by another allocator, or they must not call cudaMalloc because it
synchronizes the device, or they only hold the buffers a host hands them): its
scratch is built into the library.  Two calls in a row must both reproduce the
dE of staple_embed_bwd for the same dh, and a size beyond the built-in scratch
must be refused (STAPLE_EUNSUPPORTED) before anything runs.  This file is collected last so that a
run stopping at the first failure has already run every other test."""
import ctypes as C

import numpy as np
import pytest

import synthetic as syn
from tests.helpers import TOL, assert_close

pytestmark = pytest.mark.gpu


def _case(stp, ctx, T, D, F, V, seed):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)

    def rnd(*shape, std=1.0):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    ids = torch.from_numpy(syn.zipf_ids(T, V, 1.1, seed=seed)).cuda()
    i32 = dict(dtype=torch.int32, device="cuda")
    unique, inverse, sorted_pos = (torch.empty(T, **i32) for _ in range(3))
    seg, U = torch.empty(T + 1, **i32), torch.empty(1, **i32)
    stp.staple_dedup(ctx, ids, T, V, unique, inverse, seg, sorted_pos, U)
    dy, gs, hs, wd = rnd(T, D), rnd(T, F), rnd(T, F), rnd(D, F, std=0.05)
    dgh = torch.empty((T, 2 * F), dtype=torch.bfloat16, device="cuda")
    dE_ref = torch.full((T, F), float("nan"), dtype=torch.float32, device="cuda")
    wsb = stp.staple_workspace_bytes(T, D, F)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")   # zero-filled once, as documented
    stp.staple_embed_bwd(ctx, stp.STAPLE_BF16, T, D, F, dy, gs, hs, wd, sorted_pos, inverse, seg,
                         U, dgh, dE_ref, ws, wsb)
    assert stp.staple_get_error(ctx) == 0
    u = int(U.item())
    ref = dE_ref[:u].double().cpu().numpy()
    dh_addr = dgh.data_ptr() + F * 2          # the dh half of dgh, row pitch 2F
    for call in range(2):                     # two calls in a row share the static scratch
        dE = torch.full((T, F), float("nan"), dtype=torch.float32, device="cuda")
        stp.staple_embed_grad_static(stp.STAPLE_BF16, T, F, dh_addr, 2 * F, sorted_pos, inverse,
                                     seg, dE)
        torch.cuda.synchronize()
        got = dE[:u].double().cpu().numpy()
        assert_close(got, ref, TOL["bf16"], f"dE call {call}")
        assert np.isnan(dE[u:].cpu().numpy()).all()   # rows >= U untouched


@pytest.fixture(scope="module")
def stp():
    import token_indexed_sparse_staple_b200 as m
    return m


@pytest.fixture(scope="module")
def ctx(stp):
    c = stp.staple_context_create(0)
    yield c
    stp.staple_context_destroy(c)


def test_static_scratch_matches_workspace_entry(stp, ctx):
    _case(stp, ctx, T=3000, D=128, F=512, V=5000, seed=11)


def test_static_scratch_at_its_largest_size(stp, ctx):
    # 2 * ceil(16384 / 64) * 8192 * 4 bytes = 16 MiB: exactly the built-in scratch
    _case(stp, ctx, T=16384, D=64, F=8192, V=100352, seed=12)


def test_static_scratch_refuses_larger_sizes(stp, ctx):
    """An oversize request is refused with STAPLE_EUNSUPPORTED before any
    pointer is looked at or anything is launched (the NULL pointers would give
    STAPLE_EINVAL otherwise), and the next call still works."""
    lib = stp.lib()
    st = lib.staple_embed_grad_static(stp.STAPLE_BF16, 16448, 8192, None, 8192, None, None, None,
                                      None, None)
    assert st == stp.STAPLE_EUNSUPPORTED
    _case(stp, ctx, T=700, D=64, F=256, V=3000, seed=13)
