"""Failure detection on the GPU without a fault: every kernel wait is bounded
by the context's wait limit.  A layer whose weight stream takes far longer
than a tiny limit makes the kernels' waits run out; the call must report
STAPLE_ETIMEOUT through the device error word, and the same context must then
compute the next layer correctly (the kernels let their copies and MMAs finish
and free their tensor memory before returning)."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from tests.helpers import TOL, assert_close
from tests.layer_runner import run_layer

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 4_000_000_000
TINY_LIMIT_NS = 10_000


@pytest.fixture(scope="module")
def stp():
    import token_indexed_sparse_staple_b200 as m
    return m


@pytest.fixture(scope="module")
def ctx(stp):
    c = stp.staple_context_create(0)
    yield c
    stp.staple_context_destroy(c)


def _small_layer_matches_oracle(stp, ctx, T):
    w = syn.Workload("after-timeout", T=T, D=256, F=576, V=4000, layers=1, dtype="bf16",
                     w_std=0.05, e_std=0.05, x_std=1.0, dy_std=1.0, table="device",
                     cache_frac=0.0, group=1, training=False)
    inp = syn.make_layer_inputs(w, with_dy=False)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", training=False)
    x, wg, wu, wd = (inp.f64(k) for k in ("x", "w_gate", "w_up", "w_down"))
    ref = oracle.ffn_forward(x, inp.ids, wg, wu, wd, inp.f64("table"))
    for k in ("z", "y"):
        assert_close(got[k], ref[k], TOL["bf16"], k)


@pytest.mark.parametrize("T,D,F", [(64, 8192, 256), (64, 4096, 512), (384, 32768, 256)])
def test_wait_limit_runs_out_then_context_recovers(stp, ctx, T, D, F):
    """A long d_model makes every gate/up tile stream megabytes of weights
    through one SM before its accumulator is ready: 2 MB per tile in the decode
    kernel's two-launch path (T = 64, d_model 8192: 64 down tiles, more than
    the clusters the device holds at once), 1 MB in its cluster path (d_model
    4096, d_ff 512), 24 MB in the tiled GEMM (T = 384, d_model 32768), tens of
    microseconds at least, so a 10 us limit runs out in the first wait for an
    accumulator."""
    import torch
    V = 100
    g = torch.Generator(device="cuda")
    g.manual_seed(5)

    def rnd(*shape, std=0.02):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    x, wg, wu, wd = rnd(T, D, std=1.0), rnd(F, D), rnd(F, D), rnd(D, F)
    table = rnd(V, F)
    ids = torch.randint(0, V, (T,), generator=g, device="cuda", dtype=torch.int32)
    z = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    emb = stp.make_embed(stp.STAPLE_EMBED_TABLE, table, F, ids, V)
    wsb = stp.staple_workspace_bytes(T, D, F)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    assert stp.staple_get_error(ctx) == 0
    stp.staple_set_wait_limit(ctx, TINY_LIMIT_NS)
    try:
        stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, T, D, F, x, emb, wg, wu, wd, z, y, None, None,
                           ws, wsb)
        err = stp.staple_get_error(ctx)
    finally:
        stp.staple_set_wait_limit(ctx, DEFAULT_LIMIT_NS)
    assert err == stp.STAPLE_ETIMEOUT, stp.staple_status_string(err)
    # the error word was cleared by the read; the context computes again
    ws.zero_()
    stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, T, D, F, x, emb, wg, wu, wd, z, y, None, None, ws,
                       wsb)
    assert stp.staple_get_error(ctx) == 0
    torch.cuda.synchronize()

    def f64(t):
        return t.float().cpu().numpy().astype(np.float64)

    ref = oracle.ffn_forward(f64(x), ids.cpu().numpy(), f64(wg), f64(wu), f64(wd), f64(table))
    for k, got in (("z", z), ("y", y)):
        assert_close(f64(got), ref[k], TOL["bf16"], k)
    _small_layer_matches_oracle(stp, ctx, T)


def test_wait_limit_arguments(stp, ctx):
    with pytest.raises(stp.StapleError) as e:
        stp.staple_set_wait_limit(ctx, 0)
    assert e.value.status == stp.STAPLE_EINVAL
    with pytest.raises(stp.StapleError):
        stp.staple_set_wait_limit(ctx, 61_000_000_000)
    stp.staple_set_wait_limit(ctx, DEFAULT_LIMIT_NS)
