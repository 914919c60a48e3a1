"""GPU parity of the STAPLE FFN layer (forward and backward) against the
oracle, at sizes the oracle finishes in seconds that span several tiles and
ragged tails, plus the exact identities of the method (E = 0 is the dense
FFN; gathered rows and direct table rows give the same result)."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from tests.helpers import TOL, assert_close
from tests.layer_runner import run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def stp():
    import token_indexed_sparse_staple_b200 as m
    return m


@pytest.fixture(scope="module")
def ctx(stp):
    c = stp.staple_context_create(0)
    yield c
    stp.staple_context_destroy(c)


def oracle_layer(inp, training=True, zero_table=False):
    x, wg, wu, wd = (inp.f64(k) for k in ("x", "w_gate", "w_up", "w_down"))
    E = None if inp.table is None else inp.f64("table")
    if zero_table and E is not None:
        E = np.zeros_like(E)
    fw = oracle.ffn_forward(x, inp.ids, wg, wu, wd, E)
    if not training:
        return fw
    bw = oracle.ffn_backward(inp.f64("dy"), x, inp.ids, wg, wu, wd, fw)
    return {**fw, **bw}


def compare(got, ref, tol, keys):
    for k in keys:
        assert_close(got[k], ref[k], tol, k)


FWD = ("z", "y")
SAVED = ("g", "h")
BWD = ("dg", "dh", "dE", "dx", "dW_gate", "dW_up", "dW_down")


# ---------------------------------------------------------------- fp32 path

@pytest.mark.parametrize("embed", ["table", "rows"])
def test_tiny_f32_layer(stp, ctx, embed):
    w = syn.WORKLOADS["tiny-f32"]
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed=embed)
    ref = oracle_layer(inp)
    np.testing.assert_array_equal(got["unique"], ref["unique"])
    compare(got, ref, TOL["f32"], FWD + SAVED + BWD)


def test_tiny_f32_zero_table_is_dense(stp, ctx):
    w = syn.WORKLOADS["tiny-f32"]
    inp = syn.make_layer_inputs(w, zero_table=True)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
    dense = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="none")
    for k in FWD + SAVED + BWD:
        np.testing.assert_array_equal(got[k] + 0.0, dense[k] + 0.0, err_msg=k)
    compare(got, oracle_layer(inp), TOL["f32"], FWD + BWD)


# ---------------------------------------------------------------- bf16 path

SMALL = [
    # (T, D, F, V): several M tiles with a ragged tail; F not a multiple of the
    # 128-feature gate/up tile or the 256-wide tile; D below one tile
    (300, 128, 320, 1000),
    (129, 64, 64, 50),
    (1, 64, 128, 10),
    (640, 256, 512, 3000),
    # more tokens than the SMs' worth of 128-row tiles' k blocks: the
    # weight-gradient GEMMs run 18 k blocks over the tokens, the last ragged
    (1100, 128, 320, 1000),
]


def _bf16_workload(T, D, F, V):
    return syn.Workload("bf16-small", T=T, D=D, F=F, V=V, layers=1, dtype="bf16", w_std=0.05,
                        e_std=0.05, x_std=1.0, dy_std=1.0, table="device", cache_frac=0.0,
                        group=1, training=True)


@pytest.mark.parametrize("T,D,F,V", SMALL)
def test_bf16_layer_matches_oracle(stp, ctx, T, D, F, V):
    w = _bf16_workload(T, D, F, V)
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, D, F, V, embed="table")
    ref = oracle_layer(inp)
    np.testing.assert_array_equal(got["unique"], ref["unique"])
    compare(got, ref, TOL["bf16"], FWD + SAVED + BWD)


def test_bf16_zero_table_is_bitwise_dense(stp, ctx):
    w = _bf16_workload(300, 128, 320, 1000)
    inp = syn.make_layer_inputs(w, zero_table=True)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
    dense = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="none")
    for k in FWD + SAVED + BWD:
        np.testing.assert_array_equal(got[k] + 0.0, dense[k] + 0.0, err_msg=k)


@pytest.mark.parametrize("T", [64, 300])
def test_bf16_dense_run_matches_oracle(stp, ctx, T):
    """The E path switched off (STAPLE_EMBED_NONE), the comparison run of the
    "within 3%" claim (ai4snews summary, Interpretation), is the dense SwiGLU
    FFN: the fused decode kernel (T = 64) and the tiled GEMMs (T = 300)
    against the oracle with no table, forward and backward."""
    w = _bf16_workload(T, 256, 576, 4000)
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="none")
    x, wg, wu, wd = (inp.f64(k) for k in ("x", "w_gate", "w_up", "w_down"))
    fw = oracle.ffn_forward(x, inp.ids, wg, wu, wd, None)
    ref = {**fw, **oracle.ffn_backward(inp.f64("dy"), x, inp.ids, wg, wu, wd, fw)}
    np.testing.assert_array_equal(got["unique"], ref["unique"])
    compare(got, ref, TOL["bf16"], FWD + SAVED + BWD)


def test_bf16_gathered_rows_equal_table_rows(stp, ctx):
    w = _bf16_workload(640, 256, 512, 3000)
    inp = syn.make_layer_inputs(w)
    direct = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
    freq = syn.calibration_freq(w.V, n_tokens=1 << 18)
    gathered = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="rows", rows_table=inp.table,
                         cache_frac=0.05, freq=freq)
    assert gathered["miss_count"] > 0
    for k in FWD + SAVED + BWD:
        np.testing.assert_array_equal(gathered[k], direct[k], err_msg=k)


def test_bf16_frozen_up_projection(stp, ctx):
    w = _bf16_workload(300, 128, 320, 1000)
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", freeze_up=True)
    ref = oracle_layer(inp)
    compare(got, ref, TOL["bf16"], ("dW_gate", "dW_down", "dE", "dx"))
    assert np.all(got["dW_up"] == 7.0)   # untouched


@pytest.mark.parametrize("T,D,F,V", [(640, 256, 512, 3000), (1100, 128, 320, 1000)])
def test_bf16_deterministic(stp, ctx, T, D, F, V):
    """Two runs give the same bits."""
    w = _bf16_workload(T, D, F, V)
    inp = syn.make_layer_inputs(w)
    a = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
    b = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
    for k in FWD + SAVED + BWD:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_bf16_out_of_range_id_reported(stp, ctx):
    w = _bf16_workload(129, 64, 64, 50)
    inp = syn.make_layer_inputs(w)
    inp.ids[5] = 50
    with pytest.raises(AssertionError, match="EIDRANGE"):
        run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", training=False)


def test_bf16_rejects_unsupported_shapes(stp, ctx):
    import torch
    t = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    e = stp.make_embed(stp.STAPLE_EMBED_NONE)
    with pytest.raises(stp.StapleError) as ex:
        stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, 4, 96, 64, t, e, t, t, t, t, t)
    assert ex.value.status == stp.STAPLE_EINVAL


def test_trace_records_every_kernel(stp, ctx):
    w = _bf16_workload(300, 128, 320, 1000)
    inp = syn.make_layer_inputs(w)
    stp.staple_trace_enable(ctx, True)
    try:
        run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
        rec = stp.staple_trace_read(ctx)
    finally:
        stp.staple_trace_enable(ctx, False)
    names = [n for n, _ in rec]
    for k in ("k1_dedup", "k5_gateup", "k6_down", "k7_dz", "k8_seg_reduce", "k9_dx",
              "k10_dw_gate_up", "k10_dw_down"):
        assert k in names, (k, names)
    assert all(ms > 0 for _, ms in rec)
    assert stp.staple_trace_read(ctx) == []


# ----------------------------------------------------- decode-shaped path

@pytest.mark.parametrize("T", [1, 17, 64, 200, 256])
def test_bf16_decode_sizes_match_oracle(stp, ctx, T):
    """T <= 256 runs the fused weight-streaming kernel (weights on the MMA's M
    side, stream-K down projection whose fp32 partials are summed in piece
    order)."""
    w = _bf16_workload(T, 256, 576, 4000)
    inp = syn.make_layer_inputs(w, with_dy=False)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", training=False)
    ref = oracle_layer(inp, training=False)
    compare(got, ref, TOL["bf16"], FWD)


def test_bf16_decode_saves_g_and_h(stp, ctx):
    w = _bf16_workload(64, 256, 512, 1000)
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table")
    compare(got, oracle_layer(inp), TOL["bf16"], FWD + SAVED + BWD)


@pytest.mark.parametrize("D,F", [(2048, 1024), (1024, 8192), (4096, 11008), (4096, 1024),
                                 (128, 192), (4352, 1024), (4032, 1024), (4416, 1024)])
def test_bf16_decode_split_k_shapes(stp, ctx, D, F):
    """Both decode paths.  Two launches (the split-k sum in its own kernel):
    down tiles whose K is split over a few to many blocks (d_model 2048 and
    1024), d_ff 192 (fewer k units per down tile than a cluster has blocks),
    d_model 4352 and 4416 (more down tiles, 34 and 35, than clusters fit on the
    device at once; 4416 ends in a half tile of 64 rows).  One launch in
    clusters (one cluster per down tile, the sum in shared memory): d_model
    4096 and 4032 (32 tiles, the last of 64 rows) with d_ff 1024, and the 7B
    shape (d_ff 11008 = 172 gate/up tiles over 128 blocks, so some blocks make
    two)."""
    w = _bf16_workload(64, D, F, 2000)
    inp = syn.make_layer_inputs(w, with_dy=False)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", training=False)
    compare(got, oracle_layer(inp, training=False), TOL["bf16"], FWD)


def test_olmo2_1b_decode_layer_full_size(stp, ctx):
    """The bench workload itself: T = 64, d_model 2048, d_ff 8192, vocab 100352,
    the whole table in HBM, every output row checked against the oracle."""
    w = syn.WORKLOADS["olmo2-1b-decode-layer"]
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", training=False)
    x, wg, wu, wd = (inp.f64(k) for k in ("x", "w_gate", "w_up", "w_down"))
    E_rows = syn.bf16_bits_to_f32(inp.table[inp.ids]).astype(np.float64)
    ref = oracle.ffn_forward(x, np.arange(w.T), wg, wu, wd, E_rows)
    compare(got, ref, TOL["bf16"], FWD)


def test_split_table_gradient_matches_fused(stp, ctx):
    """staple_embed_bwd with dE == NULL, then staple_embed_grad on another
    stream, gives the dE of the fused call bit for bit."""
    import torch
    T, D, F, V = 3000, 128, 512, 5000
    g = torch.Generator(device="cuda")
    g.manual_seed(21)

    def rnd(*shape, std=1.0):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    ids = torch.from_numpy(syn.zipf_ids(T, V, 1.1, seed=21)).cuda()
    i32 = dict(dtype=torch.int32, device="cuda")
    unique, inverse, sorted_pos = (torch.empty(T, **i32) for _ in range(3))
    seg, U = torch.empty(T + 1, **i32), torch.empty(1, **i32)
    stp.staple_dedup(ctx, ids, T, V, unique, inverse, seg, sorted_pos, U)
    dy, gs, hs, wd = rnd(T, D), rnd(T, F), rnd(T, F), rnd(D, F, std=0.05)
    wsb = stp.staple_workspace_bytes(T, D, F)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    dgh = torch.empty((T, 2 * F), dtype=torch.bfloat16, device="cuda")
    ref = torch.zeros((T, F), dtype=torch.float32, device="cuda")
    stp.staple_embed_bwd(ctx, stp.STAPLE_BF16, T, D, F, dy, gs, hs, wd, sorted_pos, inverse, seg, U,
                         dgh, ref, ws, wsb)
    dgh2 = torch.empty_like(dgh)
    got = torch.zeros_like(ref)
    stp.staple_embed_bwd(ctx, stp.STAPLE_BF16, T, D, F, dy, gs, hs, wd, sorted_pos, inverse, seg, U,
                         dgh2, None, ws, wsb)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    stp.staple_embed_grad(ctx, stp.STAPLE_BF16, T, D, F, dgh2.data_ptr() + F * 2, 2 * F,
                          sorted_pos, inverse, seg, U, got, ws, wsb, stream=side)
    torch.cuda.synchronize()
    assert stp.staple_get_error(ctx) == 0
    assert torch.equal(dgh, dgh2)
    u = int(U.item())
    assert torch.equal(got[:u], ref[:u])


@pytest.mark.parametrize("D,F", [(512, 1024), (4096, 512)])
def test_bf16_decode_workspace_reused_across_calls_and_shapes(stp, ctx, D, F):
    """One workspace, zero-filled once, serves a burst of decode calls of
    different token counts and inputs issued back to back on one stream (no
    host synchronisation between them): each call's flags must be told apart
    from every earlier call's, so every output matches the oracle.  d_model
    512 takes the two-launch path (its sum kernel clears the flags), 4096 the
    cluster path (the last block past its poll clears them)."""
    import torch
    V = 3000
    Ts = [64, 17, 64, 200, 1, 64, 256, 64]
    g = torch.Generator(device="cuda")
    g.manual_seed(11)

    def rnd(*shape, std):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    wg, wu, wd = rnd(F, D, std=0.05), rnd(F, D, std=0.05), rnd(D, F, std=0.05)
    table = rnd(V, F, std=0.05)
    wsb = max(stp.staple_workspace_bytes(T, D, F) for T in Ts)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    calls = []
    for T in Ts:
        x = rnd(T, D, std=1.0)
        ids = torch.randint(0, V, (T,), generator=g, device="cuda", dtype=torch.int32)
        z = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
        emb = stp.make_embed(stp.STAPLE_EMBED_TABLE, table, F, ids, V)
        stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, T, D, F, x, emb, wg, wu, wd, z, y, None, None,
                           ws, wsb)
        calls.append((x, ids, z, y))
    torch.cuda.synchronize()
    assert stp.staple_get_error(ctx) == 0

    def f64(t):
        return t.float().cpu().numpy().astype(np.float64)

    for x, ids, z, y in calls:
        ref = oracle.ffn_forward(f64(x), ids.cpu().numpy(), f64(wg), f64(wu), f64(wd), f64(table))
        assert_close(f64(z), ref["z"], TOL["bf16"], "z")
        assert_close(f64(y), ref["y"], TOL["bf16"], "y")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_empty_batch(stp, ctx, dtype):
    """T = 0 (a step with no tokens): every call of the layer succeeds, writes
    no activation, and the weight gradients of the empty batch are zero (a
    sum over no tokens)."""
    import torch
    D, F, V = 256, 512, 100
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sdt = stp.STAPLE_BF16 if dtype == "bf16" else stp.STAPLE_F32
    g = torch.Generator(device="cuda")
    g.manual_seed(21)

    def rnd(*shape):
        return (torch.randn(shape, generator=g, device="cuda") * 0.05).to(tdt)

    wg, wu, wd, table = rnd(F, D), rnd(F, D), rnd(D, F), rnd(V, F)
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    emb = stp.make_embed(stp.STAPLE_EMBED_TABLE, table, F, ids, V)
    x, dy, dx = (torch.full((1, D), 7.0, dtype=tdt, device="cuda") for _ in range(3))
    z, gs, hs = (torch.full((1, F), 7.0, dtype=tdt, device="cuda") for _ in range(3))
    y = torch.full((1, D), 7.0, dtype=tdt, device="cuda")
    dgh = torch.full((1, 2 * F), 7.0, dtype=tdt, device="cuda")
    dE = torch.full((1, F), 7.0, dtype=torch.float32, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    sorted_pos, inverse, seg, U = (torch.zeros(2, **i32) for _ in range(4))
    dwg, dwu, dwd = (torch.full(s, 3.0, dtype=torch.float32, device="cuda")
                     for s in ((F, D), (F, D), (D, F)))
    wsb = stp.staple_workspace_bytes(0, D, F)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    stp.staple_ffn_fwd(ctx, sdt, 0, D, F, x, emb, wg, wu, wd, z, y, gs, hs, ws, wsb)
    stp.staple_embed_bwd(ctx, sdt, 0, D, F, dy, gs, hs, wd, sorted_pos, inverse, seg, U, dgh, dE,
                         ws, wsb)
    stp.staple_ffn_bwd(ctx, sdt, 0, D, F, dy, x, z, dgh, wg, wu, dx, dwg, dwu, dwd, ws, wsb)
    torch.cuda.synchronize()
    assert stp.staple_get_error(ctx) == 0
    for t in (y, z, gs, hs, dgh, dx):
        assert bool((t.float() == 7.0).all())
    assert bool((dE == 7.0).all())
    for t in (dwg, dwu, dwd):
        assert bool((t == 0.0).all())


def test_table_gradient_refuses_more_tokens_than_one_dedup(stp, ctx):
    """The reduction's counters cover the 32768 tokens one staple_dedup takes;
    a longer batch with dE requested is refused before anything runs (the
    addresses below are never touched)."""
    fake = 1 << 12
    wsb = stp.staple_workspace_bytes(32769, 64, 64)
    for call in (
            lambda: stp.staple_embed_bwd(ctx, stp.STAPLE_BF16, 32769, 64, 64, fake, fake, fake, fake,
                                         fake, fake, fake, fake, fake, fake, fake, wsb),
            lambda: stp.staple_embed_grad(ctx, stp.STAPLE_BF16, 32769, 64, 64, fake, 64, fake, fake,
                                          fake, fake, fake, fake, wsb)):
        with pytest.raises(stp.StapleError) as ex:
            call()
        assert ex.value.status == stp.STAPLE_EUNSUPPORTED
    assert stp.staple_get_error(ctx) == 0
