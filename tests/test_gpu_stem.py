"""GPU parity of the STEM variant (STAPLE_EMBED_REPLACE_UP: the token's row
replaces the up-projection, h = E[id]; abstract, ai4snews summary,
Interpretation) against the oracle's stem_forward / stem_backward, forward
and full backward, on the fp32 path, the tiled bf16 path and decode sizes."""
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


def stem_oracle(inp, training=True):
    x, wg, wd = (inp.f64(k) for k in ("x", "w_gate", "w_down"))
    fw = oracle.stem_forward(x, inp.ids, wg, wd, inp.f64("table"))
    if not training:
        return fw
    return {**fw, **oracle.stem_backward(inp.f64("dy"), x, inp.ids, wg, wd, fw)}


FWD = ("z", "y", "g", "h")
BWD = ("dg", "dh", "dE", "dx", "dW_gate", "dW_down")


def _w(T, D, F, V, dtype="bf16"):
    return syn.Workload("stem", T=T, D=D, F=F, V=V, layers=1, dtype=dtype, w_std=0.05,
                        e_std=0.05, x_std=1.0, dy_std=1.0, table="device", cache_frac=0.0,
                        group=1, training=True)


@pytest.mark.parametrize("embed", ["table", "rows"])
def test_stem_f32(stp, ctx, embed):
    w = syn.WORKLOADS["tiny-f32"]
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed=embed, stem=True)
    ref = stem_oracle(inp)
    np.testing.assert_array_equal(got["unique"], ref["unique"])
    for k in FWD + BWD:
        assert_close(got[k], ref[k], TOL["f32"], k)
    assert np.all(got["dW_up"] == 7.0)   # no up-projection: its gradient is never written


@pytest.mark.parametrize("T,D,F,V", [(300, 128, 320, 1000), (640, 256, 512, 3000), (64, 256, 576, 4000),
                                     (1, 64, 128, 10), (64, 4096, 1024, 2000)])
def test_stem_bf16(stp, ctx, T, D, F, V):
    inp = syn.make_layer_inputs(_w(T, D, F, V))
    got = run_layer(stp, ctx, inp, D, F, V, embed="table", stem=True)
    ref = stem_oracle(inp)
    np.testing.assert_array_equal(got["unique"], ref["unique"])
    for k in FWD + BWD:
        assert_close(got[k], ref[k], TOL["bf16"], k)


def test_stem_bf16_gathered_rows_from_a_host_table(stp, ctx):
    w = _w(640, 256, 512, 3000)
    inp = syn.make_layer_inputs(w)
    freq = syn.calibration_freq(w.V, n_tokens=1 << 18)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="rows", rows_table=inp.table,
                    cache_frac=0.05, freq=freq, stem=True)
    assert got["miss_count"] > 0
    ref = stem_oracle(inp)
    for k in FWD + BWD:
        assert_close(got[k], ref[k], TOL["bf16"], k)


def test_stem_olmo2_1b_decode_layer_full_size(stp, ctx):
    """The decode workload's shape (T = 64, d_model 2048, d_ff 8192, vocab
    100352, table in HBM) as STEM, every output row against the oracle."""
    w = syn.WORKLOADS["olmo2-1b-decode-layer"]
    inp = syn.make_layer_inputs(w)
    got = run_layer(stp, ctx, inp, w.D, w.F, w.V, embed="table", training=False, stem=True)
    x, wg, wd = (inp.f64(k) for k in ("x", "w_gate", "w_down"))
    E_rows = syn.bf16_bits_to_f32(inp.table[inp.ids]).astype(np.float64)
    ref = oracle.stem_forward(x, np.arange(w.T), wg, wd, E_rows)
    for k in ("z", "y"):
        assert_close(got[k], ref[k], TOL["bf16"], k)


def test_stem_rejects_a_missing_table(stp, ctx):
    import torch
    t = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    e = stp.make_embed(stp.STAPLE_EMBED_NONE, flags=stp.STAPLE_EMBED_REPLACE_UP)
    with pytest.raises(stp.StapleError) as ex:
        stp.staple_ffn_fwd(ctx, stp.STAPLE_BF16, 4, 64, 64, t, e, t, None, t, t, t)
    assert ex.value.status == stp.STAPLE_EINVAL
