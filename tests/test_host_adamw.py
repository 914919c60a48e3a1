"""The library's host AdamW (staple_adamw_rows) against the oracle's fp64
AdamW, on the CPU: no GPU is involved.

fp32 tables: table and moments within 1e-6 relative to the oracle after
several steps.  bf16 tables: the library updates in fp32 and rounds to bf16,
the oracle in fp64; each value may differ from the oracle's value rounded to
bf16 by at most one bf16 step.  The moments (fp32 in both cases) stay within
1e-6.  Rows that got no gradient must not change, bit for bit.  Tables use a
grouped layout (one layer's slice of a [V][G][F] array)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synthetic as syn

HP = dict(lr=3e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
# the library receives the hyperparameters as fp32; the oracle gets the same
# values (0.999 is 0.99900001287 in fp32, so 1 - beta2 differs by 1.3e-5
# from the decimal)
HP32 = {k: float(np.float32(x)) for k, x in HP.items()}


@pytest.fixture(scope="module")
def stp():
    import token_indexed_sparse_staple_b200 as m
    return m


def _run(stp, dtype, threads, steps=3, V=700, F=96, G=3, layer=1, U=150, seed=41):
    rng = np.random.default_rng(seed)
    if dtype == "bf16":
        full = syn.bf16_normal((V, G * F), 0.05, seed)[0]          # [V][G*F] bf16 bits
        w_ref = syn.bf16_bits_to_f32(full[:, layer * F:(layer + 1) * F]).astype(np.float64)
        sdt = stp.STAPLE_BF16
    else:
        full = (rng.standard_normal((V, G * F)) * 0.05).astype(np.float32)
        w_ref = full[:, layer * F:(layer + 1) * F].astype(np.float64)
        sdt = stp.STAPLE_F32
    before = full.copy()
    m = np.zeros((V, F), np.float32)
    v = np.zeros((V, F), np.float32)
    m_ref, v_ref = np.zeros((V, F)), np.zeros((V, F))
    touched = np.zeros(V, bool)
    for step in range(1, steps + 1):
        ids = np.sort(rng.choice(V, U, replace=False)).astype(np.int32)
        touched[ids] = True
        g = (rng.standard_normal((U, F)) * 0.1).astype(np.float32)
        base = full.ctypes.data + layer * F * full.itemsize
        stp.staple_adamw_rows(base, G * F, sdt, F, ids, U, g, F, m, v, F, step=step,
                              threads=threads, **HP)
        w_new, m_ref, v_ref = oracle.adamw_rows(w_ref, ids, g.astype(np.float64), m_ref, v_ref,
                                                step=step, **HP32)
        got = full[:, layer * F:(layer + 1) * F]
        if dtype == "bf16":
            # one bf16 step (8 significant bits) at the oracle's value
            got_f = syn.bf16_bits_to_f32(got).astype(np.float64)
            step_size = np.exp2(np.floor(np.log2(np.maximum(np.abs(w_new), 1e-30))) - 7)
            off = np.abs(got_f - w_new) / step_size
            assert off.max() <= 1.0, f"step {step}: bf16 table off by {off.max():.2f} steps"
            w_ref = got_f                 # the next step starts from the stored table
        else:
            np.testing.assert_allclose(got.astype(np.float64), w_new, rtol=1e-6,
                                       atol=1e-6 * np.abs(w_new).max())
            w_ref = got.astype(np.float64)
        np.testing.assert_allclose(m, m_ref, rtol=1e-5, atol=1e-6 * np.abs(m_ref).max())
        np.testing.assert_allclose(v, v_ref, rtol=1e-5, atol=1e-6 * np.abs(v_ref).max())
        m_ref, v_ref = m.astype(np.float64), v.astype(np.float64)
    # untouched rows, and the other layers of every row, are bit for bit unchanged
    other = np.ones(G * F, bool)
    other[layer * F:(layer + 1) * F] = False
    np.testing.assert_array_equal(full[:, other], before[:, other])
    np.testing.assert_array_equal(full[~touched], before[~touched])
    assert not np.any(m[~touched]) and not np.any(v[~touched])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("threads", [1, 4])
def test_host_adamw_matches_oracle(stp, dtype, threads):
    _run(stp, dtype, threads)


def test_host_adamw_rejects_bad_arguments(stp):
    import ctypes as C
    hp = stp.staple_adamw(1e-3, 0.9, 0.999, 1e-8, 0.0, 0)     # step 0 is not a step
    buf = np.zeros(16, np.float32)
    ids = np.zeros(1, np.int32)
    st = stp.lib().staple_adamw_rows(buf.ctypes.data, 4, stp.STAPLE_F32, 4, ids.ctypes.data, 1,
                                     buf.ctypes.data, 4, buf.ctypes.data, buf.ctypes.data, 4,
                                     C.byref(hp), 1)
    assert st == stp.STAPLE_EINVAL


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_adamw_paths_agree_bit_for_bit(stp, dtype, monkeypatch):
    """The vector paths (AVX-512, AVX2, where the CPU has them) perform the
    scalar path's IEEE operations in the same order, so all give the same
    bits.  F = 100 leaves ragged tails after 16- and 8-lane blocks, and one
    NaN gradient takes a bf16 value through the NaN branch of the rounding."""
    V, F, U = 300, 100, 120
    rng = np.random.default_rng(5)
    if dtype == "bf16":
        table0 = syn.bf16_normal((V, F), 0.05, 77)[0]
        sdt = stp.STAPLE_BF16
    else:
        table0 = (rng.standard_normal((V, F)) * 0.05).astype(np.float32)
        sdt = stp.STAPLE_F32
    grads = [(rng.standard_normal((U, F)) * 0.1).astype(np.float32) for _ in range(2)]
    grads[1][3, 17] = np.nan
    ids = [np.sort(rng.choice(V, U, replace=False)).astype(np.int32) for _ in range(2)]
    out = {}
    for isa in ("scalar", "avx2", "avx512"):
        monkeypatch.setenv("STAPLE_ADAMW_ISA", isa)
        table = table0.copy()
        m = np.zeros((V, F), np.float32)
        v = np.zeros((V, F), np.float32)
        for step in (1, 2):
            stp.staple_adamw_rows(table.ctypes.data, F, sdt, F, ids[step - 1], U, grads[step - 1],
                                  F, m, v, F, step=step, threads=3, **HP)
        out[isa] = (table.view(np.uint8), m.view(np.uint32), v.view(np.uint32))
    for isa in ("avx2", "avx512"):
        for a, b in zip(out[isa], out["scalar"]):
            np.testing.assert_array_equal(a, b, err_msg=isa)
    # the NaN reached the table, as a NaN
    r = ids[1][3]
    got = out["scalar"][0].view(np.uint16 if dtype == "bf16" else np.float32)[r, 17]
    val = syn.bf16_bits_to_f32(np.array([got]))[0] if dtype == "bf16" else got
    assert np.isnan(val)


def test_host_adamw_rejects_negative_ids_before_updating(stp):
    F, V, U = 16, 8, 3
    table = np.ones((V, F), np.float32)
    m = np.zeros((V, F), np.float32)
    v = np.zeros((V, F), np.float32)
    g = np.ones((U, F), np.float32)
    ids = np.array([1, -2, 5], np.int32)
    with pytest.raises(stp.StapleError) as ex:
        stp.staple_adamw_rows(table.ctypes.data, F, stp.STAPLE_F32, F, ids, U, g, F, m, v, F,
                              step=1, threads=1, **HP)
    assert ex.value.status == stp.STAPLE_EINVAL
    assert np.all(table == 1.0) and not np.any(m) and not np.any(v)
