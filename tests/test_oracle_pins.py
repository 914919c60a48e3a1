"""Pins of the CPU oracle to things other than itself.

Brute-force per-token loops in plain Python floats (no numpy matmul), the
identity E = 0 => dense FFN, the single-token closed form of the table
gradient, fp64 central finite differences, conservation and permutation
properties, brute-force dedup / top-K / probe, and the sizes the pages print.
"""
import json
import math
import os
import random

import numpy as np
import pytest

import oracle
import synthetic as syn

HERE = os.path.dirname(os.path.abspath(__file__))


# --------------------------------------------------------------------------
# Brute-force references: plain Python loops, math.exp, no numpy arithmetic
# --------------------------------------------------------------------------

def _sig(v):
    return 1.0 / (1.0 + math.exp(-v))


def brute_forward(x, ids, wg, wu, wd, E):
    T, D = len(x), len(x[0])
    F = len(wg)
    out = {k: [] for k in ("g", "h", "z", "y")}
    for t in range(T):
        g = [sum(wg[f][d] * x[t][d] for d in range(D)) for f in range(F)]
        u = [sum(wu[f][d] * x[t][d] for d in range(D)) for f in range(F)]
        h = [u[f] + (E[ids[t]][f] if E is not None else 0.0) for f in range(F)]
        z = [g[f] * _sig(g[f]) * h[f] for f in range(F)]
        y = [sum(wd[d][f] * z[f] for f in range(F)) for d in range(D)]
        for k, v in (("g", g), ("h", h), ("z", z), ("y", y)):
            out[k].append(v)
    return {k: np.array(v) for k, v in out.items()}


def brute_backward(dy, x, ids, wg, wu, wd, E):
    T, D = len(x), len(x[0])
    F = len(wg)
    fw = brute_forward(x, ids, wg, wu, wd, E)
    dE = {}
    dx = [[0.0] * D for _ in range(T)]
    dWg = [[0.0] * D for _ in range(F)]
    dWu = [[0.0] * D for _ in range(F)]
    dWd = [[0.0] * F for _ in range(D)]
    for t in range(T):
        for f in range(F):
            g = fw["g"][t][f]
            h = fw["h"][t][f]
            s = _sig(g)
            dz = sum(wd[d][f] * dy[t][d] for d in range(D))
            dh = dz * g * s
            dg = dz * h * (s + g * s * (1.0 - s))
            row = dE.setdefault(ids[t], [0.0] * F)
            row[f] += dh
            for d in range(D):
                dx[t][d] += wg[f][d] * dg + wu[f][d] * dh
                dWg[f][d] += dg * x[t][d]
                dWu[f][d] += dh * x[t][d]
        for d in range(D):
            for f in range(F):
                dWd[d][f] += dy[t][d] * fw["z"][t][f]
    keys = sorted(dE)
    return {"unique": np.array(keys), "dE": np.array([dE[k] for k in keys]),
            "dx": np.array(dx), "dW_gate": np.array(dWg), "dW_up": np.array(dWu),
            "dW_down": np.array(dWd)}


def _tiny(seed=0, T=7, D=5, F=6, V=11, ids=None, zero_table=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D))
    wg = rng.standard_normal((F, D)) * 0.7
    wu = rng.standard_normal((F, D)) * 0.7
    wd = rng.standard_normal((D, F)) * 0.7
    E = np.zeros((V, F)) if zero_table else rng.standard_normal((V, F)) * 0.5
    if ids is None:
        ids = rng.integers(0, V, size=T)
    dy = rng.standard_normal((T, D))
    return x, np.asarray(ids), wg, wu, wd, E, dy


def _lists(*arrs):
    return [a.tolist() for a in arrs]


# --------------------------------------------------------------------------
# Forward / backward against brute force
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_forward_matches_brute_force(seed):
    x, ids, wg, wu, wd, E, _ = _tiny(seed)
    got = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    ref = brute_forward(*_lists(x), ids.tolist(), *_lists(wg, wu, wd, E))
    for k in ("g", "h", "z", "y"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-12, atol=1e-12, err_msg=k)


@pytest.mark.parametrize("seed", [0, 3])
def test_backward_matches_brute_force(seed):
    x, ids, wg, wu, wd, E, dy = _tiny(seed, ids=[3, 1, 3, 7, 1, 3, 0])
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    got = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    ref = brute_backward(*_lists(dy, x), ids.tolist(), *_lists(wg, wu, wd, E))
    np.testing.assert_array_equal(got["unique"], ref["unique"])
    for k in ("dE", "dx", "dW_gate", "dW_up", "dW_down"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-11, atol=1e-11, err_msg=k)


def test_zero_table_gives_dense_ffn():
    """E = 0 restores the seed model's computation (zero-initialised tables)."""
    x, ids, wg, wu, wd, E, dy = _tiny(5, zero_table=True)
    staple = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    dense_ref = brute_forward(*_lists(x), ids.tolist(), *_lists(wg, wu, wd), None)
    np.testing.assert_array_equal(staple["y"], oracle.ffn_forward(x, ids, wg, wu, wd, None)["y"])
    np.testing.assert_allclose(staple["y"], dense_ref["y"], rtol=1e-12, atol=1e-13)


def test_single_token_table_gradient_closed_form():
    """T = 1: the table gradient is SiLU(W_gate x) * (W_down^T dY), one row."""
    x, ids, wg, wu, wd, E, dy = _tiny(9, T=1)
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    D, F = wd.shape
    xs, dys = x[0].tolist(), dy[0].tolist()
    expect = []
    for f in range(F):
        g = sum(wg[f][d] * xs[d] for d in range(D))
        expect.append(g * _sig(g) * sum(wd[d][f] * dys[d] for d in range(D)))
    assert bw["dE"].shape == (1, F)
    np.testing.assert_allclose(bw["dE"][0], expect, rtol=1e-12, atol=1e-14)


def _loss(x, ids, wg, wu, wd, E, dy):
    return float(np.sum(dy * oracle.ffn_forward(x, ids, wg, wu, wd, E)["y"]))


def test_gradients_match_finite_differences():
    x, ids, wg, wu, wd, E, dy = _tiny(11, T=6, D=4, F=5, V=9, ids=[2, 5, 2, 8, 5, 2])
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    eps = 1e-6
    rnd = random.Random(0)
    arrays = {"x": x, "wg": wg, "wu": wu, "wd": wd, "E": E}
    grads = {"x": bw["dx"], "wg": bw["dW_gate"], "wu": bw["dW_up"], "wd": bw["dW_down"]}
    uniq = list(bw["unique"])
    for name, arr in arrays.items():
        for _ in range(6):
            if name == "E":
                r = rnd.choice(uniq)
                idx = (r, rnd.randrange(arr.shape[1]))
                analytic = bw["dE"][uniq.index(r), idx[1]]
            else:
                idx = tuple(rnd.randrange(n) for n in arr.shape)
                analytic = grads[name][idx]
            old = arr[idx]
            arr[idx] = old + eps
            lp = _loss(**arrays, ids=ids, dy=dy)
            arr[idx] = old - eps
            lm = _loss(**arrays, ids=ids, dy=dy)
            arr[idx] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - analytic) <= 1e-6 * max(1.0, abs(analytic)), (name, idx, fd, analytic)
    # rows of E that no token uses get no gradient: U rows only
    assert len(uniq) == 3


def test_table_gradient_conservation_and_independence_from_E():
    x, ids, wg, wu, wd, E, dy = _tiny(13, T=40, V=12)
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    np.testing.assert_allclose(bw["dE"].sum(axis=0), bw["dh"].sum(axis=0), rtol=1e-12, atol=1e-12)
    fw0 = oracle.ffn_forward(x, ids, wg, wu, wd, np.zeros_like(E))
    bw0 = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw0)
    np.testing.assert_array_equal(bw["dE"], bw0["dE"])
    # linearity of y in E: y(E) - y(0) = W_down (SiLU(g) * E[ids])
    lin = (fw["a"] * E[ids]) @ wd.T
    np.testing.assert_allclose(fw["y"] - fw0["y"], lin, rtol=1e-10, atol=1e-12)


def test_permutation_invariance():
    x, ids, wg, wu, wd, E, dy = _tiny(17, T=30, V=8)
    perm = np.random.default_rng(1).permutation(len(ids))
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    fwp = oracle.ffn_forward(x[perm], ids[perm], wg, wu, wd, E)
    bwp = oracle.ffn_backward(dy[perm], x[perm], ids[perm], wg, wu, wd, fwp)
    np.testing.assert_allclose(fwp["y"], fw["y"][perm], rtol=1e-13, atol=1e-14)
    for k in ("dE", "dW_gate", "dW_up", "dW_down"):
        np.testing.assert_allclose(bwp[k], bw[k], rtol=1e-11, atol=1e-12, err_msg=k)


def test_all_distinct_ids_table_gradient_is_dh_permuted():
    x, ids, wg, wu, wd, E, dy = _tiny(19, T=6, V=10, ids=[9, 2, 4, 0, 7, 5])
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    order = np.argsort(ids)
    np.testing.assert_array_equal(bw["dE"], bw["dh"][order])


def test_silu_special_values():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert oracle.silu_grad(np.array([0.0]))[0] == 0.5
    big = np.array([40.0, -40.0])
    np.testing.assert_allclose(oracle.silu(big), [40.0, -40.0 * math.exp(-40.0)], rtol=1e-12)
    g = np.linspace(-6, 6, 25)
    fd = (oracle.silu(g + 1e-6) - oracle.silu(g - 1e-6)) / 2e-6
    np.testing.assert_allclose(oracle.silu_grad(g), fd, rtol=1e-7, atol=1e-9)


# --------------------------------------------------------------------------
# Sampled forms agree with the full definitions
# --------------------------------------------------------------------------

def test_sampled_forms_match_full_definitions():
    x, ids, wg, wu, wd, E, dy = _tiny(23, T=50, D=6, F=7, V=9)
    fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
    bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
    rows = [0, 7, 49]
    np.testing.assert_allclose(oracle.forward_rows(rows, x, ids, wg, wu, wd, E)["y"], fw["y"][rows], rtol=1e-13)
    np.testing.assert_allclose(oracle.dx_rows(rows, dy, x, ids, wg, wu, wd, E), bw["dx"][rows], rtol=1e-12, atol=1e-13)
    uids = bw["unique"][[0, -1]]
    np.testing.assert_allclose(oracle.embed_grad_rows(uids, dy, x, ids, wg, wu, wd, E), bw["dE"][[0, -1]],
                               rtol=1e-12, atol=1e-13)
    ent = [("gate", 3, 2), ("up", 6, 0), ("down", 5, 4), ("gate", 3, 5)]
    got = oracle.weight_grad_entries(ent, dy, x, ids, wg, wu, wd, E)
    want = [bw["dW_gate"][3, 2], bw["dW_up"][6, 0], bw["dW_down"][5, 4], bw["dW_gate"][3, 5]]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Retrieval steps against brute force
# --------------------------------------------------------------------------

@pytest.mark.parametrize("ids", [
    [5, 3, 5, 5, 0, 9, 3],
    [4],
    [2, 2, 2, 2],
    list(range(20))[::-1],
    [],
])
def test_dedup_brute_force(ids):
    u, inv, seg, sp = oracle.dedup(np.array(ids, dtype=np.int32))
    ref_u = sorted(set(ids))
    assert u.tolist() == ref_u
    assert [ref_u[i] for i in inv] == list(ids)
    assert seg[0] == 0 and seg[-1] == len(ids) and len(seg) == len(ref_u) + 1
    for j, val in enumerate(ref_u):
        pos = [p for p, v in enumerate(ids) if v == val]
        assert sp[seg[j]:seg[j + 1]].tolist() == pos


def test_hot_set_and_probe_brute_force():
    rnd = random.Random(3)
    V = 50
    freq = np.array([rnd.choice([0, 1, 1, 2, 5, 5, 9]) for _ in range(V)], dtype=np.int64)
    for frac in (0.0, 0.05, 0.1, 0.33, 1.0):
        hot, slot_of = oracle.hot_set(freq, frac)
        K = math.ceil(frac * V)
        ref = sorted(range(V), key=lambda i: (-freq[i], i))[:K]
        assert hot.tolist() == ref
        for i in range(V):
            assert slot_of[i] == (ref.index(i) if i in ref else -1)
        uniq = np.array(sorted(rnd.sample(range(V), 12)), dtype=np.int32)
        slot, miss = oracle.probe(uniq, slot_of)
        assert slot.tolist() == [ref.index(i) if i in ref else -1 for i in uniq]
        assert miss.tolist() == [j for j, i in enumerate(uniq) if i not in ref]
    assert oracle.hot_set(freq, 0.05)[0].size == 3   # ceil(2.5) = 3


def test_gather_is_a_bit_copy():
    bits, _ = syn.bf16_normal((40, 24), 0.01, 5)
    uniq = np.array([0, 7, 39], dtype=np.int32)
    rows = oracle.gather_rows(bits, uniq)
    assert rows.dtype == np.uint16
    np.testing.assert_array_equal(rows, bits[[0, 7, 39]])
    grouped = oracle.gather_rows(bits, uniq, row_offset=8, width=8)
    np.testing.assert_array_equal(grouped, bits[[0, 7, 39], 8:16])
    # the cache image: slot k holds the row of the k-th hot id, element by element
    freq = np.array([3, 9, 1, 9, 0, 4] + [0] * 34, dtype=np.int64)
    hot, _ = oracle.hot_set(freq, 0.1)                  # 4 slots: ids 1, 3, 5, 0
    cache = oracle.cache_rows_for(bits, hot)
    assert list(hot) == [1, 3, 5, 0]
    for k, i in enumerate([1, 3, 5, 0]):
        for f in range(bits.shape[1]):
            assert cache[k, f] == bits[i, f]


# --------------------------------------------------------------------------
# Sizes the pages print
# --------------------------------------------------------------------------

def test_paper_printed_sizes():
    with open(os.path.join(HERE, "golden", "paper_numbers.json")) as f:
        gold = json.load(f)
    s = oracle.paper_shapes()

    def check(key, got):
        g = gold[key]
        assert abs(got - g["value"]) <= g["tol"], (key, got, g)

    check("table_bytes_12L", s["table_bytes"])
    check("table_plus_moments_GiB_12L", s["table_plus_moments_bytes"] / 2**30)
    check("cache_GB_12L_at_5pct", s["cache_bytes"] / 1e9)
    check("dense_linear_flops_per_token", s["dense_linear_flops_per_token"])
    check("stem_linear_flops_per_token", s["stem_linear_flops_per_token"])
    check("dense_weight_GB", s["dense_weight_bytes"] / 1e9)
    check("stem_weight_GB", s["stem_weight_bytes"] / 1e9)
    assert s["cache_rows"] == 5018


def test_zipf_stream_hit_rate_is_plausible():
    """The top 5% of a Zipf(1.1) vocabulary carries ~85% of tokens; the pages
    report ~80% hits for a 5-6% cache.  Plausibility, not parity."""
    with open(os.path.join(HERE, "golden", "paper_numbers.json")) as f:
        g = json.load(f)["hit_rate_at_5_6pct_vocab"]
    V = 100352
    m = syn.top_mass(V, 1.1, 0.05)
    assert abs(m - g["value"]) <= g["tol"]
    freq = syn.calibration_freq(V, n_tokens=1 << 21)
    _, slot_of = oracle.hot_set(freq, 0.05)
    ids = syn.zipf_ids(1 << 16, V, seed=99)
    hit = float(np.mean(slot_of[ids] >= 0))
    assert abs(hit - m) < 0.02


# --------------------------------------------------------------------------
# Planted mistakes: each plausible slip in the oracle must fail a pin above
# --------------------------------------------------------------------------

def _mutant_backward(kind):
    real = oracle.ffn_backward

    def bad(dy, x, ids, wg, wu, wd, fw):
        out = real(dy, x, ids, wg, wu, wd, fw)
        if kind == "dg_sign":
            out["dx"] = -out["dg"] @ wg + out["dh"] @ wu
        elif kind == "dh_uses_sigmoid":
            dh = out["dz"] / (1 + np.exp(-fw["g"]))
            out["dE"] = real(dy, x, ids, wg, wu, wd, {**fw, "a": dh / np.where(out["dz"] == 0, 1, out["dz"])})["dE"]
        elif kind == "dWd_transposed":
            out["dW_down"] = (fw["z"].T @ dy).T[::-1].copy()
        return out
    return bad


def _mutant_forward(kind):
    real = oracle.ffn_forward

    def bad(x, ids, wg, wu, wd, table=None):
        if kind == "drop_E":
            return real(x, ids, wg, wu, wd, None)
        if kind == "E_on_gate":
            out = real(x, ids, wg, wu, wd, None)
            g = out["g"] + table[np.asarray(ids)]
            out["z"] = oracle.silu(g) * out["h"]
            out["y"] = out["z"] @ wd.T
            return out
        if kind == "wrong_row":
            return real(x, (np.asarray(ids) + 1) % table.shape[0], wg, wu, wd, table)
        raise ValueError(kind)
    return bad


@pytest.mark.parametrize("kind", ["drop_E", "E_on_gate", "wrong_row"])
def test_planted_forward_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(oracle, "ffn_forward", _mutant_forward(kind))
    with pytest.raises(AssertionError):
        test_forward_matches_brute_force(0)


@pytest.mark.parametrize("kind", ["dg_sign", "dh_uses_sigmoid", "dWd_transposed"])
def test_planted_backward_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(oracle, "ffn_backward", _mutant_backward(kind))
    with pytest.raises(AssertionError):
        test_backward_matches_brute_force(0)


# --------------------------------------------------------------------------
# Host AdamW on the touched rows
# --------------------------------------------------------------------------

_HP = dict(lr=1e-2, beta1=0.9, beta2=0.99, eps=1e-8, weight_decay=0.1)


def test_adamw_dense_matches_torch_adamw():
    """All rows touched every step: the oracle is torch.optim.AdamW (fp64)."""
    import torch
    rng = np.random.default_rng(31)
    V, F = 6, 5
    w0 = rng.standard_normal((V, F))
    p = torch.nn.Parameter(torch.tensor(w0, dtype=torch.float64))
    opt = torch.optim.AdamW([p], lr=_HP["lr"], betas=(_HP["beta1"], _HP["beta2"]),
                            eps=_HP["eps"], weight_decay=_HP["weight_decay"])
    w, m, v = w0.copy(), np.zeros((V, F)), np.zeros((V, F))
    ids = np.arange(V)
    for step in range(1, 4):
        g = rng.standard_normal((V, F))
        p.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        w, m, v = oracle.adamw_rows(w, ids, g, m, v, step=step, **_HP)
        np.testing.assert_allclose(w, p.detach().numpy(), rtol=1e-12, atol=1e-14)


def test_adamw_first_step_closed_form_and_untouched_rows():
    """From zero moments, step 1 moves w by lr (g / (|g| + eps) + wd w); rows
    without a gradient keep their value and moments."""
    rng = np.random.default_rng(32)
    V, F = 10, 7
    w0 = rng.standard_normal((V, F))
    m0, v0 = np.zeros((V, F)), np.zeros((V, F))
    m0[1], v0[1] = 0.5, 0.25                      # an untouched row with state
    ids = np.array([3, 7, 0])
    g = rng.standard_normal((3, F))
    w, m, v = oracle.adamw_rows(w0, ids, g, m0, v0, step=1, **_HP)
    expect = w0[ids] - _HP["lr"] * (g / (np.abs(g) + _HP["eps"]) + _HP["weight_decay"] * w0[ids])
    np.testing.assert_allclose(w[ids], expect, rtol=1e-12)
    rest = np.setdiff1d(np.arange(V), ids)
    np.testing.assert_array_equal(w[rest], w0[rest])
    np.testing.assert_array_equal(m[rest], m0[rest])
    np.testing.assert_array_equal(v[rest], v0[rest])


def test_planted_adamw_mistake_is_caught(monkeypatch):
    """Without the bias corrections the closed form above fails."""
    def no_bias_correction(table, ids, grad, m, v, lr, beta1, beta2, eps, weight_decay, step):
        w, m, v = np.array(table, float), np.array(m, float), np.array(v, float)
        g = np.asarray(grad, float)
        m[ids] = beta1 * m[ids] + (1 - beta1) * g
        v[ids] = beta2 * v[ids] + (1 - beta2) * g * g
        w[ids] = w[ids] - lr * (m[ids] / (np.sqrt(v[ids]) + eps) + weight_decay * w[ids])
        return w, m, v
    monkeypatch.setattr(oracle, "adamw_rows", no_bias_correction)
    with pytest.raises(AssertionError):
        test_adamw_first_step_closed_form_and_untouched_rows()


# --------------------------------------------------------------------------
# STEM, the replacement variant (the row replaces the up-projection)
# --------------------------------------------------------------------------

def brute_stem(dy, x, ids, wg, wd, E):
    """Per-token plain-Python loops of the STEM layer and its gradients."""
    T, D = len(x), len(x[0])
    F = len(wg)
    out = {k: [] for k in ("g", "h", "z", "y")}
    dE, dx = {}, [[0.0] * D for _ in range(T)]
    dWg = [[0.0] * D for _ in range(F)]
    dWd = [[0.0] * F for _ in range(D)]
    for t in range(T):
        g = [sum(wg[f][d] * x[t][d] for d in range(D)) for f in range(F)]
        h = [E[ids[t]][f] for f in range(F)]
        z = [g[f] * _sig(g[f]) * h[f] for f in range(F)]
        y = [sum(wd[d][f] * z[f] for f in range(F)) for d in range(D)]
        for k, v in (("g", g), ("h", h), ("z", z), ("y", y)):
            out[k].append(v)
        for f in range(F):
            s = _sig(g[f])
            dz = sum(wd[d][f] * dy[t][d] for d in range(D))
            dh = dz * g[f] * s
            dg = dz * h[f] * (s + g[f] * s * (1.0 - s))
            row = dE.setdefault(ids[t], [0.0] * F)
            row[f] += dh
            for d in range(D):
                dx[t][d] += wg[f][d] * dg
                dWg[f][d] += dg * x[t][d]
        for d in range(D):
            for f in range(F):
                dWd[d][f] += dy[t][d] * z[f]
    keys = sorted(dE)
    res = {k: np.array(v) for k, v in out.items()}
    res.update(unique=np.array(keys), dE=np.array([dE[k] for k in keys]), dx=np.array(dx),
               dW_gate=np.array(dWg), dW_down=np.array(dWd))
    return res


@pytest.mark.parametrize("seed", [0, 4])
def test_stem_matches_brute_force(seed):
    x, ids, wg, _, wd, E, dy = _tiny(seed)
    fw = oracle.stem_forward(x, ids, wg, wd, E)
    bw = oracle.stem_backward(dy, x, ids, wg, wd, fw)
    ref = brute_stem(*_lists(dy, x), ids.tolist(), *_lists(wg, wd, E))
    for k in ("g", "h", "z", "y"):
        np.testing.assert_allclose(fw[k], ref[k], rtol=1e-12, atol=1e-12, err_msg=k)
    np.testing.assert_array_equal(bw["unique"], ref["unique"])
    for k in ("dE", "dx", "dW_gate", "dW_down"):
        np.testing.assert_allclose(bw[k], ref[k], rtol=1e-11, atol=1e-11, err_msg=k)


def test_stem_is_staple_with_a_zero_up_projection():
    """h = W_up x + E[id] with W_up = 0 is h = E[id]: the two definitions agree
    exactly on everything STEM has (the STAPLE oracle is pinned on its own)."""
    x, ids, wg, wu, wd, E, dy = _tiny(2)
    zero = np.zeros_like(wu)
    st = oracle.stem_forward(x, ids, wg, wd, E)
    sp = oracle.ffn_forward(x, ids, wg, zero, wd, E)
    for k in ("g", "h", "z", "y"):
        np.testing.assert_array_equal(st[k], sp[k], err_msg=k)
    bs = oracle.stem_backward(dy, x, ids, wg, wd, st)
    bp = oracle.ffn_backward(dy, x, ids, wg, zero, wd, sp)
    for k in ("dh", "dg", "dE", "dx", "dW_gate", "dW_down"):
        np.testing.assert_array_equal(bs[k], bp[k], err_msg=k)
    # with a nonzero up-projection the layers differ (STEM drops it)
    assert not np.allclose(oracle.ffn_forward(x, ids, wg, wu, wd, E)["y"], st["y"])


def test_stem_gradients_match_finite_differences():
    x, ids, wg, _, wd, E, dy = _tiny(5, T=4, D=3, F=4, V=6)

    def loss(x_, wg_, wd_, E_):
        return float(np.sum(dy * oracle.stem_forward(x_, ids, wg_, wd_, E_)["y"]))

    fw = oracle.stem_forward(x, ids, wg, wd, E)
    bw = oracle.stem_backward(dy, x, ids, wg, wd, fw)
    eps = 1e-6
    for name, arr, grad in (("x", x, bw["dx"]), ("W_gate", wg, bw["dW_gate"]),
                            ("W_down", wd, bw["dW_down"])):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a = arr.copy()
            a[idx] += eps
            args_p = [x, wg, wd, E]
            args_p[["x", "W_gate", "W_down"].index(name)] = a
            lp = loss(*args_p)
            a[idx] -= 2 * eps
            args_m = [x, wg, wd, E]
            args_m[["x", "W_gate", "W_down"].index(name)] = a
            lm = loss(*args_m)
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)
    numE = np.zeros_like(E)
    for idx in np.ndindex(E.shape):
        a = E.copy()
        a[idx] += eps
        lp = loss(x, wg, wd, a)
        a[idx] -= 2 * eps
        lm = loss(x, wg, wd, a)
        numE[idx] = (lp - lm) / (2 * eps)
    np.testing.assert_allclose(bw["dE"], numE[bw["unique"]], rtol=1e-6, atol=1e-8)


def test_stem_single_token_table_gradient_closed_form():
    x, ids, wg, _, wd, E, dy = _tiny(6, T=1)
    fw = oracle.stem_forward(x, ids, wg, wd, E)
    bw = oracle.stem_backward(dy, x, ids, wg, wd, fw)
    closed = oracle.silu(wg @ x[0]) * (wd.T @ dy[0])
    np.testing.assert_allclose(bw["dE"][0], closed, rtol=1e-13, atol=1e-13)


def _mutant_stem(kind):
    real = oracle.stem_forward

    def bad(x, ids, wg, wd, table):
        out = real(x, ids, wg, wd, table)
        if kind == "adds_to_gate":
            g = out["g"] + out["h"]
            out["z"] = oracle.silu(g) * out["h"]
        elif kind == "ungated":
            out["z"] = out["h"]
        elif kind == "wrong_row":
            out["z"] = out["a"] * np.asarray(table)[(np.asarray(ids) + 1) % table.shape[0]]
        out["y"] = out["z"] @ np.asarray(wd).T
        return out
    return bad


@pytest.mark.parametrize("kind", ["adds_to_gate", "ungated", "wrong_row"])
def test_planted_stem_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(oracle, "stem_forward", _mutant_stem(kind))
    with pytest.raises(AssertionError):
        test_stem_matches_brute_force(0)
