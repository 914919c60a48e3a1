"""Stacks of augmented layers through token_indexed_sparse_staple_b200.stack.
Tables are grouped four layers per host row, in pinned host memory with a 5 %
cache.  The batch is deduplicated once per step and each group is gathered on
prefetch streams.

Each layer is checked against the oracle on its own inputs as the GPU produced
them: its x, and in training the gradient passed down from the layer above.
So errors do not compound down the stack.  Retrieval is checked bit for bit
per group.  The training stack also returns every layer's dE to host memory,
which is compared with the oracle's dE.  The decode stack runs from a
captured CUDA graph, replayed for several id batches."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synthetic as syn
from tests.helpers import TOL, assert_close, bits, dev, f64

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


def _stack_inputs(L, G, D, F, V, w_std=0.05, e_std=0.05):
    """Per-layer weights and tables (numpy bf16 bits), tables grouped G per host row."""
    layers = []
    for l in range(L):
        wg = syn.bf16_normal((F, D), w_std, syn.SEED_W + 3 * l)[0]
        wu = syn.bf16_normal((F, D), w_std, syn.SEED_W + 3 * l + 1)[0]
        wd = syn.bf16_normal((D, F), w_std, syn.SEED_W + 3 * l + 2)[0]
        E = syn.bf16_normal((V, F), e_std, syn.SEED_E + l)[0]
        layers.append((wg, wu, wd, E))
    groups = [np.ascontiguousarray(np.stack([layers[g * G + j][3] for j in range(G)], axis=1)
                                   .reshape(V, G * F)) for g in range(L // G)]
    return layers, groups


def _build(stp, ctx, layers, groups, V, F, G, freq):
    import torch
    from token_indexed_sparse_staple_b200.stack import GroupedTables, LayerWeights
    W = [LayerWeights(dev(wg, "bf16"), dev(wu, "bf16"), dev(wd, "bf16")) for wg, wu, wd, _ in layers]
    host = [torch.from_numpy(gr.view(np.int16)).pin_memory() for gr in groups]
    return W, GroupedTables(ctx, host, V, F, G, freq, 0.05)


def _f64b(a):
    return syn.bf16_bits_to_f32(a).astype(np.float64)


@pytest.mark.parametrize("de_return", ["dma", "kernel"])
def test_train_stack_matches_oracle_per_layer(stp, ctx, de_return):
    import torch

    from token_indexed_sparse_staple_b200.stack import TrainStack
    L, G, T, D, F, V = 8, 4, 300, 128, 256, 1000
    layers, groups = _stack_inputs(L, G, D, F, V)
    freq = syn.calibration_freq(V, n_tokens=1 << 18)
    W, tables = _build(stp, ctx, layers, groups, V, F, G, freq)
    try:
        s = TrainStack(ctx, W, tables, T, D, F, V, keep_dy=True, de_return=de_return)
        for step in range(2):       # two steps: the second finds its head prefetched
            ids = syn.zipf_ids(T, V, 1.1, seed=50 + step)
            nxt = syn.zipf_ids(T, V, 1.1, seed=51 + step)
            x0 = dev(syn.bf16_normal((T, D), 1.0, 60 + step)[0], "bf16")
            dyt = dev(syn.bf16_normal((T, D), 1.0, 70 + step)[0], "bf16")
            r = s.step(torch.from_numpy(ids).cuda(), x0, dyt,
                       next_ids=torch.from_numpy(nxt).cuda() if step == 0 else None)
            s.host_ready.synchronize()   # this step's dE rows are in host memory
            torch.cuda.synchronize()
            assert stp.staple_get_error(ctx) == 0
            u_ref, _, _, _ = oracle.dedup(ids)
            U = int(r.U.item())
            assert U == u_ref.size
            np.testing.assert_array_equal(r.unique.cpu().numpy()[:U], u_ref)
            for g in range(L // G):
                np.testing.assert_array_equal(bits(r.rows[g])[:U], oracle.gather_rows(groups[g], u_ref))
            b = s.b
            for l in range(L):
                wg, wu, wd, E = (_f64b(a) for a in layers[l])
                x = f64(b.xs[l])
                fw = oracle.ffn_forward(x, ids, wg, wu, wd, E)
                assert_close(f64(b.xs[l + 1]), fw["y"], TOL["bf16"], f"y layer {l}")
                assert_close(f64(b.z[l]), fw["z"], TOL["bf16"], f"z layer {l}")
                dy = f64(dyt) if l == L - 1 else f64(b.dy[l + 1])
                bw = oracle.ffn_backward(dy, x, ids, wg, wu, wd, fw)
                assert int(b.host_U[l][0]) == U
                np.testing.assert_array_equal(b.host_unique[l].numpy()[:U], u_ref)
                assert_close(b.host_dE[l].numpy()[:U].astype(np.float64), bw["dE"], TOL["bf16"],
                             f"host dE layer {l}")
                dwg, dwu, dwd = b.dW[l]
                assert_close(f64(dwg), bw["dW_gate"], TOL["bf16"], f"dW_gate layer {l}")
                assert_close(f64(dwu), bw["dW_up"], TOL["bf16"], f"dW_up layer {l}")
                assert_close(f64(dwd), bw["dW_down"], TOL["bf16"], f"dW_down layer {l}")
                assert_close(f64(b.dy[l]), bw["dx"], TOL["bf16"], f"dx layer {l}")
    finally:
        tables.close()


def test_decode_stack_graph_matches_oracle_per_layer(stp, ctx):
    import torch

    from token_indexed_sparse_staple_b200.stack import DecodeStack
    L, G, T, D, F, V = 8, 4, 64, 128, 256, 1000
    layers, groups = _stack_inputs(L, G, D, F, V)
    freq = syn.calibration_freq(V, n_tokens=1 << 18)
    W, tables = _build(stp, ctx, layers, groups, V, F, G, freq)
    try:
        s = DecodeStack(ctx, W, tables, T, D, F, V)
        st = torch.cuda.Stream()
        # warm up once outside the graph, then capture
        with torch.cuda.stream(st):
            s.run(st)
        torch.cuda.synchronize()
        s.capture(st)
        for rep in range(3):
            ids = syn.zipf_ids(T, V, 1.1, seed=80 + rep)
            s.ids_buf.copy_(torch.from_numpy(ids))
            s.xs[0].copy_(dev(syn.bf16_normal((T, D), 1.0, 90 + rep)[0], "bf16"))
            torch.cuda.synchronize()
            with torch.cuda.stream(st):
                s.replay()
            torch.cuda.synchronize()
            assert stp.staple_get_error(ctx) == 0
            u_ref = oracle.dedup(ids)[0]
            U = int(s.r.U.item())
            assert U == u_ref.size
            for g in range(L // G):
                np.testing.assert_array_equal(bits(s.r.rows[g])[:U], oracle.gather_rows(groups[g], u_ref))
            for l in range(L):
                wg, wu, wd, E = (_f64b(a) for a in layers[l])
                fw = oracle.ffn_forward(f64(s.xs[l]), ids, wg, wu, wd, E)
                assert_close(f64(s.xs[l + 1]), fw["y"], TOL["bf16"], f"replay {rep} y layer {l}")
        s.release()
    finally:
        tables.close()


def test_decode_stack_graphs_with_recorded_inputs(stp, ctx):
    """One captured step graph per batch, each copying its own ids and x in
    (capture with ids_src / x_src): replayed out of capture order, every
    replay computes its own batch, checked per layer against the oracle."""
    import torch

    from token_indexed_sparse_staple_b200.stack import DecodeStack
    L, G, T, D, F, V = 4, 4, 64, 128, 256, 1000
    layers, groups = _stack_inputs(L, G, D, F, V)
    freq = syn.calibration_freq(V, n_tokens=1 << 18)
    W, tables = _build(stp, ctx, layers, groups, V, F, G, freq)
    try:
        s = DecodeStack(ctx, W, tables, T, D, F, V)
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            s.run(st)
        torch.cuda.synchronize()
        batches = [syn.zipf_ids(T, V, 1.1, seed=180 + k) for k in range(3)]
        ids_src = [torch.from_numpy(b).cuda() for b in batches]
        x_src = [dev(syn.bf16_normal((T, D), 1.0, 190 + k)[0], "bf16") for k in range(3)]
        graphs = [s.capture(st, ids_src[k], x_src[k]) for k in range(3)]
        for k in (2, 0, 1, 2):
            with torch.cuda.stream(st):
                graphs[k].replay()
            torch.cuda.synchronize()
            assert stp.staple_get_error(ctx) == 0
            assert torch.equal(s.ids_buf, ids_src[k])
            for l in range(L):
                wg, wu, wd, E = (_f64b(a) for a in layers[l])
                fw = oracle.ffn_forward(f64(s.xs[l]), batches[k], wg, wu, wd, E)
                assert_close(f64(s.xs[l + 1]), fw["y"], TOL["bf16"], f"batch {k} y layer {l}")
            np.testing.assert_array_equal(f64(s.xs[0]), f64(x_src[k]))
        del graphs
        s.release()
    finally:
        tables.close()
