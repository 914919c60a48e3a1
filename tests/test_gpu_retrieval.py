"""GPU parity of the retrieval path (dedup, cache build, probe, hit and miss
gathers) against the oracle: bit-exact for every index and every row byte."""
import numpy as np
import pytest

import oracle
import synthetic as syn
from tests.helpers import bits, dev, empty, read_device

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


def run_dedup(stp, ctx, ids, V):
    import torch
    T = len(ids)
    d_ids = torch.from_numpy(np.asarray(ids, dtype=np.int32)).cuda()
    out = {k: empty(max(T, 1), "i32") for k in ("unique", "inverse", "sorted_pos")}
    seg = empty(T + 1, "i32")
    U = empty(1, "i32")
    stp.staple_dedup(ctx, d_ids, T, V, out["unique"], out["inverse"], seg, out["sorted_pos"], U)
    assert stp.staple_get_error(ctx) == 0
    u = int(U.item())
    return (out["unique"].cpu().numpy()[:u], out["inverse"].cpu().numpy()[:T],
            seg.cpu().numpy()[:u + 1], out["sorted_pos"].cpu().numpy()[:T])


CASES = {
    "empty": ([], 10),
    "one": ([7], 10),
    "all_equal": ([3] * 1000, 10),
    "all_distinct": (list(range(999, -1, -1)), 1000),
    "edges": ([0, 99999, 0, 99999, 5], 100000),
    "V_is_1": ([0, 0, 0], 1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_dedup_edge_cases(stp, ctx, name):
    ids, V = CASES[name]
    got = run_dedup(stp, ctx, ids, V)
    ref = oracle.dedup(np.array(ids, dtype=np.int32))
    for g, r, what in zip(got, ref, ("unique", "inverse", "seg_off", "sorted_pos")):
        np.testing.assert_array_equal(g, r, err_msg=what)


@pytest.mark.parametrize("T,V", [(64, 100352), (256, 1000), (1025, 100352), (4097, 50000),
                                 (16384, 100352), (32768, 100352), (16384, 1 << 20)])
def test_dedup_zipf(stp, ctx, T, V):
    ids = syn.zipf_ids(T, V, 1.1, seed=T + V)
    got = run_dedup(stp, ctx, ids, V)
    ref = oracle.dedup(ids)
    for g, r, what in zip(got, ref, ("unique", "inverse", "seg_off", "sorted_pos")):
        np.testing.assert_array_equal(g, r, err_msg=what)


def test_dedup_reports_out_of_range_ids(stp, ctx):
    import torch
    ids = torch.tensor([1, 2, 10, 3], dtype=torch.int32, device="cuda")
    bufs = [empty(4, "i32") for _ in range(3)]
    seg, U = empty(5, "i32"), empty(1, "i32")
    stp.staple_dedup(ctx, ids, 4, 10, bufs[0], bufs[1], seg, bufs[2], U)
    assert stp.staple_get_error(ctx) == stp.STAPLE_EIDRANGE
    assert stp.staple_get_error(ctx) == 0   # reading clears the word


def _table(w, layer=0, groups=1):
    """[V][groups*F] bf16 table (groups stacked layers, token-major)."""
    parts = [syn.bf16_normal((w.V, w.F), w.e_std, syn.SEED_E + layer + g)[0] for g in range(groups)]
    return np.ascontiguousarray(np.stack(parts, axis=1).reshape(w.V, groups * w.F))


@pytest.mark.parametrize("where", ["device", "host"])
@pytest.mark.parametrize("frac", [0.0, 0.05, 1.0])
@pytest.mark.parametrize("groups", [1, 4])
def test_cache_and_gather(stp, ctx, where, frac, groups):
    import torch
    w = syn.Workload("small", T=3000, D=64, F=128, V=5000, layers=groups, dtype="bf16",
                     w_std=0.02, e_std=0.01, x_std=1.0, dy_std=1.0, table=where, cache_frac=frac,
                     group=groups, training=False)
    E = _table(w, groups=groups)
    if where == "device":
        t_store = dev(E, "bf16")
        flags = stp.STAPLE_TABLE_DEVICE
    else:
        t_store = torch.from_numpy(E.view(np.int16)).pin_memory()
        flags = stp.STAPLE_TABLE_HOST_PINNED
    table = stp.staple_table_register(ctx, t_store, E.nbytes, w.V, w.F, groups, stp.STAPLE_BF16, flags)
    freq = syn.calibration_freq(w.V, n_tokens=1 << 18)
    cache = stp.staple_cache_build(ctx, table, freq, frac)
    try:
        hot_ref, slot_of = oracle.hot_set(freq, frac)
        np.testing.assert_array_equal(stp.staple_cache_hot_ids(cache), hot_ref)
        K, cap = stp.staple_cache_info(cache)
        assert K == hot_ref.size and cap >= 2 * K and cap & (cap - 1) == 0
        if K:
            raw = read_device(stp.staple_cache_rows(cache), K * groups * w.F * 2)
            np.testing.assert_array_equal(raw.view(np.uint16).reshape(K, groups * w.F),
                                          oracle.cache_rows_for(E, hot_ref))

        ids = syn.zipf_ids(w.T, w.V, 1.1, seed=5)
        T = w.T
        d_ids = torch.from_numpy(ids).cuda()
        unique, inverse, sorted_pos, slot, miss = (empty(T, "i32") for _ in range(5))
        seg, U, mc = empty(T + 1, "i32"), empty(1, "i32"), empty(1, "i32")
        rows = torch.zeros((T, groups * w.F), dtype=torch.bfloat16, device="cuda")
        side = torch.cuda.Stream()
        stp.staple_gather_rows(ctx, cache, table, d_ids, T, unique, inverse, seg, sorted_pos, U,
                               slot, miss, mc, rows, side=side)
        assert stp.staple_get_error(ctx) == 0
        u_ref, inv_ref, _, _ = oracle.dedup(ids)
        slot_ref, miss_ref = oracle.probe(u_ref, slot_of)
        Ug = int(U.item())
        assert Ug == u_ref.size
        np.testing.assert_array_equal(slot.cpu().numpy()[:Ug], slot_ref)
        assert int(mc.item()) == miss_ref.size
        np.testing.assert_array_equal(miss.cpu().numpy()[:miss_ref.size], miss_ref)
        np.testing.assert_array_equal(bits(rows)[:Ug], oracle.gather_rows(E, u_ref))
        if frac == 0.05:
            # Zipf stream: most tokens hit a 5% cache
            hit_tokens = np.mean(slot_ref[inv_ref] >= 0)
            assert hit_tokens > 0.6
    finally:
        stp.staple_cache_free(cache)
        stp.staple_table_unregister(table)


def test_register_pageable_host_table(stp, ctx):
    import torch
    import mmap
    E = syn.bf16_normal((300, 64), 0.01, 3)[0]
    mm = mmap.mmap(-1, E.nbytes)   # page-aligned pageable memory
    host = np.frombuffer(mm, dtype=np.uint16).reshape(E.shape)
    host[:] = E
    table = stp.staple_table_register(ctx, host, host.nbytes, 300, 64, 1, stp.STAPLE_BF16,
                                      stp.STAPLE_TABLE_HOST_REGISTER)
    try:
        ids = np.array([5, 299, 5, 0], dtype=np.int32)
        T = 4
        d_ids = torch.from_numpy(ids).cuda()
        bufs = [empty(T, "i32") for _ in range(5)]
        seg, U, mc = empty(T + 1, "i32"), empty(1, "i32"), empty(1, "i32")
        rows = torch.zeros((T, 64), dtype=torch.bfloat16, device="cuda")
        stp.staple_gather_rows(ctx, None, table, d_ids, T, bufs[0], bufs[1], seg, bufs[2], U,
                               bufs[3], bufs[4], mc, rows)
        assert stp.staple_get_error(ctx) == 0
        np.testing.assert_array_equal(bits(rows)[:3], E[[0, 5, 299]])
        assert int(mc.item()) == 3
    finally:
        stp.staple_table_unregister(table)


def test_cache_refresh_after_host_adamw(stp, ctx):
    """After the host AdamW updates a batch's rows, staple_cache_refresh
    re-reads the cached ones: cached copies of the batch's hot ids equal the
    updated table rows, the other cached rows are untouched, and a new gather
    returns the updated table bit for bit (hits from the cache, misses from the
    host).  Two grouped layers per host row; the optimizer updates layer 1."""
    import torch
    V, F, G, T = 4000, 128, 2, 2500
    parts = [syn.bf16_normal((V, F), 0.05, 500 + g)[0] for g in range(G)]
    E = np.ascontiguousarray(np.stack(parts, axis=1).reshape(V, G * F))
    host = torch.from_numpy(E.view(np.int16)).pin_memory()
    table = stp.staple_table_register(ctx, host, E.nbytes, V, F, G, stp.STAPLE_BF16,
                                      stp.STAPLE_TABLE_HOST_PINNED)
    freq = syn.calibration_freq(V, n_tokens=1 << 18)
    cache = stp.staple_cache_build(ctx, table, freq, 0.05)
    try:
        hot = stp.staple_cache_hot_ids(cache)
        K = hot.size
        ids = syn.zipf_ids(T, V, 1.1, seed=77)
        d_ids = torch.from_numpy(ids).cuda()
        unique, inverse, sorted_pos, slot, miss = (empty(T, "i32") for _ in range(5))
        seg, U, mc = empty(T + 1, "i32"), empty(1, "i32"), empty(1, "i32")
        rows = torch.zeros((T, G * F), dtype=torch.bfloat16, device="cuda")
        stp.staple_gather_rows(ctx, cache, table, d_ids, T, unique, inverse, seg, sorted_pos, U,
                               slot, miss, mc, rows)
        torch.cuda.synchronize()
        u = int(U.item())
        uniq = unique.cpu().numpy()[:u].copy()
        cache_before = read_device(stp.staple_cache_rows(cache), K * G * F * 2).view(np.uint16)
        cache_before = cache_before.reshape(K, G * F).copy()
        # host AdamW on layer 1 of the batch's rows (the pinned buffer itself)
        rng = np.random.default_rng(78)
        grad = (rng.standard_normal((u, F)) * 0.1).astype(np.float32)
        m = np.zeros((V, F), np.float32)
        v = np.zeros((V, F), np.float32)
        stp.staple_adamw_rows(host.data_ptr() + F * 2, G * F, stp.STAPLE_BF16, F, uniq, u, grad, F,
                              m, v, F, lr=1e-2, beta1=0.9, beta2=0.999, eps=1e-8,
                              weight_decay=0.0, step=1, threads=4)
        updated = host.numpy().view(np.uint16).reshape(V, G * F).copy()
        assert not np.array_equal(updated[uniq], E[uniq])          # the rows did change
        stp.staple_cache_refresh(ctx, cache, table, unique, slot, U)
        torch.cuda.synchronize()
        assert stp.staple_get_error(ctx) == 0
        cache_after = read_device(stp.staple_cache_rows(cache), K * G * F * 2).view(np.uint16)
        cache_after = cache_after.reshape(K, G * F)
        in_batch = np.isin(hot, uniq)
        assert in_batch.any() and (~in_batch).any()
        np.testing.assert_array_equal(cache_after[in_batch], updated[hot[in_batch]])
        np.testing.assert_array_equal(cache_after[~in_batch], cache_before[~in_batch])
        # a new gather sees the updated rows, hits and misses alike
        rows2 = torch.zeros_like(rows)
        stp.staple_gather_rows(ctx, cache, table, d_ids, T, unique, inverse, seg, sorted_pos, U,
                               slot, miss, mc, rows2)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bits(rows2)[:u], updated[uniq])
    finally:
        stp.staple_cache_free(cache)
        stp.staple_table_unregister(table)


@pytest.mark.parametrize("frac,groups,chunk,threads", [(0.05, 1, 256, 4), (0.0, 1, 7, 1),
                                                       (0.05, 4, 1, 0), (1.0, 2, 64, 2),
                                                       # one chunk larger than the batch, and
                                                       # the largest chunk size the call takes
                                                       (0.05, 1, 5000, 2), (0.0, 1, 2**31 - 1, 0)])
def test_bulk_miss_path_equals_zero_copy(stp, ctx, frac, groups, chunk, threads):
    """The prefill path (misses packed on the host, bulk copy, scatter) gives
    the same rows, hit/miss map and miss list as the zero-copy gather, bit for
    bit, and both equal the oracle's rows; two calls in a row on one stream
    reuse the staging buffers."""
    import torch
    V, F, T = 3000, 128, 2000
    w = syn.Workload("bulk", T=T, D=64, F=F, V=V, layers=groups, dtype="bf16", w_std=0.02,
                     e_std=0.05, x_std=1.0, dy_std=1.0, table="host", cache_frac=frac,
                     group=groups, training=False)
    E = _table(w, groups=groups)
    host = torch.from_numpy(E.view(np.int16)).pin_memory()
    table = stp.staple_table_register(ctx, host, E.nbytes, V, F, groups, stp.STAPLE_BF16,
                                      stp.STAPLE_TABLE_HOST_PINNED)
    cache = stp.staple_cache_build(ctx, table, syn.calibration_freq(V, n_tokens=1 << 18), frac)
    try:
        st = torch.cuda.Stream()
        staging_h = torch.empty((T, groups * F), dtype=torch.bfloat16).pin_memory()
        staging_d = torch.empty((T, groups * F), dtype=torch.bfloat16, device="cuda")
        list_h = torch.empty(1 + 2 * T, dtype=torch.int32).pin_memory()
        for rep in range(2):
            ids = syn.zipf_ids(T, V, 1.1, seed=90 + rep)
            d_ids = torch.from_numpy(ids).cuda()
            unique, inverse, sorted_pos = (empty(T, "i32") for _ in range(3))
            seg, U = empty(T + 1, "i32"), empty(1, "i32")
            stp.staple_dedup(ctx, d_ids, T, V, unique, inverse, seg, sorted_pos, U, stream=st)
            out = {}
            for path in ("zero_copy", "bulk"):
                slot, miss = empty(T, "i32"), empty(T, "i32")
                mc = empty(1, "i32")
                rows = torch.zeros((T, groups * F), dtype=torch.bfloat16, device="cuda")
                if path == "bulk":
                    stp.staple_gather_unique_rows_bulk(ctx, cache, table, unique, U, T, slot, miss,
                                                       mc, rows, staging_h, staging_d, list_h,
                                                       chunk_rows=chunk, threads=threads, stream=st)
                else:
                    stp.staple_gather_unique_rows(ctx, cache, table, unique, U, T, slot, miss, mc,
                                                  rows, stream=st, side=st)
                st.synchronize()
                u = int(U.item())
                out[path] = (bits(rows)[:u], slot.cpu().numpy()[:u], int(mc.item()),
                             miss.cpu().numpy()[:int(mc.item())])
            assert stp.staple_get_error(ctx, st) == 0
            zr, zs, zc, zm = out["zero_copy"]
            br, bs, bc, bm = out["bulk"]
            np.testing.assert_array_equal(br, zr)
            np.testing.assert_array_equal(bs, zs)
            assert bc == zc
            np.testing.assert_array_equal(bm, zm)
            u_ref = oracle.dedup(ids)[0]
            np.testing.assert_array_equal(br, oracle.gather_rows(E, u_ref))
    finally:
        stp.staple_cache_free(cache)
        stp.staple_table_unregister(table)


def test_injected_allocation_failures_return_enomem(stp, ctx, monkeypatch):
    """Fault injection on the host: STAPLE_FAIL_ALLOC names an allocation
    site, and that allocation fails as if the device were out of memory.  The
    call returns STAPLE_ENOMEM, frees what it had allocated, and works again
    once the variable is gone."""
    V, F = 64, 64
    table = dev(syn.bf16_normal((V, F), 0.01, 3)[0], "bf16")
    th = stp.staple_table_register(ctx, table, V * F * 2, V, F, 1, stp.STAPLE_BF16,
                                   stp.STAPLE_TABLE_DEVICE)
    freq = np.arange(V, dtype=np.int64)
    try:
        for site in ("cache_rows", "cache_hash", "cache_hot", "all"):
            monkeypatch.setenv("STAPLE_FAIL_ALLOC", site)
            with pytest.raises(stp.StapleError) as ex:
                stp.staple_cache_build(ctx, th, freq, 0.25)
            assert ex.value.status == stp.STAPLE_ENOMEM, site
        monkeypatch.setenv("STAPLE_FAIL_ALLOC", "context_err")
        with pytest.raises(stp.StapleError) as ex:
            stp.staple_context_create(0)
        assert ex.value.status == stp.STAPLE_ENOMEM
        monkeypatch.delenv("STAPLE_FAIL_ALLOC")
        cache = stp.staple_cache_build(ctx, th, freq, 0.25)
        np.testing.assert_array_equal(stp.staple_cache_hot_ids(cache),
                                      oracle.hot_set(freq, 0.25)[0])
        stp.staple_cache_free(cache)
        assert stp.staple_get_error(ctx) == 0
    finally:
        stp.staple_table_unregister(th)
