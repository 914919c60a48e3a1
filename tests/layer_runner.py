"""Run one STAPLE layer (forward, optionally backward) through the C ABI on
seeded inputs and return every output as numpy; the GPU parity tests compare
these against the oracle."""
from __future__ import annotations

import numpy as np

from tests.helpers import dev, empty, f64


def run_layer(stp, ctx, inp, D, F, V, *, embed="table", training=True, rows_table=None,
              freeze_up=False, cache_frac=None, freq=None, stem=False):
    """inp: synthetic.LayerInputs.  embed in {"none", "table", "rows"}.
    rows_table: host numpy table registered as pinned host memory for the
    "rows" mode (default: the device table).  stem: the STEM layer (the row
    replaces the up-projection; W_up is passed as NULL)."""
    import torch
    dt = inp.dtype
    sdt = stp.STAPLE_BF16 if dt == "bf16" else stp.STAPLE_F32
    T = inp.ids.size
    x, wg, wu, wd = (dev(getattr(inp, k), dt) for k in ("x", "w_gate", "w_up", "w_down"))
    embed_flags = stp.STAPLE_EMBED_REPLACE_UP if stem else 0
    if stem:
        wu = None
    ids = torch.from_numpy(inp.ids).cuda()
    z, g, h = (empty((T, F), dt) for _ in range(3))
    y = empty((T, D), dt)
    out = {}
    keep = []
    unique = inverse = sorted_pos = seg = U = None
    table_handle = cache = None
    if embed == "none":
        e = stp.make_embed(stp.STAPLE_EMBED_NONE)
    elif embed == "table":
        tab = dev(inp.table, dt)
        keep.append(tab)
        e = stp.make_embed(stp.STAPLE_EMBED_TABLE, tab, F, ids, V, flags=embed_flags)
    else:
        unique, inverse, sorted_pos, slot, miss = (empty(max(T, 1), "i32") for _ in range(5))
        seg, U, mc = empty(T + 1, "i32"), empty(1, "i32"), empty(1, "i32")
        if rows_table is None:
            tab = dev(inp.table, dt)
            flags = stp.STAPLE_TABLE_DEVICE
        else:
            tab = torch.from_numpy(rows_table.view(np.int16) if dt == "bf16" else rows_table).pin_memory()
            flags = stp.STAPLE_TABLE_HOST_PINNED
        keep.append(tab)
        esz = 2 if dt == "bf16" else 4
        table_handle = stp.staple_table_register(ctx, tab, V * F * esz, V, F, 1, sdt, flags)
        if cache_frac is not None:
            cache = stp.staple_cache_build(ctx, table_handle, freq, cache_frac)
        rows = empty((max(T, 1), F), dt)
        side = torch.cuda.Stream()
        stp.staple_gather_rows(ctx, cache, table_handle, ids, T, unique, inverse, seg, sorted_pos, U,
                               slot, miss, mc, rows, side=side)
        e = stp.make_embed(stp.STAPLE_EMBED_ROWS, rows, F, inverse, max(T, 1), flags=embed_flags)
        keep.append(rows)
        out["miss_count"] = int(mc.item())
    wsb = stp.staple_workspace_bytes(T, D, F)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    try:
        stp.staple_ffn_fwd(ctx, sdt, T, D, F, x, e, wg, wu, wd, z, y,
                           g if training else None, h if training else None, ws, wsb)
        err = stp.staple_get_error(ctx)
        assert err == 0, stp.staple_status_string(err)
        out.update(z=f64(z), y=f64(y))
        if training:
            out.update(g=f64(g), h=f64(h))
            if unique is None:
                unique, inverse, sorted_pos = (empty(max(T, 1), "i32") for _ in range(3))
                seg, U = empty(T + 1, "i32"), empty(1, "i32")
                stp.staple_dedup(ctx, ids, T, V, unique, inverse, seg, sorted_pos, U)
            dy = dev(inp.dy, dt)
            dgh = empty((T, 2 * F), dt)
            dE = torch.zeros((max(T, 1), F), dtype=torch.float32, device="cuda")
            stp.staple_embed_bwd(ctx, sdt, T, D, F, dy, g, h, wd, sorted_pos, inverse, seg, U, dgh,
                                 dE, ws, wsb)
            dx = empty((T, D), dt)
            dwg = torch.empty((F, D), dtype=torch.float32, device="cuda")
            dwu = torch.full((F, D), 7.0, dtype=torch.float32, device="cuda")
            dwd = torch.empty((D, F), dtype=torch.float32, device="cuda")
            stp.staple_ffn_bwd(ctx, sdt, T, D, F, dy, x, z, dgh, wg, wu, dx, dwg,
                               None if (freeze_up or stem) else dwu, dwd)
            err = stp.staple_get_error(ctx)
            assert err == 0, stp.staple_status_string(err)
            u = int(U.item())
            out.update(U=u, unique=unique.cpu().numpy()[:u], dE=f64(dE)[:u], dg=f64(dgh)[:, :F],
                       dh=f64(dgh)[:, F:], dx=f64(dx), dW_gate=f64(dwg), dW_up=f64(dwu),
                       dW_down=f64(dwd))
    finally:
        if cache is not None:
            stp.staple_cache_free(cache)
        if table_handle is not None:
            stp.staple_table_unregister(table_handle)
    return out
