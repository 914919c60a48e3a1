"""Stacks of STAPLE layers driven through the C ABI: the per-step
orchestration of several augmented layers (host logic only; every step of
the computation runs in the library's kernels).

- x_{l+1} = y_l, and every layer sees the same token ids.  So the batch is
  deduplicated once per step, and one inverse map serves every layer
  (retrieval-path table, Prefill row: dedup once, reuse the inverse map).
- Tables are grouped G adjacent layers per host row, token-major: host array
  [V][G][F] per group (retrieval-path table, Decode row).  One gather per
  group fetches the rows of all G layers.  Later groups are gathered on
  prefetch streams while earlier layers compute, and a layer waits only for
  its own group (Decode row: synchronise when a group is first consumed).
- Training: the backward pass runs the layers in reverse.  Each layer's U
  table-gradient rows go back to host memory on a copy stream while the next
  layer's backward runs.  By default the copy engine moves exactly U rows:
  U reaches pinned host memory right after the dedup, long before the
  backward needs it.  SM stores over the host link (staple_embed_grad_to_host,
  which reads U on the device and so also works inside a captured graph)
  would occupy every SM's store path with slow posted writes and stall the
  concurrent GEMMs' epilogues.  The next step's dedup
  and first-group gather run during this step's backward (successive batches
  are pipelined: retrieval-path table, Prefill row).  No table optimizer runs
  here, so nothing the prefetch reads changes in between.
- Decode: one step (dedup, group gathers, all layers) is captured once in a
  multi-stream CUDA graph and replayed (Decode row: grouped lookups and the
  model in one multi-stream CUDA graph).

torch supplies device memory, pinned host memory, streams and events.
"""
from __future__ import annotations

from dataclasses import dataclass

import token_indexed_sparse_staple_b200 as stp


@dataclass
class LayerWeights:
    w_gate: object   # [F][D] bf16
    w_up: object     # [F][D] bf16
    w_down: object   # [D][F] bf16


class GroupedTables:
    """The host tables of L layers, G layers per host row: group k is a
    page-locked [V][G * F] bf16 array (layer G*k + j in columns [j F, (j+1) F)),
    registered with the library, each with its own hot-row cache."""

    def __init__(self, ctx, host_groups, V: int, F: int, G: int, freq, frac: float):
        self.ctx, self.V, self.F, self.G = ctx, V, F, G
        self.host = list(host_groups)
        self.handles, self.caches = [], []
        try:
            for t in self.host:
                h = stp.staple_table_register(ctx, t, t.numel() * t.element_size(), V, F, G,
                                              stp.STAPLE_BF16, stp.STAPLE_TABLE_HOST_PINNED)
                self.handles.append(h)
                self.caches.append(stp.staple_cache_build(ctx, h, freq, frac))
        except Exception:
            self.close()
            raise

    @property
    def n_groups(self) -> int:
        return len(self.host)

    def close(self):
        for c in self.caches:
            stp.staple_cache_free(c)
        for h in self.handles:
            stp.staple_table_unregister(h)
        self.caches, self.handles = [], []


class Retrieval:
    """One step's retrieval state: a dedup and, per group, the probe results
    and the gathered rows [T][G * F]."""

    def __init__(self, T: int, F: int, G: int, n_groups: int):
        import torch
        i32 = dict(dtype=torch.int32, device="cuda")
        self.T, self.F, self.G = T, F, G
        self.unique, self.inverse, self.sorted_pos = (torch.empty(max(T, 1), **i32) for _ in range(3))
        self.seg, self.U = torch.empty(T + 1, **i32), torch.empty(1, **i32)
        self.slot = [torch.empty(max(T, 1), **i32) for _ in range(n_groups)]
        self.miss = [torch.empty(max(T, 1), **i32) for _ in range(n_groups)]
        self.mc = [torch.empty(1, **i32) for _ in range(n_groups)]
        self.rows = [torch.empty((max(T, 1), G * F), dtype=torch.bfloat16, device="cuda")
                     for _ in range(n_groups)]
        self.ready = [torch.cuda.Event() for _ in range(n_groups)]
        self.free = torch.cuda.Event()   # recorded after the last reader of this step
        self.U_host = torch.zeros(1, dtype=torch.int32, pin_memory=True)
        self.U_known = torch.cuda.Event()  # U_host holds this step's U

    def embed(self, layer: int):
        """The embed argument of layer `layer`: its G-slice of its group's rows,
        indexed by the inverse map."""
        g, j = divmod(layer, self.G)
        base = self.rows[g].data_ptr() + j * self.F * self.rows[g].element_size()
        return stp.make_embed(stp.STAPLE_EMBED_ROWS, base, self.G * self.F, self.inverse, self.T)


def issue_dedup(ctx, r: Retrieval, ids, V: int, stream, u_to_host: bool = True):
    """The batch's dedup on `stream`; with u_to_host, U is also copied to pinned
    host memory (the training stack reads it there; a decode step does not,
    and the copy would sit between the dedup and the first gather)."""
    import torch
    stp.staple_dedup(ctx, ids, r.T, V, r.unique, r.inverse, r.seg, r.sorted_pos, r.U,
                     stream=stream)
    if u_to_host:
        with torch.cuda.stream(stream):
            r.U_host.copy_(r.U, non_blocking=True)   # 4 bytes; read by the host much later
        r.U_known.record(stream)


def issue_group(ctx, r: Retrieval, tables: GroupedTables, g: int, stream, side):
    stp.staple_gather_unique_rows(ctx, tables.caches[g], tables.handles[g], r.unique, r.U, r.T,
                                  r.slot[g], r.miss[g], r.mc[g], r.rows[g], stream=stream,
                                  side=side)
    r.ready[g].record(stream)


# --------------------------------------------------------------------------
# Training stack
# --------------------------------------------------------------------------

@dataclass
class TrainBuffers:
    xs: list                       # x_0 .. x_L: [T][D] bf16 (x_{l+1} = y_l)
    z: list
    g: list
    h: list                        # per layer [T][F] bf16, saved for the backward
    dy: list                       # [T][D] bf16 gradients passed down (two alternating, or L)
    dgh: object                    # [T][2F] bf16, one layer at a time
    dE: list                       # two fp32 [T][F] buffers alternating (copy-out overlap)
    dE_copied: list                # events: the copy of dE[i] to the host has been issued and run
    dW: list                       # per layer (dW_gate, dW_up, dW_down) fp32
    host_dE: list                  # per layer page-locked fp32 [T][F]
    host_unique: list              # per layer page-locked int32 [T]
    host_U: list                   # per layer page-locked int32 [1]
    ws: object
    wsb: int


class TrainStack:
    """L augmented layers, forward and full backward per step, with dE of
    every layer returned to host memory."""

    def __init__(self, ctx, weights: list, tables: GroupedTables, T: int, D: int, F: int, V: int,
                 freeze_up: bool = False, keep_dy: bool = False, de_return: str = "dma"):
        """keep_dy keeps every layer's incoming gradient (L buffers instead of
        two alternating ones), so each layer can be checked on its own inputs.
        de_return: "dma" (copy engine, U known on the host) or "kernel"
        (staple_embed_grad_to_host, U read on the device)."""
        assert de_return in ("dma", "kernel")
        self.de_return = de_return
        import torch
        self.ctx, self.W, self.tables = ctx, weights, tables
        self.T, self.D, self.F, self.V, self.G = T, D, F, V, tables.G
        self.L = len(weights)
        assert self.L == tables.n_groups * self.G
        self.freeze_up = freeze_up
        bf = dict(dtype=torch.bfloat16, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        L = self.L
        wsb = stp.staple_workspace_bytes(T, D, F)
        self.b = TrainBuffers(
            xs=[torch.empty((T, D), **bf) for _ in range(L + 1)],
            z=[torch.empty((T, F), **bf) for _ in range(L)],
            g=[torch.empty((T, F), **bf) for _ in range(L)],
            h=[torch.empty((T, F), **bf) for _ in range(L)],
            dy=[torch.empty((T, D), **bf) for _ in range(L if keep_dy else 2)],
            dgh=torch.empty((T, 2 * F), **bf),
            dE=[torch.empty((T, F), **f32) for _ in range(2)],
            dE_copied=[torch.cuda.Event() for _ in range(2)],
            dW=[(torch.empty((F, D), **f32), None if freeze_up else torch.empty((F, D), **f32),
                 torch.empty((D, F), **f32)) for _ in range(L)],
            host_dE=[torch.empty((T, F), dtype=torch.float32).pin_memory() for _ in range(L)],
            host_unique=[torch.empty(T, dtype=torch.int32).pin_memory() for _ in range(L)],
            host_U=[torch.zeros(1, dtype=torch.int32).pin_memory() for _ in range(L)],
            ws=torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda"), wsb=wsb)
        self.retr = [Retrieval(T, F, self.G, tables.n_groups) for _ in range(2)]
        self.pf, self.pf_side, self.copy = (torch.cuda.Stream() for _ in range(3))
        self.host_ready = torch.cuda.Event()   # the last step's dE rows are in host memory
        self.step_no = 0
        self._primed = None   # (step, ids) whose dedup + group 0 are in flight

    def _prefetch_head(self, r: Retrieval, ids):
        """Dedup and group 0 of a step, on the prefetch streams, once the
        previous user of `r` is done with it."""
        self.pf.wait_event(r.free)
        issue_dedup(self.ctx, r, ids, self.V, self.pf)
        issue_group(self.ctx, r, self.tables, 0, self.pf, self.pf_side)

    def step(self, ids, x0, dy_top, next_ids=None, stream=None):
        """One training step on `stream` (default: torch's current stream).
        ids [T] int32, x0 [T][D] and dy_top [T][D] bf16 on the device.
        next_ids, when given, lets the next step's dedup and first gather run
        during this step's backward; the next step then uses those ids (its
        own `ids` argument is not read again).  Returns the Retrieval used
        (its U_dev, unique ids and hit/miss maps stay valid until the step
        after next).  The step's dE rows reach host memory when host_ready
        completes (wait on it before reading host_dE): later work on `stream`,
        such as the next step's forward, does not wait for the last layer's
        copy-out, since no table optimizer runs between the steps here."""
        import torch
        st = stream or torch.cuda.current_stream()
        b, T, D, F = self.b, self.T, self.D, self.F
        r = self.retr[self.step_no % 2]
        if self._primed is None or self._primed[0] != self.step_no:
            self.pf.wait_stream(st)               # ids may come from this stream
            self._prefetch_head(r, ids)
        for gi in range(1, self.tables.n_groups):
            issue_group(self.ctx, r, self.tables, gi, self.pf, self.pf_side)
        if x0.data_ptr() != b.xs[0].data_ptr():
            with torch.cuda.stream(st):
                b.xs[0].copy_(x0)
        # forward
        for l in range(self.L):
            gi = l // self.G
            if l % self.G == 0:
                st.wait_event(r.ready[gi])
            w = self.W[l]
            stp.staple_ffn_fwd(self.ctx, stp.STAPLE_BF16, T, D, F, b.xs[l], r.embed(l), w.w_gate,
                               w.w_up, w.w_down, b.z[l], b.xs[l + 1], b.g[l], b.h[l], b.ws, b.wsb,
                               stream=st)
        # the next step's dedup and first group while the backward runs
        if next_ids is not None:
            rn = self.retr[(self.step_no + 1) % 2]
            self.pf.wait_stream(st)
            self._prefetch_head(rn, next_ids)
            self._primed = (self.step_no + 1, next_ids)
        # backward, layers in reverse
        if self.de_return == "dma":
            r.U_known.synchronize()               # completed long ago: the dedup ran first
            U = int(r.U_host[0])
        dy = dy_top
        for l in reversed(range(self.L)):
            w = self.W[l]
            k = l % 2
            st.wait_event(b.dE_copied[k])          # dE[k]'s previous copy-out is done
            stp.staple_embed_bwd(self.ctx, stp.STAPLE_BF16, T, D, F, dy, b.g[l], b.h[l], w.w_down,
                                 r.sorted_pos, r.inverse, r.seg, r.U, b.dgh, b.dE[k], b.ws, b.wsb,
                                 stream=st)
            self.copy.wait_stream(st)
            if self.de_return == "dma":
                with torch.cuda.stream(self.copy):
                    b.host_dE[l][:U].copy_(b.dE[k][:U], non_blocking=True)
                    b.host_unique[l][:U].copy_(r.unique[:U], non_blocking=True)
                b.host_U[l][0] = U
            else:
                stp.staple_embed_grad_to_host(self.ctx, F, T, b.dE[k], r.unique, r.U,
                                              b.host_dE[l], b.host_unique[l], b.host_U[l],
                                              stream=self.copy)
            b.dE_copied[k].record(self.copy)
            dx = b.dy[l % len(b.dy)]   # the gradient layer l passes down (layer l-1's dy)
            dwg, dwu, dwd = b.dW[l]
            stp.staple_ffn_bwd(self.ctx, stp.STAPLE_BF16, T, D, F, dy, b.xs[l], b.z[l], b.dgh,
                               w.w_gate, w.w_up, dx, dwg, dwu, dwd, stream=st)
            dy = dx
        r.free.record(self.copy)                   # after the last reader (layer 0's copy-out)
        self.host_ready.record(self.copy)
        self.step_no += 1
        return r


# --------------------------------------------------------------------------
# Decode stack
# --------------------------------------------------------------------------

class DecodeStack:
    """L augmented layers at decode sizes (T <= 256): one step = dedup,
    group gathers on prefetch streams, the L fused decode layers.  capture()
    records a step into a CUDA graph; replay() runs it for the ids currently
    in `ids_buf`."""

    def __init__(self, ctx, weights: list, tables: GroupedTables, T: int, D: int, F: int, V: int):
        import torch
        self.ctx, self.W, self.tables = ctx, weights, tables
        self.T, self.D, self.F, self.V, self.G = T, D, F, V, tables.G
        self.L = len(weights)
        assert self.L == tables.n_groups * self.G
        bf = dict(dtype=torch.bfloat16, device="cuda")
        self.ids_buf = torch.zeros(T, dtype=torch.int32, device="cuda")
        self.xs = [torch.empty((T, D), **bf) for _ in range(self.L + 1)]
        self.z = torch.empty((T, F), **bf)
        self.wsb = stp.staple_workspace_bytes(T, D, F)
        self.ws = torch.zeros(self.wsb, dtype=torch.uint8, device="cuda")
        self.r = Retrieval(T, F, self.G, tables.n_groups)
        self.pf, self.pf_side = torch.cuda.Stream(), torch.cuda.Stream()
        self.graph = None

    def run(self, stream=None):
        """One step for ids_buf and xs[0]; y of the last layer in xs[L]."""
        import torch
        st = stream or torch.cuda.current_stream()
        r = self.r
        self.pf.wait_stream(st)
        issue_dedup(self.ctx, r, self.ids_buf, self.V, self.pf, u_to_host=False)
        for gi in range(self.tables.n_groups):
            issue_group(self.ctx, r, self.tables, gi, self.pf, self.pf_side)
        for l in range(self.L):
            if l % self.G == 0:
                st.wait_event(r.ready[l // self.G])
            w = self.W[l]
            stp.staple_ffn_fwd(self.ctx, stp.STAPLE_BF16, self.T, self.D, self.F, self.xs[l],
                               r.embed(l), w.w_gate, w.w_up, w.w_down, self.z, self.xs[l + 1],
                               None, None, self.ws, self.wsb, stream=st)
        st.wait_stream(self.pf)                    # join the prefetch streams (graph capture)

    def capture(self, stream, ids_src=None, x_src=None):
        """Record a step into a CUDA graph (kept for replay() and returned).
        With ids_src / x_src the graph first copies them into ids_buf /
        xs[0], so that a set of graphs feeds recorded inputs with no copy
        outside the graphs."""
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            if ids_src is not None:
                self.ids_buf.copy_(ids_src)
            if x_src is not None:
                self.xs[0].copy_(x_src)
            self.run(stream)
        self.graph = g
        return g

    def replay(self):
        self.graph.replay()

    def release(self):
        self.graph = None
