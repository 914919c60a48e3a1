"""fp64 definition of the STAPLE FFN layer, its retrieval steps and gradients.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may import it and
for the source tags [ABS], [AIS], [RADIO], [TLA]).

Notation: T tokens, D = d_model, F = d_ff, V = vocabulary, U = distinct ids in
the batch.  Weights use the [out][in] layout: W_gate, W_up in [F][D],
W_down in [D][F]; the table E is [V][F].  All real arithmetic is float64 on
the exact values the GPU receives (bf16 or fp32 storage widened to fp64); the
oracle rounds nothing.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "silu", "silu_grad", "dedup", "hot_set", "probe", "gather_rows",
    "ffn_forward", "ffn_backward", "forward_rows", "embed_grad_rows",
    "weight_grad_entries", "dx_rows", "cache_rows_for", "paper_shapes", "adamw_rows",
    "stem_forward", "stem_backward",
]


# --------------------------------------------------------------------------
# Activation
# --------------------------------------------------------------------------

def silu(g: np.ndarray) -> np.ndarray:
    """SiLU(g) = g * sigmoid(g), the gate non-linearity of a SwiGLU FFN.
    Reading: OLMo-2's FFN is SwiGLU with no biases; the pages add nothing to it."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d SiLU / dg = s(g) * (1 + g * (1 - s(g))), s the logistic sigmoid."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


# --------------------------------------------------------------------------
# Retrieval: dedup, hot-row cache, gather  ([TLA] retrieval-path table)
# --------------------------------------------------------------------------

def dedup(ids: np.ndarray):
    """Deduplicate a batch's token ids once ([TLA] retrieval-path table,
    Prefill row; the inverse map is reused by every augmented layer).

    Returns (unique, inverse, seg_off, sorted_pos), all int32:
      unique[U]      distinct ids in ascending order (reading: the pages do not
                     fix an order; ascending is the sorted-unique convention)
      inverse[T]     unique[inverse[i]] == ids[i]
      seg_off[U+1]   tokens with id unique[j] are sorted_pos[seg_off[j]:seg_off[j+1]]
      sorted_pos[T]  token positions ordered by (id, position)
    """
    ids = np.asarray(ids, dtype=np.int64).reshape(-1)
    unique, inverse = np.unique(ids, return_inverse=True)
    sorted_pos = np.argsort(ids, kind="stable")
    counts = np.bincount(inverse.reshape(-1), minlength=unique.size)
    seg_off = np.concatenate([[0], np.cumsum(counts)])
    return (unique.astype(np.int32), inverse.reshape(-1).astype(np.int32),
            seg_off.astype(np.int32), sorted_pos.astype(np.int32))


def hot_set(freq: np.ndarray, frac: float):
    """The frequency-aware GPU cache: the ceil(frac * V) most frequent rows
    ([ABS]: about 5% of embeddings cached on the GPU; [RADIO]: 5-6% of the
    vocabulary gives roughly an 80% hit rate).

    Readings: the pages call the cache both "most frequent" and "LFU" without
    an eviction rule, so the hot set is static for a run, chosen from a given
    frequency count; ties go to the smaller id; K rounds up; a row's slot is
    its rank in (frequency descending, id ascending) order.

    Returns (hot_ids[K] int32 in slot order, slot_of_id[V] int32, -1 = not cached).
    """
    freq = np.asarray(freq, dtype=np.int64).reshape(-1)
    V = freq.size
    K = min(V, int(math.ceil(frac * V - 1e-9))) if frac > 0 else 0
    order = np.lexsort((np.arange(V), -freq))     # primary: -freq, secondary: id
    hot = order[:K].astype(np.int32)
    slot_of_id = np.full(V, -1, dtype=np.int32)
    slot_of_id[hot] = np.arange(K, dtype=np.int32)
    return hot, slot_of_id


def probe(unique: np.ndarray, slot_of_id: np.ndarray):
    """Cache probe per distinct id ([TLA] retrieval-path table: probe the GPU
    cache, fetch only the misses).  Returns (slot[U] with -1 for a miss,
    miss_list = positions j in `unique` order whose row is not cached)."""
    slot = slot_of_id[np.asarray(unique, dtype=np.int64)].astype(np.int32)
    miss_list = np.nonzero(slot < 0)[0].astype(np.int32)
    return slot, miss_list


def gather_rows(table: np.ndarray, unique: np.ndarray, row_offset: int = 0,
                width: int | None = None) -> np.ndarray:
    """The U active rows, copied bit for bit ([RADIO]: only the U x d_ff active
    rows are materialised on the GPU).  `table` is any storage dtype; with a
    grouped host layout [V][G*F] pass row_offset = g*F and width = F."""
    t = np.asarray(table)
    width = t.shape[1] - row_offset if width is None else width
    return t[np.asarray(unique, dtype=np.int64), row_offset:row_offset + width].copy()


def cache_rows_for(table: np.ndarray, hot: np.ndarray) -> np.ndarray:
    """Contents of the HBM cache: row slot k holds E[hot[k]] (bit copy)."""
    return np.asarray(table)[np.asarray(hot, dtype=np.int64)].copy()


# --------------------------------------------------------------------------
# Forward  ([ABS], [AIS] Synopsis/Interpretation)
# --------------------------------------------------------------------------

def ffn_forward(x, ids, w_gate, w_up, w_down, table=None) -> dict:
    """STAPLE FFN: the pretrained up-projection is kept and the token-indexed
    embedding is added to its output as a residual pathway ([ABS]; [AIS]
    Interpretation), inside a SwiGLU FFN:

        g = W_gate x,  u = W_up x,  h = u + E[id],  z = SiLU(g) * h,  y = W_down z.

    With table=None (or E = 0) this is the dense FFN: a zero-initialised table
    restores the seed model's computation ([AIS] Interpretation).
    Inputs are fp64 arrays; returns g, u, a = SiLU(g), h, z, y.
    """
    x = np.asarray(x, dtype=np.float64)
    g = x @ np.asarray(w_gate, dtype=np.float64).T
    u = x @ np.asarray(w_up, dtype=np.float64).T
    a = silu(g)
    if table is None:
        h = u.copy()
    else:
        h = u + np.asarray(table, dtype=np.float64)[np.asarray(ids, dtype=np.int64)]
    z = a * h
    y = z @ np.asarray(w_down, dtype=np.float64).T
    return {"g": g, "u": u, "a": a, "h": h, "z": z, "y": y}


# --------------------------------------------------------------------------
# Backward  ([RADIO]: U active rows form the leaf whose gradient is per row)
# --------------------------------------------------------------------------

def ffn_backward(dy, x, ids, w_gate, w_up, w_down, fwd: dict) -> dict:
    """Gradients of <dY, y> for the layer above.

        dz = W_down^T dY,  dh = dz * SiLU(g),  dg = dz * h * SiLU'(g)
        dE[j] = sum over tokens i with ids_i == unique_j of dh_i   (U rows only)
        dx = W_gate^T dg + W_up^T dh
        dW_gate = sum_i dg_i x_i^T,  dW_up = sum_i dh_i x_i^T,  dW_down = sum_i dY_i z_i^T

    The table gradient exists only for the U distinct ids of the batch, one
    row each, in ascending-id order (the order `dedup` returns).
    """
    dy = np.asarray(dy, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    wg = np.asarray(w_gate, dtype=np.float64)
    wu = np.asarray(w_up, dtype=np.float64)
    wd = np.asarray(w_down, dtype=np.float64)
    dz = dy @ wd
    dh = dz * fwd["a"]
    dg = dz * fwd["h"] * silu_grad(fwd["g"])
    unique, inverse, _, _ = dedup(ids)
    dE = np.zeros((unique.size, dh.shape[1]), dtype=np.float64)
    np.add.at(dE, inverse.astype(np.int64), dh)
    return {
        "dz": dz, "dh": dh, "dg": dg, "unique": unique, "dE": dE,
        "dx": dg @ wg + dh @ wu,
        "dW_gate": dg.T @ x, "dW_up": dh.T @ x, "dW_down": dy.T @ fwd["z"],
    }


# --------------------------------------------------------------------------
# STEM, the replacement variant STAPLE builds on ([ABS]; [AIS] Interpretation)
# --------------------------------------------------------------------------

def stem_forward(x, ids, w_gate, w_down, table) -> dict:
    """STEM's FFN: the token-indexed row replaces the up-projection instead of
    being added to it ([ABS]: STEM replaces FFN up-projections with
    token-indexed embeddings; [AIS] Interpretation: the replacement drops the
    up-projection), still gated by SiLU of the gate projection:

        g = W_gate x,  h = E[id],  z = SiLU(g) * h,  y = W_down z.

    Reading: the pages give no formula for STEM beyond "replace the
    up-projection"; the gate and down projections are kept as in the SwiGLU
    FFN (its FLOPs and weights then drop by one d_model x d_ff matrix per
    layer, which is what [TLA] Table 4 prints for STEM-12L).
    Returns g, a = SiLU(g), h, z, y (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    g = x @ np.asarray(w_gate, dtype=np.float64).T
    a = silu(g)
    h = np.asarray(table, dtype=np.float64)[np.asarray(ids, dtype=np.int64)]
    z = a * h
    y = z @ np.asarray(w_down, dtype=np.float64).T
    return {"g": g, "a": a, "h": h, "z": z, "y": y}


def stem_backward(dy, x, ids, w_gate, w_down, fwd: dict) -> dict:
    """Gradients of <dY, y> for stem_forward:

        dz = W_down^T dY,  dh = dz * SiLU(g),  dg = dz * h * SiLU'(g)
        dE[j] = sum of dh over the tokens whose id is unique_j   (U rows)
        dx = W_gate^T dg,  dW_gate = sum_i dg_i x_i^T,  dW_down = sum_i dY_i z_i^T

    (no up-projection, so no dW_up and no W_up^T dh term in dx)."""
    dy = np.asarray(dy, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    wg = np.asarray(w_gate, dtype=np.float64)
    wd = np.asarray(w_down, dtype=np.float64)
    dz = dy @ wd
    dh = dz * fwd["a"]
    dg = dz * fwd["h"] * silu_grad(fwd["g"])
    unique, inverse, _, _ = dedup(ids)
    dE = np.zeros((unique.size, dh.shape[1]), dtype=np.float64)
    np.add.at(dE, inverse.astype(np.int64), dh)
    return {"dz": dz, "dh": dh, "dg": dg, "unique": unique, "dE": dE, "dx": dg @ wg,
            "dW_gate": dg.T @ x, "dW_down": dy.T @ fwd["z"]}


# --------------------------------------------------------------------------
# Sampled forms for full-size workloads (exact definitions on subsets)
# --------------------------------------------------------------------------

def forward_rows(rows, x, ids, w_gate, w_up, w_down, table=None) -> dict:
    """ffn_forward restricted to the token positions `rows` (each token's
    output depends on that token alone)."""
    rows = np.asarray(rows, dtype=np.int64)
    tab = None if table is None else table
    return ffn_forward(np.asarray(x)[rows], np.asarray(ids)[rows], w_gate, w_up, w_down, tab)


def _columns(f, x, ids, w_gate, w_up, w_down, table, dy):
    """g, h, z, dz, dh, dg over all tokens for the single feature column f."""
    x = np.asarray(x, dtype=np.float64)
    g = x @ np.asarray(w_gate[f], dtype=np.float64)
    u = x @ np.asarray(w_up[f], dtype=np.float64)
    h = u if table is None else u + np.asarray(table[np.asarray(ids, dtype=np.int64), f], dtype=np.float64)
    a = silu(g)
    dz = np.asarray(dy, dtype=np.float64) @ np.asarray(w_down[:, f], dtype=np.float64)
    return {"g": g, "h": h, "z": a * h, "dz": dz, "dh": dz * a, "dg": dz * h * silu_grad(g)}


def embed_grad_rows(uids, dy, x, ids, w_gate, w_up, w_down, table=None) -> np.ndarray:
    """dE rows for the listed distinct ids only: for each id, the sum of dh
    over the tokens that carry it.  Returns [len(uids)][F] fp64."""
    ids = np.asarray(ids, dtype=np.int64)
    out = []
    for uid in np.asarray(uids, dtype=np.int64):
        toks = np.nonzero(ids == uid)[0]
        fw = forward_rows(toks, x, ids, w_gate, w_up, w_down, table)
        dz = np.asarray(dy, dtype=np.float64)[toks] @ np.asarray(w_down, dtype=np.float64)
        out.append((dz * fw["a"]).sum(axis=0))
    return np.array(out, dtype=np.float64).reshape(len(out), np.asarray(w_gate).shape[0])


def weight_grad_entries(entries, dy, x, ids, w_gate, w_up, w_down, table=None) -> np.ndarray:
    """Selected weight-gradient entries.  `entries` is a list of
    (which, r, c) with which in {"gate", "up", "down"}; gate/up entries are
    dW[f=r][d=c], down entries are dW_down[d=r][f=c]."""
    cache = {}
    vals = []
    x64 = np.asarray(x, dtype=np.float64)
    dy64 = np.asarray(dy, dtype=np.float64)
    for which, r, c in entries:
        f = r if which in ("gate", "up") else c
        if f not in cache:
            cache[f] = _columns(f, x, ids, w_gate, w_up, w_down, table, dy)
        col = cache[f]
        if which == "gate":
            vals.append(float(col["dg"] @ x64[:, c]))
        elif which == "up":
            vals.append(float(col["dh"] @ x64[:, c]))
        else:
            vals.append(float(dy64[:, r] @ col["z"]))
    return np.array(vals, dtype=np.float64)


def dx_rows(rows, dy, x, ids, w_gate, w_up, w_down, table=None) -> np.ndarray:
    """dx for the listed token positions: W_gate^T dg_i + W_up^T dh_i."""
    rows = np.asarray(rows, dtype=np.int64)
    fw = forward_rows(rows, x, ids, w_gate, w_up, w_down, table)
    bw = ffn_backward(np.asarray(dy)[rows], np.asarray(x)[rows], np.asarray(ids)[rows],
                      w_gate, w_up, w_down, fw)
    return bw["dx"]


# --------------------------------------------------------------------------
# Host optimizer step on the touched rows ([TLA] Table 4 caption: the tables
# are offloaded with their AdamW moments; [AIS] Interpretation: the table is
# the trained parameter, per-row gradients)
# --------------------------------------------------------------------------

def adamw_rows(table, ids, grad, m, v, lr, beta1, beta2, eps, weight_decay, step):
    """One AdamW step on the rows `ids` of a table, the others untouched.

    The pages train the tables with AdamW, fp32 moments in host memory, but
    print no update formula or hyperparameters.  Reading: the standard AdamW
    with decoupled weight decay (Loshchilov & Hutter, "Decoupled Weight Decay
    Regularization"), applied only to the rows that got a gradient:

        m = b1 m + (1 - b1) g,    v = b2 v + (1 - b2) g^2
        m_hat = m / (1 - b1^t),   v_hat = v / (1 - b2^t)
        w = w - lr (m_hat / (sqrt(v_hat) + eps) + weight_decay w)

    table, m, v: [V][F]; ids: [U] distinct; grad: [U][F].  Returns new fp64
    copies (table, m, v); the oracle rounds nothing.
    """
    w = np.array(table, dtype=np.float64)
    m = np.array(m, dtype=np.float64)
    v = np.array(v, dtype=np.float64)
    ids = np.asarray(ids, dtype=np.int64)
    g = np.asarray(grad, dtype=np.float64)
    m[ids] = beta1 * m[ids] + (1.0 - beta1) * g
    v[ids] = beta2 * v[ids] + (1.0 - beta2) * g * g
    m_hat = m[ids] / (1.0 - beta1 ** step)
    v_hat = v[ids] / (1.0 - beta2 ** step)
    w[ids] = w[ids] - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * w[ids])
    return w, m, v


# --------------------------------------------------------------------------
# Sizes printed on the pages ([TLA] Table 4, Figure 4; [AIS] Interpretation)
# --------------------------------------------------------------------------

def paper_shapes(D=2048, F=8192, V=100352, n_layers=16, n_aug=12, frac=0.05,
                 attn_proj=4, bytes_bf16=2, bytes_moments=8) -> dict:
    """Closed-form sizes of an OLMo-2-1B-shaped model with n_aug augmented
    layers: table bytes (vocab x d_ff per augmented layer, bf16), table plus
    two fp32 AdamW moments on the host, the hot-row cache at `frac` of the
    vocabulary, dense/STEM linear FLOPs per token and GPU weight bytes.
    Reading: d_ff-wide tables (the printed 19.73 GB fixes the width); untied
    input embedding and LM head; four D x D attention projections per layer."""
    table_elems = n_aug * V * F
    per_layer_lin = attn_proj * D * D + 3 * D * F
    lin_params = n_layers * per_layer_lin + D * V          # + LM head
    all_params = lin_params + D * V                         # + input embedding
    K = int(math.ceil(frac * V - 1e-9))
    return {
        "table_bytes": table_elems * bytes_bf16,
        "table_plus_moments_bytes": table_elems * (bytes_bf16 + bytes_moments),
        "cache_rows": K,
        "cache_bytes": n_aug * K * F * bytes_bf16,
        "dense_linear_flops_per_token": 2 * lin_params,
        "stem_linear_flops_per_token": 2 * (lin_params - n_aug * D * F),
        "dense_weight_bytes": all_params * bytes_bf16,
        "stem_weight_bytes": (all_params - n_aug * D * F) * bytes_bf16,
    }
