"""Seeded synthetic inputs for the STAPLE FFN layer.

This module is shared by the CPU oracle, the tests and the benchmark.  It holds
no arithmetic of the method itself: only random draws, the bf16 storage
rounding that turns an fp32 draw into the exact bf16 value both sides receive,
and the workload presets (shapes and seeds).

Token statistics: the pages train on a web corpus and serve real prompts; no
corpus is available here, so token ids are drawn from a truncated Zipf law,
p(rank r) proportional to r**-s for r = 1..V, and ranks are mapped to ids
through a seeded random permutation so that hot rows are scattered across the
table as in a real BPE vocabulary.  The STAPLE paper ("STAPLE: Static Sparse
Upcycling of Pretrained Checkpoints via Embedding Modules", ai4snews summary,
Perspective; Table 4) measures serving on a single B200 at batch 64 and
context 256; the decode presets below use batch 64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "zipf_probs", "zipf_ids", "calibration_freq",
    "normal_f32", "f32_to_bf16_bits", "bf16_bits_to_f32", "bf16_normal",
    "LayerInputs", "make_layer_inputs",
]

# Seeds: ids = 1000 + preset index, weights = 2000 + layer, table = 3000 + layer,
# activations / upstream gradients = 4000 + step, rank permutation = 7,
# calibration stream (cache frequencies) = 1.
SEED_IDS = 1000
SEED_W = 2000
SEED_E = 3000
SEED_ACT = 4000
SEED_PERM = 7
SEED_CALIB = 1


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens per step (batch x sequence)
    D: int            # d_model
    F: int            # d_ff (also the table row width)
    V: int            # vocabulary size (table rows)
    layers: int       # stacked augmented layers
    dtype: str        # "f32" or "bf16"
    w_std: float      # std of W_gate, W_up, W_down
    e_std: float      # std of the table E
    x_std: float      # std of the layer input x
    dy_std: float     # std of the upstream gradient dY
    table: str        # "device" (whole table in HBM) or "host" (pinned host + HBM cache)
    cache_frac: float  # fraction of the vocabulary cached in HBM (host tables)
    group: int        # adjacent layers stored token-major per host row
    training: bool    # forward + backward, or forward only
    steps: int = 1    # consecutive decode steps (stacked decode preset)
    zipf_s: float = 1.1
    index: int = 0
    notes: str = field(default="", compare=False)


WORKLOADS = {
    "tiny-f32": Workload(
        "tiny-f32", T=256, D=64, F=256, V=1000, layers=1, dtype="f32",
        w_std=0.02, e_std=0.02, x_std=0.02, dy_std=1.0, table="device",
        cache_frac=0.0, group=1, training=True, index=0,
        notes="single layer, fp32 end to end, table on the GPU"),
    "olmo2-1b-decode-layer": Workload(
        "olmo2-1b-decode-layer", T=64, D=2048, F=8192, V=100352, layers=1,
        dtype="bf16", w_std=0.02, e_std=0.01, x_std=1.0, dy_std=1.0,
        table="device", cache_frac=0.0, group=1, training=False, index=1,
        notes="one OLMo-2-1B-shaped layer, batch 64 decode, table in HBM"),
    "olmo2-1b-train-layer": Workload(
        "olmo2-1b-train-layer", T=16384, D=2048, F=8192, V=100352, layers=1,
        dtype="bf16", w_std=0.02, e_std=0.01, x_std=1.0, dy_std=1.0,
        table="host", cache_frac=0.05, group=1, training=True, index=2,
        notes="4 x 4096 tokens, host table with the top 5% rows cached"),
    "olmo2-7b-decode-16l": Workload(
        "olmo2-7b-decode-16l", T=64, D=4096, F=11008, V=100352, layers=16,
        dtype="bf16", w_std=0.02, e_std=0.01, x_std=1.0, dy_std=1.0,
        table="host", cache_frac=0.05, group=4, training=False, steps=256,
        index=3, notes="16 stacked layers, tables grouped 4 per host row"),
    "olmo2-1b-train-12l": Workload(
        "olmo2-1b-train-12l", T=16384, D=2048, F=8192, V=100352, layers=12,
        dtype="bf16", w_std=0.02, e_std=0.01, x_std=1.0, dy_std=1.0,
        table="host", cache_frac=0.05, group=4, training=True, index=4,
        notes="12 stacked layers, dedup once per step, dE returned to host"),
}


# --------------------------------------------------------------------------
# Token ids
# --------------------------------------------------------------------------

def zipf_probs(V: int, s: float) -> np.ndarray:
    """Probability of each rank r = 1..V under a Zipf law truncated at V."""
    r = np.arange(1, V + 1, dtype=np.float64)
    w = r ** (-float(s))
    return w / w.sum()


def _rank_to_id(V: int, identity: bool) -> np.ndarray:
    if identity:
        return np.arange(V, dtype=np.int64)
    return np.random.default_rng(SEED_PERM).permutation(V).astype(np.int64)


def zipf_ids(T: int, V: int, s: float = 1.1, seed: int = SEED_IDS,
             identity_perm: bool = False) -> np.ndarray:
    """T token ids in [0, V), Zipf(s) over ranks, ranks scattered by a fixed
    permutation (identity_perm=True keeps rank r at id r-1)."""
    if T == 0:
        return np.zeros(0, dtype=np.int32)
    cdf = np.cumsum(zipf_probs(V, s))
    cdf[-1] = 1.0
    u = np.random.default_rng(seed).random(T)
    rank0 = np.searchsorted(cdf, u, side="right")
    rank0 = np.minimum(rank0, V - 1)
    return _rank_to_id(V, identity_perm)[rank0].astype(np.int32)


def calibration_freq(V: int, s: float = 1.1, n_tokens: int = 1 << 24,
                     seed: int = SEED_CALIB, identity_perm: bool = False) -> np.ndarray:
    """Token counts of a separate calibration stream: the frequency input of
    the hot-row cache.  Drawn in chunks to bound memory."""
    freq = np.zeros(V, dtype=np.int64)
    rng_seed = seed
    left = n_tokens
    chunk = 1 << 22
    while left > 0:
        n = min(chunk, left)
        ids = zipf_ids(n, V, s, seed=rng_seed, identity_perm=identity_perm)
        freq += np.bincount(ids, minlength=V)
        left -= n
        rng_seed += 1_000_003
    return freq


# --------------------------------------------------------------------------
# Real-valued tensors
# --------------------------------------------------------------------------

def normal_f32(shape, std: float, seed: int) -> np.ndarray:
    return (np.random.default_rng(seed).standard_normal(shape, dtype=np.float32)
            * np.float32(std))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns the raw
    16-bit patterns.  Inputs are finite draws, so NaN handling is not needed."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_normal(shape, std: float, seed: int):
    """(bits, values): bf16 bit patterns and the same values widened to fp32."""
    bits = f32_to_bf16_bits(normal_f32(shape, std, seed))
    return bits, bf16_bits_to_f32(bits)


# --------------------------------------------------------------------------
# One layer's inputs
# --------------------------------------------------------------------------

@dataclass
class LayerInputs:
    """Storage arrays as the GPU receives them (fp32 or bf16 bit patterns)
    plus the exact values widened to fp64 for the oracle."""
    dtype: str
    ids: np.ndarray
    x: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    table: np.ndarray | None
    dy: np.ndarray | None

    def f64(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        if a is None:
            return None
        if self.dtype == "bf16":
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)


def _draw(shape, std, seed, dtype):
    if dtype == "bf16":
        return bf16_normal(shape, std, seed)[0]
    return normal_f32(shape, std, seed)


def make_layer_inputs(w: Workload, layer: int = 0, step: int = 0, T: int | None = None,
                      with_table: bool = True, zero_table: bool = False,
                      with_dy: bool | None = None, identity_perm: bool = False) -> LayerInputs:
    """Draw one layer's inputs for workload `w` (T overrides the token count)."""
    T = w.T if T is None else T
    ids = zipf_ids(T, w.V, w.zipf_s, seed=SEED_IDS + w.index + 7919 * step,
                   identity_perm=identity_perm)
    x = _draw((T, w.D), w.x_std, SEED_ACT + 2 * step, w.dtype)
    wg = _draw((w.F, w.D), w.w_std, SEED_W + 3 * layer, w.dtype)
    wu = _draw((w.F, w.D), w.w_std, SEED_W + 3 * layer + 1, w.dtype)
    wd = _draw((w.D, w.F), w.w_std, SEED_W + 3 * layer + 2, w.dtype)
    table = None
    if with_table:
        if zero_table:
            table = np.zeros((w.V, w.F), dtype=np.uint16 if w.dtype == "bf16" else np.float32)
        else:
            table = _draw((w.V, w.F), w.e_std, SEED_E + layer, w.dtype)
    if with_dy is None:
        with_dy = w.training
    dy = _draw((T, w.D), w.dy_std, SEED_ACT + 2 * step + 1, w.dtype) if with_dy else None
    return LayerInputs(w.dtype, ids, x, wg, wu, wd, table, dy)


def expected_unique(T: int, V: int, s: float) -> float:
    """Expected number of distinct ids among T Zipf draws (used for sizing
    and for checking the generator, not by the method)."""
    p = zipf_probs(V, s)
    return float(np.sum(1.0 - np.exp(T * np.log1p(-np.minimum(p, 1 - 1e-16)))))


def top_mass(V: int, s: float, frac: float) -> float:
    """Probability mass of the ceil(frac*V) most frequent ranks."""
    k = int(math.ceil(frac * V))
    return float(zipf_probs(V, s)[:k].sum())
