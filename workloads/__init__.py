"""Seeded synthetic inputs for the SiTU-GLU workloads.

This module holds no SiTU arithmetic: it draws the inputs (gate_up, routing
weights, grad_out) that both the CUDA path and the fp64 oracle consume, so
that the two are compared on bit-identical data.  It imports neither of them.

Generation is deterministic and independent of threading: every tensor is cut
into blocks of ``BLOCK_ROWS`` rows and each block draws from its own numpy
``PCG64`` stream seeded by ``SeedSequence([seed, tensor_id, block])``.
Normals are numpy's ``standard_normal``; values are rounded to the storage
dtype with round-to-nearest-even (float64 -> float32 -> bf16).

The five workloads restate the synthetic configurations the measurements are
quoted on (tiny, dense FFN, routed MoE expert rows, fp32 beta sweep with no
linear clamp, large).  No dataset is involved.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

BLOCK_ROWS = 64

TENSOR_GATE_UP = 1
TENSOR_ROUTING = 2
TENSOR_GRAD_OUT = 3
TENSOR_COL_WEIGHTS = 4
TENSOR_ELEM_WEIGHTS = 5
TENSOR_FC1_X = 6
TENSOR_FC1_W = 7
TENSOR_FC1_SPLIT = 8
TENSOR_AR_VALUES = 9
TENSOR_AR_WEIGHTS = 10
TENSOR_FC2_DOUT = 11
TENSOR_FC2_W = 12
TENSOR_FC2_GU = 13


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  Standard deviations are the N(0, s) scale."""

    index: int
    name: str
    dtype: str            # "bf16" or "f32": gate_up, output, grad_out, d_gate_up
    tokens: int           # rows T
    inter: int            # intermediate size I (gate_up is [T, 2I])
    g_std: float
    u_std: float
    outlier_p: float      # probability an entry is replaced by +-U(lo, hi)
    outlier_lo: float
    outlier_hi: float
    rw_kind: str          # "uniform" U(0,1), "ones", or "topk_softmax"
    go_std: float
    betas: tuple          # gate betas to run (the sweep has several)
    linear_beta: float | None
    seed: int
    experts: int = 0      # topk_softmax only: experts per token
    topk: int = 0         # topk_softmax only: weights kept per token

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def fwd_bytes(self) -> int:
        """Algorithmic HBM bytes of one forward: read gate_up and w, write Y."""
        return self.tokens * (2 * self.inter * self.elem_bytes + 4 + self.inter * self.elem_bytes)

    def bwd_bytes(self) -> int:
        """Algorithmic HBM bytes of one backward: read gate_up, grad_out and w,
        write d_gate_up and d_w."""
        s = self.elem_bytes
        return self.tokens * (2 * self.inter * s + self.inter * s + 4 + 2 * self.inter * s + 4)

    def describe(self) -> str:
        return (f"{self.name}: gate_up {self.dtype} [{self.tokens}, {2 * self.inter}] "
                f"(I={self.inter}), beta={list(self.betas)}, linear_beta={self.linear_beta}")


WORKLOADS = (
    Workload(0, "tiny", "bf16", 256, 512, 1.0, 1.0, 0.0, 0.0, 0.0, "uniform", 1.0,
             (4.0,), 25.0, seed=0),
    Workload(1, "dense_ffn", "bf16", 4096, 3072, 2.0, 1.0, 0.0, 0.0, 0.0, "ones", 0.1,
             (4.0,), 25.0, seed=1),
    Workload(2, "routed_moe", "bf16", 32768, 2048, 3.0, 3.0, 0.01, 20.0, 60.0, "topk_softmax", 1.0,
             (4.0,), 25.0, seed=2, experts=384, topk=8),
    Workload(3, "beta_sweep_f32", "f32", 16384, 4096, 1.5, 1.5, 0.0, 0.0, 0.0, "uniform", 1.0,
             (1.0, 4.0, 16.0), None, seed=3),
    Workload(4, "large", "bf16", 131072, 4096, 2.0, 2.0, 0.0, 0.0, 0.0, "uniform", 0.05,
             (4.0,), 25.0, seed=4),
)


def workload(index: int) -> Workload:
    return WORKLOADS[index]


# ---- rounding to the storage dtype ------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns the bf16
    bit patterns as uint16.  Inputs here are finite."""
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
    return ((bits + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(values: np.ndarray, dtype: str) -> np.ndarray:
    f32 = values.astype(np.float32)
    return f32_to_bf16_bits(f32) if dtype == "bf16" else f32


# ---- per-block streams ---------------------------------------------------------

def _rng(seed: int, tensor_id: int, block: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, block])))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _fill_blocks(rows: int, fill_block, n_threads: int | None = None) -> None:
    blocks = (rows + BLOCK_ROWS - 1) // BLOCK_ROWS
    n_threads = n_threads or _threads()
    if blocks <= 2 or n_threads == 1:
        for b in range(blocks):
            fill_block(b)
        return
    with ThreadPoolExecutor(max_workers=n_threads) as pool:
        list(pool.map(fill_block, range(blocks)))


def _gate_up_block(wl: Workload, tokens: int, inter: int, b: int) -> np.ndarray:
    # Always a whole block of draws, so that a row's values do not depend on T.
    r0 = b * BLOCK_ROWS
    n = BLOCK_ROWS
    rng = _rng(wl.seed, TENSOR_GATE_UP, b)
    v = rng.standard_normal((n, 2 * inter))
    v[:, :inter] *= wl.g_std
    v[:, inter:] *= wl.u_std
    if wl.outlier_p > 0.0:
        hit = rng.random((n, 2 * inter)) < wl.outlier_p
        sign = np.where(rng.random((n, 2 * inter)) < 0.5, -1.0, 1.0)
        mag = rng.uniform(wl.outlier_lo, wl.outlier_hi, size=(n, 2 * inter))
        v = np.where(hit, sign * mag, v)
    return v[:min(BLOCK_ROWS, tokens - r0)]


def gate_up(wl: Workload, tokens: int | None = None, inter: int | None = None) -> np.ndarray:
    """gate_up [T, 2I]: gate half ~ N(0, g_std), up half ~ N(0, u_std), with the
    workload's outliers; bf16 bit patterns (uint16) or float32."""
    tokens = wl.tokens if tokens is None else tokens
    inter = wl.inter if inter is None else inter
    out = np.empty((tokens, 2 * inter), dtype=np.uint16 if wl.dtype == "bf16" else np.float32)

    def fill(b):
        r0 = b * BLOCK_ROWS
        blk = _gate_up_block(wl, tokens, inter, b)
        out[r0:r0 + blk.shape[0]] = _store(blk, wl.dtype)

    _fill_blocks(tokens, fill)
    return out


def grad_out(wl: Workload, tokens: int | None = None, inter: int | None = None) -> np.ndarray:
    """grad_out [T, I] ~ N(0, go_std) in the workload's dtype."""
    tokens = wl.tokens if tokens is None else tokens
    inter = wl.inter if inter is None else inter
    out = np.empty((tokens, inter), dtype=np.uint16 if wl.dtype == "bf16" else np.float32)

    def fill(b):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, tokens - r0)
        v = _rng(wl.seed, TENSOR_GRAD_OUT, b).standard_normal((BLOCK_ROWS, inter))[:n] * wl.go_std
        out[r0:r0 + n] = _store(v, wl.dtype)

    _fill_blocks(tokens, fill)
    return out


def routing_weights(wl: Workload, tokens: int | None = None) -> np.ndarray:
    """Row-aligned routing weights [T] float32.

    "uniform": U(0, 1).  "ones": 1.0.  "topk_softmax": rows are token-major
    expert assignments (row = token * topk + k); per token, ``experts``
    N(0, 1) logits, softmax over all experts, then the ``topk`` largest
    probabilities in descending order (ties to the lower expert index), not
    renormalised."""
    tokens = wl.tokens if tokens is None else tokens
    if wl.rw_kind == "ones":
        return np.ones(tokens, dtype=np.float32)
    if wl.rw_kind == "uniform":
        out = np.empty(tokens, dtype=np.float32)

        def fill(b):
            r0 = b * BLOCK_ROWS
            n = min(BLOCK_ROWS, tokens - r0)
            out[r0:r0 + n] = _rng(wl.seed, TENSOR_ROUTING, b).random(BLOCK_ROWS)[:n].astype(np.float32)

        _fill_blocks(tokens, fill, n_threads=1)
        return out
    if wl.rw_kind == "topk_softmax":
        k, e = wl.topk, wl.experts
        n_tok = (tokens + k - 1) // k
        probs = np.empty((n_tok, k), dtype=np.float64)
        for b in range((n_tok + BLOCK_ROWS - 1) // BLOCK_ROWS):
            t0 = b * BLOCK_ROWS
            n = min(BLOCK_ROWS, n_tok - t0)
            logits = _rng(wl.seed, TENSOR_ROUTING, b).standard_normal((BLOCK_ROWS, e))[:n]
            z = np.exp(logits - logits.max(axis=1, keepdims=True))
            p = z / z.sum(axis=1, keepdims=True)
            order = np.argsort(-p, axis=1, kind="stable")[:, :k]
            probs[t0:t0 + n] = np.take_along_axis(p, order, axis=1)
        return probs.reshape(-1)[:tokens].astype(np.float32)
    raise ValueError(f"unknown routing-weight kind {wl.rw_kind!r}")


def column_weights(wl: Workload, inter: int | None = None) -> np.ndarray:
    """Per-column routing weights [I] float32 ~ U(0, 1): one weight shared by
    every row of a column (the [I] broadcast form of routing_weights)."""
    inter = wl.inter if inter is None else inter
    return _rng(wl.seed, TENSOR_COL_WEIGHTS, 0).random(inter).astype(np.float32)


def element_weights(wl: Workload, tokens: int | None = None, inter: int | None = None) -> np.ndarray:
    """Per-element routing weights [T, I] float32 ~ U(0, 1), drawn in whole
    64-row blocks like gate_up."""
    tokens = wl.tokens if tokens is None else tokens
    inter = wl.inter if inter is None else inter
    out = np.empty((tokens, inter), dtype=np.float32)

    def fill(b):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, tokens - r0)
        out[r0:r0 + n] = _rng(wl.seed, TENSOR_ELEM_WEIGHTS, b).random((BLOCK_ROWS, inter))[:n]

    _fill_blocks(tokens, fill)
    return out


def inputs(wl: Workload, tokens: int | None = None, inter: int | None = None) -> dict:
    """All three inputs of a workload: gate_up, routing_weights [T], grad_out."""
    return {
        "gate_up": gate_up(wl, tokens, inter),
        "routing_weights": routing_weights(wl, tokens),
        "grad_out": grad_out(wl, tokens, inter),
    }


# ---- FC1 (grouped GEMM) inputs -----------------------------------------------------

def expert_offsets(tokens: int, experts: int, seed: int, skew: float = 1.0) -> np.ndarray:
    """Row offsets [E + 1] of ``tokens`` token rows grouped by expert: expert
    sizes from a Dirichlet(skew) share of the rows (uneven, some possibly
    empty), rounded so that they add up to ``tokens``."""
    rng = _rng(seed, TENSOR_FC1_SPLIT, 0)
    share = rng.dirichlet(np.full(experts, float(skew)))
    sizes = np.floor(share * tokens).astype(np.int64)
    sizes[: tokens - int(sizes.sum())] += 1
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


def fc1_inputs(tokens: int, hidden: int, inter: int, experts: int, seed: int, w_std: float | None = None):
    """x bf16 [T, H] ~ N(0, 1); w1 bf16 [E * 2I, H] ~ N(0, w_std) (default
    3 / sqrt(H), so that G and U ~ N(0, 3) like the routed-MoE rows); row
    offsets from expert_offsets; per-row weights U(0, 1) float32.  x is drawn
    in 64-row blocks, w1 in 64-row blocks of its own."""
    w_std = 3.0 / np.sqrt(hidden) if w_std is None else w_std
    x = np.empty((tokens, hidden), dtype=np.uint16)

    def fill_x(b):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, tokens - r0)
        x[r0:r0 + n] = f32_to_bf16_bits(_rng(seed, TENSOR_FC1_X, b).standard_normal((BLOCK_ROWS, hidden))[:n]
                                        .astype(np.float32))

    _fill_blocks(tokens, fill_x)
    rows_w = experts * 2 * inter
    w1 = np.empty((rows_w, hidden), dtype=np.uint16)

    def fill_w(b):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, rows_w - r0)
        v = _rng(seed, TENSOR_FC1_W, b).standard_normal((BLOCK_ROWS, hidden))[:n] * w_std
        w1[r0:r0 + n] = f32_to_bf16_bits(v.astype(np.float32))

    _fill_blocks(rows_w, fill_w)
    offsets = expert_offsets(tokens, experts, seed)
    rw = np.empty(tokens, dtype=np.float32)
    for b in range((tokens + BLOCK_ROWS - 1) // BLOCK_ROWS):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, tokens - r0)
        rw[r0:r0 + n] = _rng(seed, TENSOR_ROUTING, b).random(BLOCK_ROWS)[:n].astype(np.float32)
    return {"x": x, "w1": w1, "offsets": offsets, "routing_weights": rw}


# ---- attention-residual mixing inputs -----------------------------------------------

def attn_res_inputs(tokens: int, blocks: int, hidden: int, seed: int, dtype: str = "bf16"):
    """Stored block sums [T, B, H] and the current prefix sum [T, H] (bf16 bits
    or float32): source b ~ N(0, s_b) with s_b = 1 + b / 2, as sums over more
    layers grow; norm_weight ~ 1 + 0.1 N(0, 1) and proj_weight ~ N(0, 1 /
    sqrt(H)) float32 [H], so that logits are a few units.  64-row blocks."""
    store = (lambda v: f32_to_bf16_bits(v.astype(np.float32))) if dtype == "bf16" else (lambda v: v.astype(np.float32))
    kind = np.uint16 if dtype == "bf16" else np.float32
    blk = np.empty((tokens, blocks, hidden), dtype=kind)
    pre = np.empty((tokens, hidden), dtype=kind)
    scale = (1.0 + 0.5 * np.arange(blocks + 1))[None, :, None]

    def fill(b):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, tokens - r0)
        v = _rng(seed, TENSOR_AR_VALUES, b).standard_normal((BLOCK_ROWS, blocks + 1, hidden))[:n] * scale
        blk[r0:r0 + n] = store(v[:, :blocks])
        pre[r0:r0 + n] = store(v[:, blocks])

    _fill_blocks(tokens, fill)
    rng = _rng(seed, TENSOR_AR_WEIGHTS, 0)
    norm_w = (1.0 + 0.1 * rng.standard_normal(hidden)).astype(np.float32)
    proj_w = (rng.standard_normal(hidden) / np.sqrt(hidden)).astype(np.float32)
    return {"blocks": blk, "prefix": pre, "norm_weight": norm_w, "proj_weight": proj_w}


# ---- FC2 data-gradient inputs ---------------------------------------------------------

def fc2_inputs(tokens: int, hidden: int, inter: int, experts: int, seed: int):
    """dout bf16 [T, H] ~ N(0, 1); w2t bf16 [E * I, H] ~ N(0, 1 / sqrt(H)) (FC2's
    weight transposed per expert, so dY ~ N(0, 1)); gate_up bf16 [T, 2I] ~
    N(0, 3) (the saved FC1 output); offsets as expert_offsets; per-row
    weights U(0, 1).  64-row blocks."""
    def block_fill(out, rows, cols, tensor, std):
        def fill(b):
            r0 = b * BLOCK_ROWS
            n = min(BLOCK_ROWS, rows - r0)
            v = _rng(seed, tensor, b).standard_normal((BLOCK_ROWS, cols))[:n] * std
            out[r0:r0 + n] = f32_to_bf16_bits(v.astype(np.float32))
        _fill_blocks(rows, fill)

    dout = np.empty((tokens, hidden), dtype=np.uint16)
    block_fill(dout, tokens, hidden, TENSOR_FC2_DOUT, 1.0)
    w2t = np.empty((experts * inter, hidden), dtype=np.uint16)
    block_fill(w2t, experts * inter, hidden, TENSOR_FC2_W, 1.0 / np.sqrt(hidden))
    gu = np.empty((tokens, 2 * inter), dtype=np.uint16)
    block_fill(gu, tokens, 2 * inter, TENSOR_FC2_GU, 3.0)
    rw = np.empty(tokens, dtype=np.float32)
    for b in range((tokens + BLOCK_ROWS - 1) // BLOCK_ROWS):
        r0 = b * BLOCK_ROWS
        n = min(BLOCK_ROWS, tokens - r0)
        rw[r0:r0 + n] = _rng(seed, TENSOR_ROUTING, b).random(BLOCK_ROWS)[:n].astype(np.float32)
    return {"dout": dout, "w2t": w2t, "gate_up": gu, "offsets": expert_offsets(tokens, experts, seed),
            "routing_weights": rw}
