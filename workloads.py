"""Seeded synthetic inputs for MoE expert-parallel dispatch / combine.

This module only draws random inputs.  It holds none of the dispatch /
combine arithmetic: both the CPU oracle (in its tests) and the CUDA path
are fed the very same arrays from here, so it is the one piece of code the
two sides share.

The workloads follow the DeepEP V2 README, section "Performance": a
V3-style batch of 8K tokens, hidden size 7168, top-8 experts, FP8 dispatch
and BF16 combine.  That page measures no dataset, so every input is drawn
here from fixed seeds:

* ``x``: bf16, N(0, 1) drawn in float32 and rounded once to bf16 (torch's
  round-to-nearest-even cast).  The "skewed" workload scales a seeded 1 %
  of the rows by 100 in float32 before the rounding, to stress the FP8
  block scales.
* ``topk_idx``: k distinct experts per token by Gumbel-top-k (sampling
  without replacement from the popularity distribution, Plackett-Luce
  order: slot j holds the j-th largest key).  Uniform popularity, or
  Zipf(s) over a seeded permutation of the experts.  A seeded, exact number
  of slots can be set to -1 (dropped).
* ``topk_weights``: float32 softmax (computed in float64) of k N(0, 1)
  router logits per token.
* ``y``: bf16 N(0, 1) stand-in for the expert outputs that combine reads,
  one row per possible receive row (``T*k + E*(align-1)``).

Every stream comes from ``numpy.random.SeedSequence(seed).spawn``, so the
draws do not depend on one another's sizes.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_y", "make_prequant", "y_rows"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # experts
    S: int            # logical segments ("ranks") the experts are split into
    k: int            # experts per token (top-k)
    align: int        # expert_alignment
    x_mode: str       # "bf16" or "fp8_quant" (bf16 x quantised to e4m3 on the fly)
    drop_frac: float = 0.0     # fraction of slots set to -1, exact count round(frac*T*k)
    zipf_s: float = 0.0        # 0 -> uniform expert popularity
    outlier_frac: float = 0.0  # fraction of rows of x scaled by outlier_scale
    outlier_scale: float = 1.0
    pairs: int = 1             # dispatch->combine pairs per step (decode graph)


WORKLOADS = {
    "tiny": Workload("tiny", T=128, H=256, E=16, S=4, k=2, align=1, x_mode="bf16"),
    "mid": Workload("mid", T=4096, H=4096, E=64, S=8, k=6, align=128, x_mode="fp8_quant",
                    drop_frac=0.05),
    "v3": Workload("v3", T=8192, H=7168, E=256, S=8, k=8, align=128, x_mode="fp8_quant"),
    "skewed": Workload("skewed", T=8192, H=7168, E=256, S=8, k=8, align=128,
                       x_mode="fp8_quant", zipf_s=1.2, outlier_frac=0.01, outlier_scale=100.0),
    "decode": Workload("decode", T=128, H=7168, E=256, S=8, k=8, align=1, x_mode="fp8_quant",
                       pairs=256),
}

# Sub-stream order; new streams are only ever appended.
_X, _EXPERTS, _LOGITS, _DROPS, _OUTLIERS, _Y, _PERM = range(7)
_N_STREAMS = 7


def _streams(seed: int):
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(_N_STREAMS)]


def _to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), torch's RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def y_rows(w: Workload) -> int:
    """Rows of the y buffer: one per possible receive row, T*k + E*(align-1)."""
    return w.T * w.k + w.E * (w.align - 1)


def _draw_x(w: Workload, g_x, g_out, T: int) -> np.ndarray:
    x = g_x.standard_normal((T, w.H), dtype=np.float32)
    n_out = int(round(w.outlier_frac * T))
    if n_out:
        rows = g_out.choice(T, size=n_out, replace=False)
        x[rows] *= np.float32(w.outlier_scale)
    return _to_bf16_bits(x)


def _draw_topk(w: Workload, g_e, g_perm, g_drop, T: int):
    if w.zipf_s > 0.0:
        perm = g_perm.permutation(w.E)
        ranks = np.empty(w.E, dtype=np.float64)
        ranks[perm] = np.arange(1, w.E + 1, dtype=np.float64)
        logp = -w.zipf_s * np.log(ranks)          # p_e proportional to rank(e)^-s
    else:
        logp = np.zeros(w.E, dtype=np.float64)
    keys = logp[None, :] + g_e.gumbel(size=(T, w.E))
    idx = np.argsort(-keys, axis=1, kind="stable")[:, : w.k].astype(np.int64)
    n_drop = int(round(w.drop_frac * T * w.k))
    if n_drop:
        flat = g_drop.choice(T * w.k, size=n_drop, replace=False)
        idx.reshape(-1)[flat] = -1
    return idx


def _draw_weights(w: Workload, g_l, T: int) -> np.ndarray:
    logits = g_l.standard_normal((T, w.k))
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def make_inputs(w: Workload | str, seed: int = 0, T: int | None = None) -> dict:
    """x (bf16 bits, uint16 [T,H]), topk_idx (int64 [T,k]), topk_weights (f32 [T,k]).

    ``T`` overrides the workload's token count (same shapes otherwise)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    T = w.T if T is None else T
    g = _streams(seed)
    return {
        "x": _draw_x(w, g[_X], g[_OUTLIERS], T),
        "topk_idx": _draw_topk(w, g[_EXPERTS], g[_PERM], g[_DROPS], T),
        "topk_weights": _draw_weights(w, g[_LOGITS], T),
    }


def make_y(w: Workload | str, seed: int = 0, rows: int | None = None) -> np.ndarray:
    """Expert outputs, bf16 bits (uint16 [rows, H]); rows defaults to y_rows(w)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    rows = y_rows(w) if rows is None else rows
    g = _streams(seed)[_Y]
    out = np.empty((rows, w.H), dtype=np.uint16)
    step = max(1, (1 << 24) // w.H)
    for r0 in range(0, rows, step):           # chunked: bounded float32 temporaries
        r1 = min(rows, r0 + step)
        out[r0:r1] = _to_bf16_bits(g.standard_normal((r1 - r0, w.H), dtype=np.float32))
    return out


def make_prequant(T: int, H: int, seed: int = 0):
    """An already-quantised (x_fp8, scales) pair: random finite e4m3 bytes
    (never the NaN codes 0x7F / 0xFF) and positive f32 scales [T, H/128]."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0xF8])))
    q = g.integers(0, 254, size=(T, H), dtype=np.uint8)
    q = q + (q >= 0x7F)                        # skip 0x7F; 253 -> 254 and 0xFF never drawn
    scales = g.uniform(1e-3, 1.0, size=(T, H // 128)).astype(np.float32)
    return q.astype(np.uint8), scales
