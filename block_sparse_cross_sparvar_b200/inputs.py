"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module only draws and lays out numbers; it holds none of the attention,
mask or index-mapping arithmetic.  Both the CUDA path and the CPU oracle are
fed the exact same bf16 bytes produced here.

Workloads imitate the Infinity-2B/8B 1024x1024 generation that the SparVAR
pages describe ("SparVAR: Exploring Sparsity in Visual AutoRegressive
Modeling", ai.info summary, "What This Paper Is About" and "Main Findings"):
trained weights and prompt sets are not available, so activations are drawn
from N(0, 1) with two structures added so that the attention maps show the
sink and locality behaviour the pages report ("Key Contributions" item 1):

* a per-head shared vector (N(0,1) * sink_amp) added to K at every token of the
  first ``n_sink_scales`` scales (sink tokens);
* an optional 2D sin/cos positional component (amplitude ``pe_amp``) added to
  Q and K at each token's position upscaled to the final grid, so that nearby
  tokens of any scale score higher (locality).

Draw order (numpy PCG64, ``default_rng(seed)``): Q, K, V as float32
[B, H, L_total, D] standard normals, then the sink vectors [H, D], then any
block-mask Bernoulli draws.  Values are rounded to bf16 (round to nearest,
ties to even) after the structures are added.
"""
from __future__ import annotations

import numpy as np

# Scale schedules (square side lengths) of the workloads.
INFINITY_SIDES = (1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64)
TINY_SIDES = (1, 2, 4, 8, 16)


def token_offsets(sides):
    """Start index of every scale in the concatenated token sequence (len n+1)."""
    off = [0]
    for s in sides:
        off.append(off[-1] + int(s) * int(s))
    return off


def bf16_round(x: np.ndarray):
    """Round float32 values to bf16 (RNE).  Returns (bits uint16, values float32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    bits = rounded.astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    return bits, vals


def _sincos_2d(y: np.ndarray, x: np.ndarray, D: int, amp: float) -> np.ndarray:
    """[n, D] positional component: first half encodes y, second half x.

    Each half uses D/4 frequencies w_f = 10000^(-f / (D/4)), with a sin and a
    cos channel per frequency.
    """
    nf = D // 4
    f = np.arange(nf, dtype=np.float64)
    w = 10000.0 ** (-f / nf)
    ay = y[:, None] * w[None, :]
    ax = x[:, None] * w[None, :]
    pe = np.concatenate([np.sin(ay), np.cos(ay), np.sin(ax), np.cos(ax)], axis=1)
    return (amp * pe).astype(np.float32)


def positional_table(sides, D: int, amp: float = 1.0) -> np.ndarray:
    """[L_total, D] positional component at each token's upscaled coordinate."""
    final = float(sides[-1])
    ys, xs = [], []
    for s in sides:
        a, b = np.divmod(np.arange(s * s), s)
        ys.append(a * final / s)
        xs.append(b * final / s)
    return _sincos_2d(np.concatenate(ys), np.concatenate(xs), D, amp)


def make_qkv(seed: int, B: int, H: int, sides, D: int, n_sink_scales: int,
             sink_amp: float = 3.0, pe: bool = True, pe_amp: float = 1.0):
    """Draw Q, K, V for the whole multi-scale sequence.

    Returns a dict with ``q``, ``k``, ``v`` as bf16 bit patterns (uint16,
    [B, H, L_total, D]) and ``qf``, ``kf``, ``vf`` as the same values in
    float32, plus ``offsets``.
    """
    rng = np.random.default_rng(seed)
    off = token_offsets(sides)
    L = off[-1]
    q = rng.standard_normal((B, H, L, D), dtype=np.float32)
    k = rng.standard_normal((B, H, L, D), dtype=np.float32)
    v = rng.standard_normal((B, H, L, D), dtype=np.float32)
    sink = rng.standard_normal((H, D), dtype=np.float32) * np.float32(sink_amp)
    n_sink_tok = off[min(n_sink_scales, len(sides))]
    k[:, :, :n_sink_tok, :] += sink[None, :, None, :]
    if pe:
        table = positional_table(sides, D, pe_amp)
        q += table[None, None]
        k += table[None, None]
    out = {"offsets": off, "rng": rng}
    for name, arr in (("q", q), ("k", k), ("v", v)):
        bits, vals = bf16_round(arr)
        out[name] = bits
        out[name + "f"] = vals
    return out


def bernoulli_keep(rng: np.random.Generator, shape, density: float) -> np.ndarray:
    """Independent Bernoulli(density) draws (bool array of ``shape``)."""
    return rng.random(shape) < density


# Workload descriptors.  Sizes follow the Infinity-2B/8B 1024x1024 schedule.
WORKLOADS = {
    # tiny: 1,2,4,8,16 schedule, B1 H2 D64, 16-token blocks, sinks = 2 scales.
    "tiny": dict(sides=TINY_SIDES, B=1, H=2, D=64, n_sink_scales=2, pe=False,
                 radius_prev=1, radius_own=1, block=16),
    # Infinity-2B-like last scale: 64x64 queries over 10521 keys, B2 H16 D128.
    "infinity2b_last": dict(sides=INFINITY_SIDES, B=2, H=16, D=128, n_sink_scales=5,
                            pe=True, radius_prev=2, radius_own=4, block=128),
    # Infinity-8B-like last two scales: B2 H32 D128.
    "infinity8b_last2": dict(sides=INFINITY_SIDES, B=2, H=32, D=128, n_sink_scales=5,
                             pe=True, radius_prev=2, radius_own=4, block=128),
}
