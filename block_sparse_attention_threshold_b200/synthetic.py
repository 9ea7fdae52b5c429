"""Seeded synthetic Q/K/V for the Sol-Attn workloads.

This module only draws inputs. It holds none of the operator's arithmetic
(no pooling, scoring, thresholding or attention), so both the CPU oracle's
tests and the CUDA path can consume it without sharing method code.

The pages run Sol-Attn inside the LTX-2.5 refine stage at 1344x768, 121
frames (Sol-H3 DGX Spark release, arex-research 3d0ff631, section "latent
hand-off: 384p draft to 768p refine"), and the LTX VAE compresses 32x
spatially (Sol-H3 overview, yanziyuan 171844, section 2.1 "how the latent
pass-through works"), which gives a 24x42 latent grid per frame.  The packed sequence is
[text | cond | audio prefix | target video] (yanziyuan 171844, "safety rail"
paragraph).  No model weights exist here, so Q/K/V are synthetic:

* prefix tokens: Q, K, V ~ N(0, 1);
* video tokens, in (t, h, w) raster order over a T x 24 x 42 grid:
  Q = 0.5 * e(t, h, w) @ P_h + sigma * eps_q and K = 0.5 * e @ P_h + sigma * eps_k,
  where e is a 96-wide sinusoidal embedding (16 frequencies
  omega_k = 10000^(-k/16) per axis, sin and cos) and P_h ~ N(0, 1/D) is one
  96 x D matrix per head shared by Q and K, so nearby tokens get correlated
  queries and keys (video locality);
* V ~ N(0, 1).

Draw order from ``numpy.random.default_rng(seed)`` (PCG64): all P_h first
(shape [H, 96, D]), then for each (b, h) in order the Q noise [N, D], the K
noise [N, D] and V [N, D].  Values are generated in fp64 and rounded once to
bf16 with round-to-nearest-even (ties to even on the fp64 bits).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Iterator, Sequence

import numpy as np

BLOCK = 64
N_FREQ = 16
EMB_DIM = 6 * N_FREQ  # (sin, cos) x (t, h, w)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, prefix, video grid, noise and taus."""

    name: str
    B: int
    H: int
    N: int
    D: int
    prefix_len: int
    grid: tuple  # (T, Hg, Wg): the video grid; the first N - prefix_len cells are used
    sigma: float
    taus: tuple
    seed: int
    source_dtype: str = "bf16"  # the workload's declared input precision

    @property
    def M(self) -> int:
        return self.N // BLOCK

    @property
    def P(self) -> int:
        return self.prefix_len // BLOCK

    @property
    def video_len(self) -> int:
        return self.N - self.prefix_len

    def dense_flops(self) -> float:
        """Dense-equivalent attention FLOPs: 4 * N^2 * D per (b, h)."""
        return 4.0 * self.N * self.N * self.D * self.B * self.H

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


NEG_INF = float("-inf")

WORKLOADS = {
    # Tiny case the oracle finishes in well under a second.
    "tiny_n1024": Workload("tiny_n1024", 1, 2, 1024, 64, 128, (4, 16, 16), 1.0,
                           (1.0,), 20260001, "fp32"),
    # Draft-like: 512-token prefix, 16x24x42 grid truncated to 15,616 cells.
    "draft_n16128": Workload("draft_n16128", 1, 40, 16128, 128, 512, (16, 24, 42), 1.0,
                             (1.0,), 20260002),
    # Refine-like: 1,024-token prefix, 32x24x42 grid truncated to 31,744 cells.
    "refine_n32768": Workload("refine_n32768", 1, 40, 32768, 128, 1024, (32, 24, 42), 0.7,
                              (1.25,), 20260003),
    # Long clip: 2,048-token prefix (512 text + 512 cond + 1,024 audio),
    # 63x24x42 grid truncated to 63,488 cells.
    "long_n65536": Workload("long_n65536", 1, 40, 65536, 128, 2048, (63, 24, 42), 0.7,
                            (1.5,), 20260004),
    # Sparsity sweep: 2,048-token prefix, 128x24x42 = 129,024 cells exactly.
    "sweep_n131072": Workload("sweep_n131072", 1, 24, 131072, 128, 2048, (128, 24, 42), 0.7,
                              (NEG_INF, 0.5, 1.0, 1.25, 1.5, 2.0), 20260005),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def video_positions(grid: Sequence[int], count: int) -> np.ndarray:
    """(t, h, w) of the first ``count`` cells of the grid in raster order -> [count, 3]."""
    T, Hg, Wg = grid
    if count > T * Hg * Wg:
        raise ValueError(f"grid {grid} has only {T * Hg * Wg} cells, {count} requested")
    c = np.arange(count, dtype=np.int64)
    return np.stack([c // (Hg * Wg), (c // Wg) % Hg, c % Wg], axis=1)


def sinusoidal_embedding(pos: np.ndarray) -> np.ndarray:
    """[n, 3] integer positions -> [n, 96] fp64 features (sin, cos per axis)."""
    omega = 10000.0 ** (-np.arange(N_FREQ, dtype=np.float64) / N_FREQ)
    feats = []
    for a in range(3):
        ang = pos[:, a:a + 1].astype(np.float64) * omega[None, :]
        feats.append(np.sin(ang))
        feats.append(np.cos(ang))
    return np.concatenate(feats, axis=1)


def fp64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 (nearest, ties to even) in one step; returns uint16 bits.

    Finite inputs of ordinary magnitude only (no NaN/inf handling is needed for
    the generator's values).
    """
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    # bf16 keeps 7 of fp64's 52 mantissa bits: drop 45 bits with RNE.
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    r = (b + (np.uint64((1 << 44) - 1) + lsb)) & ~np.uint64((1 << 45) - 1)
    f32 = r.view(np.float64).astype(np.float32)  # exact: fits in fp32
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_fp64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bits (uint16) to fp64 exactly."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


E4M3_MAX = 448.0  # largest finite OCP FP8 E4M3 value, 1.75 * 2^8


def fp64_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 to OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3
    mantissa bits; no infinities) with round-to-nearest-even in one step,
    saturating at +-448; returns uint8 bits.

    A value's quantum is 2^(e - 3) for its binade exponent e, with e taken as
    at least -6 so that the subnormals (quantum 2^-9) share the smallest
    normal binade's spacing.  x / quantum is exact in fp64, so rounding it
    with numpy's rint (ties to even) is exact RNE.
    """
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, ex = np.frexp(a)                       # a = m * 2^ex, m in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)
    q = np.ldexp(1.0, (e - 3).astype(np.int64))
    r = np.rint(a / q) * q                    # representable; may step up one binade
    _, er = np.frexp(r)
    er = er - 1
    normal = r >= 2.0 ** -6
    exp_field = np.where(normal, er + 7, 0)
    mant = np.where(normal, np.rint(np.ldexp(r, -er.astype(np.int64)) * 8) - 8, np.rint(r * 2.0 ** 9))
    bits = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    bits = np.where(neg, bits | 0x80, bits)
    return bits.astype(np.uint8)


def e4m3_bits_to_fp64(bits: np.ndarray) -> np.ndarray:
    """Decode E4M3 bits (uint8) exactly; the two NaN codes (S.1111.111) give NaN."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    e = (b >> 3) & 15
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, np.ldexp(8.0 + m, (e - 10).astype(np.int64)))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(b & 0x80, -mag, mag)


def _heads(w: Workload, rng: np.random.Generator) -> Iterator[tuple]:
    """Yield (b, h, q64, k64, v64) in draw order, fp64 [N, D] each."""
    proj = rng.standard_normal((w.H, EMB_DIM, w.D)) / math.sqrt(w.D)
    emb = sinusoidal_embedding(video_positions(w.grid, w.video_len))
    L = w.prefix_len
    for b in range(w.B):
        for h in range(w.H):
            signal = 0.5 * (emb @ proj[h])
            q = rng.standard_normal((w.N, w.D))
            k = rng.standard_normal((w.N, w.D))
            v = rng.standard_normal((w.N, w.D))
            q[L:] = signal + w.sigma * q[L:]
            k[L:] = signal + w.sigma * k[L:]
            yield b, h, q, k, v


def generate_bf16(w: Workload) -> tuple:
    """Q, K, V as bf16 bit patterns, uint16 [B, H, N, D] each (C-contiguous)."""
    shape = (w.B, w.H, w.N, w.D)
    q = np.empty(shape, np.uint16)
    k = np.empty(shape, np.uint16)
    v = np.empty(shape, np.uint16)
    for b, h, q64, k64, v64 in _heads(w, np.random.default_rng(w.seed)):
        q[b, h] = fp64_to_bf16_bits(q64)
        k[b, h] = fp64_to_bf16_bits(k64)
        v[b, h] = fp64_to_bf16_bits(v64)
    return q, k, v


def generate_e4m3(w: Workload, scales=(1.0, 1.0, 1.0)) -> tuple:
    """Q, K, V as E4M3 bits, uint8 [B, H, N, D] each: the same draws as
    generate_bf16, each value divided by its tensor's scale and rounded once
    from fp64 to E4M3 (the real value is then the decoded byte times the
    scale)."""
    shape = (w.B, w.H, w.N, w.D)
    q = np.empty(shape, np.uint8)
    k = np.empty(shape, np.uint8)
    v = np.empty(shape, np.uint8)
    sq, sk, sv = (float(x) for x in scales)
    for b, h, q64, k64, v64 in _heads(w, np.random.default_rng(w.seed)):
        q[b, h] = fp64_to_e4m3_bits(q64 / sq)
        k[b, h] = fp64_to_e4m3_bits(k64 / sk)
        v[b, h] = fp64_to_e4m3_bits(v64 / sv)
    return q, k, v


def generate_fp64(w: Workload) -> tuple:
    """Q, K, V before rounding, fp64 [B, H, N, D] (small workloads only)."""
    if w.B * w.H * w.N * w.D > (1 << 26):
        raise ValueError("generate_fp64 is meant for small workloads")
    shape = (w.B, w.H, w.N, w.D)
    q = np.empty(shape)
    k = np.empty(shape)
    v = np.empty(shape)
    for b, h, q64, k64, v64 in _heads(w, np.random.default_rng(w.seed)):
        q[b, h], k[b, h], v[b, h] = q64, k64, v64
    return q, k, v


def sample_query_blocks(M: int, P: int, count: int, seed: int) -> np.ndarray:
    """Sorted, distinct query-block indices: 0, P, M-1 plus seeded others."""
    must = sorted({0, min(P, M - 1), M - 1})
    if count >= M:
        return np.arange(M, dtype=np.int64)
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(M), must)
    extra = rng.choice(rest, size=max(0, count - len(must)), replace=False)
    return np.sort(np.concatenate([np.array(must, np.int64), extra.astype(np.int64)]))
