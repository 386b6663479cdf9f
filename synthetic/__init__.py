"""Seeded synthetic inputs for the GPTQ layer solver.

This module is shared by the CUDA path's tests and benchmark and by the oracle's
tests.  It holds no arithmetic of the method itself: it only draws the calibration
activations X and the weights W that both sides consume, in the shapes the GPTQ
pages use (a [1024, 4096] layer from "skillmd.com/skills/artubss/gptq",
section "Quantização group-wise"; Llama-shaped blocks; a few hundred calibration
sequences of 512 tokens from "dev.ayinedjimi-consultants.fr ... ia-quantization-
gptq-gguf-awq", section "Calibration et dataset").

The pages calibrate on C4 / WikiText-2 activations of trained models.  Neither the
datasets nor the weights exist here, so X is drawn from an outlier-heavy,
low-rank-plus-identity generator that stands in for them:

    X = diag(s) . (G . Z_r + Z_n)

* ``s_i ~ LogNormal(0, 1)`` per feature, and ``round(p.n)`` features chosen
  without replacement are multiplied by ``k`` (outlier channels);
* ``G ~ N(0, 1) / sqrt(r)`` is [n, r]; ``Z_r`` [r, N] and ``Z_n`` [n, N] are N(0, 1),
  i.e. ``A = [G | I_n]`` applied to a standard normal ``Z``;
* the result is rounded to bf16 (round to nearest even) and stored [n, N]
  row-major, tokens contiguous, as the raw 16-bit patterns (``numpy.uint16``).

W is drawn N(0, sigma^2) in fp32 and kept fp32 or rounded to fp16.

Every tensor comes from its own ``numpy.random.SeedSequence`` sub-stream keyed by
(seed, stream tag, chunk index), so any token range of X can be regenerated on its
own and the bytes never depend on how they were produced.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# Tokens per independently seeded chunk of X.  Fixed, so that a sub-range of
# tokens regenerates to the same bytes as the full matrix.
X_CHUNK = 4096

# Stream tags (the second word of every SeedSequence entropy key).
_TAG_SCALE = 1
_TAG_OUTLIER = 2
_TAG_LOWRANK = 3
_TAG_ZR = 4
_TAG_ZN = 5
_TAG_W = 6


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, key)])))


# --------------------------------------------------------------------------- #
# bf16 / fp16 storage helpers (input preparation only)
# --------------------------------------------------------------------------- #
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the bit patterns."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    nan = np.isnan(u.view(np.float32))
    _round_bf16_inplace(u)
    if nan.any():
        u[nan] = 0x7FC0
    return u.astype(np.uint16)


def _round_bf16_inplace(u: np.ndarray) -> None:
    """u: uint32 view of finite fp32 values; leaves the bf16 pattern in the low 16 bits."""
    t = np.right_shift(u, 16)
    np.bitwise_and(t, 1, out=t)
    t += np.uint32(0x7FFF)
    u += t
    np.right_shift(u, 16, out=u)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------- #
# X: calibration activations
# --------------------------------------------------------------------------- #
@dataclasses.dataclass(frozen=True)
class XSpec:
    n: int                 # features (the layer's input width)
    tokens: int            # calibration tokens N
    rank: int              # r of the low-rank component
    outlier_frac: float    # p
    outlier_mult: float    # k
    seed: int
    stream: int            # distinguishes the X of different layers in one block


def _x_feature_terms(spec: XSpec) -> Tuple[np.ndarray, np.ndarray]:
    n = spec.n
    s = np.exp(_rng(spec.seed, spec.stream, _TAG_SCALE).standard_normal(n))
    n_out = int(round(spec.outlier_frac * n))
    if n_out > 0:
        idx = _rng(spec.seed, spec.stream, _TAG_OUTLIER).choice(n, size=n_out, replace=False)
        s[idx] *= spec.outlier_mult
    r = max(int(spec.rank), 0)
    G = _rng(spec.seed, spec.stream, _TAG_LOWRANK).standard_normal((n, r)) / math.sqrt(max(r, 1))
    return s.astype(np.float64), G.astype(np.float64)


def make_x(spec: XSpec, t0: int = 0, t1: Optional[int] = None) -> np.ndarray:
    """Tokens [t0, t1) of X as bf16 bit patterns, shape [n, t1 - t0], row-major."""
    if t1 is None:
        t1 = spec.tokens
    if not (0 <= t0 <= t1 <= spec.tokens):
        raise ValueError("token range out of bounds")
    s, G = _x_feature_terms(spec)
    s32 = s.astype(np.float32)
    G32 = G.astype(np.float32)
    out = np.empty((spec.n, t1 - t0), dtype=np.uint16)

    def fill(c: int) -> None:
        a = c * X_CHUNK
        b = min(a + X_CHUNK, spec.tokens)
        w = b - a
        zr = _rng(spec.seed, spec.stream, _TAG_ZR, c).standard_normal((G.shape[1], w), dtype=np.float32)
        zn = _rng(spec.seed, spec.stream, _TAG_ZN, c).standard_normal((spec.n, w), dtype=np.float32)
        blk = G32 @ zr
        blk += zn
        del zn
        blk *= s32[:, None]
        u = blk.view(np.uint32)
        _round_bf16_inplace(u)
        lo, hi = max(a, t0), min(b, t1)
        out[:, lo - t0:hi - t0] = u[:, lo - a:hi - a]

    chunks = range(t0 // X_CHUNK, (t1 + X_CHUNK - 1) // X_CHUNK)
    workers = max(1, min(len(chunks), os.cpu_count() or 1, 16))
    if workers == 1:
        for c in chunks:
            fill(c)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, chunks))
    return out


# --------------------------------------------------------------------------- #
# W: layer weights
# --------------------------------------------------------------------------- #
@dataclasses.dataclass(frozen=True)
class WSpec:
    out: int
    n: int
    sigma: float
    dtype: str   # "f32" or "f16"
    seed: int
    stream: int


def make_w(spec: WSpec) -> np.ndarray:
    """W [out, n] row-major, fp32 or fp16."""
    w = _rng(spec.seed, spec.stream, _TAG_W).standard_normal((spec.out, spec.n), dtype=np.float32)
    w *= np.float32(spec.sigma)
    if spec.dtype == "f16":
        return w.astype(np.float16)
    if spec.dtype == "f32":
        return w
    raise ValueError(spec.dtype)


# --------------------------------------------------------------------------- #
# The same recipe drawn on the device (benchmarks)
# --------------------------------------------------------------------------- #
def make_x_device(spec: XSpec, device, chunk: int = 8192):
    """X [n, tokens] as a torch bf16 tensor drawn on ``device`` with torch's generator.

    Same recipe as ``make_x`` (the per-feature scales and the low-rank factor are
    make_x's own; Z is drawn by torch), so the values differ from make_x's but the
    distribution does not.  For benchmarks of large workloads, where generating X on
    the host would take longer than the work itself; parity tests use make_x.
    """
    import torch
    s, G = _x_feature_terms(spec)
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(spec.seed) * 1000003 + int(spec.stream) * 7919 + 17)
    s32 = torch.from_numpy(s.astype(np.float32)).to(dev)[:, None]
    G32 = torch.from_numpy(G.astype(np.float32)).to(dev)
    ld = (spec.tokens + 7) // 8 * 8
    out = torch.empty((spec.n, ld), dtype=torch.bfloat16, device=dev)
    for a in range(0, spec.tokens, chunk):
        w = min(chunk, spec.tokens - a)
        zr = torch.randn((G32.shape[1], w), generator=gen, device=dev, dtype=torch.float32)
        blk = torch.randn((spec.n, w), generator=gen, device=dev, dtype=torch.float32)
        blk.addmm_(G32, zr)
        blk.mul_(s32)
        out[:, a:a + w] = blk.to(torch.bfloat16)       # round to nearest even
    return out[:, :spec.tokens]


def make_w_device(spec: WSpec, device):
    """W [out, n] drawn on ``device`` with torch's generator (make_w's recipe; other values)."""
    import torch
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(spec.seed) * 1000003 + int(spec.stream) * 7919 + 29)
    w = torch.randn((spec.out, spec.n), generator=gen, device=dev, dtype=torch.float32)
    w.mul_(float(spec.sigma))
    return w.half() if spec.dtype == "f16" else w


# --------------------------------------------------------------------------- #
# Workloads
# --------------------------------------------------------------------------- #
@dataclasses.dataclass(frozen=True)
class QuantSettings:
    bits: int
    group_size: int
    sym: bool
    desc_act: bool
    damp_percent: float = 0.01
    block: int = 128


@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    w: WSpec
    x: XSpec


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[Layer, ...]
    settings: Tuple[QuantSettings, ...]

    @property
    def params(self) -> int:
        return sum(l.w.out * l.w.n for l in self.layers)


def _block(name: str, dims: Sequence[Tuple[str, int, int, int]], tokens: int, rank: int,
           frac: float, mult: float, sigma: float, settings: Sequence[QuantSettings],
           seed: int = 0) -> Workload:
    layers = []
    for i, (lname, out, n, xstream) in enumerate(dims):
        layers.append(Layer(lname, WSpec(out, n, sigma, "f16", seed, 100 + i),
                            XSpec(n, tokens, rank, frac, mult, seed, xstream)))
    return Workload(name, tuple(layers), tuple(settings))


def workloads(seed: int = 0) -> Dict[str, Workload]:
    """The five workloads, by name.

    * ``layer-256x512``: one fp32 layer [256, 512], 2048 tokens, rank 32,
      1 % outliers x20; 4-bit asymmetric g128, no act-order.
    * ``layer-1024x4096``: the pages' worked-example shape [1024, 4096] fp16
      (32,768 groups of 128), 65,536 tokens (128 sequences x 512), rank 64;
      4-bit asymmetric g128, no act-order.
    * ``llama2-7b-block``: q, k, v, o [4096, 4096], gate, up [11008, 4096],
      down [4096, 11008]; 65,536 tokens; 4-bit symmetric g128, act-order.
    * ``llama2-7b-mlp-lowbit``: gate [11008, 4096] and down [4096, 11008],
      32,768 tokens, 2 % outliers x30; bits {3, 2} x group {128, 64},
      asymmetric, act-order.
    * ``llama2-70b-block``: q, o [8192, 8192], k, v [1024, 8192], gate, up
      [28672, 8192], down [8192, 28672]; 65,536 tokens, rank 128; 4-bit
      symmetric g128, act-order.

    Layers of one block that read the same activations (q/k/v; gate/up) share
    an X stream; o and down have their own.
    """
    w: Dict[str, Workload] = {}
    w["layer-256x512"] = Workload(
        "layer-256x512",
        (Layer("linear", WSpec(256, 512, 0.02, "f32", seed, 100), XSpec(512, 2048, 32, 0.01, 20.0, seed, 1)),),
        (QuantSettings(4, 128, False, False),))
    w["layer-1024x4096"] = Workload(
        "layer-1024x4096",
        (Layer("linear", WSpec(1024, 4096, 0.02, "f16", seed, 100), XSpec(4096, 65536, 64, 0.01, 20.0, seed, 1)),),
        (QuantSettings(4, 128, False, False),))
    w["llama2-7b-block"] = _block(
        "llama2-7b-block",
        [("q", 4096, 4096, 1), ("k", 4096, 4096, 1), ("v", 4096, 4096, 1), ("o", 4096, 4096, 2),
         ("gate", 11008, 4096, 3), ("up", 11008, 4096, 3), ("down", 4096, 11008, 4)],
        65536, 64, 0.01, 20.0, 0.02, [QuantSettings(4, 128, True, True)], seed)
    w["llama2-7b-mlp-lowbit"] = _block(
        "llama2-7b-mlp-lowbit",
        [("gate", 11008, 4096, 3), ("down", 4096, 11008, 4)],
        32768, 64, 0.02, 30.0, 0.02,
        [QuantSettings(b, g, False, True) for b in (3, 2) for g in (128, 64)], seed)
    w["llama2-70b-block"] = _block(
        "llama2-70b-block",
        [("q", 8192, 8192, 1), ("k", 1024, 8192, 1), ("v", 1024, 8192, 1), ("o", 8192, 8192, 2),
         ("gate", 28672, 8192, 3), ("up", 28672, 8192, 3), ("down", 8192, 28672, 4)],
        65536, 128, 0.01, 20.0, 0.015, [QuantSettings(4, 128, True, True)], seed)
    return w


def small_case(out: int, n: int, tokens: int, seed: int, rank: int = 8, frac: float = 0.02,
               mult: float = 20.0, sigma: float = 0.02, wdtype: str = "f32") -> Tuple[np.ndarray, np.ndarray]:
    """A small (W, X) pair from the same generator, for tests."""
    x = make_x(XSpec(n, tokens, rank, frac, mult, seed, 1))
    wt = make_w(WSpec(out, n, sigma, wdtype, seed, 100))
    return wt, x


__all__: List[str] = [
    "X_CHUNK", "XSpec", "WSpec", "QuantSettings", "Layer", "Workload",
    "make_x", "make_w", "make_x_device", "make_w_device", "workloads", "small_case", "f32_to_bf16_bits", "bf16_bits_to_f32",
]
