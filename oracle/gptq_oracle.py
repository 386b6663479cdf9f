"""Plain fp64 CPU oracle of the GPTQ layer solver.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module: only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and reference
legs may call it.  It shares no code with the CUDA library (no headers, tables,
helpers or pre/post-processing); both sides only consume the same seeded inputs.

It restates, step by step and in the pages' order, what the GPTQ pages describe:

* the layer objective, min ||W.X - What.X||^2 ("polydesk.ai/glossaire/gptq",
  section "Comment fonctionne l'algorithme GPTQ");
* the Hessian proxy H = 2.X.X^T (same page, "Etape 2 : Compensation d'erreur via
  la Hessienne");
* a fixed column order, shared by every row (same page, "Etape 1 : Ordre
  arbitraire"), or decreasing activation magnitude with desc_act (same page,
  "Parametres cles de GPTQ", desc_act);
* quantize a column, take its error, push it onto the remaining columns through
  the inverse Hessian via a Cholesky decomposition (same page, "Etape 2");
* lazy batches of 128 columns (same page, "Etape 3 : Mises a jour par blocs");
* groups with their own scale and zero point ("skillmd.com/skills/artubss/gptq",
  "Quantizacao group-wise"; "polydesk.ai/glossaire/gptq", group_size), the
  symmetric range [-2^(b-1)+1, 2^(b-1)-1] with zero exact and the asymmetric
  non-zero zero point (polydesk, "sym"), scale and zero stored in FP16
  ("dev.ayinedjimi-consultants.fr ... ia-quantization-gptq-gguf-awq",
  "Calibration et dataset").

Everything the pages leave open is decided by the readings listed in the
functions below (each says "reading").  Floating point that decides an integer
(a code, a zero point) is taken in fp32, the precision the kernels decide it in;
everything else is fp64.

Library primitives used as steps: matrix products (numpy), the Cholesky
factorization and the triangular inverse (numpy / scipy LAPACK).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np
import scipy.linalg
import scipy.linalg.lapack

__all__ = [
    "bf16_bits_to_f64", "hessian", "hessian_chunked", "hessian_diag", "hessian_matvec", "damped_matvec",
    "act_order", "prepare", "prepare_trailing", "prepare_trailing_x", "Prepared",
    "group_params", "quantize_codes", "dequant_value", "sweep", "SweepResult",
    "g_idx", "unpermute_codes", "pack", "unpack", "dequantize", "layer_error",
    "rtn", "quantize_layer", "LayerResult", "gptq_layer", "pad_layer", "pack_zeros", "unpack_zeros",
    "silu", "mlp_hidden", "mlp_residual",
]

F16_MIN_SUBNORMAL = np.float32(2.0 ** -24)
F16_MAX = np.float32(65504.0)


# --------------------------------------------------------------------------- #
# 1. Hessian  (polydesk, "Etape 2": H = 2.X.X^T from the calibration activations)
# --------------------------------------------------------------------------- #
def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def hessian(x_bits: np.ndarray) -> np.ndarray:
    """H = 2 . X . X^T in fp64.  X is [n, N] (features x tokens) as bf16 bits.

    Every bf16 value and every product of two of them is exact in fp64; only the
    summation over tokens rounds.
    """
    x = bf16_bits_to_f64(x_bits)
    return 2.0 * (x @ x.T)


def hessian_chunked(x_bits: np.ndarray, chunk: int = 8192) -> np.ndarray:
    """``hessian`` summed over token chunks, so that a wide X never has to exist in
    fp64 all at once (the same fp64 sum, taken in another order)."""
    n, N = x_bits.shape
    H = np.zeros((n, n))
    for t0 in range(0, N, chunk):
        H += hessian(x_bits[:, t0:t0 + chunk])
    return H


def hessian_diag(x_bits: np.ndarray, chunk: int = 8192) -> np.ndarray:
    """diag(H) = 2 . sum_t x_it^2 in fp64 (every bf16 square is exact in fp64)."""
    n, N = x_bits.shape
    d = np.zeros(n)
    for t0 in range(0, N, chunk):
        x = bf16_bits_to_f64(x_bits[:, t0:t0 + chunk])
        d += 2.0 * np.einsum("ij,ij->i", x, x)
    return d


def hessian_matvec(x_bits: np.ndarray, V: np.ndarray, chunk: int = 4096) -> np.ndarray:
    """H . V = 2 . X . (X^T . V) in fp64 without forming H (V is [n, k]).

    For layers whose H the oracle cannot form in seconds: O(n.N.k) instead of O(n^2.N).
    """
    n, N = x_bits.shape
    V = np.asarray(V, np.float64)
    out = np.zeros_like(V)
    for t0 in range(0, N, chunk):
        x = bf16_bits_to_f64(x_bits[:, t0:t0 + chunk])
        out += x @ (x.T @ V)
    return 2.0 * out


def damped_matvec(x_bits: np.ndarray, perm: np.ndarray, lam: float, V: np.ndarray) -> np.ndarray:
    """H_d . V for the permuted, damped Hessian of ``prepare`` (no dead inputs), without
    forming it: (H_d . V)[k] = (H . V')[perm[k]] + lam . V[k], V'[perm[k]] = V[k]."""
    V = np.asarray(V, np.float64)
    Vp = np.zeros_like(V)
    Vp[perm] = V
    return hessian_matvec(x_bits, Vp)[perm] + lam * V


# --------------------------------------------------------------------------- #
# 2. Preparation: dead inputs, act-order, damping, Cholesky chain
# --------------------------------------------------------------------------- #
def act_order(diag: np.ndarray) -> np.ndarray:
    """Processing order for desc_act: decreasing activation magnitude.

    Reading (polydesk, desc_act): the activation magnitude of input i is
    diag(H)_i = 2.sum_t x_it^2.  Order by decreasing diag(H); equal keys keep
    their original relative order (lower index first).
    """
    return np.argsort(-np.asarray(diag, dtype=np.float64), kind="stable").astype(np.int64)


@dataclasses.dataclass
class Prepared:
    U: np.ndarray          # [n, n] upper Cholesky factor of (H_p + lam.I)^-1, fp64
    perm: np.ndarray       # [n] processing order: position k holds input column perm[k]
    dead: np.ndarray       # [n] bool, input columns with diag(H) == 0
    lam: float             # damping added to the diagonal
    Hd: np.ndarray         # [n, n] permuted, damped Hessian (fp64)


def prepare(H: np.ndarray, damp_percent: float, desc_act: bool,
            order_key: Optional[np.ndarray] = None) -> Prepared:
    """Damping, act-order permutation and the Cholesky factor of the inverse.

    Steps, in this order:

    1. Dead inputs (reading; the pages are silent): an input whose diag(H) is 0
       never reaches the output; set H_ii = 1 and mark it dead (its weights are
       zeroed before quantization).
    2. desc_act (polydesk, desc_act): perm = act_order(diag(H)); H <- H[perm, perm].
       ``order_key`` may override the sort key (same meaning, e.g. a more
       exactly accumulated diag(H)); it is indexed by original column.
    3. Damping (skillmd, ``damp_percent``, the "fator de amortecimento"):
       reading: lam = damp_percent . mean(diag(H)), added to the diagonal.  Relative
       to the mean diagonal, the result does not change when H is scaled.
    4. Cholesky chain (polydesk, "Etape 2": the inverse Hessian via a Cholesky
       decomposition): L = chol(H_d); H_d^-1 = L^-T . L^-1; U = the upper factor
       with H_d^-1 = U^T . U.
    """
    H = np.array(H, dtype=np.float64, copy=True)
    n = H.shape[0]
    d = np.diag(H).copy()
    dead = d == 0.0
    H[dead, dead] = 1.0
    if desc_act:
        key = np.diag(H).copy() if order_key is None else np.asarray(order_key, np.float64).copy()
        if order_key is not None:
            key[dead] = 1.0
        perm = act_order(key)
    else:
        perm = np.arange(n, dtype=np.int64)
    Hp = H[np.ix_(perm, perm)]
    lam = float(damp_percent) * float(np.mean(np.diag(Hp)))
    Hd = Hp + lam * np.eye(n)
    L = np.linalg.cholesky(Hd)                                            # H_d = L L^T
    Linv, info = scipy.linalg.lapack.dtrtri(L, lower=1)                  # L^-1
    if info != 0:
        raise np.linalg.LinAlgError("triangular inverse failed")
    Hinv = Linv.T @ Linv                                                 # H_d^-1
    Hinv = 0.5 * (Hinv + Hinv.T)
    U = np.linalg.cholesky(Hinv).T                                       # H_d^-1 = U^T U
    return Prepared(U=U, perm=perm, dead=dead, lam=lam, Hd=Hd)


def prepare_trailing(H: np.ndarray, damp_percent: float, desc_act: bool, m: int,
                     order_key: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """The last m rows and columns of U (processing order) and the order, for large n.

    Same steps as ``prepare``; steps 1-3 need only the diagonal of H, and step 4 is
    taken on the trailing m x m block of the permuted, damped H alone.  Why that
    block suffices: H_d^-1 = U^T U gives H_d = V V^T with V = U^-1 upper triangular,
    and for an upper triangular V the trailing block of V V^T is V_22 V_22^T; so
    V_22 is the same factor of H_d's trailing block, and U_22 = V_22^-1 is the upper
    factor of that block's inverse, the last m rows and columns of U.
    """
    H = np.asarray(H)
    return _trailing(np.diag(H).astype(np.float64), lambda idx: np.array(H[np.ix_(idx, idx)], np.float64),
                     damp_percent, desc_act, m, order_key)


def prepare_trailing_x(x_bits: np.ndarray, damp_percent: float, desc_act: bool, m: int,
                       order_key: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """``prepare_trailing`` of H = 2.X.X^T formed from X itself: only the exact
    diagonal and the trailing m x m block of H are computed (for layers whose whole H
    the oracle cannot form in seconds)."""
    return _trailing(hessian_diag(x_bits), lambda idx: hessian_chunked(x_bits[idx]), damp_percent, desc_act, m,
                     order_key)


def _trailing(d: np.ndarray, block, damp_percent: float, desc_act: bool, m: int,
              order_key: Optional[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Steps 1-3 of ``prepare`` from diag(H) ``d``; step 4 on ``block(tail)`` = H[tail, tail]."""
    n = d.shape[0]
    d = d.copy()
    dead = d == 0.0
    d[dead] = 1.0
    if desc_act:
        key = d.copy() if order_key is None else np.asarray(order_key, np.float64).copy()
        if order_key is not None:
            key[dead] = 1.0
        perm = act_order(key)
    else:
        perm = np.arange(n, dtype=np.int64)
    lam = float(damp_percent) * float(np.mean(d))
    tail = perm[n - m:]
    Hs = block(tail)
    Hs[np.arange(m), np.arange(m)] = d[tail] + lam
    L = np.linalg.cholesky(Hs)
    Linv, info = scipy.linalg.lapack.dtrtri(L, lower=1)
    if info != 0:
        raise np.linalg.LinAlgError("triangular inverse failed")
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T, perm


# --------------------------------------------------------------------------- #
# 3. Quantizer (decisions in fp32)
# --------------------------------------------------------------------------- #
def _to_f16_scale(s32: np.ndarray) -> np.ndarray:
    """Round a scale to FP16 (the stored precision), kept within fp16's positive range.

    Reading: the scale is rounded to fp16 *before* it is used, so the value that
    drives the error compensation is the one storage reconstructs.  A scale that
    would round to 0 takes the smallest fp16 subnormal; one beyond fp16's range
    takes its largest finite value.
    """
    s32 = np.asarray(s32, dtype=np.float32)
    s16 = np.clip(s32, F16_MIN_SUBNORMAL, F16_MAX).astype(np.float16).astype(np.float32)
    return np.maximum(s16, F16_MIN_SUBNORMAL)


def group_params(wg: np.ndarray, bits: int, sym: bool) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row scale and zero point of one group.  ``wg`` is [rows, width].

    fp32 arithmetic, one rounding per operation (as IEEE does).

    * Symmetric (polydesk, "sym": the grid [-2^(b-1)+1, 2^(b-1)-1], zero exact):
      a = max |w| (a = 0 -> 1); s = fp16(a / (2^(b-1) - 1)); z = 2^(b-1), so codes
      c = q + z lie in [1, 2^b - 1].
    * Asymmetric (polydesk, "sym": a non-zero zero point): reading: the range
      always includes 0, lo = min(min w, 0), hi = max(max w, 0) (lo = -1, hi = 1 when
      they are equal); s = fp16((hi - lo) / (2^b - 1)); z = clamp(rint(-lo / s), 0,
      2^b - 1).

    Returns (scale, zero) as fp32 arrays of shape [rows]; both are exactly
    representable in fp16.
    """
    wg = np.asarray(wg, dtype=np.float32)
    maxq = np.float32(2 ** bits - 1)
    if sym:
        a = np.max(np.abs(wg), axis=1)
        a = np.where(a == 0, np.float32(1.0), a).astype(np.float32)
        s = _to_f16_scale(a / np.float32(2 ** (bits - 1) - 1))
        z = np.full(wg.shape[0], np.float32(2 ** (bits - 1)), dtype=np.float32)
    else:
        lo = np.minimum(np.min(wg, axis=1), np.float32(0.0)).astype(np.float32)
        hi = np.maximum(np.max(wg, axis=1), np.float32(0.0)).astype(np.float32)
        same = hi == lo
        lo = np.where(same, np.float32(-1.0), lo).astype(np.float32)
        hi = np.where(same, np.float32(1.0), hi).astype(np.float32)
        s = _to_f16_scale((hi - lo) / maxq)
        z = np.clip(np.rint(-lo / s), np.float32(0.0), maxq).astype(np.float32)
    return s, z


def quantize_codes(w: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int, sym: bool) -> np.ndarray:
    """Integer codes of one column (per row), decided in fp32.

    Round to nearest, ties to even (reading; the pages only say "arrondi").
    asym: c = clamp(rint(w / s) + z, 0, 2^b - 1);
    sym:  c = clamp(rint(w / s), -(2^(b-1) - 1), 2^(b-1) - 1) + z.
    """
    w32 = np.asarray(w, dtype=np.float32)
    q = np.rint(w32 / s)
    if sym:
        h = np.float32(2 ** (bits - 1) - 1)
        c = np.clip(q, -h, h) + z
    else:
        c = np.clip(q + z, np.float32(0.0), np.float32(2 ** bits - 1))
    return c.astype(np.int64)


def dequant_value(c: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """What = s . (c - z) (exact in fp64)."""
    return np.asarray(s, np.float64) * (np.asarray(c, np.float64) - np.asarray(z, np.float64))


# --------------------------------------------------------------------------- #
# 4. The column sweep with error compensation and lazy batches
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class SweepResult:
    codes: np.ndarray      # [out, n] uint8, processing order
    scales: np.ndarray     # [G, out] fp32 values exactly representable in fp16
    zeros: np.ndarray      # [G, out] same
    err: np.ndarray        # [out, n] fp64, e_j = (w_j - what_j) / U_jj
    W_final: np.ndarray    # [out, n] fp64, the compensated weights at the time each column was quantized


def sweep(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int, sym: bool,
          block: Optional[int] = 128) -> SweepResult:
    """Quantize the columns of ``Wp`` (already permuted, dead columns zeroed) in order.

    For every column j (polydesk, "Etape 2"):

    * at a group start (j % group_size == 0), the group's per-row scale and zero
      are computed from the *current*, already compensated W[:, j:j+group_size]
      (reading: per-row, per-group parameters); with group_size = -1 one group
      spans the row and is computed at j = 0 (polydesk, group_size -1: per channel);
    * c = quantize(w_j); what = s.(c - z); e = (w_j - what) / U_jj;
    * the remaining columns absorb the error: W[:, k] -= e . U[j, k] for k > j.

    ``block`` = B applies the last step lazily (polydesk, "Etape 3"): inside the
    block immediately, and to the columns after the block once, as
    W[:, end:] -= Err . U[block, end:].  ``block=None`` is the unblocked form.
    For the two to agree exactly, groups must not straddle blocks (B % group_size == 0).
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    out, n = W.shape
    gs = n if group_size == -1 else int(group_size)
    if n % gs != 0:
        raise ValueError("n must be a multiple of group_size")
    B = n if block is None else int(block)
    G = n // gs
    codes = np.zeros((out, n), dtype=np.uint8)
    scales = np.zeros((G, out), dtype=np.float32)
    zeros = np.zeros((G, out), dtype=np.float32)
    err = np.zeros((out, n), dtype=np.float64)
    Wfin = np.zeros((out, n), dtype=np.float64)
    s = z = None
    for b0 in range(0, n, B):
        b1 = min(b0 + B, n)
        for j in range(b0, b1):
            if j % gs == 0:
                g = j // gs
                s, z = group_params(W[:, j:j + gs], bits, sym)
                scales[g], zeros[g] = s, z
            w = W[:, j].copy()
            Wfin[:, j] = w
            c = quantize_codes(w, s, z, bits, sym)
            codes[:, j] = c
            e = (w - dequant_value(c, s, z)) / U[j, j]
            err[:, j] = e
            if j + 1 < b1:
                W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
        if b1 < n:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return SweepResult(codes=codes, scales=scales, zeros=zeros, err=err, W_final=Wfin)


# --------------------------------------------------------------------------- #
# 5. Storage: un-permute, group index, bit-packing, dequantization
# --------------------------------------------------------------------------- #
def g_idx(perm: np.ndarray, group_size: int) -> np.ndarray:
    """Group of every input column (original order).

    Reading: groups are contiguous runs of ``group_size`` columns in *processing*
    order, so with act-order an input column's group is where it was processed:
    g_idx[perm[k]] = k // group_size (0 for group_size = -1).
    """
    n = len(perm)
    gi = np.zeros(n, dtype=np.int32)
    if group_size != -1:
        gi[np.asarray(perm)] = (np.arange(n) // group_size).astype(np.int32)
    return gi


def unpermute_codes(codes_p: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Codes in the original input order: orig[:, perm[k]] = processed[:, k]."""
    orig = np.empty_like(codes_p)
    orig[:, np.asarray(perm)] = codes_p
    return orig


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [out, n] (original order) into qweight int32 [n.bits/32, out].

    Reading (the pages give no layout): along the input dimension, per output
    row, the codes form a little-endian bit stream: input column k occupies bits
    k.bits ... k.bits + bits - 1 of the stream, i.e. bit (k.bits) mod 32 onward of
    32-bit word floor(k.bits / 32); a 3-bit code may continue into the next word.
    """
    codes = np.asarray(codes)
    out, n = codes.shape
    if (n * bits) % 32 != 0:
        raise ValueError("n.bits must be a multiple of 32")
    words = np.zeros((n * bits // 32, out), dtype=np.uint64)
    for k in range(n):
        c = codes[:, k].astype(np.uint64)
        pos = k * bits
        wi, off = pos // 32, pos % 32
        words[wi] |= (c << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            words[wi + 1] |= c >> np.uint64(32 - off)
    return words.astype(np.uint32).view(np.int32)


def unpack(qweight: np.ndarray, bits: int, n: int) -> np.ndarray:
    """Inverse of ``pack``: qweight [n.bits/32, out] -> codes [out, n] uint8."""
    q = np.asarray(qweight).view(np.uint32).astype(np.uint64)
    out = q.shape[1]
    codes = np.zeros((out, n), dtype=np.uint8)
    mask = np.uint64(2 ** bits - 1)
    for k in range(n):
        pos = k * bits
        wi, off = pos // 32, pos % 32
        v = q[wi] >> np.uint64(off)
        if off + bits > 32:
            v |= q[wi + 1] << np.uint64(32 - off)
        codes[:, k] = (v & mask).astype(np.uint8)
    return codes


def dequantize(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray, gidx: np.ndarray,
               bits: int, n: int) -> np.ndarray:
    """What [out, n] (original order, fp64) from the stored format."""
    codes = unpack(qweight, bits, n).astype(np.float64)
    s = np.asarray(scales, np.float64)[np.asarray(gidx)].T      # [out, n]
    z = np.asarray(zeros, np.float64)[np.asarray(gidx)].T
    return s * (codes - z)


def layer_error(W: np.ndarray, What: np.ndarray, H: np.ndarray) -> float:
    """||W.X - What.X||^2 / ||W.X||^2 through H = 2.X.X^T (polydesk, the objective).

    With D = W - What: ||D.X||^2 = tr(D.X.X^T.D^T) = tr(D.H.D^T) / 2, and the 2
    cancels in the ratio.
    """
    W = np.asarray(W, np.float64)
    D = W - np.asarray(What, np.float64)
    num = np.einsum("ij,ij->", D @ H, D)
    den = np.einsum("ij,ij->", W @ H, W)
    return float(num / den) if den != 0 else 0.0


def rtn(W: np.ndarray, bits: int, group_size: int, sym: bool,
        perm: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Round-to-nearest with the same quantizer and groups, no compensation.

    The comparison point the pages dismiss at 4 bits (polydesk, "Le probleme que
    GPTQ resout").  Groups are contiguous in the given processing order.
    Returns (codes [out, n] processing order, scales [G, out], zeros [G, out]).
    """
    W = np.asarray(W, np.float64)
    if perm is not None:
        W = W[:, np.asarray(perm)]
    out, n = W.shape
    gs = n if group_size == -1 else group_size
    G = n // gs
    codes = np.zeros((out, n), dtype=np.uint8)
    scales = np.zeros((G, out), np.float32)
    zeros = np.zeros((G, out), np.float32)
    for g in range(G):
        wg = W[:, g * gs:(g + 1) * gs]
        s, z = group_params(wg, bits, sym)
        scales[g], zeros[g] = s, z
        w32 = wg.astype(np.float32)
        q = np.rint(w32 / s[:, None])
        if sym:
            h = np.float32(2 ** (bits - 1) - 1)
            c = np.clip(q, -h, h) + z[:, None]
        else:
            c = np.clip(q + z[:, None], 0, 2 ** bits - 1)
        codes[:, g * gs:(g + 1) * gs] = c.astype(np.uint8)
    return codes, scales, zeros


# --------------------------------------------------------------------------- #
# 6. The whole layer
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class LayerResult:
    qweight: np.ndarray     # int32 [n.bits/32, out]
    scales: np.ndarray      # float16 [G, out]
    zeros: np.ndarray       # float16 [G, out]
    g_idx: np.ndarray       # int32 [n]
    codes: np.ndarray       # uint8 [out, n], original order
    perm: np.ndarray        # int64 [n]
    prep: Prepared
    sw: SweepResult
    rel_err: float          # layer error of the stored result against the undamped H
    rel_err_rtn: float      # the same for round-to-nearest


def quantize_layer(W: np.ndarray, prep: Prepared, bits: int, group_size: int, sym: bool,
                   block: Optional[int] = 128) -> Tuple[SweepResult, np.ndarray]:
    """Permute W, zero dead inputs, sweep.  Returns (sweep result, codes in original order)."""
    Wp = np.asarray(W, dtype=np.float64).copy()
    Wp[:, prep.dead] = 0.0
    Wp = Wp[:, prep.perm]
    sw = sweep(Wp, prep.U, bits, group_size, sym, block)
    return sw, unpermute_codes(sw.codes, prep.perm)


def gptq_layer(W: np.ndarray, x_bits: Optional[np.ndarray], bits: int, group_size: int, sym: bool,
               desc_act: bool, damp_percent: float = 0.01, block: Optional[int] = 128,
               H: Optional[np.ndarray] = None, with_rtn: bool = True) -> LayerResult:
    """The whole path for one layer: H, prepare, sweep, pack, metrics."""
    if H is None:
        H = hessian(x_bits)
    prep = prepare(H, damp_percent, desc_act)
    sw, codes = quantize_layer(W, prep, bits, group_size, sym, block)
    n = codes.shape[1]
    qw = pack(codes, bits)
    gi = g_idx(prep.perm, group_size)
    scales16 = sw.scales.astype(np.float16)
    zeros16 = sw.zeros.astype(np.float16)
    What = dequantize(qw, scales16, zeros16, gi, bits, n)
    rel = layer_error(W, What, H)
    rel_rtn = float("nan")
    if with_rtn:
        rc, rs, rz = rtn(W, bits, group_size, sym, prep.perm)
        qr = pack(unpermute_codes(rc, prep.perm), bits)
        rel_rtn = layer_error(W, dequantize(qr, rs.astype(np.float16), rz.astype(np.float16), gi, bits, n), H)
    return LayerResult(qweight=qw, scales=scales16, zeros=zeros16, g_idx=gi, codes=codes,
                       perm=prep.perm, prep=prep, sw=sw, rel_err=rel, rel_err_rtn=rel_rtn)


# --------------------------------------------------------------------------- #
# 7. Checkpoint variants: zero padding, packed zero points
# --------------------------------------------------------------------------- #
def pad_layer(W: np.ndarray, x_bits: Optional[np.ndarray], n: int) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """The layer zero-padded to n inputs.

    polydesk, "Limites de GPTQ" (divisibility): a width that the group size does
    not divide is handled by padding the weights with zeros.  Reading: W gets
    n - in zero columns and X (bf16 bit patterns) n - in zero rows, i.e. the padded
    inputs carry no activation; the padded layer then goes through the ordinary
    path, where those inputs are dead (zero diagonal) and count in the damping's
    mean diagonal like any other input.
    """
    W = np.asarray(W)
    out, k = W.shape
    if n < k:
        raise ValueError("padded width smaller than the layer")
    Wp = np.zeros((out, n), dtype=W.dtype)
    Wp[:, :k] = W
    xp = None
    if x_bits is not None:
        x_bits = np.asarray(x_bits)
        xp = np.zeros((n, x_bits.shape[1]), dtype=x_bits.dtype)     # bit pattern 0 is +0.0
        xp[:k] = x_bits
    return Wp, xp


def pack_zeros(zeros: np.ndarray, bits: int, zero_offset: int = 0) -> np.ndarray:
    """Zero points [G, out] -> int32 [G, out.bits/32], packed along the output dimension.

    The pages store zero points in FP16 (ayinedjimi-consultants, "Calibration et
    dataset") and warn that checkpoints of different tool versions differ
    (polydesk, "Limites de GPTQ").  Reading for the packed integer form: per group,
    the values (zero - zero_offset) mod 2^bits form a little-endian bit stream
    along the outputs, output o at stream bits o.bits ... (the stream of ``pack``,
    taken along the other dimension); zero_offset 1 is the older convention of
    storing zero - 1.
    """
    z = np.asarray(zeros, dtype=np.float64)
    if z.ndim != 2:
        raise ValueError("zeros must be [G, out]")
    if np.any(z != np.rint(z)) or np.any(z < 0) or np.any(z > 2 ** bits - 1):
        raise ValueError("zero points must be integers in [0, 2^bits - 1]")
    if zero_offset not in (0, 1):
        raise ValueError("zero_offset must be 0 or 1")
    G, out = z.shape
    if (out * bits) % 32 != 0:
        raise ValueError("out.bits must be a multiple of 32")
    v = ((z.astype(np.int64) - zero_offset) % (2 ** bits)).astype(np.uint64)
    words = np.zeros((G, out * bits // 32), dtype=np.uint64)
    for o in range(out):
        pos = o * bits
        wi, off = pos // 32, pos % 32
        words[:, wi] |= (v[:, o] << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            words[:, wi + 1] |= v[:, o] >> np.uint64(32 - off)
    return words.astype(np.uint32).view(np.int32)


def unpack_zeros(qzeros: np.ndarray, bits: int, out: int, zero_offset: int = 0) -> np.ndarray:
    """Inverse of ``pack_zeros``: int32 [G, out.bits/32] -> zero points [G, out] (float64)."""
    q = np.asarray(qzeros).view(np.uint32).astype(np.uint64)
    G = q.shape[0]
    z = np.zeros((G, out), dtype=np.float64)
    mask = np.uint64(2 ** bits - 1)
    for o in range(out):
        pos = o * bits
        wi, off = pos // 32, pos % 32
        v = q[:, wi] >> np.uint64(off)
        if off + bits > 32:
            v |= q[:, wi + 1] << np.uint64(32 - off)
        z[:, o] = ((v & mask).astype(np.int64) + zero_offset) % (2 ** bits)
    return z


# --------------------------------------------------------------------------- #
# The forward pass of a quantized MLP block (the sequential pipeline)
# --------------------------------------------------------------------------- #
# Reading: the pages quantize layer by layer, each layer calibrated on the outputs of
# the layers quantized before it (polydesk, GPTQ works layer by layer); the blocks are
# Llama-shaped (the workloads'), whose MLP is down(silu(gate x) . up x) with a
# residual connection around it.  In fp64 from the dequantized weights.
def silu(g: np.ndarray) -> np.ndarray:
    """silu(g) = g / (1 + exp(-g))."""
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g))


def mlp_hidden(x_bits: np.ndarray, What_gate: np.ndarray, What_up: np.ndarray) -> np.ndarray:
    """h = silu(What_gate . X) * (What_up . X), X [d, tokens] as bf16 bits, h [d_ff, tokens]."""
    x = bf16_bits_to_f64(x_bits)
    return silu(np.asarray(What_gate, np.float64) @ x) * (np.asarray(What_up, np.float64) @ x)


def mlp_residual(x_bits: np.ndarray, What_down: np.ndarray, h: np.ndarray) -> np.ndarray:
    """The block's output X + What_down . h (fp64)."""
    return bf16_bits_to_f64(x_bits) + np.asarray(What_down, np.float64) @ np.asarray(h, np.float64)
