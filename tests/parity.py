"""Comparison helpers shared by the GPU parity tests and the smoke check.

The tolerances are those of the method's statement: codes may differ from the
oracle's for at most 0.5 % of the weights (floating-point ties flip and the
flips cascade through the compensation), the layer error ||WX - What X||^2 /
||WX||^2 must be within 2 % of the oracle's, and scales / zeros within 1e-3
relative on groups whose codes match (read as: the group's codes and those of
every earlier column of its row, since the group's parameters are computed from
weights all those decisions compensated).  Packing and g_idx are bit-exact.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from oracle import gptq_oracle as O

CODE_MISMATCH_MAX = 0.005
REL_ERR_TOL = 0.02
SCALE_TOL = 1e-3

# The Hessian kernel's summation, which the Hessian bound below follows: every
# 16-token tensor-core instruction adds 16 exact bf16 products to its fp32
# accumulator; an accumulator starts from zero every 1024 tokens (a chunk); the
# finished chunks are added into fp32 registers with round-to-nearest; at the end
# of a call H_ij += 2 . sum (one more rounding).
HESS_MMA_K = 16
HESS_CHUNK = 1024


def hessian_bound(token_counts) -> float:
    """c such that |H_gpu[i, j] - H[i, j]| <= c . sqrt(H_ii . H_jj), H the exact 2.X.X^T.

    ``token_counts``: the tokens of each accumulate call (kernel launch) that formed H.
    Derivation, with S = sum_t |x_it x_jt| and u = 2^-23 (one fp32 ulp, relative):
    * inside a chunk, each instruction sums 17 terms (16 products and the accumulator),
      each at most sum-so-far <= S_chunk in magnitude; whether the tensor core rounds or
      truncates after aligning them, each term loses at most one ulp: <= 17 u S_chunk per
      instruction, 64 instructions per 1024-token chunk: 1088 u S_chunk;
    * each addition of a chunk into the fp32 register sum rounds to nearest: <= u/2 S
      each, one per chunk, plus the final H += 2 . sum, one per call;
    * 2 S <= sqrt(H_ii H_jj) (Cauchy-Schwarz), the factor 2 being exact.
    So c = 17 . 64 . u + (chunks + calls) . u/2.  At 65,536 tokens in one call,
    c = 1.3e-4: a kernel that dropped one 1024-token chunk (1.6 % of the sum) fails.
    """
    counts = [int(t) for t in token_counts if int(t) > 0]
    chunks = sum((t + HESS_CHUNK - 1) // HESS_CHUNK for t in counts)
    per_chunk = (HESS_MMA_K + 1) * (HESS_CHUNK // HESS_MMA_K)
    return per_chunk * 2.0 ** -23 + (chunks + len(counts)) * 2.0 ** -24


def u_residual_bound(n: int) -> float:
    """Bound on ||U . H_d . U^T . v - v|| / ||v|| for the GPU's U and the exact H_d.

    U H_d U^T = I exactly (H_d^-1 = U^T U); a computed U = (I + F) U_exact gives
    U H_d U^T - I = F + F^T + O(F^2), with F the factor's backward error, which does
    not carry H_d's condition number.  Rounding errors of a length-n fp32 chain grow
    like sqrt(n) times the unit roundoff (fp32 LAPACK factors measured 0.07-0.08 .
    sqrt(n) . 2^-23 for n = 2048 and 4096); the tensor-core products keep operands to
    2^-21 (the TF32 low parts), so the bound is 8 . sqrt(n) . 2^-21.
    """
    return 8.0 * float(np.sqrt(n)) * 2.0 ** -21


@dataclasses.dataclass
class Comparison:
    code_mismatch: float
    rel_err_gpu: float
    rel_err_oracle: float
    rel_err_ratio: float
    scale_max_rel: float
    zero_max_rel: float
    groups_compared: int
    pack_exact: bool
    gidx_exact: bool
    perm_equal: bool

    def ok(self) -> bool:
        return (self.code_mismatch <= CODE_MISMATCH_MAX and abs(self.rel_err_ratio - 1.0) <= REL_ERR_TOL
                and self.scale_max_rel <= SCALE_TOL and self.zero_max_rel <= SCALE_TOL and self.pack_exact
                and self.gidx_exact and self.perm_equal)


def compare_layer(W: np.ndarray, H64: np.ndarray, ora: "O.LayerResult", qweight: np.ndarray, scales16: np.ndarray,
                  zeros16: np.ndarray, gidx: np.ndarray, codes: np.ndarray, perm: np.ndarray, bits: int,
                  group_size: int) -> Comparison:
    n = W.shape[1]
    perm_equal = np.array_equal(perm.astype(np.int64), ora.perm)
    mism = float(np.mean(codes != ora.codes))
    What = O.dequantize(qweight, scales16, zeros16, gidx, bits, n)
    rel_g = O.layer_error(W, What, H64)
    ratio = rel_g / ora.rel_err if ora.rel_err > 0 else (1.0 if rel_g == 0 else np.inf)
    pack_exact = np.array_equal(O.pack(codes, bits).view(np.uint32), qweight.view(np.uint32))
    gidx_exact = np.array_equal(O.g_idx(perm.astype(np.int64), group_size), gidx)
    # Groups (processing order) whose codes match, together with every earlier
    # column of the same row: a group's scale and zero are computed from weights
    # that every earlier decision of the row has compensated, so they are only
    # determined up to rounding when all those decisions agree.
    gs = n if group_size == -1 else group_size
    cp_g = codes[:, ora.perm]
    cp_o = ora.codes[:, ora.perm]
    G = n // gs
    gmatch = (cp_g == cp_o).reshape(codes.shape[0], G, gs).all(axis=2)      # [out, G]
    same = np.logical_and.accumulate(gmatch, axis=1).T                     # [G, out]
    sg = scales16.astype(np.float64)
    so = ora.scales.astype(np.float64)
    zg = zeros16.astype(np.float64)
    zo = ora.zeros.astype(np.float64)
    if same.any():
        s_rel = float(np.max(np.abs(sg[same] - so[same]) / np.maximum(np.abs(so[same]), 1e-30)))
        z_rel = float(np.max(np.abs(zg[same] - zo[same]) / np.maximum(np.abs(zo[same]), 1.0)))
    else:
        s_rel = z_rel = 0.0
    return Comparison(mism, rel_g, ora.rel_err, ratio, s_rel, z_rel, int(same.sum()), pack_exact, gidx_exact,
                      perm_equal)
