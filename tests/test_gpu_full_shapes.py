"""Full-size layers of the Llama-2-7B and Llama-2-70B blocks, CUDA path against the oracle.

Layer shapes (W, H, U) and calibration token counts are the workloads' own.  (With
fewer tokens than input features H is singular: the damping makes it definite, but
directions in X's null space leave the loss unchanged, so rounding differences
flip codes freely there without changing the layer error.  That is why no test
here cuts the tokens below the features.)

Where the oracle cannot redo a stage in seconds at these sizes, it checks what it
can compute exactly:

* Hessian: sampled entries, each the oracle's 2.x_i.x_j^T from the same bits;
* act-order: the order from the oracle's exact diagonal;
* U: for n <= 4096 the oracle's whole preparation of the GPU's H; beyond, the last
  m rows and columns of U, which depend only on the trailing principal block of the
  permuted, damped H (``prepare_trailing``), i.e. the block the blocked
  factorization reaches last;
* the sweep: sampled rows (rows are independent given U) quantized by the oracle
  with the oracle's U (n <= 4096) or the GPU's U (beyond), codes, scales, zeros,
  packing, g_idx and the layer error compared as in the other parity tests.
"""
import dataclasses

import numpy as np
import pytest

import synthetic as S
import tests.parity as P
from oracle import gptq_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_15_b200 as G


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _to_dev_x(x_bits, dev):
    n, t = x_bits.shape
    ld = (t + 7) // 8 * 8
    buf = torch.zeros((n, ld), dtype=torch.int16, device=dev)
    buf[:, :t] = torch.from_numpy(x_bits.view(np.int16)).to(dev)
    return buf.view(torch.bfloat16)[:, :t]


def _gpu_stack(x_bits, st, Ws):
    """One Hessian and one preparation on the GPU, then every W of the same input."""
    dev = _dev()
    n = x_bits.shape[0]
    status = G.new_status(dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hd = torch.zeros(n, dtype=torch.float64, device=dev) if st.desc_act else None
    X = _to_dev_x(x_bits, dev)
    G.hessian_accumulate(H, X, hd, status)
    del X
    prep = G.prepare(H, st.damp_percent, st.desc_act, hd, status)
    qs = [G.quantize_layer(torch.from_numpy(np.ascontiguousarray(W)).to(dev), prep, st.bits, st.group_size, st.sym,
                           st.block, want_codes=True) for W in Ws]
    torch.cuda.synchronize()
    G.raise_on_status(status, "full-shape stack")
    return H, prep, qs


def _exact_diag(x_bits):
    """diag(H) from the oracle, one feature at a time (exact products, fp64 sums)."""
    return np.array([O.hessian(x_bits[i:i + 1])[0, 0] for i in range(x_bits.shape[0])])


def _check_hessian_samples(H, x_bits, d_exact, k=192, seed=0):
    n, N = x_bits.shape
    rng = np.random.default_rng(seed)
    a, b = rng.integers(0, n, k), rng.integers(0, n, k)
    i, j = np.minimum(a, b), np.maximum(a, b)
    i[:16] = j[:16]                                   # a few diagonal entries too
    Hg = H[torch.from_numpy(i).to(H.device), torch.from_numpy(j).to(H.device)].cpu().numpy().astype(np.float64)
    ex = np.array([O.hessian(x_bits[[p, q]])[0, 1] for p, q in zip(i, j)])
    # fp32 accumulation of N exact products, each addition off by at most one ulp:
    # |error| <= N . 2^-23 . sqrt(H_ii H_jj) (Cauchy-Schwarz)
    bound = N * 2.0 ** -23 * np.sqrt(d_exact[i] * d_exact[j])
    assert np.all(np.abs(Hg - ex) <= bound), float(np.max(np.abs(Hg - ex) / bound))


def _symmetric(H):
    return torch.triu(H) + torch.triu(H, 1).T


def _rel_err(Wr, What, Hs64):
    """||(W - What).X||^2 / ||W.X||^2 through H (the objective), fp64 on the device."""
    dev = Hs64.device
    Wt = torch.from_numpy(np.asarray(Wr, np.float64)).to(dev)
    D = Wt - torch.from_numpy(np.asarray(What, np.float64)).to(dev)
    num = ((D @ Hs64) * D).sum()
    den = ((Wt @ Hs64) * Wt).sum()
    return float(num / den)


def _compare_rows(W, q, perm_g, prep_o, rows, st, Hs64):
    bits, gs, sym = st.bits, st.group_size, st.sym
    n = W.shape[1]
    sw, codes_o = O.quantize_layer(W[rows], prep_o, bits, gs, sym, 128)
    codes_g = q.codes.cpu().numpy()
    qw = q.qweight.cpu().numpy()
    assert np.array_equal(O.pack(codes_g, bits).view(np.uint32), qw.view(np.uint32))
    assert np.array_equal(O.g_idx(perm_g, gs), q.g_idx.cpu().numpy())
    mism = float(np.mean(codes_g[rows] != codes_o))
    sc_g = q.scales.cpu().numpy()[:, rows]
    zr_g = q.zeros.cpu().numpy()[:, rows]
    What_g = O.dequantize(qw[:, rows], sc_g, zr_g, q.g_idx.cpu().numpy(), bits, n)
    What_o = O.dequantize(O.pack(codes_o, bits), sw.scales.astype(np.float16), sw.zeros.astype(np.float16),
                          O.g_idx(prep_o.perm, gs), bits, n)
    rel_g, rel_o = _rel_err(W[rows], What_g, Hs64), _rel_err(W[rows], What_o, Hs64)
    Gn = sc_g.shape[0]
    gsz = n if gs == -1 else gs
    cp_g, cp_o = codes_g[rows][:, prep_o.perm], codes_o[:, prep_o.perm]
    same = np.logical_and.accumulate((cp_g == cp_o).reshape(len(rows), Gn, gsz).all(axis=2), axis=1).T
    s_rel = np.max(np.abs(sc_g[same].astype(float) - sw.scales[same]) / sw.scales[same]) if same.any() else 0.0
    z_eq = np.array_equal(zr_g[same].astype(float), sw.zeros[same].astype(float))
    print(f"  {W.shape}: mismatch {mism:.5f} rel_err gpu {rel_g:.6g} oracle {rel_o:.6g} scale_rel {s_rel:.3g}")
    assert mism <= P.CODE_MISMATCH_MAX
    assert abs(rel_g / rel_o - 1) <= P.REL_ERR_TOL
    assert s_rel <= P.SCALE_TOL and z_eq


def _block_check(x_bits, st, Ws, rows_per_layer, m_tail=2048, seed=0):
    n = x_bits.shape[0]
    H, prep, qs = _gpu_stack(x_bits, st, Ws)
    d_exact = _exact_diag(x_bits)
    _check_hessian_samples(H, x_bits, d_exact, seed=seed)
    Hs = _symmetric(H)
    perm_g = prep.perm.cpu().numpy().astype(np.int64)
    dead_g = prep.dead.cpu().numpy().astype(bool)
    U_g = prep.U
    # U's bound: a relative error of n . 2^-23 (fp32 arithmetic over n-long chains)
    tol = n * 2.0 ** -23
    if n <= 4096:
        prep_o = O.prepare(Hs.cpu().numpy().astype(np.float64), st.damp_percent, st.desc_act, order_key=d_exact)
        assert np.array_equal(perm_g, prep_o.perm)
        Ug = U_g.cpu().numpy().astype(np.float64)
        err = np.abs(Ug - prep_o.U).max() / np.abs(prep_o.U).max()
        print(f"  U (n = {n}): max relative difference {err:.3g} (bound {tol:.3g})")
        assert err <= tol
    else:
        Ut_o, perm_o = O.prepare_trailing(Hs.cpu().numpy(), st.damp_percent, st.desc_act, m_tail, order_key=d_exact)
        assert np.array_equal(perm_g, perm_o)
        Ut_g = U_g[n - m_tail:, n - m_tail:].cpu().numpy().astype(np.float64)
        err = np.abs(Ut_g - Ut_o).max() / np.abs(Ut_o).max()
        print(f"  U (n = {n}): last {m_tail} rows and columns, max relative difference {err:.3g} (bound {tol:.3g})")
        assert err <= tol
        # the sweep of sampled rows is compared given the GPU's U
        prep_o = O.Prepared(U=U_g.cpu().numpy(), perm=perm_g, dead=dead_g, lam=0.0, Hd=None)
    Hs64 = Hs.double()
    del Hs
    rng = np.random.default_rng(seed + 1)
    for W, q, k in zip(Ws, qs, rows_per_layer):
        rows = np.sort(rng.choice(W.shape[0], k, replace=False))
        _compare_rows(W, q, perm_g, prep_o, rows, st, Hs64)
    del Hs64, H, prep, qs
    torch.cuda.empty_cache()


def _layers(wl_name, names):
    wl = S.workloads()[wl_name]
    by = {l.name: l for l in wl.layers}
    return [by[nm] for nm in names], wl.settings[0]


def test_llama7b_attention_and_mlp_in_shapes_full_tokens():
    """q [4096 x 4096] and gate [11008 x 4096] share X (4096 features, 65,536 tokens)."""
    (q, gate), st = _layers("llama2-7b-block", ["q", "gate"])
    x = S.make_x(q.x)
    _block_check(x, st, [S.make_w(q.w), S.make_w(gate.w)], [32, 32], seed=7)


@pytest.mark.parametrize("bits,gs", [(3, 128), (2, 64)])
def test_llama7b_down_shape_low_bit(bits, gs):
    """down [4096 x 11008] at 3 and 2 bits (asymmetric, act-order), 32,768 tokens."""
    (down,), st = _layers("llama2-7b-mlp-lowbit", ["down"])
    st = dataclasses.replace(st, bits=bits, group_size=gs)
    x = S.make_x(down.x)
    _block_check(x, st, [S.make_w(down.w)], [24], seed=bits * 100 + gs)


def test_llama70b_block_8192_input_layers():
    """q/o [8192 x 8192], k/v [1024 x 8192], gate/up [28672 x 8192]: one H, three shapes, 65,536 tokens."""
    (q, k, gate), st = _layers("llama2-70b-block", ["q", "k", "gate"])
    x = S.make_x(q.x)
    _block_check(x, st, [S.make_w(q.w), S.make_w(k.w), S.make_w(gate.w)], [16, 16, 16], seed=70)


def test_llama70b_down_28672_input():
    """down [8192 x 28672]: H and U are 28,672 x 28,672; 65,536 tokens."""
    (down,), st = _layers("llama2-70b-block", ["down"])
    x = S.make_x(down.x)
    _block_check(x, st, [S.make_w(down.w)], [8], seed=71)
