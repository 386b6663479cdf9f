"""Full-size layers of the Llama-2-7B and Llama-2-70B blocks, CUDA path against the oracle.

Layer shapes (W, H, U), settings and calibration token counts are the workloads' own:
the 7B block at 65,536 tokens (4-bit symmetric g128, act-order), the 7B MLP pair at
32,768 tokens under all four low-bit settings (3/2 bits x g128/g64, asymmetric,
act-order), the 70B block at 65,536 tokens.  (With fewer tokens than input features
H is singular: the damping makes it definite, but directions in X's null space
leave the loss unchanged, so rounding differences flip codes freely there without
changing the layer error.  That is why no test here cuts the tokens.)

Nothing the checks compare against comes from the GPU: every reference is the
oracle's, computed from the same X.

* up to 11,008 inputs the oracle forms H itself (fp64, summed over token chunks):
  every upper entry of the GPU's H within the bound derived from the kernel's
  chunked summation; the oracle's own preparation (order, damping, U) against the
  GPU's, U element by element; the sweep of sampled rows (rows are independent given
  U) with the oracle's own U, and the layer error through the oracle's H;
* beyond (the 28,672-input layer), where the oracle cannot form H in seconds: sampled
  entries of H under the same bound; the order from the oracle's exact diagonal; the
  last 2048 rows and columns of U from the oracle's own trailing block of H
  (``prepare_trailing_x``); all of U through the residual U . H_d . U^T . v - v with
  the oracle's H_d applied from X (``damped_matvec``), for random and unit vectors;
  the sweep of sampled rows given the GPU's U (which that residual has just checked),
  and the layer error through the oracle's H . v.
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

# the largest input width whose H and U the oracle forms whole (fp64, ~20 s on the host)
ORACLE_FULL_MAX = 11008


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


@dataclasses.dataclass
class Job:
    W: np.ndarray
    st: "S.QuantSettings"
    rows: int          # rows the oracle sweeps


def _gpu_stack(x_bits, damp, desc_act, jobs):
    """One Hessian and one preparation on the GPU, then every job on the same input."""
    dev = _dev()
    n = x_bits.shape[0]
    status = G.new_status(dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hd = torch.zeros(n, dtype=torch.float64, device=dev) if desc_act else None
    X = _to_dev_x(x_bits, dev)
    G.hessian_accumulate(H, X, hd, status)
    del X
    prep = G.prepare(H, damp, desc_act, hd, status)
    qs = []
    for j in jobs:
        W = torch.from_numpy(np.ascontiguousarray(j.W)).to(dev)
        qs.append(G.quantize_layer(W, prep, j.st.bits, j.st.group_size, j.st.sym, j.st.block, want_codes=True))
        del W
    torch.cuda.synchronize()
    G.raise_on_status(status, "full-shape stack")
    return H, prep, qs


def _check_hessian_full(H, H64, N):
    """Every upper entry of the GPU's H against the oracle's, in row slabs."""
    n = H64.shape[0]
    d = np.sqrt(np.diag(H64))
    c = P.hessian_bound([N])
    worst = 0.0
    for r0 in range(0, n, 1024):
        r1 = min(n, r0 + 1024)
        Hg = H[r0:r1].cpu().numpy().astype(np.float64)
        err = np.abs(Hg - H64[r0:r1]) / np.outer(d[r0:r1], d)
        err = np.triu(err, r0)                       # upper entries of these rows
        worst = max(worst, float(err.max()))
    print(f"  H: max |dH| / sqrt(H_ii H_jj) {worst:.3g} (bound {c:.3g})")
    assert worst <= c


def _check_hessian_samples(H, x_bits, d_exact, k=192, seed=0):
    n, N = x_bits.shape
    rng = np.random.default_rng(seed)
    a, b = rng.integers(0, n, k), rng.integers(0, n, k)
    i, j = np.minimum(a, b), np.maximum(a, b)
    i[:16] = j[:16]                                   # a few diagonal entries too
    Hg = H[torch.from_numpy(i).to(H.device), torch.from_numpy(j).to(H.device)].cpu().numpy().astype(np.float64)
    ex = np.array([O.hessian_chunked(x_bits[[p, q]])[0, 1] for p, q in zip(i, j)])
    err = np.abs(Hg - ex) / np.sqrt(d_exact[i] * d_exact[j])
    c = P.hessian_bound([N])
    print(f"  H ({k} sampled entries): max |dH| / sqrt(H_ii H_jj) {err.max():.3g} (bound {c:.3g})")
    assert np.all(err <= c)


def _check_u_residual(U_dev, Hd_matvec, seed=0):
    """max over test vectors of ||U . H_d . U^T . v - v|| / ||v||: 4 random vectors and
    8 unit vectors e_k spread over the rows (U^T e_k is row k of U)."""
    n = U_dev.shape[0]
    rng = np.random.default_rng(seed)
    ks = np.unique(np.concatenate([[0, 1, 127, 128], rng.integers(0, n, 3), [n - 1]]))
    V = np.zeros((n, 4 + len(ks)))
    V[:, :4] = rng.standard_normal((n, 4))
    V[ks, 4 + np.arange(len(ks))] = 1.0
    U64 = U_dev.double()
    Y = (U64.T @ torch.from_numpy(V).to(U64.device)).cpu().numpy()           # U^T v
    Z = Hd_matvec(Y)                                                       # H_d U^T v  (oracle)
    R = (U64 @ torch.from_numpy(Z).to(U64.device)).cpu().numpy() - V     # U H_d U^T v - v
    del U64
    res = float(np.max(np.linalg.norm(R, axis=0) / np.linalg.norm(V, axis=0)))
    tol = P.u_residual_bound(n)
    print(f"  U: max ||U H_d U^T v - v|| / ||v|| {res:.3g} (bound {tol:.3g})")
    assert res <= tol


def _compare_rows(job, q, perm_g, prep_o, rows, err_of):
    W, st = job.W, job.st
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
    rel_g, rel_o = err_of(W[rows], What_g), err_of(W[rows], What_o)
    Gn = sc_g.shape[0]
    gsz = n if gs == -1 else gs
    cp_g, cp_o = codes_g[rows][:, prep_o.perm], codes_o[:, prep_o.perm]
    same = np.logical_and.accumulate((cp_g == cp_o).reshape(len(rows), Gn, gsz).all(axis=2), axis=1).T
    s_rel = np.max(np.abs(sc_g[same].astype(float) - sw.scales[same]) / sw.scales[same]) if same.any() else 0.0
    z_eq = np.array_equal(zr_g[same].astype(float), sw.zeros[same].astype(float))
    print(f"  {W.shape} {bits}-bit g{gs} {'sym' if sym else 'asym'}: mismatch {mism:.5f} rel_err gpu {rel_g:.6g} "
          f"oracle {rel_o:.6g} scale_rel {s_rel:.3g}")
    assert mism <= P.CODE_MISMATCH_MAX
    assert abs(rel_g / rel_o - 1) <= P.REL_ERR_TOL
    assert s_rel <= P.SCALE_TOL and z_eq


def _input_check(x_bits, damp, desc_act, jobs, seed=0, m_tail=2048):
    """Everything computed from one input X, checked against the oracle (module docstring)."""
    n, N = x_bits.shape
    H, prep, qs = _gpu_stack(x_bits, damp, desc_act, jobs)
    perm_g = prep.perm.cpu().numpy().astype(np.int64)
    assert not prep.dead.cpu().numpy().any()
    tol_u = n * 2.0 ** -23          # U element by element: fp32-level arithmetic over n-long chains
    if n <= ORACLE_FULL_MAX:
        H64 = O.hessian_chunked(x_bits)
        _check_hessian_full(H, H64, N)
        del H
        prep_o = O.prepare(H64, damp, desc_act, order_key=np.diag(H64))
        assert np.array_equal(perm_g, prep_o.perm)
        err = 0.0
        for r0 in range(0, n, 2048):
            Ug = prep.U[r0:r0 + 2048].cpu().numpy().astype(np.float64)
            err = max(err, float(np.abs(Ug - prep_o.U[r0:r0 + 2048]).max()))
        err /= np.abs(prep_o.U).max()
        print(f"  U (n = {n}): max relative difference {err:.3g} (bound {tol_u:.3g})")
        assert err <= tol_u
        _check_u_residual(prep.U, lambda V: prep_o.Hd @ V, seed)
        Hd64 = prep_o.Hd
        prep_o = dataclasses.replace(prep_o, Hd=None)
        del Hd64

        def err_of(Wr, What):
            return O.layer_error(Wr, What, H64)
    else:
        d = O.hessian_diag(x_bits)
        _check_hessian_samples(H, x_bits, d, seed=seed)
        del H
        Ut_o, perm_o = O.prepare_trailing_x(x_bits, damp, desc_act, m_tail, order_key=d)
        assert np.array_equal(perm_g, perm_o)
        Ut_g = prep.U[n - m_tail:, n - m_tail:].cpu().numpy().astype(np.float64)
        err = np.abs(Ut_g - Ut_o).max() / np.abs(Ut_o).max()
        print(f"  U (n = {n}): last {m_tail} rows and columns, max relative difference {err:.3g} (bound {tol_u:.3g})")
        assert err <= tol_u
        lam = damp * float(np.mean(d))
        _check_u_residual(prep.U, lambda V: O.damped_matvec(x_bits, perm_o, lam, V), seed)
        # rows are swept given the GPU's U, which the residual above checked whole
        prep_o = O.Prepared(U=prep.U.cpu().numpy(), perm=perm_g, dead=np.zeros(n, bool), lam=lam, Hd=None)

        def err_of(Wr, What):
            Wr = np.asarray(Wr, np.float64)
            D = Wr - np.asarray(What, np.float64)
            return float(np.sum(D.T * O.hessian_matvec(x_bits, D.T)) / np.sum(Wr.T * O.hessian_matvec(x_bits, Wr.T)))
    rng = np.random.default_rng(seed + 1)
    for job, q in zip(jobs, qs):
        rows = np.sort(rng.choice(job.W.shape[0], job.rows, replace=False))
        _compare_rows(job, q, perm_g, prep_o, rows, err_of)
    del prep, qs
    torch.cuda.empty_cache()


def _layers(wl_name, names):
    wl = S.workloads()[wl_name]
    by = {l.name: l for l in wl.layers}
    return [by[nm] for nm in names], wl.settings


def test_llama7b_attention_and_mlp_in_shapes_full_tokens():
    """q [4096 x 4096] and gate [11008 x 4096] share X (4096 features, 65,536 tokens)."""
    (q, gate), (st,) = _layers("llama2-7b-block", ["q", "gate"])
    x = S.make_x(q.x)
    _input_check(x, st.damp_percent, st.desc_act, [Job(S.make_w(q.w), st, 32), Job(S.make_w(gate.w), st, 32)],
                 seed=7)


def test_llama7b_down_full_tokens():
    """down [4096 x 11008], 4-bit symmetric g128, act-order, at its own 65,536 tokens."""
    (down,), (st,) = _layers("llama2-7b-block", ["down"])
    x = S.make_x(down.x)
    _input_check(x, st.damp_percent, st.desc_act, [Job(S.make_w(down.w), st, 32)], seed=11)


@pytest.mark.parametrize("layer", ["gate", "down"])
def test_llama7b_mlp_low_bit_all_settings(layer):
    """The low-bit sweep: gate [11008 x 4096] or down [4096 x 11008] at 32,768 tokens, one H
    and one U, quantized under all four settings (3 and 2 bits x g128 and g64, asymmetric,
    act-order)."""
    (lay,), settings = _layers("llama2-7b-mlp-lowbit", [layer])
    assert len(settings) == 4
    x = S.make_x(lay.x)
    W = S.make_w(lay.w)
    st0 = settings[0]
    _input_check(x, st0.damp_percent, st0.desc_act, [Job(W, st, 24) for st in settings], seed=31)


def test_llama70b_block_8192_input_layers():
    """q/o [8192 x 8192], k/v [1024 x 8192], gate/up [28672 x 8192]: one H, three shapes, 65,536 tokens."""
    (q, k, gate), (st,) = _layers("llama2-70b-block", ["q", "k", "gate"])
    x = S.make_x(q.x)
    _input_check(x, st.damp_percent, st.desc_act,
                 [Job(S.make_w(q.w), st, 16), Job(S.make_w(k.w), st, 16), Job(S.make_w(gate.w), st, 16)], seed=70)


def test_llama70b_down_28672_input():
    """down [8192 x 28672]: H and U are 28,672 x 28,672; 65,536 tokens."""
    (down,), (st,) = _layers("llama2-70b-block", ["down"])
    x = S.make_x(down.x)
    _input_check(x, st.damp_percent, st.desc_act, [Job(S.make_w(down.w), st, 16)], seed=71)
