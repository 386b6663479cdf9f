"""Pins of the fp64 oracle against what the GPTQ pages and the mathematics fix.

None of these re-types the oracle's formulas: each checks it against a value the
pages print, a hand computation, a closed form, an invariant, a special case that
reduces to round-to-nearest, or brute force on tiny inputs.
"""
import json
import os

import numpy as np
import pytest

import synthetic as S
from oracle import gptq_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _spd_from_x(n, tokens, seed, rank=3, frac=0.2, mult=10.0):
    x = S.make_x(S.XSpec(n, tokens, rank, frac, mult, seed, 7))
    return O.hessian(x), x


# --------------------------------------------------------------------------- #
# Hessian
# --------------------------------------------------------------------------- #
def test_hessian_brute_force_and_symmetry():
    x = S.make_x(S.XSpec(5, 7, 2, 0.2, 4.0, 3, 1))
    xf = S.bf16_bits_to_f32(x).astype(float).tolist()
    H = O.hessian(x)
    for i in range(5):
        for j in range(5):
            acc = 0.0
            for t in range(7):
                acc += xf[i][t] * xf[j][t]
            assert H[i, j] == pytest.approx(2.0 * acc, rel=1e-15, abs=0)
    assert np.array_equal(H, H.T)


def test_hessian_without_forming_it_brute_force():
    # The matrix-free forms the large-layer parity tests use: chunked H, exact diagonal,
    # H . V and H_d . V, each against pure-Python sums over tokens on a tiny X.
    n, N = 6, 11
    x = S.make_x(S.XSpec(n, N, 2, 0.2, 4.0, 5, 1))
    xf = S.bf16_bits_to_f32(x).astype(float).tolist()
    rng = np.random.default_rng(2)
    V = rng.standard_normal((n, 2))
    Hc = O.hessian_chunked(x, chunk=4)          # three chunks, the last ragged
    d = O.hessian_diag(x, chunk=4)
    HV = O.hessian_matvec(x, V, chunk=3)
    for i in range(n):
        assert d[i] == pytest.approx(2.0 * sum(v * v for v in xf[i]), rel=1e-15)
        for j in range(n):
            hij = 2.0 * sum(xf[i][t] * xf[j][t] for t in range(N))
            assert Hc[i, j] == pytest.approx(hij, rel=1e-14, abs=1e-14)
        for c in range(2):
            hv = 2.0 * sum(xf[i][t] * sum(xf[j][t] * V[j, c] for j in range(n)) for t in range(N))
            assert HV[i, c] == pytest.approx(hv, rel=1e-12, abs=1e-12)
    # H_d . V with an order and a damping: (H_d V)[k] = sum_l H[perm k, perm l] V[l] + lam V[k]
    perm = np.array([3, 0, 5, 1, 4, 2])
    lam = 0.37
    HdV = O.damped_matvec(x, perm, lam, V)
    for k in range(n):
        for c in range(2):
            ref = lam * V[k, c] + sum(2.0 * sum(xf[perm[k]][t] * xf[perm[l]][t] for t in range(N)) * V[l, c]
                                      for l in range(n))
            assert HdV[k, c] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    # a planted mistake: the order applied the wrong way round
    assert not np.allclose(O.damped_matvec(x, np.argsort(perm), lam, V), HdV)


@pytest.mark.parametrize("act", [False, True])
def test_trailing_factor_from_x_inverts_the_trailing_block(act):
    # U's trailing block formed from X alone (exact diagonal + the block of H) is the
    # upper factor of the inverse of H_d's trailing block: U_t^T U_t H_d[t, t] = I, with
    # H_d from the full preparation; and it equals the full factor's block.
    n, m = 48, 20
    x = S.make_x(S.XSpec(n, 400, 3, 0.2, 10.0, 9, 7))
    full = O.prepare(O.hessian(x), 0.02, act)
    Ut, perm = O.prepare_trailing_x(x, 0.02, act, m)
    assert np.array_equal(perm, full.perm)
    assert np.all(np.tril(Ut, -1) == 0) and np.all(np.diag(Ut) > 0)
    assert np.allclose(Ut.T @ Ut @ full.Hd[n - m:, n - m:], np.eye(m), atol=1e-9)
    assert np.allclose(Ut, full.U[n - m:, n - m:], rtol=1e-10, atol=1e-12 * np.abs(full.U).max())


def test_bf16_generator_matches_torch_rounding():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(10000) * np.exp(rng.standard_normal(10000) * 3)).astype(np.float32)
    mine = S.f32_to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_generator_token_ranges_regenerate():
    spec = S.XSpec(64, 3 * S.X_CHUNK + 100, 4, 0.05, 20.0, 11, 2)
    full = S.make_x(spec)
    part = S.make_x(spec, S.X_CHUNK - 7, 2 * S.X_CHUNK + 9)
    assert np.array_equal(part, full[:, S.X_CHUNK - 7:2 * S.X_CHUNK + 9])


# --------------------------------------------------------------------------- #
# Quantizer: hand-worked groups, the page's symmetric range
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("case", ["asym", "sym", "asym2"])
def test_quantizer_hand_examples(golden_dir, case):
    g = _load(golden_dir, "quantizer_hand.json")[case]
    w = np.array([g["w"]], dtype=np.float32)
    sym = case == "sym"
    s, z = O.group_params(w, g["bits"], sym)
    assert float(s[0]) == g["scale"]
    assert float(z[0]) == g["zero"]
    k = w.shape[1]
    c = O.quantize_codes(w[0], np.full(k, s[0], np.float32), np.full(k, z[0], np.float32), g["bits"], sym)
    assert c.tolist() == g["codes"]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_symmetric_range_matches_page(golden_dir, bits):
    lo, hi = _load(golden_dir, "sym_range.json")["ranges"][str(bits)]
    rng = np.random.default_rng(bits)
    w = rng.standard_normal((64, 128)).astype(np.float32)
    w[:, 5] = 0.0
    s, z = O.group_params(w, bits, True)
    codes = np.stack([O.quantize_codes(w[:, k], s, z, bits, True) for k in range(128)], 1)
    q = codes - z[:, None].astype(np.int64)
    assert q.min() == lo and q.max() == hi               # the extremes are reached (absmax column)
    assert codes.min() >= 1 and codes.max() <= 2 ** bits - 1
    assert np.all(q[:, 5] == 0)                          # zero is exactly representable
    assert np.all(O.dequant_value(codes[:, 5], s, z) == 0.0)


def test_asymmetric_zero_point_in_code_range():
    rng = np.random.default_rng(1)
    for bits in (2, 3, 4):
        w = (rng.standard_normal((200, 64)) + rng.uniform(-2, 2, (200, 1))).astype(np.float32)
        s, z = O.group_params(w, bits, False)
        assert np.all(z >= 0) and np.all(z <= 2 ** bits - 1) and np.all(z == np.round(z))
        assert np.all(s > 0) and np.all(s.astype(np.float16).astype(np.float32) == s)
        # the grid covers [lo, hi] to within half a step: max |w - what| <= s/2 (+ rounding of s)
        codes = np.stack([O.quantize_codes(w[:, k], s, z, bits, False) for k in range(64)], 1)
        what = O.dequant_value(codes, s[:, None], z[:, None])
        assert np.all(np.abs(w - what) <= 0.5 * s[:, None] * (1 + 2e-3) + 1e-7)


# --------------------------------------------------------------------------- #
# Pages' counts and sizes
# --------------------------------------------------------------------------- #
def test_worked_example_group_count_and_bytes(golden_dir):
    g = _load(golden_dir, "worked_example.json")
    out, n, gs = g["out"], g["in"], g["group_size"]
    assert out * n == g["elements"]
    # the oracle's storage for this shape (a cheap structural run on a zero H path)
    perm = np.arange(n)
    gi = O.g_idx(perm, gs)
    G = int(gi.max()) + 1
    assert G * out == g["groups"]
    codes = np.zeros((4, n), np.uint8)
    qw = O.pack(codes, g["bits"])
    assert qw.shape == (n * g["bits"] // 32, 4)
    packed_bytes = qw.nbytes // 4 * out
    assert packed_bytes == g["packed_bytes"]
    assert g["fp16_bytes"] / packed_bytes == g["reduction"]


def test_175b_memory_claim(golden_dir):
    g = _load(golden_dir, "memory_175b.json")
    assert g["params"] * g["bits"] // 8 == g["bytes"]


# --------------------------------------------------------------------------- #
# Packing and g_idx
# --------------------------------------------------------------------------- #
def test_pack_hand_examples(golden_dir):
    for case in _load(golden_dir, "pack_hand.json")["cases"]:
        codes = np.array([case["codes"]], dtype=np.uint8)
        qw = O.pack(codes, case["bits"]).view(np.uint32)[:, 0]
        assert [int(h, 16) for h in case["words_hex"]] == [int(v) for v in qw]
        assert np.array_equal(O.unpack(O.pack(codes, case["bits"]), case["bits"], codes.shape[1]), codes)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, (37, 96)).astype(np.uint8)
    assert np.array_equal(O.unpack(O.pack(codes, bits), bits, 96), codes)


def test_g_idx_hand_example():
    assert O.g_idx(np.array([2, 0, 3, 1]), 2).tolist() == [0, 1, 0, 1]
    assert O.g_idx(np.array([2, 0, 3, 1]), -1).tolist() == [0, 0, 0, 0]


# --------------------------------------------------------------------------- #
# Preparation: U, damping, act-order, dead inputs
# --------------------------------------------------------------------------- #
def test_u_is_upper_cholesky_of_damped_inverse():
    H, _ = _spd_from_x(48, 300, 2)
    p = O.prepare(H, 0.01, True)
    U = p.U
    assert np.all(np.tril(U, -1) == 0) and np.all(np.diag(U) > 0)
    assert np.allclose(U.T @ U @ p.Hd, np.eye(48), atol=1e-9)
    Hp = H[np.ix_(p.perm, p.perm)]
    assert p.lam == pytest.approx(0.01 * np.mean(np.diag(H)), rel=1e-14)
    assert np.allclose(p.Hd - Hp, p.lam * np.eye(48), atol=1e-12 * np.abs(H).max())


@pytest.mark.parametrize("act,with_dead", [(False, False), (True, False), (True, True)])
def test_trailing_block_of_u_comes_from_the_trailing_block_of_h(act, with_dead):
    # U's last m rows and columns depend only on the trailing principal block of H_d
    # (H_d = V V^T with V = U^-1 upper triangular): the block computed from it alone
    # must equal the full factor's block.
    H, _ = _spd_from_x(40, 300, 6)
    if with_dead:
        H[5, :] = 0.0
        H[:, 5] = 0.0
        H[22, :] = 0.0
        H[:, 22] = 0.0
    key = np.diag(H) * (1.0 + 1e-9 * np.arange(40))
    full = O.prepare(H, 0.01, act, order_key=key)
    for m in (1, 7, 16, 40):
        Ut, perm = O.prepare_trailing(H, 0.01, act, m, order_key=key)
        assert np.array_equal(perm, full.perm)
        assert np.allclose(Ut, full.U[40 - m:, 40 - m:], rtol=1e-10, atol=1e-12 * np.abs(full.U).max())
    # a planted mistake (the leading block instead of the trailing one) fails
    Ul, _ = O.prepare_trailing(H[::-1, ::-1].copy(), 0.01, False, 16)
    assert not np.allclose(Ul, O.prepare(H, 0.01, False).U[24:, 24:], rtol=1e-6)


def test_act_order_descending_and_stable():
    d = np.array([3.0, 5.0, 3.0, 1.0, 5.0, 0.5])
    assert O.act_order(d).tolist() == [1, 4, 0, 2, 3, 5]
    H, _ = _spd_from_x(40, 200, 4)
    p = O.prepare(H, 0.01, True)
    dd = np.diag(H)[p.perm]
    assert np.all(np.diff(dd) <= 0)


def test_desc_act_is_identity_on_descending_diagonal():
    H, x = _spd_from_x(32, 400, 5)
    order = np.argsort(-np.diag(H), kind="stable")
    Hs = H[np.ix_(order, order)]
    W = S.make_w(S.WSpec(16, 32, 0.02, "f32", 5, 100))
    a = O.gptq_layer(W, None, 4, 8, False, True, H=Hs)
    b = O.gptq_layer(W, None, 4, 8, False, False, H=Hs)
    assert a.perm.tolist() == list(range(32))
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.qweight, b.qweight)


def test_dead_inputs_are_zeroed_and_unit_diagonal():
    H, _ = _spd_from_x(16, 100, 6)
    H[3, :] = 0
    H[:, 3] = 0
    p = O.prepare(H, 0.01, False)
    assert p.dead.tolist() == [i == 3 for i in range(16)]
    W = S.make_w(S.WSpec(8, 16, 0.02, "f32", 6, 100))
    sw, codes = O.quantize_layer(W, p, 4, 16, True, 16)
    assert np.all(O.dequant_value(sw.codes[:, 3], sw.scales[0], sw.zeros[0]) == 0.0)


# --------------------------------------------------------------------------- #
# The sweep: RTN special case, lazy == unblocked, least squares, loss identity
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("bits,gs,sym", [(4, 128, False), (4, 128, True), (3, 64, False), (2, 32, True),
                                         (3, -1, False), (2, 64, False)])
def test_identity_hessian_gives_round_to_nearest(bits, gs, sym):
    n, out = 256, 64
    W = S.make_w(S.WSpec(out, n, 0.02, "f16", 9, 100))
    for H in (np.eye(n), np.diag(np.exp(np.random.default_rng(1).standard_normal(n)))):
        r = O.gptq_layer(W, None, bits, gs, sym, False, H=H, with_rtn=False)
        rc, rs, rz = O.rtn(W, bits, gs, sym)
        assert np.array_equal(r.sw.codes, rc)
        assert np.array_equal(r.sw.scales, rs) and np.array_equal(r.sw.zeros, rz)


@pytest.mark.parametrize("bits,gs,sym,act", [(4, 128, False, False), (4, 64, True, True), (3, 32, False, True),
                                             (2, 128, True, False)])
def test_lazy_batches_equal_unblocked(bits, gs, sym, act):
    H, _ = _spd_from_x(384, 1500, 8, rank=6)
    W = S.make_w(S.WSpec(48, 384, 0.02, "f32", 8, 100))
    p = O.prepare(H, 0.01, act)
    a, ca = O.quantize_layer(W, p, bits, gs, sym, 128)
    b, cb = O.quantize_layer(W, p, bits, gs, sym, None)
    assert np.array_equal(ca, cb)
    assert np.allclose(a.W_final, b.W_final, rtol=0, atol=1e-13)


@pytest.mark.parametrize("n,bits,sym,act", [(4, 2, False, False), (5, 3, True, True), (6, 4, False, True),
                                            (6, 2, True, False)])
def test_compensation_is_brute_force_least_squares(n, bits, sym, act):
    """After columns 0..j are fixed, the remaining weights are the minimiser of
    (w - what)^T H_d (w - what) over the free columns: d_F = -H_FF^-1 H_FQ d_Q."""
    H, _ = _spd_from_x(n, 50, 10 + n, rank=2, frac=0.3)
    rng = np.random.default_rng(n)
    W = (rng.standard_normal((7, n)) * 0.3).astype(np.float32)
    p = O.prepare(H, 0.01, act)
    sw, _ = O.quantize_layer(W, p, bits, -1, sym, None)
    Wp = W.astype(np.float64)[:, p.perm]
    Hd = p.Hd
    for r in range(W.shape[0]):
        what = O.dequant_value(sw.codes[r], sw.scales[0, r], sw.zeros[0, r])
        for j in range(1, n):
            Q, F = list(range(j)), list(range(j, n))
            dQ = what[Q] - Wp[r, Q]
            dF = -np.linalg.solve(Hd[np.ix_(F, F)], Hd[np.ix_(F, Q)] @ dQ)
            assert sw.W_final[r, j] == pytest.approx(Wp[r, j] + dF[0], rel=1e-9, abs=1e-12)


def test_codes_are_nearest_grid_points_of_compensated_weights():
    H, _ = _spd_from_x(128, 600, 12)
    W = S.make_w(S.WSpec(32, 128, 0.02, "f32", 12, 100))
    p = O.prepare(H, 0.01, True)
    sw, _ = O.quantize_layer(W, p, 3, 32, False, 128)
    for g in range(4):
        cols = slice(32 * g, 32 * g + 32)
        grid = sw.scales[g][:, None] * (np.arange(8)[None, :] - sw.zeros[g][:, None])     # [out, 8]
        w = sw.W_final[:, cols].astype(np.float32).astype(np.float64)
        dist = np.abs(w[:, :, None] - grid[:, None, :])
        best = dist.min(axis=2)
        chosen = np.take_along_axis(dist, sw.codes[:, cols][:, :, None].astype(np.int64), 2)[:, :, 0]
        assert np.all(chosen <= best * (1 + 1e-6) + 1e-9)


def test_loss_identity_sum_of_squared_errors():
    """Per row, sum_j e_j^2 = (w - what)^T H_d (w - what) with e_j = (w_j - what_j)/U_jj."""
    H, _ = _spd_from_x(256, 1200, 13)
    W = S.make_w(S.WSpec(24, 256, 0.02, "f32", 13, 100))
    p = O.prepare(H, 0.01, True)
    sw, _ = O.quantize_layer(W, p, 4, 64, True, 128)
    Wp = W.astype(np.float64)[:, p.perm]
    G = 256 // 64
    what = np.concatenate([O.dequant_value(sw.codes[:, 64 * g:64 * g + 64], sw.scales[g][:, None], sw.zeros[g][:, None])
                           for g in range(G)], 1)
    d = Wp - what
    lhs = (sw.err ** 2).sum(1)
    rhs = np.einsum("ij,jk,ik->i", d, p.Hd, d)
    assert np.allclose(lhs, rhs, rtol=1e-10)


def test_power_of_two_hessian_scaling_is_exact():
    H, _ = _spd_from_x(128, 500, 14)
    W = S.make_w(S.WSpec(16, 128, 0.02, "f32", 14, 100))
    a = O.gptq_layer(W, None, 4, 32, False, True, H=H, with_rtn=False)
    b = O.gptq_layer(W, None, 4, 32, False, True, H=4.0 * H, with_rtn=False)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)


def test_layer_error_matches_direct_output_error():
    W, x = S.small_case(12, 64, 300, 15)
    H = O.hessian(x)
    r = O.gptq_layer(W, x, 4, 32, False, False, H=H)
    X = O.bf16_bits_to_f64(x)
    What = O.dequantize(r.qweight, r.scales, r.zeros, r.g_idx, 4, 64)
    direct = np.sum((W.astype(float) @ X - What @ X) ** 2) / np.sum((W.astype(float) @ X) ** 2)
    assert r.rel_err == pytest.approx(direct, rel=1e-9)


def test_stored_format_reconstructs_sweep_values():
    W, x = S.small_case(20, 128, 400, 16)
    r = O.gptq_layer(W, x, 3, 32, True, True)
    What = O.dequantize(r.qweight, r.scales, r.zeros, r.g_idx, 3, 128)[:, r.perm]
    for g in range(4):
        c = slice(32 * g, 32 * g + 32)
        assert np.array_equal(What[:, c], O.dequant_value(r.sw.codes[:, c], r.sw.scales[g][:, None], r.sw.zeros[g][:, None]))


# --------------------------------------------------------------------------- #
# GPTQ beats RTN on outlier-heavy correlated activations
# --------------------------------------------------------------------------- #
def test_gptq_beats_rtn_on_small_workload():
    wl = S.workloads()["layer-256x512"]
    L, st = wl.layers[0], wl.settings[0]
    r = O.gptq_layer(S.make_w(L.w), S.make_x(L.x), st.bits, st.group_size, st.sym, st.desc_act)
    assert r.rel_err < 0.75 * r.rel_err_rtn


@pytest.mark.parametrize("bits,gs,sym,act", [(4, 128, True, True), (3, 64, False, True), (2, 64, False, True)])
def test_gptq_beats_rtn_low_bits(bits, gs, sym, act):
    W, x = S.small_case(64, 512, 2048, 17, rank=16, frac=0.02, mult=30.0)
    r = O.gptq_layer(W, x, bits, gs, sym, act)
    assert r.rel_err < r.rel_err_rtn


# --------------------------------------------------------------------------- #
# Planted mistakes: each must trip one of the pins above
# --------------------------------------------------------------------------- #
def _least_squares_ok(sw, Wp, Hd, n):
    for r in range(Wp.shape[0]):
        what = O.dequant_value(sw.codes[r], sw.scales[0, r], sw.zeros[0, r])
        for j in range(1, n):
            Q, F = list(range(j)), list(range(j, n))
            dF = -np.linalg.solve(Hd[np.ix_(F, F)], Hd[np.ix_(F, Q)] @ (what[Q] - Wp[r, Q]))
            if abs(sw.W_final[r, j] - (Wp[r, j] + dF[0])) > 1e-9 * max(1.0, abs(Wp[r, j])):
                return False
    return True


@pytest.mark.parametrize("mistake", ["transposed_U", "negated_update", "no_damping", "lower_factor"])
def test_planted_mistakes_fail_least_squares_pin(mistake):
    n = 6
    H, _ = _spd_from_x(n, 50, 21, rank=2, frac=0.3)
    W = (np.random.default_rng(3).standard_normal((5, n)) * 0.3).astype(np.float32)
    p = O.prepare(H, 0.01, False)
    Wp = W.astype(np.float64)[:, p.perm]
    U = p.U.copy()
    Hd = p.Hd
    if mistake == "transposed_U":
        U = U.T.copy()
    elif mistake == "negated_update":
        U = -U + 2 * np.diag(np.diag(U))
    elif mistake == "no_damping":
        U = O.prepare(H, 0.0, False).U
    elif mistake == "lower_factor":
        U = np.linalg.cholesky(np.linalg.inv(Hd))
    good = O.sweep(Wp, p.U, 4, -1, False, None)
    bad = O.sweep(Wp, U, 4, -1, False, None)
    assert _least_squares_ok(good, Wp, Hd, n)
    assert not _least_squares_ok(bad, Wp, Hd, n)


def test_planted_zero_offset_mistake_fails_range_pin(golden_dir, monkeypatch):
    real = O.group_params

    def off_by_one(wg, bits, sym):
        s, z = real(wg, bits, sym)
        return s, (z - 1 if sym else z)

    monkeypatch.setattr(O, "group_params", off_by_one)
    g = _load(golden_dir, "quantizer_hand.json")["sym"]
    s, z = O.group_params(np.array([g["w"]], np.float32), 4, True)
    assert float(z[0]) != g["zero"]


# --------------------------------------------------------------------------- #
# Checkpoint variants: packed zero points, zero padding
# --------------------------------------------------------------------------- #
def test_pack_zeros_hand_examples(golden_dir):
    for case in _load(golden_dir, "pack_zeros_hand.json")["cases"]:
        z = np.array(case["zeros"], dtype=np.float64)
        bits, off = case["bits"], case["zero_offset"]
        qz = O.pack_zeros(z, bits, off).view(np.uint32).astype(np.int64)
        assert [[int(h, 16) for h in row] for row in case["words_hex"]] == qz.tolist()
        assert np.array_equal(O.unpack_zeros(O.pack_zeros(z, bits, off), bits, z.shape[1], off), z)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_zeros_is_the_code_stream_along_the_outputs(bits):
    # without the offset, group g's words are the stream the code packing forms for a
    # row of codes, here taken along the outputs: pack of the [G, out] matrix, transposed
    rng = np.random.default_rng(40 + bits)
    z = rng.integers(0, 2 ** bits, (5, 96))
    assert np.array_equal(O.pack_zeros(z, bits).view(np.uint32), O.pack(z.astype(np.uint8), bits).view(np.uint32).T)
    # with it, every value moves down by one modulo 2^bits
    assert np.array_equal(O.pack_zeros(z, bits, 1).view(np.uint32),
                          O.pack(((z - 1) % 2 ** bits).astype(np.uint8), bits).view(np.uint32).T)
    with pytest.raises(ValueError):
        O.pack_zeros(z + 0.5, bits)
    with pytest.raises(ValueError):
        O.pack_zeros(z + 2 ** bits, bits)


def _padded_case(n, n_pad, out=24, tokens=600, seed=31):
    W, x = S.small_case(out, n, tokens, seed=seed, rank=6, frac=0.03, mult=15.0)
    Wp, xp = O.pad_layer(W, x, n_pad)
    return W, x, Wp, xp


def test_padding_makes_dead_inputs_damped_by_the_padded_mean():
    n, n_pad, damp = 300, 384, 0.01
    W, x, Wp, xp = _padded_case(n, n_pad)
    assert np.array_equal(Wp[:, :n], W) and not Wp[:, n:].any()
    H, Hp = O.hessian(x), O.hessian(xp)
    assert np.array_equal(Hp[:n, :n], H) and not Hp[n:].any() and not Hp[:, n:].any()
    prep = O.prepare(Hp, damp, False)
    assert np.array_equal(np.flatnonzero(prep.dead), np.arange(n, n_pad))
    # the padded inputs' unit diagonal counts in the mean like any other input's
    lam = damp * (np.trace(H) + (n_pad - n)) / n_pad
    assert prep.lam == pytest.approx(lam, rel=1e-13)
    # U is block diagonal: the real block is the upper factor of (H + lam I)^-1
    # (numpy's inverse and Cholesky: the definition), the padded block (1 + lam)^-1/2 I
    U_ref = np.linalg.cholesky(np.linalg.inv(H + lam * np.eye(n))).T
    scale = np.abs(U_ref).max()
    assert np.abs(prep.U[:n, :n] - U_ref).max() <= 1e-10 * scale
    assert not prep.U[:n, n:].any() and not prep.U[n:, :n].any()
    assert np.allclose(prep.U[n:, n:], np.eye(n_pad - n) / np.sqrt(1.0 + lam), rtol=1e-14, atol=0)
    # planted mistake: damping by the mean over the real inputs alone misses the pin
    lam_bad = damp * np.trace(H) / n
    U_bad = np.linalg.cholesky(np.linalg.inv(H + lam_bad * np.eye(n))).T
    assert np.abs(prep.U[:n, :n] - U_bad).max() > 1e-6 * scale


@pytest.mark.parametrize("sym", [False, True])
def test_padded_layer_with_one_group_per_row_is_the_unpadded_layer(sym):
    # one group per row: its parameters come from the whole initial row, and zero
    # columns change neither its extremes (the range always holds 0) nor its largest
    # magnitude, so the padded layer's real columns are the unpadded layer quantized
    # with the padded damping
    n, n_pad, damp = 300, 320, 0.01
    W, x, Wp, xp = _padded_case(n, n_pad, seed=33)
    res = O.gptq_layer(Wp, xp, 4, -1, sym, False, damp, with_rtn=False)
    H = O.hessian(x)
    lam = damp * (np.trace(H) + (n_pad - n)) / n_pad
    prep_u = O.prepare(H, lam / np.mean(np.diag(H)), False)
    sw = O.sweep(np.asarray(W, np.float64), prep_u.U, 4, -1, sym, 128)
    assert np.array_equal(res.sw.scales, sw.scales) and np.array_equal(res.sw.zeros, sw.zeros)
    assert np.mean(res.codes[:, :n] != sw.codes) <= 1e-3
    # the padded columns take the zero point's code, which dequantizes to 0
    assert np.array_equal(res.codes[:, n:], np.repeat(res.sw.zeros[0].astype(np.uint8)[:, None], n_pad - n, 1))
    What = O.dequantize(res.qweight, res.scales, res.zeros, res.g_idx, 4, n_pad)
    assert not What[:, n:].any()


@pytest.mark.parametrize("bits,gs,sym,act", [(4, 128, False, False), (3, 64, True, True), (2, 32, False, True)])
def test_padded_columns_quantize_to_zero_and_carry_no_error(bits, gs, sym, act):
    n = 300
    n_pad = -(-n // max(32, gs)) * max(32, gs)
    W, x, Wp, xp = _padded_case(n, n_pad, seed=35 + bits)
    res = O.gptq_layer(Wp, xp, bits, gs, sym, act, with_rtn=False)
    pad = np.arange(n, n_pad)
    What = O.dequantize(res.qweight, res.scales, res.zeros, res.g_idx, bits, n_pad)
    assert not What[:, pad].any()
    # processing positions of the padded columns: no error leaves them
    pos = np.argsort(res.perm)[pad]
    assert not res.sw.err[:, pos].any()
    # their groups continue the processing order's numbering
    assert np.array_equal(res.g_idx[pad], (pos // gs).astype(np.int32))


def test_rows_are_independent_given_u(monkeypatch):
    # polydesk, "Etape 1": the inverse-Hessian work is shared by all rows, and each row is
    # quantized on its own; the full-size parity tests compare sampled rows on this basis.
    W, x = S.small_case(64, 384, 1024, seed=5)
    prep = O.prepare(O.hessian(x), 0.01, True)
    rows = np.array([3, 17, 18, 40, 63])
    sw, codes = O.quantize_layer(W, prep, 4, 128, False, 128)
    sw_r, codes_r = O.quantize_layer(W[rows], prep, 4, 128, False, 128)
    assert np.array_equal(codes[rows], codes_r)
    assert np.array_equal(sw.scales[:, rows], sw_r.scales) and np.array_equal(sw.zeros[:, rows], sw_r.zeros)
    assert np.allclose(sw.err[rows], sw_r.err, rtol=0, atol=1e-12)
    # planted mistake: parameters shared by all rows of a group (a per-tensor range) couple
    # the rows, and the subset no longer reproduces them
    real = O.group_params

    def shared(wg, bits, sym):
        s, z = real(np.broadcast_to(np.asarray(wg, np.float32).reshape(1, -1), (wg.shape[0], wg.size)), bits, sym)
        return s, z

    monkeypatch.setattr(O, "group_params", shared)
    _, codes_all = O.quantize_layer(W, prep, 4, 128, False, 128)
    _, codes_sub = O.quantize_layer(W[rows], prep, 4, 128, False, 128)
    assert not np.array_equal(codes_all[rows], codes_sub)


def test_mlp_forward_closed_forms_and_brute_force():
    # silu: 0 at 0, g . sigmoid(g), odd part g/2, tends to g and to 0
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert O.silu(np.array([1.0]))[0] == pytest.approx(1.0 / (1.0 + np.exp(-1.0)), rel=1e-15)
    g = np.array([-3.0, -0.5, 0.25, 2.0])
    assert np.allclose(O.silu(g) - O.silu(-g), g, rtol=1e-14)
    assert O.silu(np.array([40.0]))[0] == pytest.approx(40.0, rel=1e-15) and abs(O.silu(np.array([-40.0]))[0]) < 1e-15
    # the hidden activations and the residual output, against loops over a tiny block
    rng = np.random.default_rng(4)
    x = S.f32_to_bf16_bits(rng.standard_normal((3, 5)).astype(np.float32))
    xf = S.bf16_bits_to_f32(x).astype(float)
    Wg, Wu, Wd = rng.standard_normal((4, 3)), rng.standard_normal((4, 3)), rng.standard_normal((3, 4))
    h = O.mlp_hidden(x, Wg, Wu)
    out = O.mlp_residual(x, Wd, h)
    for i in range(4):
        for t in range(5):
            gv = sum(Wg[i, k] * xf[k, t] for k in range(3))
            uv = sum(Wu[i, k] * xf[k, t] for k in range(3))
            assert h[i, t] == pytest.approx(gv / (1 + np.exp(-gv)) * uv, rel=1e-12, abs=1e-14)
    for r in range(3):
        for t in range(5):
            assert out[r, t] == pytest.approx(xf[r, t] + sum(Wd[r, i] * h[i, t] for i in range(4)), rel=1e-12,
                                              abs=1e-14)
    # a planted mistake (the gate and up roles swapped) changes the result
    assert not np.allclose(O.mlp_hidden(x, Wu, Wg), h)
