"""CUDA path against the fp64 oracle, element by element, through the C ABI.

Every input comes from the seeded generator; every expected value from the oracle.
"""
import numpy as np
import pytest

import synthetic as S
from oracle import gptq_oracle as O
from tests.parity import CODE_MISMATCH_MAX, REL_ERR_TOL, compare_layer, hessian_bound

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_15_b200 as G


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _to_dev_x(x_bits, dev):
    """X on the device as a [n, tokens] view of a buffer whose row stride is a multiple of 8."""
    n, t = x_bits.shape
    ld = (t + 7) // 8 * 8
    buf = torch.zeros((n, ld), dtype=torch.int16, device=dev)
    buf[:, :t] = torch.from_numpy(x_bits.view(np.int16)).to(dev)
    return buf.view(torch.bfloat16)[:, :t]


def _w_tensor(W, dev):
    return torch.from_numpy(np.ascontiguousarray(W)).to(dev)


def _run_gpu(W, x_bits, bits, gs, sym, act, damp=0.01):
    dev = _dev()
    q, prep, H = G.gptq_quantize(_w_tensor(W, dev), _to_dev_x(x_bits, dev), bits, gs, sym, act, damp,
                                 want_codes=True, want_err=True)
    torch.cuda.synchronize()
    return q, prep, H


def _compare(W, x_bits, bits, gs, sym, act, H64=None):
    q, prep, Hg = _run_gpu(W, x_bits, bits, gs, sym, act)
    if H64 is None:
        H64 = O.hessian(x_bits)
    ora = O.gptq_layer(W, None, bits, gs, sym, act, H=H64)
    c = compare_layer(W, H64, ora, q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                      q.g_idx.cpu().numpy(), q.codes.cpu().numpy(), prep.perm.cpu().numpy(), bits, gs)
    return c, q, prep, Hg, H64, ora


# --------------------------------------------------------------------------- #
# Whole path
# --------------------------------------------------------------------------- #
def test_small_workload_full_path():
    wl = S.workloads()["layer-256x512"]
    L, st = wl.layers[0], wl.settings[0]
    W, x = S.make_w(L.w), S.make_x(L.x)
    c, *_ = _compare(W, x, st.bits, st.group_size, st.sym, st.desc_act)
    print(c)
    assert c.ok(), c


@pytest.mark.parametrize("out,n,tokens,bits,gs,sym,act", [
    (200, 384, 1000, 4, 128, False, True),      # ragged rows, 3 blocks, ragged tokens, act-order
    (77, 256, 700, 3, 64, True, False),
    (130, 320, 900, 2, 32, False, True),        # n = 2.5 blocks (ragged last block)
    (64, 512, 1500, 8, 128, True, True),
    (96, 256, 1024, 4, -1, False, False),       # one group per row
    (5000, 128, 600, 4, 128, True, True),       # many rows: 4 lanes per row
])
def test_ragged_shapes_and_settings(out, n, tokens, bits, gs, sym, act):
    W, x = S.small_case(out, n, tokens, seed=out + n, rank=8, frac=0.02, mult=20.0)
    c, q, prep, Hg, H64, ora = _compare(W, x, bits, gs, sym, act)
    print(c)
    assert c.ok(), c


def test_hessian_and_diag_against_oracle():
    dev = _dev()
    W, x = S.small_case(8, 300, 2504, seed=3)          # n not a multiple of any tile, ragged tokens
    X = _to_dev_x(x, dev)
    H = torch.zeros((300, 300), dtype=torch.float32, device=dev)
    hd = torch.zeros(300, dtype=torch.float64, device=dev)
    G.hessian_accumulate(H, X[:, :1200], hd)              # two chunks
    G.hessian_accumulate(H, X[:, 1200:].contiguous(), hd)
    torch.cuda.synchronize()
    H64 = O.hessian(x)
    Hg = H.cpu().numpy().astype(np.float64)
    iu = np.triu_indices(300)
    # the bound derived from the kernel's chunked summation (tests/parity.py), two calls
    rel = np.abs(Hg[iu] - H64[iu]) / np.sqrt(np.outer(np.diag(H64), np.diag(H64)))[iu]
    assert rel.max() <= hessian_bound([1200, 1304]), rel.max()
    print("hessian max normalised error", rel.max())
    assert np.allclose(hd.cpu().numpy(), np.diag(H64), rtol=1e-13, atol=0)


def test_hessian_from_host_memory_in_chunks():
    # X stays in pinned host memory; a small staging area forces five chunks, the last ragged
    dev = _dev()
    W, x = S.small_case(8, 300, 2504, seed=3)
    X_host = torch.from_numpy(x.view(np.int16)).pin_memory()
    H = torch.zeros((300, 300), dtype=torch.float32, device=dev)
    hd = torch.zeros(300, dtype=torch.float64, device=dev)
    staging = G.workspace(2 * 300 * 512 * 2, dev)
    st = G.new_status(dev)
    G.hessian_accumulate_host(H, X_host, hd, st, staging=staging)
    G.raise_on_status(st, "host Hessian")
    H64 = O.hessian(x)
    Hg = H.cpu().numpy().astype(np.float64)
    iu = np.triu_indices(300)
    rel = np.abs(Hg[iu] - H64[iu]) / np.sqrt(np.outer(np.diag(H64), np.diag(H64)))[iu]
    # one launch per staged chunk of 512 tokens (the staging area's halves)
    assert rel.max() <= hessian_bound([512] * 4 + [2504 - 4 * 512]), rel.max()
    assert np.allclose(hd.cpu().numpy(), np.diag(H64), rtol=1e-13, atol=0)
    # the whole path from host tensors gives the device path's result
    W, x = S.small_case(48, 320, 2504, seed=4)
    Wt = torch.from_numpy(np.ascontiguousarray(W))
    X_host = torch.from_numpy(x.view(np.int16)).pin_memory()
    q_h, p_h, _ = G.gptq_quantize(Wt.pin_memory(), X_host, 4, 32, False, True, want_codes=True)
    q_d, p_d, _ = G.gptq_quantize(Wt.to(dev), _to_dev_x(x, dev), 4, 32, False, True, want_codes=True)
    assert np.array_equal(p_h.perm.cpu().numpy(), p_d.perm.cpu().numpy())
    assert float(np.mean(q_h.codes.cpu().numpy() != q_d.codes.cpu().numpy())) <= CODE_MISMATCH_MAX


def test_prepare_u_and_perm():
    dev = _dev()
    _, x = S.small_case(8, 384, 3000, seed=4)
    H64 = O.hessian(x)
    Ht = torch.from_numpy(H64.astype(np.float32)).to(dev)
    hd = torch.from_numpy(np.diag(H64).copy()).to(dev)
    p = G.prepare(Ht, 0.01, True, hd)
    G.raise_on_status(p.status, "prepare")
    ora = O.prepare(H64, 0.01, True)
    assert np.array_equal(p.perm.cpu().numpy(), ora.perm)
    U = p.U.cpu().numpy().astype(np.float64)
    assert np.all(np.tril(U, -1) == 0) and np.all(np.diag(U) > 0)
    R = U.T @ U @ ora.Hd
    assert np.abs(R - np.eye(384)).max() < 1e-3
    assert np.abs(U - ora.U).max() / np.abs(ora.U).max() < 1e-4


@pytest.mark.parametrize("act", [False, True])
def test_prepare_replayed_as_a_graph(act):
    """gptq_prepare captures the stage as a CUDA graph the second time it sees the same
    arguments and replays it afterwards: every replay equals a direct call bit for bit,
    and a replay reads the buffers' current contents (new H values in the same buffer)."""
    dev = _dev()
    n = 1024
    Hs = []
    for seed in (11, 12):
        _, x = S.small_case(8, n, 2 * n, seed=seed)
        Hs.append(torch.from_numpy(O.hessian(x).astype(np.float32)).to(dev))
    hd = [torch.diagonal(h).double().contiguous() for h in Hs]
    def direct(i):        # graph replay off: enqueued launch by launch
        old = G.set_graph_replay(0)
        try:
            p = G.prepare(Hs[i].clone(), 0.01, act, hd[i].clone(), status=G.new_status(dev))
            torch.cuda.synchronize()
        finally:
            G.set_graph_replay(old)
        return p.U.clone(), p.perm.clone()
    ref = [direct(0), direct(1)]
    H = Hs[0].clone()
    h = hd[0].clone()
    st = G.new_status(dev)
    ws = G.workspace(G.lib().gptq_prepare_workspace_size(n), dev)
    out = None
    launches = []
    for call in range(5):
        src = 0 if call < 3 else 1
        H.copy_(Hs[src])
        h.copy_(hd[src])
        l0 = G.kernel_launches()
        out = G.prepare(H, 0.01, act, h, status=st, ws=ws, out=out)
        torch.cuda.synchronize()
        launches.append(G.kernel_launches() - l0)
        G.raise_on_status(st, "prepare")
        assert torch.equal(out.U, ref[src][0]) and torch.equal(out.perm, ref[src][1]), call
    assert len(set(launches)) == 1   # a replay counts the kernels it runs


@pytest.mark.parametrize("bits,gs,out", [(4, 128, 300), (3, 64, 257), (2, 32, 64), (8, 128, 33), (3, -1, 130),
                                         (4, 32, 1000)])
def test_packing_fused_into_the_sweep_matches_the_pack_kernel(bits, gs, out):
    """Without act-order the sweep can write qweight itself (fused_pack: the perm argument
    is NULL, the identity); by default the separate pack kernel does.  Same bits."""
    dev = _dev()
    n = 1536
    W, x = S.small_case(out, n, 3000, seed=bits * 100 + out)
    H = torch.from_numpy(O.hessian(x).astype(np.float32)).to(dev)
    p = G.prepare(H, 0.01, False)
    assert torch.equal(p.perm.cpu(), torch.arange(n, dtype=torch.int32))
    Wt = _w_tensor(W, dev)
    fused = G.quantize_layer(Wt, p, bits, gs, False, want_codes=True, fused_pack=True)
    packed = G.quantize_layer(Wt, p, bits, gs, False, want_codes=True)
    torch.cuda.synchronize()
    G.raise_on_status(p.status, "fused packing")
    for name in ("qweight", "scales", "zeros", "g_idx", "codes"):
        assert torch.equal(getattr(fused, name), getattr(packed, name)), name
    assert np.array_equal(O.pack(fused.codes.cpu().numpy(), bits).view(np.int32), fused.qweight.cpu().numpy())
    # the stacked and zero-padded entry points take the same path
    W2 = _w_tensor(S.make_w(S.WSpec(out, n, 0.02, "f32", 3, 77)), dev)
    _, (a, b) = G.quantize_layers([Wt, W2], p, bits, gs, False, fused_pack=True)
    _, (c, d) = G.quantize_layers([Wt, W2], p, bits, gs, False)
    assert torch.equal(a.qweight, c.qweight) and torch.equal(b.qweight, d.qweight)
    Wn = Wt[:, : n - 32].contiguous()
    e = G.quantize_layer(Wn, p, bits, gs, False, fused_pack=True)
    f = G.quantize_layer(Wn, p, bits, gs, False)
    assert torch.equal(e.qweight, f.qweight)


def test_quantize_replayed_as_a_graph():
    """The quantize stage is captured as a CUDA graph at the second call with the same
    arguments: replays equal direct calls bit for bit, with new weights in the same buffer."""
    dev = _dev()
    n, out = 1536, 700
    _, x = S.small_case(8, n, 3000, seed=31)
    H = torch.from_numpy(O.hessian(x).astype(np.float32)).to(dev)
    hd = torch.diagonal(H).double().contiguous()
    p = G.prepare(H, 0.01, True, hd)
    Ws = [_w_tensor(S.make_w(S.WSpec(out, n, 0.02, "f16", 3, 40 + i)), dev) for i in range(2)]
    def direct(i):        # graph replay off: enqueued launch by launch
        old = G.set_graph_replay(0)
        try:
            q = G.quantize_layer(Ws[i].clone(), p, 4, 128, True, want_codes=True, want_err=True)
            torch.cuda.synchronize()
        finally:
            G.set_graph_replay(old)
        return q
    ref = [direct(0), direct(1)]
    W = Ws[0].clone()
    st = G.new_status(dev)
    ws = G.workspace(G.quantize_workspace_size(out, n, 128), dev)
    qo = G.alloc_quantized(out, n, 4, 128, True, dev, want_codes=True, want_err=True)
    for call in range(5):
        src = 0 if call < 3 else 1
        W.copy_(Ws[src])
        p.status = st
        q = G.quantize_layer(W, p, 4, 128, True, ws=ws, out=qo, want_codes=True, want_err=True)
        torch.cuda.synchronize()
        G.raise_on_status(st, "quantize")
        for name in ("qweight", "scales", "zeros", "g_idx", "codes", "err_sq"):
            assert torch.equal(getattr(q, name), getattr(ref[src], name)), (call, name)


@pytest.mark.parametrize("n,act", [(1600, True), (2048, False), (2600, True)])
def test_prepare_outer_panels_against_the_oracle(n, act):
    """The deferred form of the preparation (bulk updates grouped by 512-wide outer panels,
    the form large layers take) forced at sizes the oracle factors in seconds: several outer
    panels, a partial last one (1600 = 3 x 512 + 64; 2600 = 5 x 512 + 40), the rings of
    buffers reused.  U element by element against the oracle's own U (fp32 chains of length
    n: n 2^-23 relative), and against the per-panel form."""
    dev = _dev()
    _, x = S.small_case(8, n, 2 * n, seed=n)
    H64 = O.hessian(x)
    Ht = torch.from_numpy(H64.astype(np.float32)).to(dev)
    hd = torch.from_numpy(np.diag(H64).copy()).to(dev)
    ora = O.prepare(H64, 0.01, act)
    old = G.prepare_set_deferred_min_n(1)
    try:
        pd = G.prepare(Ht, 0.01, act, hd)
        torch.cuda.synchronize()
    finally:
        G.prepare_set_deferred_min_n(old)
    pp = G.prepare(Ht, 0.01, act, hd)       # the per-panel form (n below the default threshold)
    G.raise_on_status(pd.status, "prepare (outer panels)")
    G.raise_on_status(pp.status, "prepare (panels)")
    assert np.array_equal(pd.perm.cpu().numpy(), ora.perm)
    Ud = pd.U.cpu().numpy().astype(np.float64)
    Up = pp.U.cpu().numpy().astype(np.float64)
    assert np.all(np.tril(Ud, -1) == 0) and np.all(np.diag(Ud) > 0)
    scale = np.abs(ora.U).max()
    err_d = np.abs(Ud - ora.U).max() / scale
    err_p = np.abs(Up - ora.U).max() / scale
    print(f"n={n}: |U - U_oracle| / max|U|: outer panels {err_d:.3g}, panels {err_p:.3g} (bound {n * 2.0 ** -23:.3g})")
    assert err_d <= n * 2.0 ** -23
    assert np.abs(Ud - Up).max() / scale <= n * 2.0 ** -23


@pytest.mark.parametrize("act", [False, True])
def test_dead_inputs(act):
    # features whose activations are all zero: H_ii = 0, so the column is dead (unit
    # diagonal in the damped H, weights zeroed); act-order puts them by their unit key
    W, x = S.small_case(64, 256, 1024, seed=9)
    x = x.copy()
    x[[3, 77, 200], :] = 0
    c, q, prep, Hg, H64, ora = _compare(W, x, 4, 32, False, act)
    print(c)
    dead = prep.dead.cpu().numpy().astype(bool)
    assert np.array_equal(np.flatnonzero(dead), [3, 77, 200])
    assert c.ok(), c


def test_identity_hessian_is_bit_exact_round_to_nearest():
    dev = _dev()
    W = S.make_w(S.WSpec(300, 512, 0.02, "f16", 5, 100))
    for bits, gs, sym in [(4, 128, False), (3, 64, True), (2, 32, False), (4, -1, True)]:
        H = torch.eye(512, dtype=torch.float32, device=dev)
        p = G.prepare(H, 0.01, False)
        q = G.quantize_layer(_w_tensor(W, dev), p, bits, gs, sym, want_codes=True)
        G.raise_on_status(p.status, "rtn")
        rc, rs, rz = O.rtn(W, bits, gs, sym)
        assert np.array_equal(q.codes.cpu().numpy(), rc)
        assert np.array_equal(q.scales.cpu().numpy(), rs.astype(np.float16))
        assert np.array_equal(q.zeros.cpu().numpy(), rz.astype(np.float16))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_bit_exact_on_oracle_codes(bits):
    dev = _dev()
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, (333, 256)).astype(np.uint8)
    qg = G.pack(torch.from_numpy(codes).to(dev), bits).cpu().numpy()
    assert np.array_equal(qg.view(np.uint32), O.pack(codes, bits).view(np.uint32))


def test_err_sq_matches_loss_identity():
    """sum_j e_j^2 = (w - what)^T H_d (w - what) per row, from the GPU's own outputs."""
    W, x = S.small_case(64, 256, 1200, seed=6)
    c, q, prep, Hg, H64, ora = _compare(W, x, 4, 64, True, True)
    assert c.perm_equal
    What = O.dequantize(q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                        q.g_idx.cpu().numpy(), 4, 256)[:, ora.perm]
    d = W.astype(np.float64)[:, ora.perm] - What
    rhs = np.einsum("ij,jk,ik->i", d, ora.prep.Hd, d)
    lhs = q.err_sq.cpu().numpy().astype(np.float64)
    # the identity holds to rounding: fp32 sums of 256 squares on the GPU (~1e-7), the
    # GPU's U and compensation in 3xTF32 against the oracle's fp64 H_d (~1e-6)
    assert np.allclose(lhs, rhs, rtol=1e-4), np.max(np.abs(lhs / rhs - 1))


# --------------------------------------------------------------------------- #
# Errors
# --------------------------------------------------------------------------- #
def test_not_spd_is_reported():
    dev = _dev()
    n = 256
    H = torch.eye(n, dtype=torch.float32, device=dev)
    H[10, 10] = -50.0
    p = G.prepare(H, 0.01, False)
    rc, info = G.status_read(p.status)
    assert rc == G.gptq.ERR_NOT_SPD
    assert 0 <= info < n


def test_nonfinite_weight_is_reported():
    dev = _dev()
    W = S.make_w(S.WSpec(16, 128, 0.02, "f32", 1, 100))
    W[3, 17] = np.nan
    H = torch.eye(128, dtype=torch.float32, device=dev)
    p = G.prepare(H, 0.01, False)
    G.quantize_layer(_w_tensor(W, dev), p, 4, 128, False)
    rc, info = G.status_read(p.status)
    assert rc == G.gptq.ERR_NONFINITE and info == 17


def test_invalid_arguments_are_synchronous():
    dev = _dev()
    W = torch.zeros((8, 100), dtype=torch.float32, device=dev)    # n % 32 != 0
    H = torch.eye(100, dtype=torch.float32, device=dev)
    p = G.prepare(H, 0.01, False)
    with pytest.raises(G.GptqError) as e:
        G.quantize_layer(W, p, 4, 32, False)
    assert e.value.code == G.gptq.ERR_UNSUPPORTED
    W2 = torch.zeros((8, 128), dtype=torch.float32, device=dev)
    H2 = torch.eye(128, dtype=torch.float32, device=dev)
    p2 = G.prepare(H2, 0.01, False)
    with pytest.raises(G.GptqError) as e:
        G.quantize_layer(W2, p2, 5, 32, False)
    assert e.value.code == G.gptq.ERR_UNSUPPORTED
    with pytest.raises(G.GptqError) as e:
        G.quantize_layer(W2, p2, 4, 128, False, block=64)
    assert e.value.code == G.gptq.ERR_UNSUPPORTED


def test_empty_token_chunk_is_a_no_op():
    dev = _dev()
    H = torch.zeros((64, 64), dtype=torch.float32, device=dev)
    X = torch.zeros((64, 0), dtype=torch.bfloat16, device=dev)
    G.hessian_accumulate(H, X)
    torch.cuda.synchronize()
    assert float(H.abs().max()) == 0.0


# --------------------------------------------------------------------------- #
# The worked-example layer at full size: [1024, 4096], 65,536 tokens
# --------------------------------------------------------------------------- #
def test_worked_example_layer_full_size():
    wl = S.workloads()["layer-1024x4096"]
    L, st = wl.layers[0], wl.settings[0]
    W, x = S.make_w(L.w), S.make_x(L.x)
    c, q, prep, Hg, H64, ora = _compare(W, x, st.bits, st.group_size, st.sym, st.desc_act)
    print(c)
    assert q.scales.numel() == 32768
    assert c.code_mismatch <= CODE_MISMATCH_MAX and abs(c.rel_err_ratio - 1) <= REL_ERR_TOL
    assert c.ok(), c


# The Llama-shaped layers at their own token counts, every setting: test_gpu_full_shapes.py.


@pytest.mark.parametrize("n", [200, 256, 520])     # the single-CTA kernel; CTA pairs (one tile; ragged tiles)
def test_bounded_wait_reports_timeout_and_the_context_survives(monkeypatch, n):
    """The Hessian producers withhold their loads (host-side test switch); the MMA
    side's bounded waits run out, the kernel drains, frees TMEM and reports
    GPTQ_ERR_TIMEOUT; the next call on the same context works."""
    dev = _dev()
    _, x = S.small_case(8, n, 1024, seed=9)
    X = _to_dev_x(x, dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    st = G.new_status(dev)
    monkeypatch.setenv("GPTQ_FAULT_INJECT", "hessian_stall")
    G.hessian_accumulate(H, X, None, st)
    rc, info = G.status_read(st)
    assert rc == G.gptq.ERR_TIMEOUT
    monkeypatch.delenv("GPTQ_FAULT_INJECT")
    G.status_reset(st)
    H.zero_()
    G.hessian_accumulate(H, X, None, st)
    rc, _ = G.status_read(st)
    assert rc == G.gptq.OK
    H64 = O.hessian(x)
    iu = np.triu_indices(n)
    rel = np.abs(H.cpu().numpy().astype(np.float64)[iu] - H64[iu]) / np.sqrt(np.outer(np.diag(H64), np.diag(H64)))[iu]
    assert rel.max() <= hessian_bound([1024])


@pytest.mark.parametrize("n,tokens", [(256, 64), (384, 1000), (768, 4096), (1300, 777)])
def test_hessian_tile_pairs_against_oracle(n, tokens):
    """The CTA-pair kernel (n >= 256): whole tiles, ragged tiles, one stage, ragged tokens."""
    dev = _dev()
    _, x = S.small_case(8, n, tokens, seed=n + tokens)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hd = torch.zeros(n, dtype=torch.float64, device=dev)
    st = G.new_status(dev)
    G.hessian_accumulate(H, _to_dev_x(x, dev), hd, st)
    G.raise_on_status(st, "pair Hessian")
    H64 = O.hessian(x)
    iu = np.triu_indices(n)
    rel = np.abs(H.cpu().numpy().astype(np.float64)[iu] - H64[iu]) / np.sqrt(np.outer(np.diag(H64), np.diag(H64)))[iu]
    assert rel.max() <= hessian_bound([tokens]), rel.max()
    assert np.allclose(hd.cpu().numpy(), np.diag(H64), rtol=1e-13, atol=0)


@pytest.mark.parametrize("sym", [True, False])
def test_rounding_boundaries_are_bit_exact(sym):
    """Weights placed on and within a few ulps of (k + 1/2).s, where the fp32 quotient
    decides the code by its last bit; with H = I there is no compensation, so the
    codes must equal round-to-nearest of the IEEE quotient exactly."""
    dev = _dev()
    rng = np.random.default_rng(7 + sym)
    out, n, gs = 512, 512, 128
    s0 = np.float16(np.exp(rng.uniform(-9, -3, (out, n // gs)))).astype(np.float32)   # fp16 scales
    W = np.zeros((out, n), np.float32)
    for g in range(n // gs):
        s = s0[:, g:g + 1]
        k = rng.integers(-7, 7, (out, gs)).astype(np.float32)
        base = ((k + np.float32(0.5)) * s).astype(np.float32)
        steps = rng.integers(-3, 4, (out, gs))
        w = base.copy()
        for _ in range(3):
            move = np.abs(steps) > _
            w = np.where(move, np.nextafter(w, np.where(steps > 0, np.inf, -np.inf).astype(np.float32)), w)
        if sym:
            w[:, 0] = 7 * s[:, 0]          # amax = 7 s  ->  scale = fp16(7 s / 7) = s
            w[:, 1] = -7 * s[:, 0]
        else:
            w[:, 0] = -7 * s[:, 0]         # lo = -7 s, hi = 8 s  ->  scale = fp16(15 s / 15) = s, zero = 7
            w[:, 1] = 8 * s[:, 0]
        W[:, g * gs:(g + 1) * gs] = np.clip(w, -7 * s, (7 if sym else 8) * s)
    H = torch.eye(n, dtype=torch.float32, device=dev)
    p = G.prepare(H, 0.01, False)
    q = G.quantize_layer(_w_tensor(W, dev), p, 4, gs, sym, want_codes=True)
    G.raise_on_status(p.status, "boundaries")
    rc, rs, rz = O.rtn(W, 4, gs, sym)
    assert np.array_equal(rs, s0.T)
    assert np.array_equal(q.codes.cpu().numpy(), rc)


# --------------------------------------------------------------------------- #
# Checkpoint variants: zero padding, packed zero points
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("n,bits,gs,sym,act", [
    (300, 4, 128, False, False),
    (300, 4, 128, True, True),
    (300, 3, 64, False, True),
    (300, 4, -1, False, False),     # one group per row: padded to a multiple of 32
    (100, 4, 128, True, False),     # fewer rows in X than one tile of the Hessian
])
def test_zero_padded_layer(n, bits, gs, sym, act):
    """W [72, n] and X [n, 1000] zero-padded to the group size through the *_padded
    entry points, against the oracle on the explicitly padded arrays."""
    dev = _dev()
    W, x = S.small_case(72, n, 1000, seed=n + bits, rank=8, frac=0.02, mult=20.0)
    n_pad = G.padded_width(n, gs)
    q, prep, Hg = G.gptq_quantize(_w_tensor(W, dev), _to_dev_x(x, dev), bits, gs, sym, act, want_codes=True,
                                  want_err=True, pad=True)
    torch.cuda.synchronize()
    assert tuple(Hg.shape) == (n_pad, n_pad) and q.g_idx.numel() == n_pad and q.codes.shape[1] == n_pad
    Hu = torch.triu(Hg).cpu().numpy()
    assert not Hu[n:].any() and not Hu[:, n:].any()        # the padded rows and columns receive nothing
    assert np.array_equal(np.flatnonzero(prep.dead.cpu().numpy()), np.arange(n, n_pad))
    Wp, xp = O.pad_layer(W, x, n_pad)
    H64 = O.hessian(xp)
    ora = O.gptq_layer(Wp, None, bits, gs, sym, act, H=H64)
    c = compare_layer(Wp, H64, ora, q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                      q.g_idx.cpu().numpy(), q.codes.cpu().numpy(), prep.perm.cpu().numpy(), bits, gs)
    print(c)
    assert c.ok(), c
    What = O.dequantize(q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                        q.g_idx.cpu().numpy(), bits, n_pad)
    assert not What[:, n:].any()


def test_zero_padded_layer_from_host_memory():
    dev = _dev()
    n = 300
    W, x = S.small_case(48, n, 2504, seed=6)
    Wt = torch.from_numpy(np.ascontiguousarray(W))
    X_host = torch.from_numpy(x.view(np.int16)).pin_memory()
    # a small staging area: several chunks of 300 rows
    n_pad = G.padded_width(n, 64)
    H = torch.zeros((n_pad, n_pad), dtype=torch.float32, device=dev)
    hd = torch.zeros(n_pad, dtype=torch.float64, device=dev)
    st = G.new_status(dev)
    G.hessian_accumulate_host(H, X_host, hd, st, staging=G.workspace(2 * n * 512 * 2, dev))
    G.raise_on_status(st, "padded host Hessian")
    H64 = O.hessian(O.pad_layer(W, x, n_pad)[1])
    Hg = H.cpu().numpy().astype(np.float64)
    iu = np.triu_indices(n_pad)
    norm = np.sqrt(np.maximum(np.outer(np.diag(H64), np.diag(H64)), 1e-300))[iu]
    # one launch per staged chunk of at least 64 tokens: at most ceil(2504 / 64) launches
    assert (np.abs(Hg[iu] - H64[iu]) / norm).max() <= hessian_bound([64] * 39 + [8])
    assert not Hg[iu][H64[iu] == 0].any()
    assert np.allclose(hd.cpu().numpy(), np.diag(H64), rtol=1e-13, atol=0)
    # the whole padded path from host tensors gives the device path's result
    q_h, p_h, _ = G.gptq_quantize(Wt.pin_memory(), X_host, 4, 64, False, True, want_codes=True, pad=True)
    q_d, p_d, _ = G.gptq_quantize(Wt.to(dev), _to_dev_x(x, dev), 4, 64, False, True, want_codes=True, pad=True)
    assert np.array_equal(p_h.perm.cpu().numpy(), p_d.perm.cpu().numpy())
    assert float(np.mean(q_h.codes.cpu().numpy() != q_d.codes.cpu().numpy())) <= CODE_MISMATCH_MAX


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("offset", [0, 1])
def test_pack_zeros_bit_exact(bits, offset):
    dev = _dev()
    rng = np.random.default_rng(10 * bits + offset)
    z = rng.integers(0, 2 ** bits, (7, 352)).astype(np.float16)
    st = G.new_status(dev)
    qz = G.pack_zeros(torch.from_numpy(z).to(dev), bits, offset, st)
    G.raise_on_status(st, "pack_zeros")
    assert np.array_equal(qz.cpu().numpy().view(np.uint32), O.pack_zeros(z, bits, offset).view(np.uint32))


def test_pack_zeros_of_a_quantized_layer():
    dev = _dev()
    W, x = S.small_case(96, 256, 1024, seed=12)
    q, prep, _ = _run_gpu(W, x, 3, 64, False, True)
    zg = q.zeros.cpu().numpy()
    qz = G.pack_zeros(q.zeros, 3, 1, prep.status)
    G.raise_on_status(prep.status, "pack_zeros")
    assert np.array_equal(qz.cpu().numpy().view(np.uint32), O.pack_zeros(zg, 3, 1).view(np.uint32))
    assert np.array_equal(O.unpack_zeros(qz.cpu().numpy(), 3, 96, 1), zg.astype(np.float64))


def test_pack_zeros_reports_a_zero_that_is_not_a_code():
    dev = _dev()
    z = np.full((3, 64), 5, dtype=np.float16)
    z[1, 17] = 2.5
    st = G.new_status(dev)
    G.pack_zeros(torch.from_numpy(z).to(dev), 4, 0, st)
    rc, info = G.status_read(st)
    assert rc == G.gptq.ERR_INVALID_ARG and info == 64 + 17


# --------------------------------------------------------------------------- #
# Ordering: the multi-stream stages are deterministic and calls queue safely
# --------------------------------------------------------------------------- #
def test_repeated_and_back_to_back_calls_are_bit_identical():
    """Every stage computes each element in a fixed order, so repeated runs give the same
    bits.  prepare() forks onto four library streams and the host Hessian onto a copy
    stream shared by all calls of a host thread; calls queued back to back without a
    synchronization must give the bits of calls run one at a time."""
    dev = _dev()
    W, x = S.small_case(1024, 1536, 3000, seed=21, rank=16)
    Wt, X = _w_tensor(W, dev), _to_dev_x(x, dev)
    X2 = _to_dev_x(S.small_case(8, 1536, 2000, seed=22, rank=16)[1], dev)

    def one(Xa, act):
        st = G.new_status(dev)
        H = torch.zeros((1536, 1536), dtype=torch.float32, device=dev)
        hd = torch.zeros(1536, dtype=torch.float64, device=dev)
        G.hessian_accumulate(H, Xa, hd, st)
        p = G.prepare(H, 0.01, act, hd, st)
        q = G.quantize_layer(Wt, p, 4, 128, False, want_codes=True)
        return st, H, p, q

    ref = []
    for Xa, act in [(X, True), (X2, False)]:
        st, H, p, q = one(Xa, act)
        torch.cuda.synchronize()
        G.raise_on_status(st, "reference run")
        ref.append((H.clone(), p.U.clone(), p.perm.clone(), q.qweight.clone(), q.scales.clone(), q.zeros.clone()))
    for _ in range(2):
        runs = [one(X, True), one(X2, False), one(X, True)]      # queued back to back
        torch.cuda.synchronize()
        for (st, H, p, q), r in zip(runs, [ref[0], ref[1], ref[0]]):
            G.raise_on_status(st, "back-to-back run")
            got = (torch.triu(H), p.U, p.perm, q.qweight, q.scales, q.zeros)
            exp = (torch.triu(r[0]),) + r[1:]
            for a, b in zip(got, exp):
                assert torch.equal(a, b)


def test_host_hessian_calls_back_to_back_are_bit_identical():
    # the copy stream and its events are shared by the calls of a host thread; two calls
    # sharing one staging area, queued without a synchronization, give the bits of one call
    dev = _dev()
    _, x = S.small_case(8, 640, 5000, seed=23, rank=16)
    X_host = torch.from_numpy(x.view(np.int16)).pin_memory()
    staging = G.workspace(2 * 640 * 1024 * 2, dev)
    st = G.new_status(dev)
    H0 = torch.zeros((640, 640), dtype=torch.float32, device=dev)
    G.hessian_accumulate_host(H0, X_host, None, st, staging=staging)
    torch.cuda.synchronize()
    Hs = [torch.zeros((640, 640), dtype=torch.float32, device=dev) for _ in range(3)]
    for H in Hs:
        G.hessian_accumulate_host(H, X_host, None, st, staging=staging)
    torch.cuda.synchronize()
    G.raise_on_status(st, "host Hessian back to back")
    for H in Hs:
        assert torch.equal(torch.triu(H), torch.triu(H0))


def test_bf16_weights():
    # W given in bf16: the oracle quantizes exactly the values the library reads
    dev = _dev()
    W32, x = S.small_case(96, 1024, 1200, seed=44)
    Wb = torch.from_numpy(W32).to(torch.bfloat16)
    W = Wb.float().numpy()
    q, prep, _ = G.gptq_quantize(Wb.to(dev), _to_dev_x(x, dev), 4, 128, False, True, want_codes=True)
    torch.cuda.synchronize()
    H64 = O.hessian(x)
    ora = O.gptq_layer(W, None, 4, 128, False, True, H=H64)
    c = compare_layer(W, H64, ora, q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                      q.g_idx.cpu().numpy(), q.codes.cpu().numpy(), prep.perm.cpu().numpy(), 4, 128)
    print(c)
    assert c.ok(), c


@pytest.mark.parametrize("bits,gs,sym", [(4, 128, False), (4, 128, True), (2, 32, False), (3, -1, True),
                                         (8, 64, False)])
def test_degenerate_groups_are_bit_exact_round_to_nearest(bits, gs, sym):
    """Rows whose groups hit the quantizer's special cases: all zero (asymmetric range
    taken as [-1, 1], symmetric magnitude 1), constant of either sign (one end of the
    range at 0), tiny (the scale clamps to fp16's smallest subnormal), huge (the scale
    clamps to fp16's largest value and codes saturate), one non-zero weight per group.
    With H = I the method reduces to round-to-nearest, so codes, scales and zeros must
    equal the oracle's bit for bit."""
    dev = _dev()
    n = 512
    rng = np.random.default_rng(bits * 10 + int(sym))
    rows = [np.zeros(n), np.full(n, 0.01), np.full(n, -0.03), 1e-9 * rng.standard_normal(n),
            1e6 * rng.standard_normal(n), 3e-6 * rng.standard_normal(n)]
    lone = np.zeros(n)
    lone[::32] = 0.05 * rng.standard_normal(n // 32)
    rows.append(lone)
    W = np.stack(rows * 5).astype(np.float32)                 # 35 rows
    H = torch.eye(n, dtype=torch.float32, device=dev)
    p = G.prepare(H, 0.01, False)
    q = G.quantize_layer(_w_tensor(W, dev), p, bits, gs, sym, want_codes=True)
    G.raise_on_status(p.status, "degenerate groups")
    rc, rs, rz = O.rtn(W, bits, gs, sym)
    assert np.array_equal(q.scales.cpu().numpy(), rs.astype(np.float16))
    assert np.array_equal(q.zeros.cpu().numpy(), rz.astype(np.float16))
    assert np.array_equal(q.codes.cpu().numpy(), rc)


# --------------------------------------------------------------------------- #
# Layers that share an input, stacked in one call
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("outs,n,bits,gs,sym,act,wdtype", [
    ((300, 64, 64), 512, 4, 128, True, True, "f16"),       # q / k / v-like: one wide, two narrow
    ((2000, 600), 384, 3, 64, False, True, "f16"),         # the stacked rows change the lanes per row
    ((5000, 200, 77), 256, 2, 32, False, False, "f32"),
])
def test_stacked_layers_equal_separate_calls_bit_for_bit(outs, n, bits, gs, sym, act, wdtype):
    """Rows are independent given U ("Etape 1"): quantizing layers of one input stacked
    along the outputs gives exactly the per-layer results."""
    dev = _dev()
    _, x = S.small_case(8, n, 3 * n, seed=n + len(outs))
    X = _to_dev_x(x, dev)
    st = G.new_status(dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hd = torch.zeros(n, dtype=torch.float64, device=dev)
    G.hessian_accumulate(H, X, hd, st)
    prep = G.prepare(H, 0.01, act, hd, st)
    Ws = [_w_tensor(S.make_w(S.WSpec(o, n, 0.02, wdtype, 5, 100 + i)), dev) for i, o in enumerate(outs)]
    sep = [G.quantize_layer(W, prep, bits, gs, sym, want_codes=True, want_err=True) for W in Ws]
    stacked, views = G.quantize_layers(Ws, prep, bits, gs, sym, want_codes=True, want_err=True)
    G.raise_on_status(st, "stacked layers")
    for a, b in zip(views, sep):
        for name in ("qweight", "scales", "zeros", "g_idx", "codes"):
            x_, y_ = getattr(a, name).contiguous().cpu().numpy(), getattr(b, name).cpu().numpy()
            assert np.array_equal(x_.view(np.uint8), y_.view(np.uint8)), name
        # err_sq is a per-row fp32 sum across the lanes of its row, whose count depends on
        # the rows per launch: equal up to the order of that sum
        assert np.allclose(a.err_sq.cpu().numpy(), b.err_sq.cpu().numpy(), rtol=1e-6, atol=0)


def test_timing_trace_records_every_stage_on_its_stream():
    dev = _dev()
    W, x = S.small_case(256, 1536, 2048, seed=9)
    G.trace_read()
    G.trace_enable(True)
    q, prep, H = _run_gpu(W, x, 4, 128, False, True)
    G.trace_enable(False)
    tr = G.trace_read()
    for k in ("hessian_tc", "hessian_diag64", "potrf_inv", "prepare_gemm3", "ingest", "sweep", "trailing_update",
              "u_operand", "pack"):
        assert k in tr and tr[k]["launches"] > 0 and tr[k]["ms"] > 0, k
    assert tr["sweep"]["launches"] == 3 and tr["potrf_inv"]["launches"] == 12
    assert tr["hessian_tc"]["work"] == pytest.approx(1536 * 1537 * 2048)
    # with the trace off nothing is recorded
    _run_gpu(W, x, 4, 128, False, True)
    assert G.trace_read() == {}


def test_timing_trace_timeline_orders_each_stream():
    dev = _dev()
    W, x = S.small_case(256, 1536, 2048, seed=9)
    G.trace_read()
    G.trace_enable(True)
    _run_gpu(W, x, 4, 128, False, True)
    G.trace_enable(False)
    tl = G.trace_read_timeline()
    assert tl and min(e[2] for e in tl) == 0.0
    assert all(0.0 <= e[2] <= e[3] for e in tl)
    # the diagonal-block chain: 12 launches on one stream, one after the other
    chain = [e for e in tl if e[0] == "potrf_inv"]
    assert len(chain) == 12 and len({e[1] for e in chain}) == 1
    assert all(a[3] <= b[2] + 1e-3 for a, b in zip(chain, chain[1:]))
    # the stages run in order: the Hessian before the preparation, the preparation before the sweep
    hess_end = max(e[3] for e in tl if e[0] == "hessian_tc")
    assert hess_end <= chain[0][2] + 1e-3
    assert chain[-1][3] <= min(e[2] for e in tl if e[0] == "sweep") + 1e-3
    assert G.trace_read_timeline() == []


def test_layer_split_over_two_ranks_on_one_device():
    """The two-rank split of sharded.py, both ranks' kernels on one device (no
    collective: the all-reduce of two partial H is their sum, one fp32 addition per
    entry, and the gather is the concatenation of the row shards).  H from the two
    token halves stays within the derived bound of the oracle's H; the rows quantized
    in two shards equal the unsplit call bit for bit."""
    from post_weight_quantization_15_b200 import sharded as SH
    dev = _dev()
    out, n, N = 333, 512, 3000
    W, x = S.small_case(out, n, N, seed=21)
    X = _to_dev_x(x, dev)
    st = G.new_status(dev)
    Hs, ds, spans = [], [], []
    for r in range(2):
        t0, t1 = SH.split_range(N, 2, r, align=8)
        spans.append(t1 - t0)
        H = torch.zeros((n, n), dtype=torch.float32, device=dev)
        hd = torch.zeros(n, dtype=torch.float64, device=dev)
        G.hessian_accumulate(H, X[:, t0:t1], hd, st)
        Hs.append(H)
        ds.append(hd)
    H = Hs[0] + Hs[1]
    hd = ds[0] + ds[1]
    H64 = O.hessian(x)
    iu = np.triu_indices(n)
    rel = np.abs(H.cpu().numpy().astype(np.float64)[iu] - H64[iu]) / np.sqrt(np.outer(np.diag(H64), np.diag(H64)))[iu]
    # each rank's own summation, and one more addition (counted as one more call)
    assert rel.max() <= hessian_bound(spans + [1]), rel.max()
    assert np.allclose(hd.cpu().numpy(), np.diag(H64), rtol=1e-13, atol=0)
    prep = G.prepare(H, 0.01, True, hd, st)
    Wt = _w_tensor(W, dev)
    whole = G.quantize_layer(Wt, prep, 4, 128, True, want_codes=True, want_err=True)
    parts = []
    for r in range(2):
        o0, o1 = SH.split_range(out, 2, r)
        parts.append(G.quantize_layer(Wt[o0:o1].contiguous(), prep, 4, 128, True, want_codes=True, want_err=True))
    G.raise_on_status(st, "split layer")
    for name, dim in (("qweight", 1), ("scales", 1), ("zeros", 1), ("codes", 0), ("err_sq", 0)):
        cat = torch.cat([getattr(p, name) for p in parts], dim=dim).cpu().numpy()
        assert np.array_equal(cat.view(np.uint8), getattr(whole, name).cpu().numpy().view(np.uint8)), name
    c = compare_layer(W, H64, O.gptq_layer(W, None, 4, 128, True, True, H=H64), whole.qweight.cpu().numpy(),
                      whole.scales.cpu().numpy(), whole.zeros.cpu().numpy(), whole.g_idx.cpu().numpy(),
                      whole.codes.cpu().numpy(), prep.perm.cpu().numpy(), 4, 128)
    assert c.ok(), c
