"""The consumer of the stored format against the oracle, through the C ABI.

gptq_dequantize must give the oracle's dequantized weights bit for bit (the fp32
product of an fp16 scale and a small integer is exact; fp16 / bf16 outputs are one
rounding of that exact value).  gptq_qmatvec must give X . What^T within the bound of
its fp32 summation, derived below.  The stored layers are the CUDA path's own
(quantized here from seeded inputs); what is compared is what the consumer makes of
them, against the oracle reading the same bits.
"""
import numpy as np
import pytest

import synthetic as S
from oracle import gptq_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_15_b200 as G


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _stored_layer(out, n, tokens, bits, gs, sym, act, seed):
    dev = _dev()
    W, x = S.small_case(out, n, tokens, seed=seed)
    Xd = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    q, prep, _ = G.gptq_quantize(torch.from_numpy(W).to(dev), Xd, bits, gs, sym, act)
    return q


def _oracle_what(q):
    n = q.g_idx.numel()
    return O.dequantize(q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                        q.g_idx.cpu().numpy(), q.bits, n)


def _matvec_bound(X64, What):
    """|Y_gpu - Y| <= c . 2^-24 . sum_k |x_k . what_k|, c the larger of the two forms' counts.

    CUDA cores: every term is an exact product of fp32 values (the activations and the exact
    What) added by one fma (one rounding of at most 2^-24 of the running sum, itself at most
    the sum of |terms|); a thread adds at most n terms, then the 8 warps' sums and the k
    splits (at most 24 more additions): c = n + 24.
    Tensor cores (4-bit codes, fp16 / bf16 activations): the products x . (code - z) are
    exact; an accumulation holds at most 8 mma.sync of 16 columns, each summing 17 aligned
    terms (16 products and the accumulator), each off by at most one ulp of that sum
    whether the hardware rounds or truncates: <= 8 . 17 . 2^-23 of the accumulation's sum of
    |terms|, which times s (> 0) is at most the sum of its |x . what|; each accumulation is
    scaled and added by one fma (at most one per 32 columns), then the warps and the splits:
    c = 272 + n / 32 + 9 + n / 256."""
    n = X64.shape[1]
    c = max(n + 24, 272 + n // 32 + 9 + n // 256)
    return c * 2.0 ** -24 * (np.abs(X64) @ np.abs(What).T)


@pytest.mark.parametrize("bits,gs,sym,act", [(4, 128, False, False), (4, 64, True, True), (2, 32, False, True),
                                             (8, -1, True, False)])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_dequantize_is_bit_exact(bits, gs, sym, act, dtype):
    q = _stored_layer(250, 512, 1536, bits, gs, sym, act, seed=bits * 10 + (gs % 7))
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    st = G.new_status(q.qweight.device)
    got = G.dequantize(q, tdt, st)
    G.raise_on_status(st, "dequantize")
    ref = _oracle_what(q)
    if dtype == "f32":
        assert np.array_equal(got.cpu().numpy(), ref.astype(np.float32))
        assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)     # exact in fp32
    elif dtype == "f16":
        assert np.array_equal(got.cpu().numpy().view(np.uint16), ref.astype(np.float16).view(np.uint16))
    else:
        bits_ref = S.f32_to_bf16_bits(ref.astype(np.float32))
        assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), bits_ref)


@pytest.mark.parametrize("M", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("bits,gs,act,xdt", [(4, 128, False, "f16"), (4, 128, True, "bf16"), (4, 64, False, "bf16"),
                                             (2, 64, True, "f16"), (8, 32, False, "f32")])
def test_qmatvec_against_the_oracle(M, bits, gs, act, xdt):
    # n = 1536: three 512-wide k splits; out = 250: a ragged last block of outputs (out % 4 != 0)
    q = _stored_layer(250, 1536, 3072, bits, gs, False, act, seed=M + bits)
    dev = q.qweight.device
    rng = np.random.default_rng(M)
    Xf = rng.standard_normal((M, 1536)).astype(np.float32)
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[xdt]
    Xt = torch.from_numpy(Xf).to(dev).to(tdt)
    st = G.new_status(dev)
    Y = G.qmatvec(q, Xt, st)
    G.raise_on_status(st, "qmatvec")
    X64 = Xt.float().cpu().numpy().astype(np.float64)       # the activations as the kernel reads them
    What = _oracle_what(q)
    ref = X64 @ What.T
    err = np.abs(Y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= _matvec_bound(X64, What)), float(np.max(err / _matvec_bound(X64, What)))


@pytest.mark.parametrize("reordered", [False, True])
def test_qmatvec_decode_shape_of_the_70b_mlp(reordered):
    """gate of the 70B block, [28672 x 8192] 4-bit g128 act-order, one token, as stored and
    reordered by group: sampled outputs against the oracle (rows are read from the stored
    bits one by one)."""
    dev = _dev()
    out, n = 28672, 8192
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    # a stored layer of that shape: random codes, positive fp16 scales, integer zeros, act-order g_idx
    q = G.QuantizedLayer(qweight=torch.randint(-2 ** 31, 2 ** 31 - 1, (n * 4 // 32, out), generator=gen, device=dev,
                                               dtype=torch.int64).to(torch.int32),
                         scales=(torch.rand((n // 128, out), generator=gen, device=dev) * 0.01 + 1e-4).half(),
                         zeros=torch.randint(0, 16, (n // 128, out), generator=gen, device=dev).half(),
                         g_idx=(torch.randperm(n, generator=gen, device=dev) // 128).to(torch.int32),
                         codes=None, err_sq=None, bits=4, group_size=128, sym=False)
    X = torch.randn((1, n), generator=gen, device=dev).half()
    st = G.new_status(dev)
    if reordered:
        qg, xperm = G.reorder_groups(q, st)
        Y = G.qmatvec(qg, X, st, xperm=xperm)
    else:
        Y = G.qmatvec(q, X, st)
    G.raise_on_status(st, "decode shape")
    cols = np.sort(np.random.default_rng(0).choice(out, 256, replace=False))
    qw = q.qweight.cpu().numpy()[:, cols]
    What = O.dequantize(qw, q.scales.cpu().numpy()[:, cols], q.zeros.cpu().numpy()[:, cols], q.g_idx.cpu().numpy(),
                        4, n)
    X64 = X.float().cpu().numpy().astype(np.float64)
    ref = X64 @ What.T
    err = np.abs(Y.cpu().numpy()[:, cols].astype(np.float64) - ref)
    assert np.all(err <= _matvec_bound(X64, What))


def test_group_index_outside_the_scales_is_reported():
    q = _stored_layer(64, 256, 512, 4, 128, False, False, seed=5)
    g = q.g_idx.clone()
    g[77] = 2                                            # only groups 0 and 1 exist
    bad = G.QuantizedLayer(q.qweight, q.scales, q.zeros, g, None, None, 4, 128, False)
    st = G.new_status(q.qweight.device)
    G.dequantize(bad, torch.float32, st)
    rc, info = G.status_read(st)
    assert rc == G.gptq.ERR_INVALID_ARG and info == 77
    st = G.new_status(q.qweight.device)
    G.qmatvec(bad, torch.zeros((2, 256), dtype=torch.float16, device=q.qweight.device), st)
    rc, info = G.status_read(st)
    assert rc == G.gptq.ERR_INVALID_ARG and info == 77


@pytest.mark.parametrize("bits,gs,M", [(4, 128, 1), (4, 32, 16), (2, 64, 5), (8, 128, 8)])
def test_reordered_act_order_layer(bits, gs, M):
    """gptq_reorder_groups on an act-order layer: xperm is a permutation sorting the columns by
    group (stable), the reordered layer dequantizes to the original's columns in that order
    bit for bit, and its product (with xperm) is the oracle's within the summation bound."""
    q = _stored_layer(260, 1024, 2048, bits, gs, False, True, seed=bits + gs + M)
    st = G.new_status(q.qweight.device)
    qg, xperm = G.reorder_groups(q, st)
    G.raise_on_status(st, "reorder")
    g = q.g_idx.cpu().numpy()
    xp = xperm.cpu().numpy()
    assert np.array_equal(np.sort(xp), np.arange(1024))
    assert np.array_equal(xp, np.argsort(g, kind="stable"))
    assert np.array_equal(qg.g_idx.cpu().numpy(), g[xp])
    What = _oracle_what(q)
    assert np.array_equal(G.dequantize(qg, torch.float32, st).cpu().numpy(), What[:, xp].astype(np.float32))
    X = torch.from_numpy(np.random.default_rng(M).standard_normal((M, 1024)).astype(np.float32)).to(
        q.qweight.device).half()
    Y = G.qmatvec(qg, X, st, xperm=xperm)
    G.raise_on_status(st, "reordered qmatvec")
    X64 = X.float().cpu().numpy().astype(np.float64)
    err = np.abs(Y.cpu().numpy().astype(np.float64) - X64 @ What.T)
    assert np.all(err <= _matvec_bound(X64, What))


@pytest.mark.parametrize("rows", [1, 2, 3])
@pytest.mark.parametrize("xdt", ["f16", "bf16"])
def test_qmatvec_with_fractional_zero_points(xdt, rows):
    """Zero points off the integers (a stored layer edited by hand) are still applied in fp32
    (one and two rows: the blocks fall back from the tensor-core form; three: the fma form):
    the product is the oracle's within the summation bound."""
    q = _stored_layer(256, 1024, 2048, 4, 128, False, False, seed=21)
    zq = (q.zeros.float() + 0.25).half()
    q2 = G.QuantizedLayer(q.qweight, q.scales, zq, q.g_idx, None, None, 4, 128, False)
    dev = q.qweight.device
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}[xdt]
    X = torch.from_numpy(np.random.default_rng(4).standard_normal((rows, 1024)).astype(np.float32)).to(dev).to(tdt)
    st = G.new_status(dev)
    Y = G.qmatvec(q2, X, st)
    G.raise_on_status(st, "fractional zeros")
    What = _oracle_what(q2)
    assert not np.array_equal(What, _oracle_what(q))
    X64 = X.float().cpu().numpy().astype(np.float64)
    err = np.abs(Y.cpu().numpy().astype(np.float64) - X64 @ What.T)
    assert np.all(err <= _matvec_bound(X64, What))
