"""The sequential block pipeline and its forward-pass kernels against the oracle.

Each stage is checked against the oracle given the same inputs as the GPU's stage
(the GPU's previous stage output), so that the comparison measures each stage, not
rounding differences compounded through earlier ones:
  gate / up   quantized on the block's input X      vs the oracle's GPTQ on that X
  h           silu(What_g X) * (What_u X)           vs the oracle's fp64 forward
  down        quantized on h                        vs the oracle's GPTQ on that h
  X_next      X + What_d h                          vs the oracle's fp64 forward
"""
import numpy as np
import pytest

import synthetic as S
from oracle import gptq_oracle as O
from tests.parity import compare_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_15_b200 as G
    from post_weight_quantization_15_b200 import pipeline as PL


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _linear_bound(K, absprod):
    """The product's summation (linear_kernel, the structure of tests/parity.py's hessian_bound):
    16-deep tensor-core steps in chunks of 256 from zero (272 ulps of the chunk's sum of
    |terms|), chunks added in fp32 with round to nearest, one store: relative to
    sum_k |a_k b_k|."""
    chunks = (K + 255) // 256
    return (272 * 2.0 ** -23 + (chunks + 1) * 2.0 ** -24) * absprod


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _as_bf16(What):
    """The dequantized weights as the forward uses them: in bf16, the activations' type (one
    tensor-core product takes one operand type).  What is exact in fp32 (an fp16 scale times
    a small integer), so this is one round to nearest even of the exact value."""
    return O.bf16_bits_to_f64(S.f32_to_bf16_bits(np.asarray(What, np.float64).astype(np.float32)))


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 520, 1000), (1100, 300, 4104)])
def test_linear_bf16_against_the_oracle(M, N, K):
    dev = _dev()
    rng = np.random.default_rng(M + N + K)
    a = S.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    b = S.f32_to_bf16_bits((rng.standard_normal((N, K)) * np.exp(rng.standard_normal((N, 1)))).astype(np.float32))
    A = torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    B = torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)
    st = G.new_status(dev)
    C = G.linear_bf16(A, B, st)
    G.raise_on_status(st, "linear")
    a64, b64 = O.bf16_bits_to_f64(a), O.bf16_bits_to_f64(b)
    ref = a64 @ b64.T
    err = np.abs(C.cpu().numpy().astype(np.float64) - ref)
    bound = _linear_bound(K, np.abs(a64) @ np.abs(b64).T)
    assert np.all(err <= bound), float(np.max(err / bound))


def test_transpose_silu_mul_residual():
    dev = _dev()
    rng = np.random.default_rng(1)
    x = S.f32_to_bf16_bits(rng.standard_normal((200, 333)).astype(np.float32))
    X = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    st = G.new_status(dev)
    assert np.array_equal(_bits(G.transpose_bf16(X, st)), x.T)
    g = (rng.standard_normal((7, 1001)) * 4).astype(np.float32)
    u = rng.standard_normal((7, 1001)).astype(np.float32)
    h = G.silu_mul(torch.from_numpy(g).to(dev), torch.from_numpy(u).to(dev), st)
    ref = O.silu(g.astype(np.float64)) * u
    # fp32 arithmetic (a few ulps), then one bf16 rounding (half an ulp of 2^-8 relative)
    got = O.bf16_bits_to_f64(_bits(h))
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
    y = rng.standard_normal((200, 333)).astype(np.float32)
    xn = G.residual_add(X, torch.from_numpy(y).to(dev), st)
    ref = O.bf16_bits_to_f64(x) + y
    assert np.all(np.abs(O.bf16_bits_to_f64(_bits(xn)) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
    G.raise_on_status(st, "elementwise")


def test_two_block_pipeline_stage_by_stage():
    dev = _dev()
    d, d_ff, N = 512, 1024, 2048
    x0 = S.make_x(S.XSpec(d, N, 16, 0.01, 20.0, 3, 1))
    blocks_np = [(S.make_w(S.WSpec(d_ff, d, 0.02, "f16", 3, 10 * b + 1)),
                  S.make_w(S.WSpec(d_ff, d, 0.02, "f16", 3, 10 * b + 2)),
                  S.make_w(S.WSpec(d, d_ff, 0.02, "f16", 3, 10 * b + 3))) for b in range(2)]
    blocks = [tuple(torch.from_numpy(w).to(dev) for w in blk) for blk in blocks_np]
    X0 = torch.from_numpy(x0.view(np.int16)).to(dev).view(torch.bfloat16)
    res, X_out = PL.quantize_mlp_blocks(X0, blocks, bits=4, group_size=128, sym=True, desc_act=True, record=True)
    xs = [r.x_in for r in res] + [X_out]
    for b, (r, (Wg, Wu, Wd)) in enumerate(zip(res, blocks_np)):
        xb = _bits(xs[b])
        # gate and up on this block's input
        Wgu = np.concatenate([Wg, Wu], axis=0)
        H64 = O.hessian(xb)
        ora = O.gptq_layer(Wgu, None, 4, 128, True, True, H=H64)
        q = r.gate_up
        c = compare_layer(Wgu, H64, ora, q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                          q.g_idx.cpu().numpy(), O.unpack(q.qweight.cpu().numpy(), 4, d).astype(np.uint8),
                          r.perm_gate_up.cpu().numpy(), 4, 128)
        print(f"block {b} gate/up:", c)
        assert c.ok(), c
        # h from the stored gate and up
        What = O.dequantize(q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.zeros.cpu().numpy(),
                            q.g_idx.cpu().numpy(), 4, d)
        Wg_hat, Wu_hat = _as_bf16(What[:d_ff]), _as_bf16(What[d_ff:])
        x64 = O.bf16_bits_to_f64(xb)
        g64, u64 = Wg_hat @ x64, Wu_hat @ x64
        h_ref = O.mlp_hidden(xb, Wg_hat, Wu_hat)
        Eg = _linear_bound(d, np.abs(Wg_hat) @ np.abs(x64))
        Eu = _linear_bound(d, np.abs(Wu_hat) @ np.abs(x64))
        s = O.silu(g64)
        # silu' is within [-0.1, 1.1]; fp32 silu a few ulps; one bf16 rounding
        tol = np.abs(s) * Eu + 1.1 * Eg * (np.abs(u64) + Eu) + 2.0 ** -20 * np.abs(h_ref) + 2.0 ** -8 * np.abs(h_ref)
        h_gpu = O.bf16_bits_to_f64(_bits(r.h))
        assert np.all(np.abs(h_gpu - h_ref) <= tol + 1e-30), float(np.max(np.abs(h_gpu - h_ref) / (tol + 1e-30)))
        # down on the GPU's h
        hb = _bits(r.h)
        Hh = O.hessian(hb)
        ora_d = O.gptq_layer(Wd, None, 4, 128, True, True, H=Hh)
        qd = r.down
        cd = compare_layer(Wd, Hh, ora_d, qd.qweight.cpu().numpy(), qd.scales.cpu().numpy(), qd.zeros.cpu().numpy(),
                           qd.g_idx.cpu().numpy(), O.unpack(qd.qweight.cpu().numpy(), 4, d_ff).astype(np.uint8),
                           r.perm_down.cpu().numpy(), 4, 128)
        print(f"block {b} down:", cd)
        assert cd.ok(), cd
        # the block's output from the stored down
        Wd_hat = _as_bf16(O.dequantize(qd.qweight.cpu().numpy(), qd.scales.cpu().numpy(), qd.zeros.cpu().numpy(),
                                       qd.g_idx.cpu().numpy(), 4, d_ff))
        x_ref = O.mlp_residual(xb, Wd_hat, h_gpu)
        tol = _linear_bound(d_ff, np.abs(Wd_hat) @ np.abs(h_gpu)) + 2.0 ** -8 * np.abs(x_ref)
        x_gpu = O.bf16_bits_to_f64(_bits(xs[b + 1]))
        assert np.all(np.abs(x_gpu - x_ref) <= tol + 1e-30)
    for r in res:
        assert r.ms["block"] > 0
