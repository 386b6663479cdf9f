"""gptq_quantize_layer_noalloc against gptq_quantize_layer, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device memory
(a plugin whose host owns all device allocations, code that may run during a
stream capture): it takes its scratch from a static device array in the library
instead of a caller workspace.  Its results must be bit-identical to the
workspace entry point's (both run the same deterministic kernels), on consecutive
calls that reuse the shared array.  This file is collected last so that a
failure here stops a `-x` run only after every other test has run.
"""
import numpy as np
import pytest

import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _setup(out, n, tokens, seed, bits, gs, sym, act):
    import post_weight_quantization_15_b200 as G
    dev = torch.device("cuda:0")
    W_np, x = S.small_case(out, n, tokens, seed=seed)
    W = torch.from_numpy(W_np).to(dev)
    X = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    st = G.new_status(dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hd = torch.zeros(n, dtype=torch.float64, device=dev)
    G.hessian_accumulate(H, X, hd, st)
    prep = G.prepare(H, 0.01, act, hd, st)
    return G, W, prep


def _assert_identical(a, b):
    """Both entry points run the same deterministic kernels: every output is bit-identical."""
    for name in ("codes", "scales", "zeros", "qweight", "g_idx", "err_sq"):
        x, y = getattr(a, name).cpu().numpy(), getattr(b, name).cpu().numpy()
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), name


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # the largest layer first, so that every later call runs over the leftover contents of a
    # larger (and different) layer in the shared array
    cases = [(256, 1536, 3072, 3, 4, 64, False, True),     # three super-blocks: both library streams
             (256, 512, 2048, 1, 4, 128, False, False),
             (200, 384, 1024, 2, 3, 64, True, True)]
    for out, n, tokens, seed, bits, gs, sym, act in cases:
        G, W, prep = _setup(out, n, tokens, seed, bits, gs, sym, act)
        ref = G.quantize_layer(W, prep, bits, gs, sym, want_codes=True, want_err=True)
        torch.cuda.synchronize()
        for _ in range(2):   # two calls in a row on the shared static scratch
            res = G.alloc_quantized(out, n, bits, gs, sym, W.device, want_codes=True, want_err=True)
            G.quantize_layer_noalloc(W, prep, res)
            G.raise_on_status(prep.status, "noalloc")
            _assert_identical(res, ref)


def test_noalloc_rejects_layers_beyond_the_static_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_quantization_15_b200 as G
    dev = torch.device("cuda:0")
    out, n = 4096, 4096                                # needs ~84 MB of scratch
    assert G.quantize_workspace_size(out, n) > G.gptq.NOALLOC_SCRATCH_BYTES
    W = torch.zeros((out, n), dtype=torch.float16, device=dev)
    prep = G.Prepared(U=torch.eye(n, device=dev), perm=torch.arange(n, dtype=torch.int32, device=dev),
                      dead=torch.zeros(n, dtype=torch.uint8, device=dev), status=G.new_status(dev), desc_act=False)
    res = G.alloc_quantized(out, n, 4, 128, False, dev)
    with pytest.raises(G.GptqError) as e:
        G.quantize_layer_noalloc(W, prep, res)
    assert e.value.code == G.gptq.ERR_WORKSPACE
