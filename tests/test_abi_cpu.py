"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol include/gptq.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "gptq.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"GPTQ_API\s+[\w\s\*]+?\b(gptq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    import post_weight_quantization_15_b200 as G
    return G.lib()


def test_header_declares_the_path():
    names = _declared()
    for required in ("gptq_hessian_accumulate", "gptq_prepare", "gptq_quantize_layer", "gptq_pack",
                     "gptq_prepare_workspace_size", "gptq_quantize_workspace_size", "gptq_status_read"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_prepare_deferred_threshold_round_trips(L):
    # host-side setting: a query (<= 0) changes nothing; a set returns the previous value
    import post_weight_quantization_15_b200 as G
    cur = G.prepare_set_deferred_min_n(0)
    assert cur == 8192
    assert G.prepare_set_deferred_min_n(1000) == cur
    assert G.prepare_set_deferred_min_n(-5) == 1000
    assert G.prepare_set_deferred_min_n(cur) == 1000
    assert G.prepare_set_deferred_min_n(0) == cur


def test_graph_replay_switch_round_trips(L):
    import post_weight_quantization_15_b200 as G
    cur = G.set_graph_replay(-1)
    assert cur == 1                          # on by default
    assert G.set_graph_replay(0) == 1
    assert G.set_graph_replay(-1) == 0
    assert G.set_graph_replay(cur) == 0
    assert G.set_graph_replay(-1) == cur


def test_version_and_status_strings(L):
    import post_weight_quantization_15_b200 as G
    assert L.gptq_version() == 1
    assert G.status_string(0) == "ok"
    assert "positive definite" in G.status_string(-3)


def test_workspace_sizes(L):
    import post_weight_quantization_15_b200 as G
    n = 4096
    assert L.gptq_prepare_workspace_size(n) >= 2 * n * n * 4
    assert G.quantize_workspace_size(1024, n) >= 1024 * n * 5
    assert L.gptq_prepare_workspace_size(0) == 0


def test_bad_arguments_rejected_without_a_gpu(L):
    P = ctypes.c_void_p
    fake = P(256)   # never dereferenced: every call below fails its argument checks first
    assert L.gptq_quantize_layer(None, 0, 8, 128, fake, None, None, 4, 128, 0, 128, fake, fake, fake, fake,
                                 None, None, fake, 1 << 30, fake, None) == -1
    assert L.gptq_quantize_layer(fake, 0, 8, 128, fake, None, None, 5, 128, 0, 128, fake, fake, fake, fake,
                                 None, None, fake, 1 << 30, fake, None) == -2
    assert L.gptq_quantize_layer(fake, 0, 8, 100, fake, None, None, 4, 32, 0, 128, fake, fake, fake, fake,
                                 None, None, fake, 1 << 30, fake, None) == -2
    assert L.gptq_quantize_layer(fake, 0, 8, 128, fake, None, None, 4, 128, 0, 64, fake, fake, fake, fake,
                                 None, None, fake, 1 << 30, fake, None) == -2
    assert L.gptq_quantize_layer(fake, 0, 8, 128, fake, None, None, 4, 128, 0, 128, fake, fake, fake, fake,
                                 None, None, fake, 16, fake, None) == -7
    assert L.gptq_prepare(fake, None, 0, ctypes.c_float(0.01), 0, fake, fake, fake, fake, 1 << 30, fake, None) == -1
    assert L.gptq_prepare(fake, None, 64, ctypes.c_float(0.01), 0, fake, fake, fake, fake, 16, fake, None) == -7
    assert L.gptq_hessian_accumulate(fake, None, 64, fake, 100, 100, None, None) == -1   # ld_x % 8 != 0
    assert L.gptq_hessian_accumulate(fake, None, 64, fake, 96, 0, None, None) == 0        # empty chunk
    assert L.gptq_pack(fake, 4, 33, 4, fake, None) == -2
    # the host-memory Hessian: ld_x < tokens, a staging area that holds less than two
    # 64-token chunks, an unaligned staging area, and the empty chunk
    assert L.gptq_hessian_accumulate_host(fake, None, 64, fake, 50, 100, fake, 1 << 20, None, None) == -1
    assert L.gptq_hessian_accumulate_host(fake, None, 64, fake, 100, 100, fake, 2 * 64 * 63 * 2, None, None) == -7
    assert L.gptq_hessian_accumulate_host(fake, None, 64, fake, 100, 100, P(258), 1 << 20, None, None) == -7
    assert L.gptq_hessian_accumulate_host(fake, None, 64, fake, 100, 0, fake, 0, None, None) == 0


def test_padded_calls_and_zero_packing_reject_bad_arguments_without_a_gpu(L):
    P = ctypes.c_void_p
    fake = P(256)
    # Hessian of X zero-padded to n rows: x_rows must lie in 1..n; the empty chunk is a no-op
    assert L.gptq_hessian_accumulate_padded(fake, None, 64, fake, 65, 96, 96, None, None) == -1
    assert L.gptq_hessian_accumulate_padded(fake, None, 64, fake, 0, 96, 96, None, None) == -1
    assert L.gptq_hessian_accumulate_padded(fake, None, 64, fake, 60, 100, 100, None, None) == -1   # ld_x % 8
    assert L.gptq_hessian_accumulate_padded(fake, None, 64, fake, 60, 96, 0, None, None) == 0
    # host form: the staging halves hold x_rows (not n) rows of at least 64 tokens
    assert L.gptq_hessian_accumulate_host_padded(fake, None, 64, fake, 65, 100, 100, fake, 1 << 20, None, None) == -1
    assert L.gptq_hessian_accumulate_host_padded(fake, None, 64, fake, 60, 100, 100, fake, 2 * 60 * 63 * 2,
                                                 None, None) == -7
    assert L.gptq_hessian_accumulate_host_padded(fake, None, 64, fake, 60, 100, 0, fake, 0, None, None) == 0
    # quantize: w_cols in 1..n, and the padded width obeys the packing and group rules
    args = (None, None, 4, 128, 0, 128, fake, fake, fake, fake, None, None, fake, 1 << 30, fake, None)
    assert L.gptq_quantize_layer_padded(fake, 0, 8, 129, 128, fake, *args) == -1
    assert L.gptq_quantize_layer_padded(fake, 0, 8, 0, 128, fake, *args) == -1
    assert L.gptq_quantize_layer_padded(fake, 0, 8, 90, 100, fake, *args) == -2
    # more output rows than the row kernels' grids hold
    assert L.gptq_quantize_layer_padded(fake, 0, 524281, 128, 128, fake, *args) == -2
    # zero points: offset 0 or 1, supported widths, out * bits % 32 == 0
    assert L.gptq_pack_zeros(None, 4, 8, 4, 0, fake, None, None) == -1
    assert L.gptq_pack_zeros(fake, 4, 8, 4, 2, fake, None, None) == -1
    assert L.gptq_pack_zeros(fake, 0, 8, 4, 0, fake, None, None) == -1
    assert L.gptq_pack_zeros(fake, 4, 8, 5, 0, fake, None, None) == -2
    assert L.gptq_pack_zeros(fake, 4, 12, 4, 0, fake, None, None) == -2


def test_padded_width():
    import post_weight_quantization_15_b200 as G
    assert G.padded_width(300, 128) == 384 and G.padded_width(300, 64) == 320 and G.padded_width(300, 32) == 320
    assert G.padded_width(300, -1) == 320 and G.padded_width(4096, 128) == 4096
    # the page's example of a width that 128 x 8 does not divide
    assert G.padded_width(29568 // 8, 128) == 3712


def test_noalloc_checks_arguments_before_the_scratch_size(L):
    """The no-alloc entry point reports argument errors exactly as gptq_quantize_layer does,
    even for a layer whose workspace would not fit its static scratch (4096 x 4096)."""
    P = ctypes.c_void_p
    fake = P(256)
    big = (4096, 4096)
    tail = (fake, fake, fake, fake, None, None, fake, None)
    assert L.gptq_quantize_layer_noalloc(None, 0, *big, fake, None, None, 4, 128, 0, 128, *tail) == -1
    assert L.gptq_quantize_layer_noalloc(fake, 0, *big, fake, None, None, 4, 128, 0, 64, *tail) == -2   # block
    assert L.gptq_quantize_layer_noalloc(fake, 0, *big, fake, None, None, 5, 128, 0, 128, *tail) == -2  # bits
    assert L.gptq_quantize_layer_noalloc(fake, 0, 524281, 128, fake, None, None, 4, 128, 0, 128, *tail) == -2
    assert L.gptq_quantize_layer_noalloc(fake, 7, *big, fake, None, None, 4, 128, 0, 128, *tail) == -1  # dtype
    # valid arguments: only now does the size decide
    assert L.gptq_quantize_layer_noalloc(fake, 0, *big, fake, None, None, 4, 128, 0, 128, *tail) == -7


def test_noalloc_binding_rejects_mismatched_buffers_without_launching():
    """Outputs sized for another layer or bit width, or a U of another size, raise
    ValueError in the binding before anything reaches the library."""
    import torch

    import post_weight_quantization_15_b200 as G
    o, n = 64, 256
    W = torch.zeros((o, n), dtype=torch.float16)

    def prep(m):
        return G.Prepared(U=torch.zeros((m, m)), perm=torch.zeros(m, dtype=torch.int32),
                          dead=torch.zeros(m, dtype=torch.uint8), status=torch.zeros(4, dtype=torch.int32),
                          desc_act=False)

    good = G.alloc_quantized(o, n, 4, 128, False, "cpu", want_codes=True, want_err=True)
    wrong_bits = G.alloc_quantized(o, n, 3, 128, False, "cpu")
    wrong_bits.bits = 4                                   # qweight sized for 3 bits
    cases = [(prep(n + 128), good, "prep.U"),             # a padded preparation
             (prep(n), G.alloc_quantized(o + 1, n, 4, 128, False, "cpu"), "qweight"),
             (prep(n), wrong_bits, "qweight"),
             (prep(n), G.alloc_quantized(o, n, 4, 64, False, "cpu"), "bits"),
             (prep(n), G.QuantizedLayer(good.qweight, good.scales, good.zeros, good.g_idx,
                                        torch.zeros((o, n + 1), dtype=torch.uint8), None, 4, 128, False), "codes")]
    cases[3][1].group_size = 128                          # scales / zeros sized for g64
    for p, out, what in cases:
        with pytest.raises(ValueError) as e:
            G.quantize_layer_noalloc(W, p, out)
        assert what in str(e.value) or "scales" in str(e.value), (what, str(e.value))
    # well-shaped host tensors still never reach the library
    with pytest.raises(ValueError, match="CUDA"):
        G.quantize_layer_noalloc(W, prep(n), good)


def test_stored_format_consumers_reject_bad_arguments_without_a_gpu(L):
    P = ctypes.c_void_p
    fake = P(256)
    # dequantize: 3-bit codes straddle words, unaligned qweight, a bad output dtype
    assert L.gptq_dequantize(fake, fake, fake, fake, 3, 128, 64, 1, 1, fake, None, None) == -2
    assert L.gptq_dequantize(P(260), fake, fake, fake, 4, 128, 64, 1, 1, fake, None, None) == -1
    assert L.gptq_dequantize(fake, fake, fake, fake, 4, 128, 64, 1, 9, fake, None, None) == -1
    assert L.gptq_dequantize(fake, fake, fake, fake, 4, 128, 64, 0, 1, fake, None, None) == -1
    # matvec: at most 16 rows, a workspace of the reported size, ld_x >= n
    need = L.gptq_qmatvec_workspace_size(4, 1024, 256)
    assert need >= 4 * 256 * 4             # at least one block's fp32 partials of Y
    assert L.gptq_qmatvec(fake, fake, fake, fake, None, 4, 1024, 256, 8, fake, 1, 17, 1024, fake, 256, fake, need,
                          None, None) == -2
    assert L.gptq_qmatvec(fake, fake, fake, fake, None, 4, 1024, 256, 8, fake, 1, 4, 1024, fake, 256, fake,
                          need - 1, None, None) == -7
    assert L.gptq_qmatvec(fake, fake, fake, fake, None, 4, 1024, 256, 8, fake, 1, 4, 1000, fake, 256, fake, need,
                          None, None) == -1
    # reordering: 3-bit, too many groups, a small workspace
    wsz = L.gptq_reorder_groups_workspace_size(8)
    assert L.gptq_reorder_groups(fake, fake, 3, 1024, 256, 8, fake, fake, fake, fake, wsz, fake, None) == -2
    assert L.gptq_reorder_groups(fake, fake, 4, 1024, 256, 2048, fake, fake, fake, fake, wsz, fake, None) == -1
    assert L.gptq_reorder_groups(fake, fake, 4, 1024, 256, 8, fake, fake, fake, fake, 0, fake, None) == -7
