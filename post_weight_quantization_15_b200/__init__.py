"""B200-native GPTQ layer solver: a C-ABI CUDA library (libgptq.so) and its binding."""
from .gptq import (  # noqa: F401
    GptqError, Prepared, QuantizedLayer, alloc_quantized, dequantize, linear_bf16, qmatvec, residual_add, silu_mul,
    transpose_bf16, gptq_quantize, hessian_accumulate, hessian_accumulate_host, kernel_launches, lib, library_path,
    new_status, pack, pack_zeros, padded_width, prepare, prepare_set_deferred_min_n, quantize_layer, quantize_layer_noalloc, quantize_layers, reorder_groups, quantize_workspace_size, raise_on_status, set_graph_replay, status_read, status_reset,
    status_string, trace_enable, trace_read, trace_read_timeline, workspace,
)

__version__ = "0.1.0"
