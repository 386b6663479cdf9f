"""Python binding of libgptq.so (ctypes): argument marshalling only.

Every step of the path runs in the library's CUDA kernels.  PyTorch is used for
device memory (the output tensors and the workspaces handed to the library) and
for the current stream.  There is no fallback: if the library or a CUDA device is
missing, every call raises.

The calls mirror include/gptq.h:

    hessian_accumulate(H, X, hdiag=None)          H += 2 . X . X^T
    prepare(H, damp_percent, desc_act, hdiag)     -> Prepared(U, perm, dead)
    quantize_layer(W, prep, bits, group_size, sym, block=128)
                                                  -> QuantizedLayer(qweight, scales, zeros, g_idx, ...)
    pack(codes, bits)                             -> qweight
    pack_zeros(zeros, bits, zero_offset=0)        -> qzeros
    gptq_quantize(W, X, ..., pad=False)           the whole path for one layer

Zero padding: H may be wider than X has rows, and U wider than W has columns; the
calls then go to the *_padded entry points, which read the missing rows / columns
as zeros (padded_width gives the width to pad to).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptq.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_NOT_SPD = -3
ERR_NONFINITE = -4
ERR_CUDA = -5
ERR_TIMEOUT = -6
ERR_WORKSPACE = -7

F32, F16, BF16 = 0, 1, 2
_DTYPE_CODE = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}

_lib = None


class _TraceRow(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("work_unit", ctypes.c_char_p), ("launches", ctypes.c_uint64),
                ("ms", ctypes.c_double), ("work", ctypes.c_double)]


class _TraceEvent(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("stream", ctypes.c_uint64), ("start_ms", ctypes.c_double),
                ("end_ms", ctypes.c_double)]


class GptqError(RuntimeError):
    def __init__(self, code: int, where: str, info: Optional[int] = None):
        self.code = code
        self.info = info
        msg = f"{where}: {status_string(code)} ({code})"
        if info is not None:
            msg += f", info={info}"
        super().__init__(msg)


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libgptq.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libgptq.so is not built ({_LIB_PATH}); run "
                           "`python -m post_weight_quantization_15_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, I64, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    L.gptq_version.restype = I
    L.gptq_version.argtypes = []
    L.gptq_kernel_launches.restype = ctypes.c_uint64
    L.gptq_kernel_launches.argtypes = []
    L.gptq_status_string.restype = ctypes.c_char_p
    L.gptq_status_string.argtypes = [I]
    L.gptq_status_reset.restype = I
    L.gptq_status_reset.argtypes = [P, P]
    L.gptq_status_read.restype = I
    L.gptq_status_read.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    L.gptq_hessian_accumulate.restype = I
    L.gptq_hessian_accumulate.argtypes = [P, P, I, P, I64, I64, P, P]
    L.gptq_hessian_accumulate_host.restype = I
    L.gptq_hessian_accumulate_host.argtypes = [P, P, I, P, I64, I64, P, SZ, P, P]
    L.gptq_prepare_workspace_size.restype = SZ
    L.gptq_prepare_workspace_size.argtypes = [I]
    L.gptq_prepare.restype = I
    L.gptq_prepare.argtypes = [P, P, I, F, I, P, P, P, P, SZ, P, P]
    L.gptq_prepare_set_deferred_min_n.restype = I
    L.gptq_prepare_set_deferred_min_n.argtypes = [I]
    L.gptq_set_graph_replay.restype = I
    L.gptq_set_graph_replay.argtypes = [I]
    L.gptq_quantize_workspace_size.restype = SZ
    L.gptq_quantize_workspace_size.argtypes = [I, I, I]
    L.gptq_quantize_layer.restype = I
    L.gptq_quantize_layer.argtypes = [P, I, I, I, P, P, P, I, I, I, I, P, P, P, P, P, P, P, SZ, P, P]
    L.gptq_quantize_layers.restype = I
    L.gptq_quantize_layers.argtypes = [P, P, I, I, I, P, P, P, I, I, I, I, P, P, P, P, P, P, P, SZ, P, P]
    L.gptq_pack.restype = I
    L.gptq_pack.argtypes = [P, I, I, I, P, P]
    L.gptq_hessian_accumulate_padded.restype = I
    L.gptq_hessian_accumulate_padded.argtypes = [P, P, I, P, I, I64, I64, P, P]
    L.gptq_hessian_accumulate_host_padded.restype = I
    L.gptq_hessian_accumulate_host_padded.argtypes = [P, P, I, P, I, I64, I64, P, SZ, P, P]
    L.gptq_quantize_layer_padded.restype = I
    L.gptq_quantize_layer_padded.argtypes = [P, I, I, I, I, P, P, P, I, I, I, I, P, P, P, P, P, P, P, SZ, P, P]
    L.gptq_pack_zeros.restype = I
    L.gptq_pack_zeros.argtypes = [P, I, I, I, I, P, P, P]
    L.gptq_trace_enable.restype = I
    L.gptq_trace_enable.argtypes = [I]
    L.gptq_trace_read.restype = I
    L.gptq_trace_read.argtypes = [ctypes.POINTER(_TraceRow), I, ctypes.POINTER(ctypes.c_int)]
    L.gptq_trace_read_timeline.restype = I
    L.gptq_trace_read_timeline.argtypes = [ctypes.POINTER(_TraceEvent), I, ctypes.POINTER(ctypes.c_int)]
    L.gptq_dequantize.restype = I
    L.gptq_dequantize.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P]
    L.gptq_qmatvec_workspace_size.restype = SZ
    L.gptq_qmatvec_workspace_size.argtypes = [I, I, I]
    L.gptq_qmatvec.restype = I
    L.gptq_qmatvec.argtypes = [P, P, P, P, P, I, I, I, I, P, I, I, I64, P, I64, P, SZ, P, P]
    L.gptq_reorder_groups_workspace_size.restype = SZ
    L.gptq_reorder_groups_workspace_size.argtypes = [I]
    L.gptq_reorder_groups.restype = I
    L.gptq_reorder_groups.argtypes = [P, P, I, I, I, I, P, P, P, P, SZ, P, P]
    L.gptq_linear_bf16.restype = I
    L.gptq_linear_bf16.argtypes = [P, I, I64, P, I, I64, I, P, I64, P, P]
    L.gptq_transpose_bf16.restype = I
    L.gptq_transpose_bf16.argtypes = [P, I, I, I64, P, I64, P, P]
    L.gptq_silu_mul.restype = I
    L.gptq_silu_mul.argtypes = [P, P, I64, P, P, P]
    L.gptq_residual_add.restype = I
    L.gptq_residual_add.argtypes = [P, P, I64, P, P, P]
    L.gptq_probe_fp32_peak.restype = I
    L.gptq_probe_fp32_peak.argtypes = [P, I, I, P]
    L.gptq_quantize_layer_noalloc.restype = I
    L.gptq_quantize_layer_noalloc.argtypes = [P, I, I, I, P, P, P, I, I, I, I, P, P, P, P, P, P, P, P]
    _lib = L
    return L


def kernel_launches() -> int:
    """Kernels enqueued by the library since it was loaded (host-side counter)."""
    return int(lib().gptq_kernel_launches())


def trace_enable(on: bool = True):
    """Start (or stop) recording CUDA events around every kernel the library launches."""
    _check(lib().gptq_trace_enable(1 if on else 0), "gptq_trace_enable")


def trace_read(max_rows: int = 64) -> dict:
    """Synchronize the recorded events and return {kernel: {launches, ms, work, unit}}; clears the record."""
    rows = (_TraceRow * max_rows)()
    n = ctypes.c_int(0)
    _check(lib().gptq_trace_read(rows, max_rows, ctypes.byref(n)), "gptq_trace_read")
    return {rows[i].kernel.decode(): {"launches": int(rows[i].launches), "ms": float(rows[i].ms),
                                      "work": float(rows[i].work), "unit": rows[i].work_unit.decode()}
            for i in range(n.value)}


def trace_read_timeline(max_events: int = 1 << 16) -> list:
    """Synchronize the recorded events and return [(kernel, stream id, start ms, end ms)] per launch, in
    enqueue order, times from the earliest recorded start; clears the record."""
    ev = (_TraceEvent * max_events)()
    n = ctypes.c_int(0)
    _check(lib().gptq_trace_read_timeline(ev, max_events, ctypes.byref(n)), "gptq_trace_read_timeline")
    return [(ev[i].kernel.decode(), int(ev[i].stream), float(ev[i].start_ms), float(ev[i].end_ms))
            for i in range(n.value)]


def probe_fp32_peak(blocks: int, iters: int, out: torch.Tensor, stream=None) -> float:
    """Enqueue the FP32 FMA probe; returns the flops it performs (time it with events)."""
    _require_cuda(out)
    if out.dtype != torch.float32 or out.numel() < blocks * 256:
        raise ValueError("out must be fp32 with at least blocks * 256 elements")
    _check(lib().gptq_probe_fp32_peak(_ptr(out), int(blocks), int(iters), _stream(stream)), "gptq_probe_fp32_peak")
    return 2.0 * blocks * 256 * iters * 128


def status_string(code: int) -> str:
    try:
        return lib().gptq_status_string(int(code)).decode()
    except RuntimeError:
        return str(code)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != OK:
        raise GptqError(rc, where)


def _require_cuda(*ts: Optional[torch.Tensor]):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte-aligned device buffer of at least nbytes (torch allocations are)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# --------------------------------------------------------------------------- #
# status block
# --------------------------------------------------------------------------- #
def new_status(device) -> torch.Tensor:
    return torch.zeros(4, dtype=torch.int32, device=device)


def status_reset(st: torch.Tensor, stream=None):
    _check(lib().gptq_status_reset(_ptr(st), _stream(stream)), "gptq_status_reset")


def status_read(st: torch.Tensor, stream=None):
    info = ctypes.c_int32(0)
    rc = lib().gptq_status_read(_ptr(st), _stream(stream), ctypes.byref(info))
    return rc, info.value


def raise_on_status(st: torch.Tensor, where: str, stream=None):
    rc, info = status_read(st, stream)
    if rc != OK:
        raise GptqError(rc, where, info)


# --------------------------------------------------------------------------- #
# K1
# --------------------------------------------------------------------------- #
def padded_width(n: int, group_size: int) -> int:
    """The width a layer of n inputs is zero-padded to: the next multiple of
    max(32, group_size) (32 for group_size -1)."""
    m = 32 if group_size == -1 else max(32, int(group_size))
    return (int(n) + m - 1) // m * m


def _check_h(H: torch.Tensor, rows: int, hdiag: Optional[torch.Tensor]) -> int:
    n = H.shape[0] if H.dim() == 2 else -1
    if H.dtype != torch.float32 or H.dim() != 2 or H.shape[1] != n or n < rows or not H.is_contiguous():
        raise ValueError("H must be a contiguous fp32 [n, n] tensor with n >= the rows of X")
    if hdiag is not None and (hdiag.dtype != torch.float64 or hdiag.numel() != n):
        raise ValueError("hdiag must be fp64 [n]")
    return n


def hessian_accumulate(H: torch.Tensor, X: torch.Tensor, hdiag: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """H += 2 . X . X^T.  H fp32 [n, n]; X bf16 [rows, tokens] (row stride may exceed tokens).

    rows < n: X is zero-padded to n rows (gptq_hessian_accumulate_padded).
    """
    _require_cuda(H, X, hdiag, status)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a bf16 [n, tokens] tensor with contiguous rows")
    rows = X.shape[0]
    n = _check_h(H, rows, hdiag)
    if rows == n:
        rc = lib().gptq_hessian_accumulate(_ptr(H), _ptr(hdiag), n, _ptr(X), X.stride(0), X.shape[1],
                                           _ptr(status), _stream(stream))
    else:
        rc = lib().gptq_hessian_accumulate_padded(_ptr(H), _ptr(hdiag), n, _ptr(X), rows, X.stride(0), X.shape[1],
                                                  _ptr(status), _stream(stream))
    _check(rc, "gptq_hessian_accumulate")
    return H


def hessian_accumulate_host(H: torch.Tensor, X_host: torch.Tensor, hdiag: Optional[torch.Tensor] = None,
                            status: Optional[torch.Tensor] = None, staging: Optional[torch.Tensor] = None,
                            chunk_tokens: int = 8192, stream=None) -> torch.Tensor:
    """H += 2 . X . X^T with X in host memory (pinned for overlap), copied in token chunks.

    ``staging`` is a device byte buffer (allocated here if None: two halves of
    n x chunk_tokens bf16); the copies of chunk i + 1 overlap the product of chunk i.
    """
    _require_cuda(H, hdiag, status, staging)
    if X_host.device.type != "cpu" or X_host.dtype not in (torch.bfloat16, torch.int16, torch.uint16) \
            or X_host.dim() != 2 or X_host.stride(1) != 1:
        raise ValueError("X_host must be a host [n, tokens] bf16 tensor with contiguous rows")
    rows = X_host.shape[0]
    n = _check_h(H, rows, hdiag)
    if staging is None:
        chunk = max(64, min(int(chunk_tokens), (X_host.shape[1] + 63) // 64 * 64)) // 64 * 64
        staging = workspace(2 * rows * chunk * 2, H.device)
    _check(lib().gptq_hessian_accumulate_host_padded(_ptr(H), _ptr(hdiag), n, ctypes.c_void_p(X_host.data_ptr()),
                                                     rows, X_host.stride(0), X_host.shape[1], _ptr(staging),
                                                     staging.numel(), _ptr(status), _stream(stream)),
           "gptq_hessian_accumulate_host")
    return H


# --------------------------------------------------------------------------- #
# K2
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class Prepared:
    U: torch.Tensor       # fp32 [n, n] upper
    perm: torch.Tensor    # int32 [n]
    dead: torch.Tensor    # uint8 [n]
    status: torch.Tensor  # int32 [4]
    desc_act: bool        # False: perm is the identity


def _perm_arg(prep: "Prepared", fused_pack: bool = False):
    """The perm argument of the quantize calls: NULL (the identity) selects the packing fused
    into the sweep; allowed only when the order is the identity (desc_act False)."""
    return None if (fused_pack and not prep.desc_act) else prep.perm


def prepare(H: torch.Tensor, damp_percent: float = 0.01, desc_act: bool = False,
            hdiag: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
            ws: Optional[torch.Tensor] = None, out: Optional[Prepared] = None, stream=None) -> Prepared:
    _require_cuda(H, hdiag, status, ws)
    n = H.shape[0]
    if H.dtype != torch.float32 or tuple(H.shape) != (n, n) or not H.is_contiguous():
        raise ValueError("H must be a contiguous fp32 [n, n] tensor")
    dev = H.device
    if status is None:
        status = new_status(dev)
    need = lib().gptq_prepare_workspace_size(n)
    if ws is None or ws.numel() < need:
        ws = workspace(need, dev)
    if out is None:
        out = Prepared(U=torch.empty((n, n), dtype=torch.float32, device=dev),
                       perm=torch.empty(n, dtype=torch.int32, device=dev),
                       dead=torch.empty(n, dtype=torch.uint8, device=dev), status=status, desc_act=bool(desc_act))
    out.status = status
    _check(lib().gptq_prepare(_ptr(H), _ptr(hdiag), n, float(damp_percent), int(bool(desc_act)), _ptr(out.U),
                              _ptr(out.perm), _ptr(out.dead), _ptr(ws), ws.numel(), _ptr(status), _stream(stream)),
           "gptq_prepare")
    return out


def prepare_set_deferred_min_n(min_n: int) -> int:
    """gptq_prepare_set_deferred_min_n: prepare groups its bulk updates by 512-wide outer
    panels for n >= min_n (default 8192).  min_n <= 0 only queries.  Returns the previous value."""
    return int(lib().gptq_prepare_set_deferred_min_n(int(min_n)))


def set_graph_replay(on: int) -> int:
    """gptq_set_graph_replay: prepare and quantize replay a captured CUDA graph for repeated
    calls with the same arguments (on by default, per host thread); on < 0 only queries.
    Returns the previous value."""
    return int(lib().gptq_set_graph_replay(int(on)))


# --------------------------------------------------------------------------- #
# K0 / K3 / K4 / K5
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class QuantizedLayer:
    qweight: torch.Tensor          # int32 [n*bits/32, out]
    scales: torch.Tensor           # fp16 [G, out]
    zeros: torch.Tensor            # fp16 [G, out]
    g_idx: torch.Tensor            # int32 [n]
    codes: Optional[torch.Tensor]  # uint8 [out, n] (original order) if requested
    err_sq: Optional[torch.Tensor]  # fp32 [out] if requested
    bits: int
    group_size: int
    sym: bool


def quantize_workspace_size(out: int, n: int, block: int = 128) -> int:
    return int(lib().gptq_quantize_workspace_size(out, n, block))


def alloc_quantized(out: int, n: int, bits: int, group_size: int, sym: bool, device, want_codes=False,
                    want_err=False) -> QuantizedLayer:
    G = 1 if group_size == -1 else n // group_size
    return QuantizedLayer(
        qweight=torch.empty((n * bits // 32, out), dtype=torch.int32, device=device),
        scales=torch.empty((G, out), dtype=torch.float16, device=device),
        zeros=torch.empty((G, out), dtype=torch.float16, device=device),
        g_idx=torch.empty(n, dtype=torch.int32, device=device),
        codes=torch.empty((out, n), dtype=torch.uint8, device=device) if want_codes else None,
        err_sq=torch.empty(out, dtype=torch.float32, device=device) if want_err else None,
        bits=bits, group_size=group_size, sym=bool(sym))


def _check_shape(t: Optional[torch.Tensor], shape, dtype, what: str):
    if t is not None and (tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous()):
        raise ValueError(f"{what} must be a contiguous {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")


def _check_prepared(prep: Prepared, n: int):
    """U fp32 [n, n], perm int32 [n], dead uint8 [n], status int32 [4]."""
    _check_shape(prep.U, (n, n), torch.float32, "prep.U")
    _check_shape(prep.perm, (n,), torch.int32, "prep.perm")
    _check_shape(prep.dead, (n,), torch.uint8, "prep.dead")
    if prep.status is None:
        raise ValueError("prep.status must be a status block")
    _check_shape(prep.status, (4,), torch.int32, "prep.status")


def _check_quantized(out: QuantizedLayer, o: int, n: int):
    """Output buffers sized for an o x n layer at out.bits / out.group_size."""
    bits, gs = int(out.bits), int(out.group_size)
    if bits not in (2, 3, 4, 8) or gs not in (-1, 32, 64, 128) or (gs > 0 and n % gs) or (n * bits) % 32:
        raise ValueError(f"unsupported bits={bits} / group_size={gs} for n={n}")
    G = 1 if gs == -1 else n // gs
    _check_shape(out.qweight, (n * bits // 32, o), torch.int32, "qweight")
    _check_shape(out.scales, (G, o), torch.float16, "scales")
    _check_shape(out.zeros, (G, o), torch.float16, "zeros")
    _check_shape(out.g_idx, (n,), torch.int32, "g_idx")
    _check_shape(out.codes, (o, n), torch.uint8, "codes")
    _check_shape(out.err_sq, (o,), torch.float32, "err_sq")


def quantize_layer(W: torch.Tensor, prep: Prepared, bits: int = 4, group_size: int = 128, sym: bool = False,
                   block: int = 128, want_codes: bool = False, want_err: bool = False,
                   ws: Optional[torch.Tensor] = None, out: Optional[QuantizedLayer] = None,
                   stream=None, fused_pack: bool = False) -> QuantizedLayer:
    """Sweep, lazy trailing update and packing of W [out, in] given ``prep`` (n = U's size).

    fused_pack: without act-order, let the sweep write qweight itself instead of a separate
    packing launch (same bits; measured slower, so off by default).

    in == n is the ordinary call.  in < n quantizes W zero-padded to n columns (the
    outputs then describe the padded layer: qweight, g_idx and codes have n columns);
    ``prep`` must then come from the padded Hessian (see hessian_accumulate).
    """
    _require_cuda(W, ws)
    if W.dim() != 2 or not W.is_contiguous() or W.dtype not in _DTYPE_CODE:
        raise ValueError("W must be a contiguous fp32/fp16/bf16 [out, n] tensor")
    o, w_cols = W.shape
    n = prep.U.shape[0]
    if w_cols > n:
        raise ValueError("W has more columns than U")
    dev = W.device
    need = quantize_workspace_size(o, n, block)
    if ws is None or ws.numel() < need:
        ws = workspace(need, dev)
    if out is None:
        out = alloc_quantized(o, n, bits, group_size, sym, dev, want_codes, want_err)
    else:
        _check_quantized(out, o, n)
    # w_cols < n: W is zero-padded to n columns (gptq_quantize_layer_padded)
    _check(lib().gptq_quantize_layer_padded(_ptr(W), _DTYPE_CODE[W.dtype], o, w_cols, n, _ptr(prep.U),
                                            _ptr(_perm_arg(prep, fused_pack)), _ptr(prep.dead), int(bits), int(group_size),
                                            int(bool(sym)), int(block), _ptr(out.qweight), _ptr(out.scales),
                                            _ptr(out.zeros), _ptr(out.g_idx), _ptr(out.codes), _ptr(out.err_sq),
                                            _ptr(ws), ws.numel(), _ptr(prep.status), _stream(stream)),
           "gptq_quantize_layer")
    return out


MAX_LAYERS = 8


def quantize_layers(Ws, prep: Prepared, bits: int = 4, group_size: int = 128, sym: bool = False,
                    block: int = 128, want_codes: bool = False, want_err: bool = False,
                    ws: Optional[torch.Tensor] = None, out: Optional[QuantizedLayer] = None, stream=None,
                    fused_pack: bool = False):
    """Several layers that read the same input (share ``prep``), in one call (fused_pack: as
    in quantize_layer).

    Returns (stacked, views): ``stacked`` is the QuantizedLayer of the layers stacked
    along the outputs, ``views`` one QuantizedLayer per layer whose tensors are views of
    it (qweight / scales / zeros: column ranges, not contiguous; codes / err_sq: row
    ranges).  Bit-identical to one quantize_layer call per layer (err_sq up to the order
    of its per-row sum).
    """
    Ws = list(Ws)
    if not 1 <= len(Ws) <= MAX_LAYERS:
        raise ValueError(f"1 to {MAX_LAYERS} layers per call")
    n = prep.U.shape[0]
    dt = Ws[0].dtype
    for W in Ws:
        if W.dim() != 2 or not W.is_contiguous() or W.dtype != dt or dt not in _DTYPE_CODE or W.shape[1] != n:
            raise ValueError("every W must be a contiguous [out_i, n] tensor of one dtype (fp32/fp16/bf16)")
    _require_cuda(*Ws, ws)
    outs = [int(W.shape[0]) for W in Ws]
    o = sum(outs)
    dev = Ws[0].device
    need = quantize_workspace_size(o, n, block)
    if ws is None or ws.numel() < need:
        ws = workspace(need, dev)
    if out is None:
        out = alloc_quantized(o, n, bits, group_size, sym, dev, want_codes, want_err)
    else:
        _check_quantized(out, o, n)
    ptrs = (ctypes.c_void_p * len(Ws))(*[W.data_ptr() for W in Ws])
    rows = (ctypes.c_int * len(Ws))(*outs)
    _check(lib().gptq_quantize_layers(ptrs, rows, len(Ws), _DTYPE_CODE[dt], n, _ptr(prep.U), _ptr(_perm_arg(prep, fused_pack)),
                                      _ptr(prep.dead), int(bits), int(group_size), int(bool(sym)), int(block),
                                      _ptr(out.qweight), _ptr(out.scales), _ptr(out.zeros), _ptr(out.g_idx),
                                      _ptr(out.codes), _ptr(out.err_sq), _ptr(ws), ws.numel(), _ptr(prep.status),
                                      _stream(stream)), "gptq_quantize_layers")
    views, r0 = [], 0
    for k in outs:
        sl = slice(r0, r0 + k)
        views.append(QuantizedLayer(out.qweight[:, sl], out.scales[:, sl], out.zeros[:, sl], out.g_idx,
                                    None if out.codes is None else out.codes[sl],
                                    None if out.err_sq is None else out.err_sq[sl], out.bits, out.group_size,
                                    out.sym))
        r0 += k
    return out, views


def _stored(q: QuantizedLayer):
    n = q.g_idx.numel()
    out = q.qweight.shape[1]
    if q.qweight.shape[0] * 32 != n * q.bits or not q.qweight.is_contiguous() or not q.scales.is_contiguous() \
            or not q.zeros.is_contiguous() or q.scales.shape != q.zeros.shape or q.scales.shape[1] != out:
        raise ValueError("a contiguous stored layer (qweight [n*bits/32, out], scales / zeros [G, out]) is needed")
    _require_cuda(q.qweight, q.scales, q.zeros, q.g_idx)
    return n, out, q.scales.shape[0]


def dequantize(q: QuantizedLayer, dtype=torch.float16, status: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """What [out, n] = scales[g_idx] . (codes - zeros[g_idx]) from the stored format."""
    n, o, groups = _stored(q)
    if out is None:
        out = torch.empty((o, n), dtype=dtype, device=q.qweight.device)
    _check_shape(out, (o, n), dtype, "What")
    _check(lib().gptq_dequantize(_ptr(q.qweight), _ptr(q.scales), _ptr(q.zeros), _ptr(q.g_idx), int(q.bits), n, o,
                                 groups, _DTYPE_CODE[dtype], _ptr(out), _ptr(status), _stream(stream)),
           "gptq_dequantize")
    return out


def reorder_groups(q: QuantizedLayer, status: Optional[torch.Tensor] = None, stream=None):
    """Once per act-order layer: (layer with its columns sorted by group, xperm) for qmatvec."""
    n, o, groups = _stored(q)
    dev = q.qweight.device
    st = status if status is not None else new_status(dev)
    qg = torch.empty_like(q.qweight)
    gg = torch.empty_like(q.g_idx)
    xperm = torch.empty_like(q.g_idx)
    ws = workspace(int(lib().gptq_reorder_groups_workspace_size(groups)), dev)
    _check(lib().gptq_reorder_groups(_ptr(q.qweight), _ptr(q.g_idx), int(q.bits), n, o, groups, _ptr(qg), _ptr(gg),
                                     _ptr(xperm), _ptr(ws), ws.numel(), _ptr(st), _stream(stream)),
           "gptq_reorder_groups")
    return QuantizedLayer(qg, q.scales, q.zeros, gg, None, None, q.bits, q.group_size, q.sym), xperm


def qmatvec(q: QuantizedLayer, X: torch.Tensor, status: Optional[torch.Tensor] = None,
            ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
            xperm: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y [M, out] (fp32) = X [M, n] . What^T for M <= 16, the weights dequantized in registers.

    xperm: for a layer from reorder_groups, its column permutation."""
    n, o, groups = _stored(q)
    _require_cuda(X, ws, out, xperm)
    if xperm is not None and (xperm.dtype != torch.int32 or xperm.numel() != n):
        raise ValueError("xperm must be int32 [n]")
    if X.dim() != 2 or X.shape[1] != n or X.stride(1) != 1 or X.dtype not in _DTYPE_CODE:
        raise ValueError("X must be an fp16/bf16/fp32 [M, n] tensor with contiguous rows")
    M = X.shape[0]
    need = int(lib().gptq_qmatvec_workspace_size(M, n, o))
    if ws is None or ws.numel() < need:
        ws = workspace(need, X.device)
    if out is None:
        out = torch.empty((M, o), dtype=torch.float32, device=X.device)
    if out.dtype != torch.float32 or out.dim() != 2 or out.shape[0] != M or out.shape[1] != o or out.stride(1) != 1:
        raise ValueError("out must be an fp32 [M, out] tensor with contiguous rows")
    _check(lib().gptq_qmatvec(_ptr(q.qweight), _ptr(q.scales), _ptr(q.zeros), _ptr(q.g_idx), _ptr(xperm),
                              int(q.bits), n, o,
                              groups, _ptr(X), _DTYPE_CODE[X.dtype], M, X.stride(0), _ptr(out), out.stride(0),
                              _ptr(ws), ws.numel(), _ptr(status), _stream(stream)), "gptq_qmatvec")
    return out


# --------------------------------------------------------------------------- #
# A quantized block's forward pass (the sequential pipeline)
# --------------------------------------------------------------------------- #
def linear_bf16(A: torch.Tensor, B: torch.Tensor, status: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """C [M, N] fp32 = A [M, K] . B [N, K]^T, bf16 operands with contiguous rows."""
    _require_cuda(A, B, status, out)
    for t in (A, B):
        if t.dtype != torch.bfloat16 or t.dim() != 2 or t.stride(1) != 1:
            raise ValueError("A and B must be bf16 2-D tensors with contiguous rows")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B must share K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    if out.dtype != torch.float32 or tuple(out.shape) != (M, N) or out.stride(1) != 1:
        raise ValueError("out must be fp32 [M, N] with contiguous rows")
    _check(lib().gptq_linear_bf16(_ptr(A), M, A.stride(0), _ptr(B), N, B.stride(0), K, _ptr(out), out.stride(0),
                                  _ptr(status), _stream(stream)), "gptq_linear_bf16")
    return out


def transpose_bf16(X: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _require_cuda(X, status)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a bf16 2-D tensor with contiguous rows")
    r, c = X.shape
    Xt = torch.empty((c, r), dtype=torch.bfloat16, device=X.device)
    _check(lib().gptq_transpose_bf16(_ptr(X), r, c, X.stride(0), _ptr(Xt), r, _ptr(status), _stream(stream)),
           "gptq_transpose_bf16")
    return Xt


def silu_mul(G: torch.Tensor, U: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16(silu(G) . U) for contiguous fp32 G, U of one shape."""
    _require_cuda(G, U, status)
    if G.dtype != torch.float32 or U.dtype != torch.float32 or G.shape != U.shape or not G.is_contiguous() \
            or not U.is_contiguous():
        raise ValueError("G and U must be contiguous fp32 tensors of one shape")
    h = torch.empty(G.shape, dtype=torch.bfloat16, device=G.device)
    _check(lib().gptq_silu_mul(_ptr(G), _ptr(U), G.numel(), _ptr(h), _ptr(status), _stream(stream)), "gptq_silu_mul")
    return h


def residual_add(X: torch.Tensor, Y: torch.Tensor, status: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """bf16(X + Y) for contiguous X bf16 and Y fp32 of one shape."""
    _require_cuda(X, Y, status)
    if X.dtype != torch.bfloat16 or Y.dtype != torch.float32 or X.shape != Y.shape or not X.is_contiguous() \
            or not Y.is_contiguous():
        raise ValueError("X (bf16) and Y (fp32) must be contiguous tensors of one shape")
    Xn = torch.empty(X.shape, dtype=torch.bfloat16, device=X.device)
    _check(lib().gptq_residual_add(_ptr(X), _ptr(Y), X.numel(), _ptr(Xn), _ptr(status), _stream(stream)),
           "gptq_residual_add")
    return Xn


def pack(codes: torch.Tensor, bits: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _require_cuda(codes, out)
    if codes.dtype != torch.uint8 or codes.dim() != 2 or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous uint8 [out, n] tensor")
    o, n = codes.shape
    if out is None:
        out = torch.empty((n * bits // 32, o), dtype=torch.int32, device=codes.device)
    _check(lib().gptq_pack(_ptr(codes), o, n, int(bits), _ptr(out), _stream(stream)), "gptq_pack")
    return out


def pack_zeros(zeros: torch.Tensor, bits: int, zero_offset: int = 0, status: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fp16 zero points [G, out] -> qzeros int32 [G, out*bits/32], packed along the outputs.

    zero_offset 1 stores zero - 1 (the convention of older checkpoints).
    """
    _require_cuda(zeros, status, out)
    if zeros.dtype != torch.float16 or zeros.dim() != 2 or not zeros.is_contiguous():
        raise ValueError("zeros must be a contiguous fp16 [G, out] tensor")
    g, o = zeros.shape
    if out is None:
        out = torch.empty((g, o * bits // 32), dtype=torch.int32, device=zeros.device)
    _check(lib().gptq_pack_zeros(_ptr(zeros), g, o, int(bits), int(zero_offset), _ptr(out), _ptr(status),
                                 _stream(stream)), "gptq_pack_zeros")
    return out


# --------------------------------------------------------------------------- #
# The whole path for one layer
# --------------------------------------------------------------------------- #
def gptq_quantize(W: torch.Tensor, X: torch.Tensor, bits: int = 4, group_size: int = 128, sym: bool = False,
                  desc_act: bool = False, damp_percent: float = 0.01, block: int = 128,
                  want_codes: bool = False, want_err: bool = False, check: bool = True, pad: bool = False):
    """H = 2.X.X^T, prepare, quantize.  Returns (QuantizedLayer, Prepared, H).

    W and X on the device, or both in host memory (pinned for overlap): then X crosses
    to the device in token chunks while the Hessian of the previous chunk is formed.
    pad: quantize the layer zero-padded to padded_width(in, group_size) inputs (the
    outputs then describe the padded layer).
    Every call allocates its buffers, so its calls run without graph replay (see
    set_graph_replay); loops that reuse buffers call prepare / quantize_layer themselves.
    """
    n = padded_width(X.shape[0], group_size) if pad else X.shape[0]
    host = X.device.type == "cpu"
    dev = torch.device("cuda", torch.cuda.current_device()) if host else X.device
    st = new_status(dev)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hdiag = torch.zeros(n, dtype=torch.float64, device=dev) if desc_act else None
    if host:
        W = W.to(dev, non_blocking=True)
        hessian_accumulate_host(H, X, hdiag, st)
    else:
        hessian_accumulate(H, X, hdiag, st)
    replay = set_graph_replay(0)
    try:
        prep = prepare(H, damp_percent, desc_act, hdiag, st)
        q = quantize_layer(W, prep, bits, group_size, sym, block, want_codes, want_err)
    finally:
        set_graph_replay(replay)
    if check:
        raise_on_status(st, "gptq_quantize")
    return q, prep, H


# --------------------------------------------------------------------------- #
# Static-scratch variant (no workspace)
# --------------------------------------------------------------------------- #
NOALLOC_SCRATCH_BYTES = 32 << 20


def quantize_layer_noalloc(W: torch.Tensor, prep: Prepared, out: QuantizedLayer, block: int = 128,
                           stream=None) -> QuantizedLayer:
    """quantize_layer for callers that cannot allocate device memory.

    The library takes its scratch from a static 32 MiB device array instead of a
    workspace, so this call allocates nothing; the caller passes preallocated
    outputs (see alloc_quantized).  Layers whose workspace would exceed the array
    raise GptqError(ERR_WORKSPACE).  Calls that overlap on the GPU race on the
    shared array.
    """
    if W.dim() != 2 or not W.is_contiguous() or W.dtype not in _DTYPE_CODE:
        raise ValueError("W must be a contiguous fp32/fp16/bf16 [out, n] tensor")
    o, n = W.shape
    _check_prepared(prep, n)
    _check_quantized(out, o, n)
    _require_cuda(W, prep.U, prep.perm, prep.dead, prep.status, out.qweight, out.scales, out.zeros, out.g_idx,
                  out.codes, out.err_sq)
    _check(lib().gptq_quantize_layer_noalloc(_ptr(W), _DTYPE_CODE[W.dtype], o, n, _ptr(prep.U), _ptr(prep.perm),
                                             _ptr(prep.dead), int(out.bits), int(out.group_size), int(out.sym),
                                             int(block), _ptr(out.qweight), _ptr(out.scales), _ptr(out.zeros),
                                             _ptr(out.g_idx), _ptr(out.codes), _ptr(out.err_sq), _ptr(prep.status),
                                             _stream(stream)), "gptq_quantize_layer_noalloc")
    return out
