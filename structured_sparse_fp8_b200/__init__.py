"""B200-native 2:4 structured-sparse FP8 GEMM.

Thin Python binding over the C ABI in ``include/sp24.h``: every function
below only allocates output tensors with torch (device memory plumbing),
marshals pointers and the current CUDA stream, and calls into
``libsp24.so``.  All arithmetic runs in the library's sm_100a kernels.

Entry points (same names as the C ABI):
    sp24_prune_compress, fp8_quantize_pertensor, slide68_decompose,
    slide68_lift, sp24_gemm, fp8_gemm_dense, sp24_pack_weights,
    sp24_prune_compress_packed, slide68_decompose_packed, sp24_gemm_packed,
    sp24_quantize_gemm_packed, slide68_lift_gemm_packed, fp8_quantize_pertoken,
    sp24_prune_compress_perchannel, sp24_gemm_packed_scaled, slide_decompose, slide_lift,
    int8_quantize_pertensor, sp24_prune_compress_int8, sp24_gemm_int8_packed
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import DTYPE_BF16, DTYPE_E4M3, Sp24Error  # noqa: F401

__all__ = [
    "sp24_prune_compress", "fp8_quantize_pertensor", "slide68_decompose", "slide68_lift",
    "sp24_gemm", "fp8_gemm_dense", "sp24_pack_weights", "sp24_prune_compress_packed", "slide68_decompose_packed",
    "sp24_gemm_packed", "sp24_quantize_gemm_packed", "slide68_lift_gemm_packed",
    "fp8_quantize_pertoken", "sp24_prune_compress_perchannel", "sp24_gemm_packed_scaled",
    "slide_decompose", "slide_lift", "int8_quantize_pertensor", "sp24_prune_compress_int8",
    "sp24_gemm_int8_packed",
    "Workspace",
    "Sp24Error", "DTYPE_E4M3", "DTYPE_BF16",
]

_DT = {"e4m3": DTYPE_E4M3, "bf16": DTYPE_BF16, DTYPE_E4M3: DTYPE_E4M3, DTYPE_BF16: DTYPE_BF16}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise Sp24Error("tensors must be contiguous CUDA tensors")


class Workspace:
    """Zero-filled device scratch shared by calls on one stream.

    Every library call leaves its workspace zero-filled, so a buffer can be
    reused by calls that do not run concurrently (one Workspace per stream).
    """

    _by_key: dict = {}

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf = torch.zeros(4096, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int):
        if nbytes > self.buf.numel():
            self.buf = torch.zeros(max(nbytes, 2 * self.buf.numel()), dtype=torch.uint8,
                                   device=self.device)
        return self.buf

    @classmethod
    def for_current_stream(cls, device) -> "Workspace":
        device = torch.device(device)
        key = (device.index, _stream(device))
        ws = cls._by_key.get(key)
        if ws is None:
            ws = cls._by_key[key] = cls(device)
        return ws


def _ws(device, op, m, n, k, dtype=DTYPE_E4M3, workspace=None):
    lib = _lib.load()
    need = lib.sp24_workspace_size(op, m, n, k, dtype)
    ws = workspace or Workspace.for_current_stream(device)
    buf = ws.get(max(need, 256))
    return buf, buf.numel()


def sp24_prune_compress(W: torch.Tensor, out_dtype="e4m3", pruned_dense: bool = False,
                        status: torch.Tensor | None = None, workspace: Workspace | None = None,
                        out: dict | None = None):
    """2:4 magnitude prune + (E4M3 quantise) + compress of W bf16 [N, K].

    Returns dict(values, meta, scale, pruned_dense); ``out`` may supply any
    of these tensors preallocated.
    """
    lib = _lib.load()
    _require_cuda(W, status)
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    dt = _DT[out_dtype]
    N, K = W.shape
    out = out or {}
    vdt = torch.uint8 if dt == DTYPE_E4M3 else torch.bfloat16
    values = out.get("values")
    if values is None:
        values = torch.empty((N, K // 2), dtype=vdt, device=W.device)
    meta = out.get("meta")
    if meta is None:
        meta = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    scale = out.get("scale")
    if scale is None and dt == DTYPE_E4M3:
        scale = torch.empty((1,), dtype=torch.float32, device=W.device)
    dense = out.get("pruned_dense")
    if dense is None and pruned_dense:
        dense = torch.empty((N, K), dtype=vdt, device=W.device)
    _require_cuda(values, meta, scale, dense)
    if values.shape != (N, K // 2) or values.dtype != vdt or meta.shape != (N, K // 8):
        raise Sp24Error("output tensors have the wrong shape or dtype")
    ws, wsn = _ws(W.device, _lib.OP_PRUNE_COMPRESS, 0, N, K, dt, workspace)
    rc = lib.sp24_prune_compress(_ptr(W), N, K, dt, _ptr(values), _ptr(meta), _ptr(scale),
                                 _ptr(dense), _ptr(ws), wsn, _ptr(status), _stream(W.device))
    _lib.check(rc, "sp24_prune_compress")
    return dict(values=values, meta=meta, scale=scale, pruned_dense=dense)


def fp8_quantize_pertensor(X: torch.Tensor, status: torch.Tensor | None = None,
                           out: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                           workspace: Workspace | None = None):
    """Per-tensor E4M3 quantisation of X bf16 [rows, cols] -> (codes u8, scale f32[1])."""
    lib = _lib.load()
    _require_cuda(X, status, out, scale)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    rows, cols = X.shape
    q = out if out is not None else torch.empty((rows, cols), dtype=torch.uint8, device=X.device)
    s = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=X.device)
    ws, wsn = _ws(X.device, _lib.OP_QUANTIZE, rows, 0, cols, DTYPE_E4M3, workspace)
    rc = lib.fp8_quantize_pertensor(_ptr(X), rows, cols, _ptr(q), _ptr(s), _ptr(ws), wsn,
                                    _ptr(status), _stream(X.device))
    _lib.check(rc, "fp8_quantize_pertensor")
    return q, s


def int8_quantize_pertensor(X: torch.Tensor, status: torch.Tensor | None = None,
                            out: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                            workspace: Workspace | None = None):
    """Symmetric per-tensor INT8 quantisation of X bf16 [rows, cols] -> (codes int8, scale f32[1])."""
    lib = _lib.load()
    _require_cuda(X, status, out, scale)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    rows, cols = X.shape
    q = out if out is not None else torch.empty((rows, cols), dtype=torch.int8, device=X.device)
    s = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=X.device)
    ws, wsn = _ws(X.device, _lib.OP_QUANTIZE, rows, 0, cols, DTYPE_E4M3, workspace)
    rc = lib.int8_quantize_pertensor(_ptr(X), rows, cols, _ptr(q), _ptr(s), _ptr(ws), wsn,
                                     _ptr(status), _stream(X.device))
    _lib.check(rc, "int8_quantize_pertensor")
    return q, s


def sp24_prune_compress_int8(W: torch.Tensor, status: torch.Tensor | None = None,
                             workspace: Workspace | None = None, out: dict | None = None):
    """2:4 magnitude prune + symmetric per-tensor INT8 quantise + compress of
    W bf16 [N, K]: returns dict(values int8 [N, K/2], meta u8 [N, K/8], scale);
    ``out`` may supply any of these preallocated."""
    lib = _lib.load()
    out = out or {}
    _require_cuda(W, status, *out.values())
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    N, K = W.shape
    values = out.get("values")
    values = values if values is not None else torch.empty((N, K // 2), dtype=torch.int8, device=W.device)
    meta = out.get("meta")
    meta = meta if meta is not None else torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    scale = out.get("scale")
    scale = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=W.device)
    ws, wsn = _ws(W.device, _lib.OP_PRUNE_COMPRESS, 0, N, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_prune_compress_int8(_ptr(W), N, K, _ptr(values), _ptr(meta), _ptr(scale), _ptr(ws), wsn,
                                      _ptr(status), _stream(W.device))
    _lib.check(rc, "sp24_prune_compress_int8")
    return dict(values=values, meta=meta, scale=scale)


def slide68_decompose(W: torch.Tensor, out_dtype="e4m3", status: torch.Tensor | None = None,
                      workspace: Workspace | None = None, out: dict | None = None):
    """6:8 prune + sliding-window decomposition of W bf16 [N, K] into 2:4 over K' = 1.5 K."""
    lib = _lib.load()
    _require_cuda(W, status)
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    dt = _DT[out_dtype]
    N, K = W.shape
    out = out or {}
    vdt = torch.uint8 if dt == DTYPE_E4M3 else torch.bfloat16
    values = out.get("values")
    if values is None:
        values = torch.empty((N, 3 * K // 4), dtype=vdt, device=W.device)
    meta = out.get("meta")
    if meta is None:
        meta = torch.empty((N, 3 * K // 16), dtype=torch.uint8, device=W.device)
    scale = out.get("scale")
    if scale is None and dt == DTYPE_E4M3:
        scale = torch.empty((1,), dtype=torch.float32, device=W.device)
    _require_cuda(values, meta, scale)
    if values.shape != (N, 3 * K // 4) or values.dtype != vdt or meta.shape != (N, 3 * K // 16):
        raise Sp24Error("output tensors have the wrong shape or dtype")
    ws, wsn = _ws(W.device, _lib.OP_SLIDE68_DECOMPOSE, 0, N, K, dt, workspace)
    rc = lib.slide68_decompose(_ptr(W), N, K, dt, _ptr(values), _ptr(meta), _ptr(scale), _ptr(ws),
                               wsn, _ptr(status), _stream(W.device))
    _lib.check(rc, "slide68_decompose")
    return dict(values=values, meta=meta, scale=scale)


def slide68_lift(X: torch.Tensor, status: torch.Tensor | None = None,
                 out: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                 workspace: Workspace | None = None):
    """Quantise X bf16 [M, K] to E4M3 and lift it to [M, 1.5 K] -> (codes, scale)."""
    lib = _lib.load()
    _require_cuda(X, status, out, scale)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    M, K = X.shape
    q = out if out is not None else torch.empty((M, 3 * K // 2), dtype=torch.uint8, device=X.device)
    s = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=X.device)
    ws, wsn = _ws(X.device, _lib.OP_SLIDE68_LIFT, M, 0, K, DTYPE_E4M3, workspace)
    rc = lib.slide68_lift(_ptr(X), M, K, _ptr(q), _ptr(s), _ptr(ws), wsn, _ptr(status),
                          _stream(X.device))
    _lib.check(rc, "slide68_lift")
    return q, s


def sp24_gemm(xq: torch.Tensor, x_scale, values: torch.Tensor, meta: torch.Tensor, w_scale,
              dtype="e4m3", out: torch.Tensor | None = None, status: torch.Tensor | None = None,
              workspace: Workspace | None = None):
    """Sparse GEMM Y[M, N] = bf16(sx * sw * Xq . W^T) with W 2:4-compressed."""
    lib = _lib.load()
    _require_cuda(xq, x_scale, values, meta, w_scale, out, status)
    dt = _DT[dtype]
    M, K = xq.shape
    N = values.shape[0]
    if values.shape[1] * 2 != K or meta.shape != (N, K // 8):
        raise Sp24Error("operand shapes disagree")
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    ws, wsn = _ws(xq.device, _lib.OP_GEMM, M, N, K, dt, workspace)
    rc = lib.sp24_gemm(_ptr(xq), _ptr(x_scale), _ptr(values), _ptr(meta), _ptr(w_scale), _ptr(y),
                       M, N, K, dt, _ptr(ws), wsn, _ptr(status), _stream(xq.device))
    _lib.check(rc, "sp24_gemm")
    return y


def sp24_pack_weights(values: torch.Tensor, meta: torch.Tensor, out: torch.Tensor | None = None):
    """Tile-packed copy of 2:4 E4M3 weights (values u8 [N, K/2], meta u8 [N, K/8])."""
    lib = _lib.load()
    _require_cuda(values, meta, out)
    N, K = values.shape[0], values.shape[1] * 2
    if meta.shape != (N, K // 8) or values.dtype != torch.uint8:
        raise Sp24Error("values/meta shapes disagree")
    packed = out if out is not None else torch.empty(N * K // 2 + N * K // 8, dtype=torch.uint8,
                                                     device=values.device)
    rc = lib.sp24_pack_weights(_ptr(values), _ptr(meta), N, K, _ptr(packed), _stream(values.device))
    _lib.check(rc, "sp24_pack_weights")
    return packed


def sp24_prune_compress_packed(W: torch.Tensor, status: torch.Tensor | None = None,
                               workspace: Workspace | None = None, out: torch.Tensor | None = None,
                               scale: torch.Tensor | None = None):
    """E4M3 2:4 prune + quantise of W bf16 [N, K] straight into the tile-packed
    layout (what sp24_pack_weights makes of sp24_prune_compress's output).

    Returns (packed u8 [N*K/2 + N*K/8], scale f32 [1]).
    """
    lib = _lib.load()
    _require_cuda(W, status, out, scale)
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    N, K = W.shape
    packed = out if out is not None else torch.empty(N * K // 2 + N * K // 8, dtype=torch.uint8,
                                                     device=W.device)
    if packed.numel() != N * K // 2 + N * K // 8 or packed.dtype != torch.uint8:
        raise Sp24Error("packed output has the wrong size or dtype")
    sc = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=W.device)
    ws, wsn = _ws(W.device, _lib.OP_PRUNE_COMPRESS, 0, N, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_prune_compress_packed(_ptr(W), N, K, _ptr(packed), _ptr(sc), _ptr(ws), wsn,
                                        _ptr(status), _stream(W.device))
    _lib.check(rc, "sp24_prune_compress_packed")
    return packed, sc


def slide68_decompose_packed(W: torch.Tensor, status: torch.Tensor | None = None,
                             workspace: Workspace | None = None, out: torch.Tensor | None = None,
                             scale: torch.Tensor | None = None):
    """E4M3 6:8 decomposition of W bf16 [N, K] straight into the tile-packed
    layout of the lifted 2:4 operand (K' = 3K/2): what sp24_pack_weights
    makes of slide68_decompose's output.

    Returns (packed u8 [N*K'/2 + N*K'/8], scale f32 [1]).
    """
    lib = _lib.load()
    _require_cuda(W, status, out, scale)
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    N, K = W.shape
    kl = 3 * K // 2
    packed = out if out is not None else torch.empty(N * kl // 2 + N * kl // 8, dtype=torch.uint8,
                                                     device=W.device)
    if packed.numel() != N * kl // 2 + N * kl // 8 or packed.dtype != torch.uint8:
        raise Sp24Error("packed output has the wrong size or dtype")
    sc = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=W.device)
    ws, wsn = _ws(W.device, _lib.OP_SLIDE68_DECOMPOSE, 0, N, K, DTYPE_E4M3, workspace)
    rc = lib.slide68_decompose_packed(_ptr(W), N, K, _ptr(packed), _ptr(sc), _ptr(ws), wsn,
                                      _ptr(status), _stream(W.device))
    _lib.check(rc, "slide68_decompose_packed")
    return packed, sc


def sp24_gemm_packed(xq: torch.Tensor, x_scale, packed: torch.Tensor, w_scale, n: int,
                     out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     workspace: Workspace | None = None):
    """Sparse E4M3 GEMM with tile-packed weights (see sp24_pack_weights)."""
    lib = _lib.load()
    _require_cuda(xq, x_scale, packed, w_scale, out, status)
    M, K = xq.shape
    if packed.numel() != n * K // 2 + n * K // 8:
        raise Sp24Error("packed weights do not match N x K")
    y = out if out is not None else torch.empty((M, n), dtype=torch.bfloat16, device=xq.device)
    ws, wsn = _ws(xq.device, _lib.OP_GEMM_PACKED, M, n, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_gemm_packed(_ptr(xq), _ptr(x_scale), _ptr(packed), _ptr(w_scale), _ptr(y), M, n, K,
                              _ptr(ws), wsn, _ptr(status), _stream(xq.device))
    _lib.check(rc, "sp24_gemm_packed")
    return y


def sp24_gemm_int8_packed(xq: torch.Tensor, x_scale, packed: torch.Tensor, w_scale, n: int,
                          out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                          workspace: Workspace | None = None):
    """INT8 W8A8 sparse GEMM: xq int8 [M, K], tile-packed INT8 2:4 weights
    (sp24_pack_weights of sp24_prune_compress_int8's values viewed as bytes,
    and its metadata) -> Y bf16 [M, n]."""
    lib = _lib.load()
    _require_cuda(xq, x_scale, packed, w_scale, out, status)
    if xq.dtype != torch.int8 or xq.dim() != 2:
        raise Sp24Error("xq must be a 2-D int8 tensor")
    M, K = xq.shape
    if packed.numel() != n * K // 2 + n * K // 8:
        raise Sp24Error("packed weights do not match N x K")
    y = out if out is not None else torch.empty((M, n), dtype=torch.bfloat16, device=xq.device)
    ws, wsn = _ws(xq.device, _lib.OP_GEMM_PACKED, M, n, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_gemm_int8_packed(_ptr(xq), _ptr(x_scale), _ptr(packed), _ptr(w_scale), _ptr(y), M, n, K,
                                   _ptr(ws), wsn, _ptr(status), _stream(xq.device))
    _lib.check(rc, "sp24_gemm_int8_packed")
    return y


def fp4_quantize_pertensor(X: torch.Tensor, status: torch.Tensor | None = None,
                           out: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                           workspace: Workspace | None = None):
    """Per-tensor FP4 (E2M1) quantisation of X bf16 [rows, cols] -> (codes u8
    [rows, cols / 2], two per byte, element 2i in the low nibble; scale f32[1])."""
    lib = _lib.load()
    _require_cuda(X, status, out, scale)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    rows, cols = X.shape
    q = out if out is not None else torch.empty((rows, cols // 2), dtype=torch.uint8, device=X.device)
    s = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=X.device)
    ws, wsn = _ws(X.device, _lib.OP_QUANTIZE, rows, 0, cols, DTYPE_E4M3, workspace)
    rc = lib.fp4_quantize_pertensor(_ptr(X), rows, cols, _ptr(q), _ptr(s), _ptr(ws), wsn,
                                    _ptr(status), _stream(X.device))
    _lib.check(rc, "fp4_quantize_pertensor")
    return q, s


def sp24_prune_compress_fp4(W: torch.Tensor, status: torch.Tensor | None = None,
                            workspace: Workspace | None = None, out: dict | None = None):
    """2:4 magnitude prune + per-tensor FP4 (E2M1) quantise + compress of W bf16
    [N, K]: returns dict(values u8 [N, K/4] (K/2 codes, two per byte), meta u8
    [N, K/8], scale); ``out`` may supply any of these preallocated."""
    lib = _lib.load()
    out = out or {}
    _require_cuda(W, status, *out.values())
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    N, K = W.shape
    values = out.get("values")
    values = values if values is not None else torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    meta = out.get("meta")
    meta = meta if meta is not None else torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    scale = out.get("scale")
    scale = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=W.device)
    ws, wsn = _ws(W.device, _lib.OP_PRUNE_COMPRESS, 0, N, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_prune_compress_fp4(_ptr(W), N, K, _ptr(values), _ptr(meta), _ptr(scale), _ptr(ws), wsn,
                                     _ptr(status), _stream(W.device))
    _lib.check(rc, "sp24_prune_compress_fp4")
    return dict(values=values, meta=meta, scale=scale)


def sp24_gemm_fp4(xq: torch.Tensor, x_scale, values: torch.Tensor, meta: torch.Tensor, w_scale,
                  out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  workspace: Workspace | None = None):
    """FP4 sparse GEMM: xq u8 [M, K/2] (fp4_quantize_pertensor), values u8 [N, K/4]
    and meta u8 [N, K/8] (sp24_prune_compress_fp4) -> Y bf16 [M, N]."""
    lib = _lib.load()
    _require_cuda(xq, x_scale, values, meta, w_scale, out, status)
    if xq.dtype != torch.uint8 or xq.dim() != 2 or values.dim() != 2:
        raise Sp24Error("xq and values must be 2-D uint8 tensors of packed FP4 codes")
    M, K = xq.shape[0], xq.shape[1] * 2
    N = values.shape[0]
    if values.shape[1] * 4 != K or meta.shape != (N, K // 8):
        raise Sp24Error("values / meta do not match N x K")
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    ws, wsn = _ws(xq.device, _lib.OP_GEMM_FP4, M, N, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_gemm_fp4(_ptr(xq), _ptr(x_scale), _ptr(values), _ptr(meta), _ptr(w_scale), _ptr(y), M, N, K,
                           _ptr(ws), wsn, _ptr(status), _stream(xq.device))
    _lib.check(rc, "sp24_gemm_fp4")
    return y


def _quant_gemm(name, op, klift, X, packed, w_scale, n, out, xq_out, x_scale_out, status, workspace):
    lib = _lib.load()
    _require_cuda(X, packed, w_scale, out, xq_out, x_scale_out, status)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    M, K = X.shape
    kg = klift(K)
    if packed.numel() != n * kg // 2 + n * kg // 8:
        raise Sp24Error("packed weights do not match N x K")
    y = out if out is not None else torch.empty((M, n), dtype=torch.bfloat16, device=X.device)
    xq = xq_out if xq_out is not None else torch.empty((M, kg), dtype=torch.uint8, device=X.device)
    if xq.numel() != M * kg or xq.dtype != torch.uint8:
        raise Sp24Error("code output has the wrong size or dtype")
    sx = x_scale_out if x_scale_out is not None else torch.empty((1,), dtype=torch.float32, device=X.device)
    ws, wsn = _ws(X.device, op, M, n, K, DTYPE_E4M3, workspace)
    rc = getattr(lib, name)(_ptr(X), M, n, K, _ptr(packed), _ptr(w_scale), _ptr(xq), _ptr(sx), _ptr(y),
                            _ptr(ws), wsn, _ptr(status), _stream(X.device))
    _lib.check(rc, name)
    return y, xq, sx


def sp24_quantize_gemm_packed(X: torch.Tensor, packed: torch.Tensor, w_scale, n: int,
                              out: torch.Tensor | None = None, xq_out: torch.Tensor | None = None,
                              x_scale_out: torch.Tensor | None = None,
                              status: torch.Tensor | None = None, workspace: Workspace | None = None):
    """Per-tensor E4M3 quantisation of X bf16 [M, K] (M <= 256) fused with the
    packed sparse GEMM: fp8_quantize_pertensor followed by sp24_gemm_packed
    in one launch.  Returns (Y bf16 [M, n], Xq u8 [M, K], x_scale f32 [1])."""
    return _quant_gemm("sp24_quantize_gemm_packed", _lib.OP_QUANTIZE_GEMM_PACKED, lambda k: k, X, packed,
                       w_scale, n, out, xq_out, x_scale_out, status, workspace)


def slide68_lift_gemm_packed(X: torch.Tensor, packed: torch.Tensor, w_scale, n: int,
                             out: torch.Tensor | None = None, xq_out: torch.Tensor | None = None,
                             x_scale_out: torch.Tensor | None = None,
                             status: torch.Tensor | None = None, workspace: Workspace | None = None):
    """slide68_lift of X bf16 [M, K] (M <= 256) fused with the packed sparse GEMM
    over K' = 3K/2 (weights from slide68_decompose_packed).  Returns
    (Y bf16 [M, n], lifted codes u8 [M, K'], x_scale f32 [1])."""
    return _quant_gemm("slide68_lift_gemm_packed", _lib.OP_LIFT_GEMM_PACKED, lambda k: 3 * k // 2, X, packed,
                       w_scale, n, out, xq_out, x_scale_out, status, workspace)


def _slide_kprime(k: int, n: int) -> int:
    if k % (2 * n):
        raise Sp24Error("K must be a multiple of 2n")
    return k // (2 * n) * 4 * (n - 1)


def slide_decompose(W: torch.Tensor, n: int, status: torch.Tensor | None = None,
                    workspace: Workspace | None = None, out: dict | None = None):
    """(2n-2):2n decomposition (n = 3, 4, 5) of W bf16 [N, K] into 2:4 E4M3 over
    K' = K (2n-2)/n: returns dict(values [N, K'/2], meta [N, K'/8], scale);
    ``out`` may supply any of these preallocated."""
    lib = _lib.load()
    out = out or {}
    _require_cuda(W, status, *out.values())
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    N, K = W.shape
    kp = _slide_kprime(K, n)
    values = out.get("values")
    values = values if values is not None else torch.empty((N, kp // 2), dtype=torch.uint8, device=W.device)
    meta = out.get("meta")
    meta = meta if meta is not None else torch.empty((N, kp // 8), dtype=torch.uint8, device=W.device)
    scale = out.get("scale")
    scale = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=W.device)
    ws, wsn = _ws(W.device, _lib.OP_SLIDE68_DECOMPOSE, 0, N, K, DTYPE_E4M3, workspace)
    rc = lib.slide_decompose(_ptr(W), N, K, n, _ptr(values), _ptr(meta), _ptr(scale), _ptr(ws), wsn,
                             _ptr(status), _stream(W.device))
    _lib.check(rc, "slide_decompose")
    return dict(values=values, meta=meta, scale=scale)


def slide_lift(X: torch.Tensor, n: int, status: torch.Tensor | None = None,
               workspace: Workspace | None = None, out: torch.Tensor | None = None,
               scale: torch.Tensor | None = None):
    """Lift of X bf16 [M, K] to K' = K (2n-2)/n fused with per-tensor E4M3
    quantisation: returns (codes u8 [M, K'], scale f32 [1])."""
    lib = _lib.load()
    _require_cuda(X, status, out, scale)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    M, K = X.shape
    kp = _slide_kprime(K, n)
    q = out if out is not None else torch.empty((M, kp), dtype=torch.uint8, device=X.device)
    sc = scale if scale is not None else torch.empty((1,), dtype=torch.float32, device=X.device)
    ws, wsn = _ws(X.device, _lib.OP_SLIDE68_LIFT, M, 0, K, DTYPE_E4M3, workspace)
    rc = lib.slide_lift(_ptr(X), M, K, n, _ptr(q), _ptr(sc), _ptr(ws), wsn, _ptr(status), _stream(X.device))
    _lib.check(rc, "slide_lift")
    return q, sc


def fp8_quantize_pertoken(X: torch.Tensor, status: torch.Tensor | None = None,
                          out: torch.Tensor | None = None, scales: torch.Tensor | None = None):
    """Per-token E4M3 quantisation of X bf16 [M, K]: returns (codes u8 [M, K],
    scales f32 [M]) with scales[m] = amax|X[m, :]| / 448."""
    lib = _lib.load()
    _require_cuda(X, status, out, scales)
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise Sp24Error("X must be a 2-D bf16 tensor")
    M, K = X.shape
    q = out if out is not None else torch.empty((M, K), dtype=torch.uint8, device=X.device)
    sc = scales if scales is not None else torch.empty((M,), dtype=torch.float32, device=X.device)
    if q.shape != (M, K) or q.dtype != torch.uint8 or sc.numel() != M or sc.dtype != torch.float32:
        raise Sp24Error("output tensors have the wrong shape or dtype")
    rc = lib.fp8_quantize_pertoken(_ptr(X), M, K, _ptr(q), _ptr(sc), _ptr(status), _stream(X.device))
    _lib.check(rc, "fp8_quantize_pertoken")
    return q, sc


def sp24_prune_compress_perchannel(W: torch.Tensor, status: torch.Tensor | None = None, out: dict | None = None):
    """2:4 prune + per-output-channel E4M3 quantise + compress of W bf16 [N, K].
    Returns dict(values u8 [N, K/2], meta u8 [N, K/8], scales f32 [N])."""
    lib = _lib.load()
    _require_cuda(W, status)
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise Sp24Error("W must be a 2-D bf16 tensor")
    N, K = W.shape
    out = dict(out or {})
    values = out.get("values")
    if values is None:
        values = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    meta = out.get("meta")
    if meta is None:
        meta = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    scales = out.get("scales")
    if scales is None:
        scales = torch.empty((N,), dtype=torch.float32, device=W.device)
    _require_cuda(values, meta, scales)
    rc = lib.sp24_prune_compress_perchannel(_ptr(W), N, K, _ptr(values), _ptr(meta), _ptr(scales),
                                            _ptr(status), _stream(W.device))
    _lib.check(rc, "sp24_prune_compress_perchannel")
    return dict(values=values, meta=meta, scales=scales)


def sp24_gemm_packed_scaled(xq: torch.Tensor, x_scales: torch.Tensor, packed: torch.Tensor,
                            w_scales: torch.Tensor, n: int, out: torch.Tensor | None = None,
                            status: torch.Tensor | None = None, workspace: Workspace | None = None):
    """sp24_gemm_packed with a per-token scale vector (x_scales of M floats,
    or one) and a per-channel one (w_scales of n floats, or one)."""
    lib = _lib.load()
    _require_cuda(xq, x_scales, packed, w_scales, out, status)
    M, K = xq.shape
    if packed.numel() != n * K // 2 + n * K // 8:
        raise Sp24Error("packed weights do not match N x K")
    xv, wv = x_scales.numel() != 1, w_scales.numel() != 1
    if (xv and x_scales.numel() != M) or (wv and w_scales.numel() != n):
        raise Sp24Error("scale vectors must hold one value or one per token / channel")
    y = out if out is not None else torch.empty((M, n), dtype=torch.bfloat16, device=xq.device)
    ws, wsn = _ws(xq.device, _lib.OP_GEMM_PACKED, M, n, K, DTYPE_E4M3, workspace)
    rc = lib.sp24_gemm_packed_scaled(_ptr(xq), _ptr(x_scales), int(xv), _ptr(packed), _ptr(w_scales), int(wv),
                                     _ptr(y), M, n, K, _ptr(ws), wsn, _ptr(status), _stream(xq.device))
    _lib.check(rc, "sp24_gemm_packed_scaled")
    return y


def fp8_gemm_dense(xq: torch.Tensor, x_scale, wq: torch.Tensor, w_scale,
                   out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                   workspace: Workspace | None = None):
    """Dense FP8 GEMM of the same kernel family (sparse-speedup baseline)."""
    lib = _lib.load()
    _require_cuda(xq, x_scale, wq, w_scale, out, status)
    M, K = xq.shape
    N = wq.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    ws, wsn = _ws(xq.device, _lib.OP_GEMM_DENSE, M, N, K, DTYPE_E4M3, workspace)
    rc = lib.fp8_gemm_dense(_ptr(xq), _ptr(x_scale), _ptr(wq), _ptr(w_scale), _ptr(y), M, N, K,
                            _ptr(ws), wsn, _ptr(status), _stream(xq.device))
    _lib.check(rc, "fp8_gemm_dense")
    return y


def debug_e4m3_encode(v: torch.Tensor) -> torch.Tensor:
    """E4M3 codes of fp32 values via the kernels' own device routine (test hook)."""
    lib = _lib.load()
    _require_cuda(v)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _lib.check(lib.sp24_debug_e4m3_encode(_ptr(v), _ptr(out), v.numel(), _stream(v.device)),
               "sp24_debug_e4m3_encode")
    return out
