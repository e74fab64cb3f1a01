"""Python binding of libmxmoe (MXFP8 routed-experts MLP for sm_100a).

Argument marshalling only: tensors are checked, output buffers allocated with
torch on the tensor's device, and the C ABI of include/mxmoe.h is called on
the current torch CUDA stream.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing or
unbuilt library raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "ROW", "COL", "PLAIN", "MMA", "lib", "MXMOEError",
    "mxfp8_quantize", "mxfp8_swiglu_quant", "mxfp8_dequantize",
    "mxfp8_grouped_gemm", "mxfp8_grouped_gemm_wgrad",
    "mxfp8_grouped_gemm_swiglu_quant", "mxfp8_grouped_gemm_dswiglu_quant",
    "moe_mlp_fwd", "moe_mlp_bwd", "device_error", "header_functions",
    "make_qweights", "mxmoe_quantize_weights", "moe_mlp_fwd_q", "moe_mlp_bwd_q", "moe_mlp_fwd_unfused_q",
    "mxmoe_route_capacity", "mxmoe_route", "mxmoe_permute_quant", "mxmoe_unpermute_combine",
    "mxmoe_combine_weight_grad", "make_layer_saved", "moe_layer_fwd_q", "moe_layer_bwd_q",
]

ROW, COL = 1, 2
PLAIN, MMA = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "mxmoe.h")


class MXMOEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"mxmoe status {status}: {msg}")
        self.status = status


class _Saved(ctypes.Structure):
    _fields_ = [("h13", ctypes.c_void_p), ("h_col_codes", ctypes.c_void_p), ("h_col_scales", ctypes.c_void_p),
                ("x_col_codes", ctypes.c_void_p), ("x_col_scales", ctypes.c_void_p)]


class _QWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w13_codes", "w13_scales", "w13t_codes", "w13t_scales",
                                                "w2_codes", "w2_scales", "w2t_codes", "w2t_scales")]


class _LayerSaved(ctypes.Structure):
    _fields_ = [("offsets", ctypes.c_void_p), ("row_slot", ctypes.c_void_p), ("slot_row", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("mlp", _Saved)]


_P, _I, _L, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "mxmoe_last_error_message": ([], ctypes.c_char_p),
    "mxmoe_version": ([], ctypes.c_char_p),
    "mxmoe_check_device_error": ([_P, _I, ctypes.POINTER(ctypes.c_int)], _I),
    "mxfp8_quantize": ([_P, _L, _L, _L, _I, _I, _P, _P, _P, _P, _P], _I),
    "mxfp8_quantize_e5m2": ([_P, _L, _L, _L, _I, _I, _P, _P, _P, _P, _P], _I),
    "mxfp8_dequantize_e5m2": ([_P, _P, _L, _L, _P, _P], _I),
    "mxfp8_swiglu_quant": ([_P, _L, _L, _I, _I, _P, _P, _P, _P, _P], _I),
    "mxfp8_dequantize": ([_P, _P, _L, _L, _P, _P], _I),
    "mxfp8_grouped_gemm": ([_P, _P, _L, _L, _P, _P, _I, _L, _P, _I, _P, _P], _I),
    "mxfp8_grouped_gemm_wgrad": ([_P, _P, _L, _P, _P, _L, _L, _P, _P, _I, _I, _P, _P], _I),
    "mxfp8_grouped_gemm_swiglu_quant": ([_P, _P, _L, _L, _P, _P, _I, _L, _P, _I, _P, _P, _P, _P, _P, _P], _I),
    "mxfp8_grouped_gemm_dswiglu_quant": ([_P, _P, _L, _L, _P, _P, _I, _L, _P, _I, _P, _P, _P, _P, _P, _P], _I),
    "mxmoe_workspace_size": ([_L, _L, _I, _L, _I], _S),
    "moe_mlp_fwd": ([_P, _L, _L, _P, _P, _I, _L, _P, _I, _P, ctypes.POINTER(_Saved), _P, _S, _P], _I),
    "moe_mlp_bwd": ([_P, _L, _L, _P, _P, _I, _L, _P, _I, ctypes.POINTER(_Saved), _P, _P, _P, _P, _S, _P], _I),
    "moe_mlp_fwd_noalloc": ([_P, _L, _L, _P, _P, _I, _L, _P, _I, _P, ctypes.POINTER(_Saved), _P], _I),
    "mxmoe_quantize_weights": ([_P, _P, _I, _L, _L, ctypes.POINTER(_QWeights), _P], _I),
    "mxmoe_selftest_wait_timeout": ([_P], _I),
    "moe_mlp_fwd_unfused_q": ([_P, _L, _L, ctypes.POINTER(_QWeights), _I, _L, _P, _I, _P, ctypes.POINTER(_Saved),
                               _P, _S, _P], _I),
    "moe_mlp_fwd_q": ([_P, _L, _L, ctypes.POINTER(_QWeights), _I, _L, _P, _I, _P, ctypes.POINTER(_Saved), _P, _S,
                       _P], _I),
    "moe_mlp_bwd_q": ([_P, _L, _L, ctypes.POINTER(_QWeights), _I, _L, _P, _I, ctypes.POINTER(_Saved), _P, _P, _P,
                       _P, _S, _P], _I),
    "mxmoe_route_capacity": ([_L, _I, _I, _I], _L),
    "mxmoe_route_workspace_size": ([_L, _I, _I], _S),
    "mxmoe_route": ([_P, _L, _I, _I, _I, _L, _P, _P, _P, _P, _S, _P], _I),
    "mxmoe_permute_quant": ([_P, _L, _L, _P, _I, _P, _L, _P, _I, _I, _P, _P, _P, _P, _P], _I),
    "mxmoe_unpermute_combine": ([_P, _L, _L, _P, _P, _L, _I, _P, _P], _I),
    "mxmoe_combine_weight_grad": ([_P, _P, _L, _L, _P, _L, _I, _P, _P], _I),
    "moe_layer_workspace_size": ([_L, _I, _L, _I, _L, _I, _I], _S),
    "moe_layer_fwd_q": ([_P, _L, _L, _P, _P, _I, ctypes.POINTER(_QWeights), _I, _L, _I, _P,
                         ctypes.POINTER(_LayerSaved), _P, _S, _P], _I),
    "moe_layer_bwd_q": ([_P, _L, _L, _P, _I, ctypes.POINTER(_QWeights), _I, _L, _I, ctypes.POINTER(_LayerSaved),
                         _P, _P, _P, _P, _P, _S, _P], _I),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmxmoe.so from the package directory (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m mxfp8_block_scaled_routed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, ret) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ret
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/mxmoe.h."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


def _check(status: int):
    if status != 0:
        raise MXMOEError(status, lib().mxmoe_last_error_message().decode())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t: torch.Tensor, shape, name: str):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _scales(t: torch.Tensor, n: int, name: str):
    """E8M0 scale bytes: a contiguous uint8 CUDA tensor of exactly n bytes."""
    _need(t, torch.uint8, name)
    if t.numel() != n:
        raise ValueError(f"{name} must hold {n} scale bytes, got {t.numel()}")


def _u8(shape, dev):
    return torch.empty(shape, dtype=torch.uint8, device=dev)


def device_error(reset: bool = True, device=None) -> int:
    """First device-side error code recorded by the kernels (0 if none)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = ctypes.c_int(0)
    _check(lib().mxmoe_check_device_error(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream),
                                    int(reset), ctypes.byref(code)))
    return code.value


# ----------------------------------------------------------------------------- casts
def mxfp8_quantize(x: torch.Tensor, modes: int = ROW | COL, scale_layout: int = PLAIN, elem: str = "e4m3"):
    """bf16 [rows, cols] or [batch, rows, cols] -> dict of MXFP8 tensors (E4M3 or E5M2 codes).

    Keys: row_codes [.., rows, cols], row_scales, col_codes [.., cols, rows],
    col_scales.  PLAIN scales are [.., rows, ceil(cols/32)] / [.., cols, rows/32];
    MMA scales are flat uint8 vectors in the tensor-core atom layout.
    """
    _need(x, torch.bfloat16, "x")
    if x.dim() not in (2, 3):
        raise ValueError("x must be 2-D or 3-D")
    batch = x.shape[0] if x.dim() == 3 else 1
    rows, cols = x.shape[-2], x.shape[-1]
    lead = (batch,) if x.dim() == 3 else ()
    out = {}
    if modes & ROW:
        out["row_codes"] = _u8(lead + (rows, cols), x.device)
        out["row_scales"] = (_u8(lead + (rows, (cols + 31) // 32), x.device) if scale_layout == PLAIN
                             else _u8((batch * rows * cols // 32,), x.device))
    if modes & COL:
        out["col_codes"] = _u8(lead + (cols, rows), x.device)
        out["col_scales"] = (_u8(lead + (cols, rows // 32), x.device) if scale_layout == PLAIN
                             else _u8((batch * rows * cols // 32,), x.device))
    fn = {"e4m3": lib().mxfp8_quantize, "e5m2": lib().mxfp8_quantize_e5m2}[elem]
    _check(fn(_ptr(x), batch, rows, cols, modes, scale_layout,
                                _ptr(out.get("row_codes")), _ptr(out.get("row_scales")),
                                _ptr(out.get("col_codes")), _ptr(out.get("col_scales")), _stream(x)))
    return out


def mxfp8_swiglu_quant(h13: torch.Tensor, modes: int = ROW | COL, scale_layout: int = PLAIN):
    """bf16 h13 [rows, 2F] -> MXFP8 of h = silu(gate) * up, as mxfp8_quantize."""
    _need(h13, torch.bfloat16, "h13")
    rows, F2 = h13.shape
    F = F2 // 2
    out = {}
    if modes & ROW:
        out["row_codes"] = _u8((rows, F), h13.device)
        out["row_scales"] = (_u8((rows, F // 32), h13.device) if scale_layout == PLAIN
                             else _u8((rows * F // 32,), h13.device))
    if modes & COL:
        out["col_codes"] = _u8((F, rows), h13.device)
        out["col_scales"] = (_u8((F, rows // 32), h13.device) if scale_layout == PLAIN
                             else _u8((rows * F // 32,), h13.device))
    _check(lib().mxfp8_swiglu_quant(_ptr(h13), rows, F, modes, scale_layout,
                                    _ptr(out.get("row_codes")), _ptr(out.get("row_scales")),
                                    _ptr(out.get("col_codes")), _ptr(out.get("col_scales")), _stream(h13)))
    return out


def mxfp8_dequantize(codes: torch.Tensor, scales: torch.Tensor, elem: str = "e4m3") -> torch.Tensor:
    """MXFP8 ROW (plain scales, E4M3 or E5M2 codes) -> bf16."""
    _need(codes, torch.uint8, "codes")
    if codes.dim() != 2:
        raise ValueError("codes must be 2-D")
    rows, cols = codes.shape
    _scales(scales, rows * ((cols + 31) // 32), "scales")
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=codes.device)
    fn = {"e4m3": lib().mxfp8_dequantize, "e5m2": lib().mxfp8_dequantize_e5m2}[elem]
    _check(fn(_ptr(codes), _ptr(scales), rows, cols, _ptr(out), _stream(codes)))
    return out


# ----------------------------------------------------------------------------- GEMMs
def _offs(offsets: torch.Tensor):
    _need(offsets, torch.int32, "expert_offsets")
    return offsets.numel() - 1


def mxfp8_grouped_gemm(a, a_scales, w, w_scales, offsets, pad_multiple=128, out=None):
    """Ragged-M grouped GEMM: a [M, K] codes, w [E, N, K] codes (MMA scales)."""
    E = _offs(offsets)
    _need(a, torch.uint8, "a")
    _need(w, torch.uint8, "w")
    M, K = a.shape
    if w.dim() != 3 or w.shape[0] != E or w.shape[2] != K:
        raise ValueError(f"w must be [E={E}, N, K={K}], got {tuple(w.shape)}")
    N = w.shape[1]
    _scales(a_scales, M * K // 32, "a_scales")
    _scales(w_scales, E * N * K // 32, "w_scales")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    _need(out, torch.bfloat16, "out")
    _shape(out, (M, N), "out")
    _check(lib().mxfp8_grouped_gemm(_ptr(a), _ptr(a_scales), M, K, _ptr(w), _ptr(w_scales), E, N,
                                    _ptr(offsets), pad_multiple, _ptr(out), _stream(a)))
    return out


def mxfp8_grouped_gemm_wgrad(gt, gt_scales, xt, xt_scales, offsets, pad_multiple=128, out=None, expert_rows=None):
    """Ragged-K grouped GEMM: gt [N, M], xt [Kx, M] COL codes -> dw bf16 [E, N, Kx].

    expert_rows (optional, int32 [E] on the device): token rows at the head of
    each expert's padded segment; the all-padding K blocks are skipped."""
    E = _offs(offsets)
    _need(gt, torch.uint8, "gt")
    _need(xt, torch.uint8, "xt")
    N, M = gt.shape
    if xt.dim() != 2 or xt.shape[1] != M:
        raise ValueError(f"xt must be [Kx, M={M}], got {tuple(xt.shape)}")
    Kx = xt.shape[0]
    _scales(gt_scales, N * M // 32, "gt_scales")
    _scales(xt_scales, Kx * M // 32, "xt_scales")
    if out is None:
        out = torch.empty(E, N, Kx, dtype=torch.bfloat16, device=gt.device)
    _need(out, torch.bfloat16, "out")
    _shape(out, (E, N, Kx), "out")
    if expert_rows is not None:
        _need(expert_rows, torch.int32, "expert_rows")
        if expert_rows.numel() != E:
            raise ValueError(f"expert_rows must hold E={E} counts, got {expert_rows.numel()}")
    _check(lib().mxfp8_grouped_gemm_wgrad(_ptr(gt), _ptr(gt_scales), N, _ptr(xt), _ptr(xt_scales), Kx, M,
                                          _ptr(offsets), _ptr(expert_rows), E, pad_multiple, _ptr(out), _stream(gt)))
    return out


def mxfp8_grouped_gemm_swiglu_quant(a, a_scales, w13, w13_scales, offsets, pad_multiple=128, want_h13=True):
    """FC1 + SwiGLU + dual quantization; returns dict(h13, h_row_codes, h_row_scales, h_col_codes, h_col_scales)."""
    E = _offs(offsets)
    _need(a, torch.uint8, "a")
    _need(w13, torch.uint8, "w13")
    M, K = a.shape
    if w13.dim() != 3 or w13.shape[0] != E or w13.shape[2] != K or w13.shape[1] % 2:
        raise ValueError(f"w13 must be [E={E}, 2F, K={K}], got {tuple(w13.shape)}")
    F = w13.shape[1] // 2
    _scales(a_scales, M * K // 32, "a_scales")
    _scales(w13_scales, E * 2 * F * K // 32, "w13_scales")
    dev = a.device
    o = dict(h13=torch.empty(M, 2 * F, dtype=torch.bfloat16, device=dev) if want_h13 else None,
             h_row_codes=_u8((M, F), dev), h_row_scales=_u8((M * F // 32,), dev),
             h_col_codes=_u8((F, M), dev), h_col_scales=_u8((M * F // 32,), dev))
    _check(lib().mxfp8_grouped_gemm_swiglu_quant(
        _ptr(a), _ptr(a_scales), M, K, _ptr(w13), _ptr(w13_scales), E, F, _ptr(offsets), pad_multiple,
        _ptr(o["h13"]), _ptr(o["h_row_codes"]), _ptr(o["h_row_scales"]), _ptr(o["h_col_codes"]),
        _ptr(o["h_col_scales"]), _stream(a)))
    return o


def mxfp8_grouped_gemm_dswiglu_quant(dy, dy_scales, w2t, w2t_scales, offsets, h13, pad_multiple=128):
    """FC2 dgrad + dSwiGLU + dual quantization; returns dict(g_row_codes, g_row_scales, g_col_codes, g_col_scales)."""
    E = _offs(offsets)
    _need(dy, torch.uint8, "dy")
    _need(w2t, torch.uint8, "w2t")
    M, D = dy.shape
    F = w2t.shape[1]
    dev = dy.device
    _need(h13, torch.bfloat16, "h13")
    _scales(dy_scales, M * D // 32, "dy_scales")
    _scales(w2t_scales, E * F * D // 32, "w2t_scales")
    if w2t.dim() != 3 or w2t.shape[0] != E or w2t.shape[2] != D:
        raise ValueError(f"w2t must be [E={E}, F, D={D}], got {tuple(w2t.shape)}")
    if tuple(h13.shape) != (M, 2 * F):
        raise ValueError(f"h13 must be [M={M}, 2F={2 * F}], got {tuple(h13.shape)}")
    o = dict(g_row_codes=_u8((M, 2 * F), dev), g_row_scales=_u8((M * 2 * F // 32,), dev),
             g_col_codes=_u8((2 * F, M), dev), g_col_scales=_u8((M * 2 * F // 32,), dev))
    _check(lib().mxfp8_grouped_gemm_dswiglu_quant(
        _ptr(dy), _ptr(dy_scales), M, D, _ptr(w2t), _ptr(w2t_scales), E, F, _ptr(offsets), pad_multiple,
        _ptr(h13), _ptr(o["g_row_codes"]), _ptr(o["g_row_scales"]), _ptr(o["g_col_codes"]),
        _ptr(o["g_col_scales"]), _stream(dy)))
    return o


# ----------------------------------------------------------------------------- composites
def workspace_bytes(M, D, E, F, which):
    return int(lib().mxmoe_workspace_size(M, D, E, F, which))


def make_saved(M, D, F, device):
    return dict(h13=torch.empty(M, 2 * F, dtype=torch.bfloat16, device=device),
                h_col_codes=_u8((F, M), device), h_col_scales=_u8((M * F // 32,), device),
                x_col_codes=_u8((D, M), device), x_col_scales=_u8((M * D // 32,), device))


def _saved_struct(s):
    return _Saved(s["h13"].data_ptr(), s["h_col_codes"].data_ptr(), s["h_col_scales"].data_ptr(),
                  s["x_col_codes"].data_ptr(), s["x_col_scales"].data_ptr())


def moe_mlp_fwd(x, w13, w2, offsets, pad_multiple=128, y=None, saved=None, workspace=None):
    """Forward of the routed-experts MLP. Returns (y bf16 [M, D], saved dict)."""
    E = _offs(offsets)
    for t, n in ((x, "x"), (w13, "w13"), (w2, "w2")):
        _need(t, torch.bfloat16, n)
    M, D = x.shape
    F = w13.shape[1] // 2
    dev = x.device
    y = torch.empty(M, D, dtype=torch.bfloat16, device=dev) if y is None else y
    saved = make_saved(M, D, F, dev) if saved is None else saved
    nb = workspace_bytes(M, D, E, F, 1)
    ws = _u8((nb,), dev) if workspace is None else workspace
    st = _saved_struct(saved)
    _check(lib().moe_mlp_fwd(_ptr(x), M, D, _ptr(w13), _ptr(w2), E, F, _ptr(offsets), pad_multiple, _ptr(y),
                             ctypes.byref(st), _ptr(ws), ws.numel(), _stream(x)))
    return y, saved


def moe_mlp_bwd(dy, w13, w2, offsets, saved, pad_multiple=128, dx=None, dw13=None, dw2=None, workspace=None):
    """Backward of the routed-experts MLP. Returns (dx, dw13, dw2) in bf16."""
    E = _offs(offsets)
    for t, n in ((dy, "dy"), (w13, "w13"), (w2, "w2")):
        _need(t, torch.bfloat16, n)
    M, D = dy.shape
    F = w13.shape[1] // 2
    dev = dy.device
    dx = torch.empty(M, D, dtype=torch.bfloat16, device=dev) if dx is None else dx
    dw13 = torch.empty_like(w13) if dw13 is None else dw13
    dw2 = torch.empty_like(w2) if dw2 is None else dw2
    nb = workspace_bytes(M, D, E, F, 2)
    ws = _u8((nb,), dev) if workspace is None else workspace
    st = _saved_struct(saved)
    _check(lib().moe_mlp_bwd(_ptr(dy), M, D, _ptr(w13), _ptr(w2), E, F, _ptr(offsets), pad_multiple,
                             ctypes.byref(st), _ptr(dx), _ptr(dw13), _ptr(dw2), _ptr(ws), ws.numel(), _stream(dy)))
    return dx, dw13, dw2


# ----------------------------------------------------------------------------- pre-quantized weights
def make_qweights(E, D, F, device):
    """Buffers for the ROW and COL MXFP8 copies of W13 [E, 2F, D] and W2 [E, D, F]."""
    return dict(w13_codes=_u8((E, 2 * F, D), device), w13_scales=_u8((E * 2 * F * D // 32,), device),
                w13t_codes=_u8((E, D, 2 * F), device), w13t_scales=_u8((E * 2 * F * D // 32,), device),
                w2_codes=_u8((E, D, F), device), w2_scales=_u8((E * D * F // 32,), device),
                w2t_codes=_u8((E, F, D), device), w2t_scales=_u8((E * D * F // 32,), device))


def _qw_struct(q):
    return _QWeights(*(q[n].data_ptr() for n, _ in _QWeights._fields_))


def mxmoe_quantize_weights(w13, w2, qw=None):
    """Dual (ROW + COL) MXFP8 casts of both expert weights, one read of each."""
    _need(w13, torch.bfloat16, "w13")
    _need(w2, torch.bfloat16, "w2")
    E, F2, D = w13.shape
    F = F2 // 2
    qw = make_qweights(E, D, F, w13.device) if qw is None else qw
    st = _qw_struct(qw)
    _check(lib().mxmoe_quantize_weights(_ptr(w13), _ptr(w2), E, D, F, ctypes.byref(st), _stream(w13)))
    return qw


def moe_mlp_fwd_q(x, qw, offsets, pad_multiple=128, y=None, saved=None, workspace=None):
    """Forward with pre-quantized weights. Returns (y, saved)."""
    E = _offs(offsets)
    _need(x, torch.bfloat16, "x")
    M, D = x.shape
    F = qw["w13_codes"].shape[1] // 2
    dev = x.device
    y = torch.empty(M, D, dtype=torch.bfloat16, device=dev) if y is None else y
    saved = make_saved(M, D, F, dev) if saved is None else saved
    ws = _u8((workspace_bytes(M, D, E, F, 3),), dev) if workspace is None else workspace
    st, q = _saved_struct(saved), _qw_struct(qw)
    _check(lib().moe_mlp_fwd_q(_ptr(x), M, D, ctypes.byref(q), E, F, _ptr(offsets), pad_multiple, _ptr(y),
                               ctypes.byref(st), _ptr(ws), ws.numel(), _stream(x)))
    return y, saved


def moe_mlp_fwd_unfused_q(x, qw, offsets, pad_multiple=128, y=None, saved=None, workspace=None):
    """Unfused forward (FC1 -> bf16 h13 -> standalone SwiGLU cast -> FC2). Returns (y, saved)."""
    E = _offs(offsets)
    _need(x, torch.bfloat16, "x")
    M, D = x.shape
    F = qw["w13_codes"].shape[1] // 2
    dev = x.device
    y = torch.empty(M, D, dtype=torch.bfloat16, device=dev) if y is None else y
    saved = make_saved(M, D, F, dev) if saved is None else saved
    ws = _u8((workspace_bytes(M, D, E, F, 3),), dev) if workspace is None else workspace
    st, q = _saved_struct(saved), _qw_struct(qw)
    _check(lib().moe_mlp_fwd_unfused_q(_ptr(x), M, D, ctypes.byref(q), E, F, _ptr(offsets), pad_multiple, _ptr(y),
                                       ctypes.byref(st), _ptr(ws), ws.numel(), _stream(x)))
    return y, saved


def moe_mlp_bwd_q(dy, qw, offsets, saved, pad_multiple=128, dx=None, dw13=None, dw2=None, workspace=None):
    """Backward with pre-quantized weights. Returns (dx, dw13, dw2)."""
    E = _offs(offsets)
    _need(dy, torch.bfloat16, "dy")
    M, D = dy.shape
    F = qw["w13_codes"].shape[1] // 2
    dev = dy.device
    dx = torch.empty(M, D, dtype=torch.bfloat16, device=dev) if dx is None else dx
    dw13 = torch.empty(E, 2 * F, D, dtype=torch.bfloat16, device=dev) if dw13 is None else dw13
    dw2 = torch.empty(E, D, F, dtype=torch.bfloat16, device=dev) if dw2 is None else dw2
    ws = _u8((workspace_bytes(M, D, E, F, 4),), dev) if workspace is None else workspace
    st, q = _saved_struct(saved), _qw_struct(qw)
    _check(lib().moe_mlp_bwd_q(_ptr(dy), M, D, ctypes.byref(q), E, F, _ptr(offsets), pad_multiple,
                               ctypes.byref(st), _ptr(dx), _ptr(dw13), _ptr(dw2), _ptr(ws), ws.numel(), _stream(dy)))
    return dx, dw13, dw2


# ----------------------------------------------------------------------------- dispatcher
def mxmoe_route_capacity(T: int, top_k: int, E: int, pad_multiple: int) -> int:
    """Rows a padded expert-major layout of T tokens x top_k can need (multiple of 128)."""
    cap = lib().mxmoe_route_capacity(T, top_k, E, pad_multiple)
    if cap < 0:
        raise ValueError("invalid routing sizes")
    return int(cap)


def mxmoe_route(topk_ids: torch.Tensor, E: int, pad_multiple: int, m_cap: int | None = None):
    """int32 [T, top_k] expert ids -> dict(offsets [E+1], row_slot [m_cap], slot_row [T*top_k])."""
    _need(topk_ids, torch.int32, "topk_ids")
    T, k = topk_ids.shape
    if m_cap is None:
        m_cap = mxmoe_route_capacity(T, k, E, pad_multiple)
    dev = topk_ids.device
    out = {"offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
           "row_slot": torch.empty(m_cap, dtype=torch.int32, device=dev),
           "slot_row": torch.empty(T * k, dtype=torch.int32, device=dev)}
    nws = lib().mxmoe_route_workspace_size(T, k, E)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    _check(lib().mxmoe_route(_ptr(topk_ids), T, k, E, pad_multiple, m_cap, _ptr(out["offsets"]),
                             _ptr(out["row_slot"]), _ptr(out["slot_row"]), _ptr(ws), ws.numel(), _stream(topk_ids)))
    return out


def mxmoe_permute_quant(x_tokens: torch.Tensor, row_slot: torch.Tensor, top_k: int, weights=None,
                        rows_dev=None, modes: int = ROW | COL, scale_layout: int = MMA):
    """Gather token rows into the padded layout and MXFP8-quantize them (optionally weighted)."""
    _need(x_tokens, torch.bfloat16, "x_tokens")
    _need(row_slot, torch.int32, "row_slot")
    if weights is not None:
        _need(weights, torch.float32, "weights")
    if rows_dev is not None:
        _need(rows_dev, torch.int32, "rows_dev")
    T, D = x_tokens.shape
    m = row_slot.numel()
    dev = x_tokens.device
    out = {}
    if modes & ROW:
        out["row_codes"] = _u8((m, D), dev)
        out["row_scales"] = _u8((m, D // 32), dev) if scale_layout == PLAIN else _u8((m * D // 32,), dev)
    if modes & COL:
        out["col_codes"] = _u8((D, m), dev)
        out["col_scales"] = _u8((D, m // 32), dev) if scale_layout == PLAIN else _u8((m * D // 32,), dev)
    _check(lib().mxmoe_permute_quant(_ptr(x_tokens), T, D, _ptr(row_slot), top_k, _ptr(weights), m,
                                     _ptr(rows_dev), modes, scale_layout,
                                     _ptr(out.get("row_codes")), _ptr(out.get("row_scales")),
                                     _ptr(out.get("col_codes")), _ptr(out.get("col_scales")), _stream(x_tokens)))
    return out


def mxmoe_unpermute_combine(y: torch.Tensor, slot_row: torch.Tensor, top_k: int, weights=None, out=None):
    """out[t] = sum_j w[t, j] * y[slot_row[t*top_k + j]] (bf16 [T, D])."""
    _need(y, torch.bfloat16, "y")
    _need(slot_row, torch.int32, "slot_row")
    if weights is not None:
        _need(weights, torch.float32, "weights")
    T = slot_row.numel() // top_k
    if out is None:
        out = torch.empty(T, y.shape[1], dtype=torch.bfloat16, device=y.device)
    _check(lib().mxmoe_unpermute_combine(_ptr(y), y.shape[0], y.shape[1], _ptr(slot_row), _ptr(weights), T, top_k,
                                         _ptr(out), _stream(y)))
    return out


def mxmoe_combine_weight_grad(dout: torch.Tensor, y: torch.Tensor, slot_row: torch.Tensor, top_k: int):
    """d w[t, j] = <dout[t], y[slot_row[t*top_k + j]]> as fp32 [T, top_k]."""
    _need(dout, torch.bfloat16, "dout")
    _need(y, torch.bfloat16, "y")
    _need(slot_row, torch.int32, "slot_row")
    T, D = dout.shape
    dw = torch.empty(T, top_k, dtype=torch.float32, device=dout.device)
    _check(lib().mxmoe_combine_weight_grad(_ptr(dout), _ptr(y), y.shape[0], D, _ptr(slot_row), T, top_k,
                                           _ptr(dw), _stream(dout)))
    return dw


# ----------------------------------------------------------------------------- layer composites
def layer_workspace_bytes(T, top_k, D, E, F, pad_multiple, which):
    return int(lib().moe_layer_workspace_size(T, top_k, D, E, F, pad_multiple, which))


def make_layer_saved(T, top_k, D, E, F, pad_multiple, device):
    """Buffers the layer forward keeps for its backward (m_cap rows each)."""
    m = mxmoe_route_capacity(T, top_k, E, pad_multiple)
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device=device)
    return dict(offsets=i32(E + 1), row_slot=i32(m), slot_row=i32(T * top_k),
                y=torch.empty(m, D, dtype=torch.bfloat16, device=device), mlp=make_saved(m, D, F, device))


def _layer_struct(s):
    return _LayerSaved(s["offsets"].data_ptr(), s["row_slot"].data_ptr(), s["slot_row"].data_ptr(),
                       s["y"].data_ptr(), _saved_struct(s["mlp"]))


def moe_layer_fwd_q(x_tokens, topk_ids, topk_weights, qw, pad_multiple=256, out=None, saved=None, workspace=None):
    """Token-major layer forward: route, gather + cast, MLP, weighted combine. Returns (out, saved)."""
    _need(x_tokens, torch.bfloat16, "x_tokens")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_weights, torch.float32, "topk_weights")
    T, D = x_tokens.shape
    k = topk_ids.shape[1]
    E, F = qw["w13_codes"].shape[0], qw["w13_codes"].shape[1] // 2
    dev = x_tokens.device
    out = torch.empty(T, D, dtype=torch.bfloat16, device=dev) if out is None else out
    saved = make_layer_saved(T, k, D, E, F, pad_multiple, dev) if saved is None else saved
    ws = _u8((layer_workspace_bytes(T, k, D, E, F, pad_multiple, 1),), dev) if workspace is None else workspace
    st, q = _layer_struct(saved), _qw_struct(qw)
    _check(lib().moe_layer_fwd_q(_ptr(x_tokens), T, D, _ptr(topk_ids), _ptr(topk_weights), k, ctypes.byref(q), E, F,
                                 pad_multiple, _ptr(out), ctypes.byref(st), _ptr(ws), ws.numel(), _stream(x_tokens)))
    return out, saved


def moe_layer_bwd_q(dout_tokens, topk_weights, qw, saved, pad_multiple=256, dx=None, dw13=None, dw2=None,
                    dweights=True, workspace=None):
    """Token-major layer backward. Returns (dx_tokens, dw13, dw2, dweights or None)."""
    _need(dout_tokens, torch.bfloat16, "dout_tokens")
    _need(topk_weights, torch.float32, "topk_weights")
    T, D = dout_tokens.shape
    k = topk_weights.shape[1]
    E, F = qw["w13t_codes"].shape[0], qw["w13t_codes"].shape[2] // 2
    dev = dout_tokens.device
    dx = torch.empty(T, D, dtype=torch.bfloat16, device=dev) if dx is None else dx
    dw13 = torch.empty(E, 2 * F, D, dtype=torch.bfloat16, device=dev) if dw13 is None else dw13
    dw2 = torch.empty(E, D, F, dtype=torch.bfloat16, device=dev) if dw2 is None else dw2
    dwr = None
    if dweights is True:
        dwr = torch.empty(T, k, dtype=torch.float32, device=dev)
    elif isinstance(dweights, torch.Tensor):
        dwr = dweights
    ws = _u8((layer_workspace_bytes(T, k, D, E, F, pad_multiple, 2),), dev) if workspace is None else workspace
    st, q = _layer_struct(saved), _qw_struct(qw)
    _check(lib().moe_layer_bwd_q(_ptr(dout_tokens), T, D, _ptr(topk_weights), k, ctypes.byref(q), E, F, pad_multiple,
                                 ctypes.byref(st), _ptr(dx), _ptr(dw13), _ptr(dw2), _ptr(dwr), _ptr(ws), ws.numel(),
                                 _stream(dout_tokens)))
    return dx, dw13, dw2, dwr
