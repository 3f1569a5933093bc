"""Python binding of libfp4q, the sm_100a block-scaled FP4 weight quantizer.

Argument marshalling only: every step of the quantization runs in the CUDA
kernels behind the C ABI of ``include/fp4q.h``.  PyTorch supplies device
memory and streams.  The functions named like the C entry points
(``fp4q_global_absmax``, ``fp4q_nvfp4_sweepmse``, ``fp4q_nvfp4_sweepwmse``,
``fp4q_mxfp4_quant``, ``fp4q_mxfp4_quant_hadamard``, ``fp4q_dequant``) take
caller-allocated CUDA tensors, check their devices, dtypes and sizes, and
enqueue the call on the current torch stream.  ``nvfp4_quantize``,
``mxfp4_quantize`` and ``dequantize`` allocate the outputs with torch and call
the same entry points.

There is no CPU fallback: if ``libfp4q.so`` has not been built, or no CUDA
device is visible, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import NamedTuple, Optional

import torch

__all__ = [
    "Fp4qError", "library_path", "load", "version", "check_status",
    "fp4q_global_absmax", "fp4q_nvfp4_sweepmse", "fp4q_nvfp4_sweepwmse", "fp4q_mxfp4_quant",
    "fp4q_mxfp4_quant_hadamard", "fp4q_mxfp4_quant_absmax", "fp4q_quantize_dual", "fp4q_dequant",
    "fp4q_probe_e2m1", "fp4q_probe_e4m3",
    "fp4q_quantize_batch", "fp4q_batch_workspace_bytes", "fp4q_quantize_batch_static", "BatchTensor",
    "fp4q_nvfp4_sweep_dynamic", "fp4q_dynamic_workspace_bytes", "nvfp4_quantize_dynamic",
    "fp4q_mma_scale_bytes", "fp4q_scales_to_mma_layout", "mma_scales",
    "fp4q_focus_quant", "fp4q_mxfp4_unrotate", "focus_quantize", "mxfp4_unrotate", "FocusResult",
    "fp4q_nvfp4_gptq", "fp4q_gptq_workspace_bytes", "nvfp4_gptq", "fp4q_probe_wait", "fp4q_probe_copy",
    "quantize_batch", "fp4q_mxfp4_quant_group", "fp4q_nvfp4_sweep_group", "GROUP_MAX",
    "NVFP4Result", "MXFP4Result", "nvfp4_quantize", "mxfp4_quantize", "quantize_dual", "dequantize",
    "FLAG_NONFINITE", "FLAG_RANGE", "FLAG_TIMEOUT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfp4q.so")
_lib = None
_lib_lock = threading.Lock()

OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_NONFINITE, ERR_CUDA, ERR_RANGE, ERR_ARG = range(9)
F32, BF16 = 0, 1
NVFP4, MXFP4 = 0, 1
FLAG_NONFINITE, FLAG_RANGE, FLAG_TIMEOUT = 1, 2, 4
BATCH_MAX = 128
GROUP_MAX = 32
NVFP4_BLOCK, MXFP4_BLOCK = 16, 32
EXPORTS = ("fp4q_version", "fp4q_status_string", "fp4q_last_cuda_error", "fp4q_global_absmax",
           "fp4q_nvfp4_sweepmse", "fp4q_nvfp4_sweepwmse", "fp4q_mxfp4_quant",
           "fp4q_mxfp4_quant_hadamard", "fp4q_mxfp4_quant_absmax", "fp4q_quantize_dual",
           "fp4q_quantize_batch", "fp4q_batch_workspace_bytes", "fp4q_quantize_batch_static", "fp4q_dequant",
           "fp4q_probe_e2m1", "fp4q_probe_e4m3", "fp4q_nvfp4_sweep_dynamic", "fp4q_dynamic_workspace_bytes",
           "fp4q_mma_scale_bytes", "fp4q_scales_to_mma_layout", "fp4q_focus_quant", "fp4q_mxfp4_unrotate",
           "fp4q_nvfp4_gptq", "fp4q_gptq_workspace_bytes", "fp4q_probe_wait",
           "fp4q_probe_copy", "fp4q_mxfp4_quant_group", "fp4q_nvfp4_sweep_group")


class BatchTensor(ctypes.Structure):
    """Mirror of fp4q_batch_tensor (include/fp4q.h)."""
    _fields_ = [("w", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("importance", ctypes.c_void_p), ("sign_masks", ctypes.c_void_p),
                ("amax", ctypes.c_void_p), ("global_scale", ctypes.c_void_p),
                ("nv_codes", ctypes.c_void_p), ("nv_scales", ctypes.c_void_p),
                ("nv_deq", ctypes.c_void_p), ("nv_loss", ctypes.c_void_p),
                ("mx_codes", ctypes.c_void_p), ("mx_scales", ctypes.c_void_p),
                ("mx_deq", ctypes.c_void_p), ("mx_loss", ctypes.c_void_p)]


class Fp4qError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.fp4q_status_string(status).decode()
        if status == ERR_CUDA:
            msg += ": " + lib.fp4q_last_cuda_error().decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libfp4q.so (raises if it has not been built).  Thread-safe: the
    first caller loads it and declares the signatures, the others wait."""
    if _lib is not None:
        return _lib
    with _lib_lock:
        return _lib if _lib is not None else _load_locked()


def _load_locked():
    global _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m fp4_post_weight_grid_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.fp4q_version.restype = I
    lib.fp4q_version.argtypes = []
    lib.fp4q_status_string.restype = ctypes.c_char_p
    lib.fp4q_status_string.argtypes = [I]
    lib.fp4q_last_cuda_error.restype = ctypes.c_char_p
    lib.fp4q_last_cuda_error.argtypes = []
    sigs = {
        "fp4q_global_absmax": [P, I, I64, P, P, P],
        "fp4q_nvfp4_sweepmse": [P, I, I64, I64, P, P, P, P, P, P, P, P],
        "fp4q_nvfp4_sweepwmse": [P, I, I64, I64, P, P, P, P, P, P, P, P, P],
        "fp4q_mxfp4_quant": [P, I, I64, I64, P, P, P, P, P, P],
        "fp4q_mxfp4_quant_hadamard": [P, I, I64, I64, P, P, P, P, P, P, P],
        "fp4q_mxfp4_quant_absmax": [P, I, I64, I64, P, P, P, P, P, P, P, P],
        "fp4q_quantize_dual": [P, I, I64, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "fp4q_dequant": [I, P, P, P, I64, I64, P, I, P],
        "fp4q_probe_e2m1": [P, P, I64, P],
        "fp4q_probe_e4m3": [P, P, I64, P],
        "fp4q_probe_wait": [P, ctypes.c_uint32, ctypes.c_uint32, P, P],
        "fp4q_probe_copy": [P, P, I64, P],
    }
    sigs["fp4q_quantize_batch"] = [ctypes.POINTER(BatchTensor), ctypes.c_int32, I, P, ctypes.c_size_t, P, P]
    sigs["fp4q_quantize_batch_static"] = [ctypes.POINTER(BatchTensor), ctypes.c_int32, I, P, P]
    sigs["fp4q_mxfp4_quant_group"] = [ctypes.POINTER(BatchTensor), ctypes.c_int32, I, P, P]
    sigs["fp4q_nvfp4_sweep_group"] = [ctypes.POINTER(BatchTensor), ctypes.c_int32, I, P, P]
    sigs["fp4q_scales_to_mma_layout"] = [P, I64, I64, P, P]
    sigs["fp4q_focus_quant"] = [I, P, I, I64, I64, P, P, P, ctypes.c_int32, P, P, P, P, P]
    sigs["fp4q_mxfp4_unrotate"] = [P, I, I64, I64, P, P, P]
    sigs["fp4q_nvfp4_gptq"] = [P, I64, I64, P, P, P, P, P, P, P, ctypes.c_size_t, P, P]
    sigs["fp4q_nvfp4_sweep_dynamic"] = [P, I, I64, I64, P, P, P, P, P, P, P, P, ctypes.c_size_t, P, P]
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.restype = I
        fn.argtypes = args
    lib.fp4q_batch_workspace_bytes.restype = ctypes.c_size_t
    lib.fp4q_batch_workspace_bytes.argtypes = []
    lib.fp4q_gptq_workspace_bytes.restype = ctypes.c_size_t
    lib.fp4q_gptq_workspace_bytes.argtypes = [I64]
    lib.fp4q_mma_scale_bytes.restype = I64
    lib.fp4q_mma_scale_bytes.argtypes = [I64, I64]
    lib.fp4q_dynamic_workspace_bytes.restype = ctypes.c_size_t
    lib.fp4q_dynamic_workspace_bytes.argtypes = []
    _lib = lib
    return lib


def version() -> int:
    return load().fp4q_version()


# --------------------------------------------------------------------------- marshalling helpers

def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _dev(t: Optional[torch.Tensor], name: str, dtype=None, numel=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU fallback)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr() if t.numel() > 0 else None


def _wdtype(w: torch.Tensor) -> int:
    if w.dtype == torch.bfloat16:
        return BF16
    if w.dtype == torch.float32:
        return F32
    raise TypeError(f"weights must be bfloat16 or float32, got {w.dtype}")


def _check(status: int, where: str):
    if status != OK:
        raise Fp4qError(status, where)


def _rc(w: torch.Tensor, block: int = 1):
    if w.dim() != 2:
        raise ValueError("weights must be a 2-D [rows, cols] tensor")
    if w.shape[1] % block:
        raise Fp4qError(ERR_SHAPE, f"cols = {w.shape[1]} is not a multiple of the block size {block}")
    return w.shape[0], w.shape[1]


# --------------------------------------------------------------------------- C entry points

def fp4q_global_absmax(x: torch.Tensor, d_amax: torch.Tensor, d_status: Optional[torch.Tensor] = None,
                       stream=None) -> None:
    """d_amax[0] = max|x| (NaN if x holds a NaN).  ScaleSweep: S = max|x|/(256*6).
    With d_status (one int32 on the device) the call also ORs FLAG_NONFINITE or
    FLAG_RANGE into it when that maximum cannot give a global scale."""
    dev = x.device
    xp = _dev(x, "x", device=dev)
    ap = _dev(d_amax, "d_amax", torch.float32, 1, dev)
    sp = _dev(d_status, "d_status", torch.int32, 1, dev)
    _check(load().fp4q_global_absmax(xp, _wdtype(x), x.numel(), ap, sp, _stream(stream)),
           "fp4q_global_absmax")


def _nvfp4_args(w, d_amax, codes, scales, d_global_scale, deq, block_loss, d_status):
    rows, cols = _rc(w, NVFP4_BLOCK)
    dev = w.device
    n = rows * cols
    return (rows, cols, _dev(w, "w", device=dev), _dev(d_amax, "d_amax", torch.float32, 1, dev),
            _dev(codes, "codes", torch.uint8, n // 2, dev),
            _dev(scales, "scales", torch.uint8, n // NVFP4_BLOCK, dev),
            _dev(d_global_scale, "d_global_scale", torch.float32, 1, dev),
            _dev(deq, "deq", w.dtype, n, dev),
            _dev(block_loss, "block_loss", torch.float32, n // NVFP4_BLOCK, dev),
            _dev(d_status, "d_status", torch.int32, 1, dev))


def fp4q_nvfp4_sweepmse(w, d_amax, codes, scales, d_global_scale, deq=None, block_loss=None,
                        d_status=None, stream=None) -> None:
    """NVFP4 ScaleSweep, MSE objective, window p-3..p+7 around s_base."""
    rows, cols, wp, ap, cp, sp, gp, dp, lp, st = _nvfp4_args(w, d_amax, codes, scales,
                                                            d_global_scale, deq, block_loss, d_status)
    _check(load().fp4q_nvfp4_sweepmse(wp, _wdtype(w), rows, cols, ap, cp, sp, gp, dp, lp, st,
                                      _stream(stream)), "fp4q_nvfp4_sweepmse")


def fp4q_nvfp4_sweepwmse(w, d_amax, importance, codes, scales, d_global_scale, deq=None,
                         block_loss=None, d_status=None, stream=None) -> None:
    """NVFP4 ScaleSweep, importance-weighted MSE, window p-8..p+7."""
    rows, cols, wp, ap, cp, sp, gp, dp, lp, st = _nvfp4_args(w, d_amax, codes, scales,
                                                            d_global_scale, deq, block_loss, d_status)
    ip = _dev(importance, "importance", torch.float32, cols, w.device)
    _check(load().fp4q_nvfp4_sweepwmse(wp, _wdtype(w), rows, cols, ap, ip, cp, sp, gp, dp, lp, st,
                                       _stream(stream)), "fp4q_nvfp4_sweepwmse")


def _mx_args(w, codes, scales, deq, block_loss, d_status):
    rows, cols = _rc(w, MXFP4_BLOCK)
    dev = w.device
    n = rows * cols
    return (rows, cols, _dev(w, "w", device=dev), _dev(codes, "codes", torch.uint8, n // 2, dev),
            _dev(scales, "scales", torch.uint8, n // MXFP4_BLOCK, dev),
            _dev(deq, "deq", w.dtype, n, dev),
            _dev(block_loss, "block_loss", torch.float32, n // MXFP4_BLOCK, dev),
            _dev(d_status, "d_status", torch.int32, 1, dev))


def fp4q_mxfp4_quant(w, codes, scales, deq=None, block_loss=None, d_status=None, stream=None) -> None:
    """MXFP4, E8M0 exponent sweep e0-1..e0+1 per 32-element block."""
    rows, cols, wp, cp, sp, dp, lp, st = _mx_args(w, codes, scales, deq, block_loss, d_status)
    _check(load().fp4q_mxfp4_quant(wp, _wdtype(w), rows, cols, cp, sp, dp, lp, st, _stream(stream)),
           "fp4q_mxfp4_quant")


def fp4q_mxfp4_quant_hadamard(w, sign_masks, codes, scales, deq=None, block_loss=None,
                              d_status=None, stream=None) -> None:
    """MXFP4 after the fused random-sign 32-point block Hadamard rotation."""
    rows, cols, wp, cp, sp, dp, lp, st = _mx_args(w, codes, scales, deq, block_loss, d_status)
    mp = _dev(sign_masks, "sign_masks", (torch.int32, torch.uint32), cols // MXFP4_BLOCK, w.device)
    _check(load().fp4q_mxfp4_quant_hadamard(wp, _wdtype(w), rows, cols, mp, cp, sp, dp, lp, st,
                                            _stream(stream)), "fp4q_mxfp4_quant_hadamard")


def fp4q_mxfp4_quant_absmax(w, sign_masks, codes, scales, d_amax, deq=None, block_loss=None,
                            d_status=None, stream=None) -> None:
    """MXFP4 (rotated when sign_masks is given) that also writes max|w| to d_amax."""
    rows, cols, wp, cp, sp, dp, lp, st = _mx_args(w, codes, scales, deq, block_loss, d_status)
    mp = _dev(sign_masks, "sign_masks", (torch.int32, torch.uint32), cols // MXFP4_BLOCK, w.device)
    ap = _dev(d_amax, "d_amax", torch.float32, 1, w.device)
    _check(load().fp4q_mxfp4_quant_absmax(wp, _wdtype(w), rows, cols, mp, cp, sp, dp, lp, ap, st,
                                          _stream(stream)), "fp4q_mxfp4_quant_absmax")


def fp4q_quantize_dual(w, importance, sign_masks, d_amax, nv_codes, nv_scales, d_global_scale,
                       nv_deq, nv_loss, mx_codes, mx_scales, mx_deq, mx_loss, d_status,
                       stream=None) -> None:
    """NVFP4 ScaleSweep and MXFP4 of the same weight in two launches."""
    rows, cols, wp, cp, sp, dp, lp, st = _mx_args(w, mx_codes, mx_scales, mx_deq, mx_loss, d_status)
    _, _, _, ap, ncp, nsp, gp, ndp, nlp, _ = _nvfp4_args(w, d_amax, nv_codes, nv_scales, d_global_scale,
                                                        nv_deq, nv_loss, d_status)
    ip = _dev(importance, "importance", torch.float32, cols, w.device)
    mp = _dev(sign_masks, "sign_masks", (torch.int32, torch.uint32), cols // MXFP4_BLOCK, w.device)
    _check(load().fp4q_quantize_dual(wp, _wdtype(w), rows, cols, ip, mp, ap, ncp, nsp, gp, ndp, nlp,
                                     cp, sp, dp, lp, st, _stream(stream)), "fp4q_quantize_dual")


def fp4q_focus_quant(fmt: int, w, scales, d_global_scale, coeffs, sub_block: int, codes, deq=None,
                     block_loss=None, d_status=None, stream=None) -> None:
    """FOCUS forward quantizer: codes of w / (S_dq * c_k) per sub-block, the
    reconstruction with S_dq.  `scales`: the stored block scale bytes;
    `coeffs`: float16 [rows, cols / sub_block]; `d_global_scale`: NVFP4 S."""
    bs = MXFP4_BLOCK if fmt == MXFP4 else NVFP4_BLOCK
    rows, cols = _rc(w, bs)
    dev = w.device
    n = rows * cols
    sub = int(sub_block)
    if sub <= 0 or bs % sub:
        raise Fp4qError(ERR_ARG, f"fp4q_focus_quant: sub_block {sub} does not divide the block of {bs}")
    args = (_dev(w, "w", device=dev), _wdtype(w), rows, cols,
            _dev(scales, "scales", torch.uint8, n // bs, dev),
            _dev(d_global_scale, "d_global_scale", torch.float32, 1, dev),
            _dev(coeffs, "coeffs", torch.float16, n // sub, dev), sub,
            _dev(codes, "codes", torch.uint8, n // 2, dev), _dev(deq, "deq", w.dtype, n, dev),
            _dev(block_loss, "block_loss", torch.float32, n // bs, dev),
            _dev(d_status, "d_status", torch.int32, 1, dev), _stream(stream))
    _check(load().fp4q_focus_quant(int(fmt), *args), "fp4q_focus_quant")


def fp4q_mxfp4_unrotate(y, sign_masks, out, stream=None) -> None:
    """Rotated-domain MXFP4 reconstruction `y` back to the original domain, into `out`."""
    rows, cols = _rc(y, MXFP4_BLOCK)
    dev = y.device
    _check(load().fp4q_mxfp4_unrotate(_dev(y, "y", device=dev), _wdtype(y), rows, cols,
                                      _dev(sign_masks, "sign_masks", (torch.int32, torch.uint32), cols // 32, dev),
                                      _dev(out, "out", y.dtype, rows * cols, dev), _stream(stream)),
           "fp4q_mxfp4_unrotate")


def fp4q_gptq_workspace_bytes(rows: int) -> int:
    return int(load().fp4q_gptq_workspace_bytes(int(rows)))


def fp4q_nvfp4_gptq(w, U, d_amax, codes, scales, d_global_scale, deq, workspace, d_status, stream=None) -> None:
    """ScaleSweep inside GPTQ.  `w` (float32, contiguous) is overwritten with
    the error-compensated values; `U` the upper Cholesky factor of H^-1."""
    rows, cols = _rc(w, NVFP4_BLOCK)
    if w.dtype != torch.float32:
        raise TypeError("fp4q_nvfp4_gptq works on a float32 copy of the weight")
    dev = w.device
    n = rows * cols
    ws = _dev(workspace, "workspace", device=dev)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().fp4q_nvfp4_gptq(_dev(w, "w", device=dev), rows, cols, _dev(U, "U", torch.float32, cols * cols, dev),
                                  _dev(d_amax, "d_amax", torch.float32, 1, dev),
                                  _dev(codes, "codes", torch.uint8, n // 2, dev),
                                  _dev(scales, "scales", torch.uint8, n // NVFP4_BLOCK, dev),
                                  _dev(d_global_scale, "d_global_scale", torch.float32, 1, dev),
                                  _dev(deq, "deq", torch.float32, n, dev), ws, nbytes,
                                  _dev(d_status, "d_status", torch.int32, 1, dev), _stream(stream)),
           "fp4q_nvfp4_gptq")


def fp4q_mma_scale_bytes(rows: int, scale_cols: int) -> int:
    return int(load().fp4q_mma_scale_bytes(int(rows), int(scale_cols)))


def fp4q_scales_to_mma_layout(scales: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """[rows][scale_cols] uint8 block scales -> the 128 x 4 tiled layout of
    Blackwell block-scaled GEMMs, written to `out` (uint8, fp4q_mma_scale_bytes)."""
    if scales.dim() != 2:
        raise ValueError("scales must be a 2-D [rows][scale_cols] tensor")
    rows, scols = scales.shape
    sp = _dev(scales, "scales", torch.uint8, device=scales.device)
    op = _dev(out, "out", torch.uint8, fp4q_mma_scale_bytes(rows, scols), scales.device)
    _check(load().fp4q_scales_to_mma_layout(sp, rows, scols, op, _stream(stream)), "fp4q_scales_to_mma_layout")


def mma_scales(scales: torch.Tensor, stream=None) -> torch.Tensor:
    """Allocating form of fp4q_scales_to_mma_layout (flat uint8 tensor)."""
    rows, scols = scales.shape
    out = torch.empty(fp4q_mma_scale_bytes(rows, scols), dtype=torch.uint8, device=scales.device)
    fp4q_scales_to_mma_layout(scales, out, stream)
    return out


def fp4q_dynamic_workspace_bytes() -> int:
    return int(load().fp4q_dynamic_workspace_bytes())


def fp4q_nvfp4_sweep_dynamic(x, importance, d_amax, codes, scales, d_global_scale, deq, block_loss,
                             workspace: torch.Tensor, d_status, stream=None) -> None:
    """Global max and NVFP4 ScaleSweep (MSE, or WMSE with `importance`) in one
    cooperative launch.  `workspace`: a zeroed CUDA tensor of at least
    fp4q_dynamic_workspace_bytes() bytes, left zeroed by the call."""
    rows, cols, xp, ap, cp, sp, gp, dp, lp, st = _nvfp4_args(x, d_amax, codes, scales,
                                                            d_global_scale, deq, block_loss, d_status)
    ip = _dev(importance, "importance", torch.float32, cols, x.device)
    wsp = _dev(workspace, "workspace", device=x.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load().fp4q_nvfp4_sweep_dynamic(xp, _wdtype(x), rows, cols, ip, ap, cp, sp, gp, dp, lp, wsp, nbytes,
                                           st, _stream(stream)), "fp4q_nvfp4_sweep_dynamic")


def fp4q_batch_workspace_bytes() -> int:
    return int(load().fp4q_batch_workspace_bytes())


def _batch_array(items):
    """fp4q_batch_tensor array of the descriptor dicts (argument marshalling)."""
    dev = items[0]["w"].device
    arr = (BatchTensor * len(items))()
    for k, it in enumerate(items):
        w = it["w"]
        if w.dtype != items[0]["w"].dtype:
            raise TypeError("all weights of a batch share one dtype")
        rows, cols = _rc(w, MXFP4_BLOCK)
        n = rows * cols
        arr[k].w = _dev(w, "w", device=dev)
        arr[k].rows, arr[k].cols = rows, cols
        arr[k].importance = _dev(it.get("importance"), "importance", torch.float32, cols, dev)
        arr[k].sign_masks = _dev(it.get("sign_masks"), "sign_masks", (torch.int32, torch.uint32),
                                 cols // MXFP4_BLOCK, dev)
        arr[k].amax = _dev(it["amax"], "amax", torch.float32, 1, dev)
        arr[k].global_scale = _dev(it["global_scale"], "global_scale", torch.float32, 1, dev)
        arr[k].nv_codes = _dev(it["nv_codes"], "nv_codes", torch.uint8, n // 2, dev)
        arr[k].nv_scales = _dev(it["nv_scales"], "nv_scales", torch.uint8, n // NVFP4_BLOCK, dev)
        arr[k].nv_deq = _dev(it.get("nv_deq"), "nv_deq", w.dtype, n, dev)
        arr[k].nv_loss = _dev(it.get("nv_loss"), "nv_loss", torch.float32, n // NVFP4_BLOCK, dev)
        arr[k].mx_codes = _dev(it["mx_codes"], "mx_codes", torch.uint8, n // 2, dev)
        arr[k].mx_scales = _dev(it["mx_scales"], "mx_scales", torch.uint8, n // MXFP4_BLOCK, dev)
        arr[k].mx_deq = _dev(it.get("mx_deq"), "mx_deq", w.dtype, n, dev)
        arr[k].mx_loss = _dev(it.get("mx_loss"), "mx_loss", torch.float32, n // MXFP4_BLOCK, dev)
    return arr, dev


def fp4q_quantize_batch_static(items, d_status: torch.Tensor, stream=None) -> None:
    """fp4q_quantize_batch with the library's own static scratch instead of a
    caller-provided workspace (at most BATCH_MAX weights; allocates nothing)."""
    if len(items) > BATCH_MAX:
        raise Fp4qError(ERR_ARG, f"fp4q_quantize_batch_static takes at most {BATCH_MAX} weights")
    if not items:
        return
    arr, dev = _batch_array(items)
    sp = _dev(d_status, "d_status", torch.int32, 1, dev)
    _check(load().fp4q_quantize_batch_static(arr, len(items), _wdtype(items[0]["w"]), sp, _stream(stream)),
           "fp4q_quantize_batch_static")


def fp4q_quantize_batch(items, workspace: torch.Tensor, d_status: torch.Tensor, stream=None) -> None:
    """Quantize a list of weights to NVFP4 and MXFP4 in one persistent launch per
    BATCH_MAX weights.  `items` is a list of dicts with the fields of
    fp4q_batch_tensor as CUDA tensors (w, amax, global_scale, nv_codes, nv_scales,
    mx_codes, mx_scales required; importance, sign_masks, nv_deq, nv_loss, mx_deq,
    mx_loss optional).  All weights share one dtype."""
    if not items:
        return
    dt = _wdtype(items[0]["w"])
    dev = items[0]["w"].device
    arr = (BatchTensor * len(items))()
    for k, it in enumerate(items):
        w = it["w"]
        if w.dtype != items[0]["w"].dtype:
            raise TypeError("all weights of a batch share one dtype")
        rows, cols = _rc(w, MXFP4_BLOCK)
        n = rows * cols
        arr[k].w = _dev(w, "w", device=dev)
        arr[k].rows, arr[k].cols = rows, cols
        arr[k].importance = _dev(it.get("importance"), "importance", torch.float32, cols, dev)
        arr[k].sign_masks = _dev(it.get("sign_masks"), "sign_masks", (torch.int32, torch.uint32),
                                 cols // MXFP4_BLOCK, dev)
        arr[k].amax = _dev(it["amax"], "amax", torch.float32, 1, dev)
        arr[k].global_scale = _dev(it["global_scale"], "global_scale", torch.float32, 1, dev)
        arr[k].nv_codes = _dev(it["nv_codes"], "nv_codes", torch.uint8, n // 2, dev)
        arr[k].nv_scales = _dev(it["nv_scales"], "nv_scales", torch.uint8, n // NVFP4_BLOCK, dev)
        arr[k].nv_deq = _dev(it.get("nv_deq"), "nv_deq", w.dtype, n, dev)
        arr[k].nv_loss = _dev(it.get("nv_loss"), "nv_loss", torch.float32, n // NVFP4_BLOCK, dev)
        arr[k].mx_codes = _dev(it["mx_codes"], "mx_codes", torch.uint8, n // 2, dev)
        arr[k].mx_scales = _dev(it["mx_scales"], "mx_scales", torch.uint8, n // MXFP4_BLOCK, dev)
        arr[k].mx_deq = _dev(it.get("mx_deq"), "mx_deq", w.dtype, n, dev)
        arr[k].mx_loss = _dev(it.get("mx_loss"), "mx_loss", torch.float32, n // MXFP4_BLOCK, dev)
    wp = _dev(workspace, "workspace", torch.uint8, None, dev)
    sp = _dev(d_status, "d_status", torch.int32, 1, dev)
    _check(load().fp4q_quantize_batch(arr, len(items), dt, wp, workspace.numel(), sp, _stream(stream)),
           "fp4q_quantize_batch")


def _group_array(items, prefix):
    """fp4q_batch_tensor array for a grouped call: w, amax and the `prefix`
    ("mx" or "nv") outputs, plus sign_masks (mx) or importance and
    global_scale (nv); the other fields stay NULL (argument marshalling)."""
    dev = items[0]["w"].device
    arr = (BatchTensor * len(items))()
    for k, it in enumerate(items):
        w = it["w"]
        if w.dtype != items[0]["w"].dtype:
            raise TypeError("all weights of a group share one dtype")
        rows, cols = _rc(w, MXFP4_BLOCK if prefix == "mx" else NVFP4_BLOCK)
        n = rows * cols
        bs = MXFP4_BLOCK if prefix == "mx" else NVFP4_BLOCK
        arr[k].w = _dev(w, "w", device=dev)
        arr[k].rows, arr[k].cols = rows, cols
        arr[k].amax = _dev(it["amax"], "amax", torch.float32, 1, dev)
        if prefix == "mx":
            arr[k].sign_masks = _dev(it.get("sign_masks"), "sign_masks", (torch.int32, torch.uint32),
                                     cols // MXFP4_BLOCK, dev)
        else:
            arr[k].importance = _dev(it.get("importance"), "importance", torch.float32, cols, dev)
            arr[k].global_scale = _dev(it["global_scale"], "global_scale", torch.float32, 1, dev)
        setattr(arr[k], prefix + "_codes", _dev(it[prefix + "_codes"], prefix + "_codes", torch.uint8, n // 2, dev))
        setattr(arr[k], prefix + "_scales", _dev(it[prefix + "_scales"], prefix + "_scales", torch.uint8, n // bs, dev))
        setattr(arr[k], prefix + "_deq", _dev(it.get(prefix + "_deq"), prefix + "_deq", w.dtype, n, dev))
        setattr(arr[k], prefix + "_loss", _dev(it.get(prefix + "_loss"), prefix + "_loss", torch.float32, n // bs, dev))
    return arr, dev


def fp4q_mxfp4_quant_group(items, d_status: torch.Tensor, stream=None) -> None:
    """fp4q_mxfp4_quant_absmax for a list of weights in one launch per GROUP_MAX
    weights of one kind.  `items`: dicts with w, amax, mx_codes, mx_scales
    (CUDA tensors) and optionally sign_masks, mx_deq, mx_loss."""
    if not items:
        return
    arr, dev = _group_array(items, "mx")
    sp = _dev(d_status, "d_status", torch.int32, 1, dev)
    _check(load().fp4q_mxfp4_quant_group(arr, len(items), _wdtype(items[0]["w"]), sp, _stream(stream)),
           "fp4q_mxfp4_quant_group")


def fp4q_nvfp4_sweep_group(items, d_status: torch.Tensor, stream=None) -> None:
    """fp4q_nvfp4_sweepmse / fp4q_nvfp4_sweepwmse for a list of weights in one
    launch per GROUP_MAX weights of one kind.  `items`: dicts with w, amax (the
    weight's max|w|, already on the device), global_scale, nv_codes, nv_scales
    (CUDA tensors) and optionally importance, nv_deq, nv_loss."""
    if not items:
        return
    arr, dev = _group_array(items, "nv")
    sp = _dev(d_status, "d_status", torch.int32, 1, dev)
    _check(load().fp4q_nvfp4_sweep_group(arr, len(items), _wdtype(items[0]["w"]), sp, _stream(stream)),
           "fp4q_nvfp4_sweep_group")


def fp4q_dequant(fmt: int, codes, scales, d_global_scale, rows: int, cols: int, out,
                 stream=None) -> None:
    """Decode codes + scales (+ S for NVFP4) into `out` (bf16 or fp32)."""
    dev = out.device
    bs = MXFP4_BLOCK if fmt == MXFP4 else NVFP4_BLOCK
    n = rows * cols
    cp = _dev(codes, "codes", torch.uint8, n // 2, dev)
    sp = _dev(scales, "scales", torch.uint8, n // bs, dev)
    gp = _dev(d_global_scale, "d_global_scale", torch.float32, 1, dev) if fmt == NVFP4 else None
    op = _dev(out, "out", None, n, dev)
    _check(load().fp4q_dequant(int(fmt), cp, sp, gp, rows, cols, op, _wdtype(out), _stream(stream)),
           "fp4q_dequant")


def fp4q_probe_e2m1(r: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    dev = r.device
    _check(load().fp4q_probe_e2m1(_dev(r, "r", torch.float32, device=dev),
                                  _dev(out, "out", torch.uint8, r.numel(), dev), r.numel(),
                                  _stream(stream)), "fp4q_probe_e2m1")


def fp4q_probe_copy(src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    """Plain streaming copy of src's bytes into dst (diagnostic: the copy
    bandwidth of the library's own loads and stores)."""
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < nbytes:
        raise ValueError("dst is smaller than src")
    _check(load().fp4q_probe_copy(_dev(src, "src", device=src.device), _dev(dst, "dst", device=src.device),
                                  nbytes, _stream(stream)), "fp4q_probe_copy")


def fp4q_probe_wait(flag: torch.Tensor, target: int, limit: int, d_status: torch.Tensor, stream=None) -> None:
    """The library's bounded spin-wait on its own (diagnostic): wait for
    flag >= target at most `limit` polls, FLAG_TIMEOUT in d_status if not."""
    fp = _dev(flag, "flag", (torch.int32, torch.uint32), 1, flag.device)
    sp = _dev(d_status, "d_status", torch.int32, 1, flag.device)
    _check(load().fp4q_probe_wait(fp, int(target), int(limit), sp, _stream(stream)), "fp4q_probe_wait")


def fp4q_probe_e4m3(v: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    dev = v.device
    _check(load().fp4q_probe_e4m3(_dev(v, "v", torch.float32, device=dev),
                                  _dev(out, "out", torch.uint8, v.numel(), dev), v.numel(),
                                  _stream(stream)), "fp4q_probe_e4m3")


# --------------------------------------------------------------------------- allocating helpers

class NVFP4Result(NamedTuple):
    codes: torch.Tensor           # uint8 [rows, cols/2]
    scales: torch.Tensor          # uint8 [rows, cols/16], E4M3 patterns
    global_scale: torch.Tensor    # float32 [1], S
    deq: Optional[torch.Tensor]   # input dtype [rows, cols]
    block_loss: Optional[torch.Tensor]  # float32 [rows, cols/16]
    amax: torch.Tensor            # float32 [1], max|w|
    status: torch.Tensor          # int32 [1], FLAG_* bits


class MXFP4Result(NamedTuple):
    codes: torch.Tensor           # uint8 [rows, cols/2]
    scales: torch.Tensor          # uint8 [rows, cols/32], E8M0 bytes
    deq: Optional[torch.Tensor]
    block_loss: Optional[torch.Tensor]
    status: torch.Tensor


def nvfp4_quantize(w: torch.Tensor, importance: Optional[torch.Tensor] = None, with_deq=True,
                   with_loss=True, stream=None) -> NVFP4Result:
    """Global absmax then the ScaleSweep (MSE, or WMSE when `importance` is given)."""
    rows, cols = _rc(w, NVFP4_BLOCK)
    dev = w.device
    kw = dict(device=dev)
    amax = torch.empty(1, dtype=torch.float32, **kw)
    S = torch.empty(1, dtype=torch.float32, **kw)
    status = torch.zeros(1, dtype=torch.int32, **kw)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, **kw)
    scales = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.uint8, **kw)
    deq = torch.empty_like(w) if with_deq else None
    loss = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.float32, **kw) if with_loss else None
    fp4q_global_absmax(w, amax, stream=stream)
    if importance is None:
        fp4q_nvfp4_sweepmse(w, amax, codes, scales, S, deq, loss, status, stream)
    else:
        fp4q_nvfp4_sweepwmse(w, amax, importance, codes, scales, S, deq, loss, status, stream)
    return NVFP4Result(codes, scales, S, deq, loss, amax, status)


def nvfp4_quantize_dynamic(x: torch.Tensor, importance: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None, with_deq=True, with_loss=True,
                           stream=None) -> NVFP4Result:
    """nvfp4_quantize in one launch (fp4q_nvfp4_sweep_dynamic).  Pass a zeroed
    `workspace` to reuse it across calls on one stream; by default a fresh one
    is allocated."""
    rows, cols = _rc(x, NVFP4_BLOCK)
    dev = x.device
    kw = dict(device=dev)
    amax = torch.empty(1, dtype=torch.float32, **kw)
    S = torch.empty(1, dtype=torch.float32, **kw)
    status = torch.zeros(1, dtype=torch.int32, **kw)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, **kw)
    scales = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.uint8, **kw)
    deq = torch.empty_like(x) if with_deq else None
    loss = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.float32, **kw) if with_loss else None
    if workspace is None:
        workspace = torch.zeros(fp4q_dynamic_workspace_bytes() // 4, dtype=torch.int32, **kw)
    fp4q_nvfp4_sweep_dynamic(x, importance, amax, codes, scales, S, deq, loss, workspace, status, stream)
    return NVFP4Result(codes, scales, S, deq, loss, amax, status)


class FocusResult(NamedTuple):
    codes: torch.Tensor           # uint8 [rows, cols/2]
    deq: Optional[torch.Tensor]   # reconstruction with the stored scales
    block_loss: Optional[torch.Tensor]
    status: torch.Tensor


def focus_quantize(w: torch.Tensor, fmt: int, scales: torch.Tensor, coeffs: torch.Tensor, sub_block: int = 8,
                   global_scale: Optional[torch.Tensor] = None, with_deq=True, with_loss=True,
                   stream=None) -> FocusResult:
    """Allocating form of fp4q_focus_quant."""
    bs = MXFP4_BLOCK if fmt == MXFP4 else NVFP4_BLOCK
    rows, cols = _rc(w, bs)
    kw = dict(device=w.device)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, **kw)
    deq = torch.empty_like(w) if with_deq else None
    loss = torch.empty((rows, cols // bs), dtype=torch.float32, **kw) if with_loss else None
    status = torch.zeros(1, dtype=torch.int32, **kw)
    fp4q_focus_quant(fmt, w, scales, global_scale, coeffs, sub_block, codes, deq, loss, status, stream)
    return FocusResult(codes, deq, loss, status)


def nvfp4_gptq(w: torch.Tensor, U: torch.Tensor, with_deq=True, stream=None) -> NVFP4Result:
    """Allocating form of fp4q_nvfp4_gptq on a float32 copy of `w` (the input is
    not modified); the global scale is that of `w`."""
    rows, cols = _rc(w, NVFP4_BLOCK)
    kw = dict(device=w.device)
    work = w.to(torch.float32).contiguous().clone()
    amax = torch.empty(1, dtype=torch.float32, **kw)
    fp4q_global_absmax(work, amax, stream=stream)
    S = torch.empty(1, dtype=torch.float32, **kw)
    status = torch.zeros(1, dtype=torch.int32, **kw)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, **kw)
    scales = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.uint8, **kw)
    deq = torch.empty((rows, cols), dtype=torch.float32, **kw) if with_deq else None
    ws = torch.empty(max(fp4q_gptq_workspace_bytes(rows), 16), dtype=torch.uint8, **kw)
    fp4q_nvfp4_gptq(work, U, amax, codes, scales, S, deq, ws, status, stream)
    return NVFP4Result(codes, scales, S, deq, None, amax, status)


def mxfp4_unrotate(y: torch.Tensor, sign_masks: torch.Tensor, stream=None) -> torch.Tensor:
    """Allocating form of fp4q_mxfp4_unrotate."""
    out = torch.empty_like(y)
    fp4q_mxfp4_unrotate(y, sign_masks, out, stream)
    return out


def mxfp4_quantize(w: torch.Tensor, sign_masks: Optional[torch.Tensor] = None, with_deq=True,
                   with_loss=True, stream=None) -> MXFP4Result:
    """MXFP4 E8M0 sweep; block Hadamard first when `sign_masks` is given."""
    rows, cols = _rc(w, MXFP4_BLOCK)
    dev = w.device
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // MXFP4_BLOCK), dtype=torch.uint8, device=dev)
    deq = torch.empty_like(w) if with_deq else None
    loss = torch.empty((rows, cols // MXFP4_BLOCK), dtype=torch.float32, device=dev) if with_loss else None
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if sign_masks is None:
        fp4q_mxfp4_quant(w, codes, scales, deq, loss, status, stream)
    else:
        fp4q_mxfp4_quant_hadamard(w, sign_masks, codes, scales, deq, loss, status, stream)
    return MXFP4Result(codes, scales, deq, loss, status)


def quantize_dual(w: torch.Tensor, importance: Optional[torch.Tensor] = None,
                  sign_masks: Optional[torch.Tensor] = None, with_deq=True, with_loss=True,
                  stream=None):
    """NVFP4 (MSE, or WMSE with `importance`) and MXFP4 (rotated with `sign_masks`)
    of the same weight; returns (NVFP4Result, MXFP4Result) sharing one status word."""
    rows, cols = _rc(w, MXFP4_BLOCK)
    dev = w.device
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    S = torch.empty(1, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nv = NVFP4Result(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                     torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.uint8, device=dev), S,
                     torch.empty_like(w) if with_deq else None,
                     torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.float32, device=dev) if with_loss else None,
                     amax, status)
    mx = MXFP4Result(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                     torch.empty((rows, cols // MXFP4_BLOCK), dtype=torch.uint8, device=dev),
                     torch.empty_like(w) if with_deq else None,
                     torch.empty((rows, cols // MXFP4_BLOCK), dtype=torch.float32, device=dev) if with_loss else None,
                     status)
    fp4q_quantize_dual(w, importance, sign_masks, amax, nv.codes, nv.scales, S, nv.deq, nv.block_loss,
                       mx.codes, mx.scales, mx.deq, mx.block_loss, status, stream)
    return nv, mx


def quantize_batch(weights, importances=None, sign_masks=None, with_deq=True, with_loss=True,
                   stream=None):
    """NVFP4 and MXFP4 of every weight in `weights` (one dtype), in one launch per
    BATCH_MAX weights; returns a list of (NVFP4Result, MXFP4Result) sharing one
    status word."""
    if not weights:
        return []
    dev = weights[0].device
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(fp4q_batch_workspace_bytes(), dtype=torch.uint8, device=dev)
    items, out = [], []
    for k, w in enumerate(weights):
        rows, cols = _rc(w, MXFP4_BLOCK)
        amax = torch.empty(1, dtype=torch.float32, device=dev)
        S = torch.empty(1, dtype=torch.float32, device=dev)
        nv = NVFP4Result(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                         torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.uint8, device=dev), S,
                         torch.empty_like(w) if with_deq else None,
                         torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.float32, device=dev)
                         if with_loss else None, amax, status)
        mx = MXFP4Result(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                         torch.empty((rows, cols // MXFP4_BLOCK), dtype=torch.uint8, device=dev),
                         torch.empty_like(w) if with_deq else None,
                         torch.empty((rows, cols // MXFP4_BLOCK), dtype=torch.float32, device=dev)
                         if with_loss else None, status)
        items.append(dict(w=w, importance=None if importances is None else importances[k],
                          sign_masks=None if sign_masks is None else sign_masks[k], amax=amax,
                          global_scale=S, nv_codes=nv.codes, nv_scales=nv.scales, nv_deq=nv.deq,
                          nv_loss=nv.block_loss, mx_codes=mx.codes, mx_scales=mx.scales,
                          mx_deq=mx.deq, mx_loss=mx.block_loss))
        out.append((nv, mx))
    fp4q_quantize_batch(items, ws, status, stream)
    return out


def dequantize(fmt: int, codes: torch.Tensor, scales: torch.Tensor, global_scale=None,
               dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    rows, half = codes.shape
    out = torch.empty((rows, half * 2), dtype=dtype, device=codes.device)
    fp4q_dequant(fmt, codes, scales, global_scale, rows, half * 2, out, stream)
    return out


def check_status(status: torch.Tensor) -> int:
    """Synchronize on the status word and raise on a device-reported flag."""
    v = int(status.item())
    if v & FLAG_NONFINITE:
        raise Fp4qError(ERR_NONFINITE, "device status")
    if v & FLAG_RANGE:
        raise Fp4qError(ERR_RANGE, "device status")
    return v
