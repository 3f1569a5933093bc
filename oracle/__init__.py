"""CPU oracle for block-scaled FP4 weight quantization (test infrastructure).

This package is test infrastructure.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  The CUDA library never
imports, links or calls it, and it shares no code with the CUDA library: the
arithmetic lives in ``fp4q_oracle.c`` (plain C, one binary32 operation at a
time, built with ``-ffp-contract=off``); this module only marshals numpy arrays.

Sources: the ScaleSweep technical summary (gist.science, arXiv 2606.07618),
"Metodologia: ScaleSweep" sections 1-3, for NVFP4; the MR-GPTQ summary
"Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization" (arXiv 2509.23202), technical summary sections 1-2, for MXFP4
and the block Hadamard; the TORQ summary (arXiv 2605.19561) section 2.B for
the MXFP4 centre exponent.  The readings taken where the pages are silent are
stated in ``fp4q_oracle.c``.

Parity pins: the functions here are pinned by tests/test_oracle_codecs.py,
tests/test_oracle_nvfp4.py and tests/test_oracle_mxfp4.py.  The optimality of
the MXFP4 exponent window e0-1..e0+1 is not claimed by the pages and is
"parity unpinned" beyond the defined computation.  ``scales_to_mma_layout``
(the tiled scale layout read by Blackwell block-scaled GEMMs, a hardware
interface the pages do not describe) is pinned on the CPU against CUTLASS's
hierarchical shape/stride definition of that layout, evaluated by a small
independent layout-algebra routine in tests/test_oracle_mxfp4.py, and on the
GPU by a library GEMM that reads it (tests/test_gpu_mma_layout.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4q_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

NVFP4_MSE_WINDOW = (-3, 7)      # Lemma 4.3 lower bound, Lemma 4.1 upper bound
NVFP4_WMSE_WINDOW = (-8, 7)     # empirical 1/2 lower bound for WMSE
NVFP4_BLOCK = 16
MXFP4_BLOCK = 32
STATUS_OK, STATUS_NONFINITE, STATUS_RANGE = 0, 5, 7


def build(force: bool = False) -> str:
    """Compile fp4q_oracle.c into liboracle.so (gcc, -O2, no FP contraction)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                   "-fno-fast-math", "-fopenmp", _SRC, "-o", _LIB + ".tmp", "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        I = ctypes.c_int
        sigs = {
            "orc_e2m1_encode": (I, [F]),
            "orc_e2m1_decode": (F, [I]),
            "orc_e4m3_value": (F, [I]),
            "orc_e4m3_encode": (I, [F]),
            "orc_e8m0_value": (F, [I]),
            "orc_bf16_rne": (ctypes.c_uint16, [F]),
            "orc_round_bf16": (None, [P, P, I64]),
            "orc_e2m1_encode_array": (None, [P, P, I64]),
            "orc_e4m3_encode_array": (None, [P, P, I64]),
            "orc_global_absmax": (F, [P, I64]),
            "orc_gmax_status": (I, [F]),
            "orc_global_scale": (F, [F]),
            "orc_nvfp4_quant": (I, [P, I64, I64, F, P, I, I, P, P, P, P, P, I]),
            "orc_nvfp4_bruteforce": (I, [P, I64, I64, F, P, P, P, P, I]),
            "orc_nvfp4_dequant": (None, [P, P, F, I64, I64, P]),
            "orc_hadamard_scale": (F, []),
            "orc_hadamard32": (None, [P, ctypes.c_uint32, P]),
            "orc_mx_centre_exponent": (I, [F]),
            "orc_mxfp4_quant": (I, [P, I64, I64, P, P, P, P, P, P, I]),
            "orc_mxfp4_dequant": (None, [P, P, I64, I64, P]),
            "orc_max_threads": (I, []),
            "orc_mma_scale_bytes": (I64, [I64, I64]),
            "orc_hadamard32_inverse": (None, [P, ctypes.c_uint32, P]),
            "orc_mxfp4_unrotate": (None, [P, I64, I64, P, P]),
            "orc_focus_quant": (I, [I, P, I64, I64, P, F, P, I, P, P, P]),
            "orc_nvfp4_gptq": (I, [P, I64, I64, P, F, I, I, P, P, P, P, I]),
            "orc_scales_to_mma_layout": (None, [P, I64, I64, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype != np.float32:
        raise TypeError("oracle inputs are float32 arrays (upcast bf16 exactly first)")
    return x


# ---------------------------------------------------------------------------
# codecs (scalar, for pins)
# ---------------------------------------------------------------------------

def e2m1_encode(r: float) -> int:
    return _load().orc_e2m1_encode(float(np.float32(r)))


def e2m1_decode(nibble: int) -> float:
    return _load().orc_e2m1_decode(int(nibble))


def e4m3_value(p: int) -> float:
    return _load().orc_e4m3_value(int(p))


def e4m3_encode(v: float) -> int:
    return _load().orc_e4m3_encode(float(np.float32(v)))


def e8m0_value(b: int) -> float:
    return _load().orc_e8m0_value(int(b))


def e2m1_encode_array(r: np.ndarray) -> np.ndarray:
    r = _f32(r)
    out = np.empty(r.shape, dtype=np.uint8)
    _load().orc_e2m1_encode_array(_ptr(r), _ptr(out), r.size)
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(_ptr(v), _ptr(out), v.size)
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    x = _f32(x)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_round_bf16(_ptr(x), _ptr(out), x.size)
    return out


def hadamard_scale() -> float:
    return _load().orc_hadamard_scale()


def hadamard32(x: np.ndarray, mask: int) -> np.ndarray:
    x = _f32(x).reshape(32)
    y = np.empty(32, dtype=np.float32)
    _load().orc_hadamard32(_ptr(x), ctypes.c_uint32(int(mask) & 0xFFFFFFFF), _ptr(y))
    return y


def mx_centre_exponent(amax: float) -> int:
    return _load().orc_mx_centre_exponent(float(np.float32(amax)))


# ---------------------------------------------------------------------------
# tensor-level routines
# ---------------------------------------------------------------------------

def global_absmax(x: np.ndarray) -> np.float32:
    x = _f32(x)
    return np.float32(_load().orc_global_absmax(_ptr(x), x.size))


def gmax_status(gmax: float) -> int:
    return _load().orc_gmax_status(float(np.float32(gmax)))


def global_scale(gmax: float) -> np.float32:
    return np.float32(_load().orc_global_scale(float(np.float32(gmax))))


def nvfp4_quant(x: np.ndarray, S=None, importance=None, window=NVFP4_MSE_WINDOW,
                threads: int = 0) -> dict:
    """NVFP4 ScaleSweep of a rows x cols fp32 matrix.

    S defaults to the global scale of x itself; pass it explicitly when x is a
    sample of rows from a larger tensor.  Returns codes, scales, S, the fp32
    reconstruction ``y``, the per-block ``loss`` and the s_base pattern ``base``.
    """
    x = _f32(x)
    rows, cols = x.shape
    if S is None:
        g = global_absmax(x)
        st = gmax_status(g)
        if st != STATUS_OK:
            return {"status": st}
        S = global_scale(g)
    S = np.float32(S)
    w = None if importance is None else _f32(importance).reshape(cols)
    nb = rows * cols // NVFP4_BLOCK
    codes = np.empty(rows * cols // 2, dtype=np.uint8)
    scales = np.empty(nb, dtype=np.uint8)
    base = np.empty(nb, dtype=np.uint8)
    y = np.empty((rows, cols), dtype=np.float32)
    loss = np.empty(nb, dtype=np.float32)
    rc = _load().orc_nvfp4_quant(_ptr(x), rows, cols, float(S), _ptr(w), int(window[0]),
                                 int(window[1]), _ptr(codes), _ptr(scales), _ptr(y),
                                 _ptr(loss), _ptr(base), int(threads))
    if rc not in (STATUS_OK,):
        raise ValueError(f"oracle nvfp4_quant failed with {rc}")
    return {"status": STATUS_OK, "codes": codes.reshape(rows, cols // 2),
            "scales": scales.reshape(rows, cols // NVFP4_BLOCK), "S": S, "y": y,
            "loss": loss.reshape(rows, cols // NVFP4_BLOCK),
            "base": base.reshape(rows, cols // NVFP4_BLOCK)}


def nvfp4_bruteforce(x: np.ndarray, S, importance=None, threads: int = 0) -> dict:
    x = _f32(x)
    rows, cols = x.shape
    w = None if importance is None else _f32(importance).reshape(cols)
    nb = rows * cols // NVFP4_BLOCK
    bp = np.empty(nb, dtype=np.uint8)
    bl = np.empty(nb, dtype=np.float32)
    nt = np.empty(nb, dtype=np.uint8)
    _load().orc_nvfp4_bruteforce(_ptr(x), rows, cols, float(np.float32(S)), _ptr(w),
                                 _ptr(bp), _ptr(bl), _ptr(nt), int(threads))
    shp = (rows, cols // NVFP4_BLOCK)
    return {"pattern": bp.reshape(shp), "loss": bl.reshape(shp), "ties": nt.reshape(shp)}


def nvfp4_dequant(codes: np.ndarray, scales: np.ndarray, S, rows: int, cols: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    y = np.empty((rows, cols), dtype=np.float32)
    _load().orc_nvfp4_dequant(_ptr(codes), _ptr(scales), float(np.float32(S)), rows, cols, _ptr(y))
    return y


def mxfp4_quant(x: np.ndarray, sign_masks=None, threads: int = 0) -> dict:
    """MXFP4 with the E8M0 e0-1..e0+1 sweep; block Hadamard when sign_masks is given."""
    x = _f32(x)
    rows, cols = x.shape
    nb = rows * cols // MXFP4_BLOCK
    m = None if sign_masks is None else np.ascontiguousarray(sign_masks, dtype=np.uint32).reshape(cols // MXFP4_BLOCK)
    codes = np.empty(rows * cols // 2, dtype=np.uint8)
    scales = np.empty(nb, dtype=np.uint8)
    y = np.empty((rows, cols), dtype=np.float32)
    loss = np.empty(nb, dtype=np.float32)
    rot = np.empty((rows, cols), dtype=np.float32)
    st = _load().orc_mxfp4_quant(_ptr(x), rows, cols, _ptr(m), _ptr(codes), _ptr(scales), _ptr(y),
                                 _ptr(loss), _ptr(rot), int(threads))
    return {"status": st, "codes": codes.reshape(rows, cols // 2),
            "scales": scales.reshape(rows, cols // MXFP4_BLOCK), "y": y,
            "loss": loss.reshape(rows, cols // MXFP4_BLOCK), "rotated": rot}


def mxfp4_dequant(codes: np.ndarray, scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    y = np.empty((rows, cols), dtype=np.float32)
    _load().orc_mxfp4_dequant(_ptr(codes), _ptr(scales), rows, cols, _ptr(y))
    return y


def nvfp4_gptq(x: np.ndarray, U: np.ndarray, S=None, window=NVFP4_MSE_WINDOW, threads: int = 0) -> dict:
    """ScaleSweep inside GPTQ (Cholesky form): `U` the upper Cholesky factor of
    the inverse dampened Gram matrix (cols x cols, fp32; U^T U = H^-1).  S
    defaults to the global scale of x.  Returns codes, scales, y and the scaled
    errors err."""
    x = _f32(x)
    rows, cols = x.shape
    U = _f32(U)
    assert U.shape == (cols, cols)
    if S is None:
        S = global_scale(global_absmax(x))
    codes = np.empty(rows * cols // 2, dtype=np.uint8)
    scales = np.empty(rows * cols // NVFP4_BLOCK, dtype=np.uint8)
    y = np.empty((rows, cols), dtype=np.float32)
    err = np.empty((rows, cols), dtype=np.float32)
    st = _load().orc_nvfp4_gptq(_ptr(x), rows, cols, _ptr(U), float(np.float32(S)), int(window[0]),
                                int(window[1]), _ptr(codes), _ptr(scales), _ptr(y), _ptr(err), int(threads))
    if st != STATUS_OK:
        raise ValueError(f"oracle nvfp4_gptq failed with {st}")
    return {"codes": codes.reshape(rows, cols // 2), "scales": scales.reshape(rows, cols // NVFP4_BLOCK),
            "y": y, "err": err, "S": np.float32(S)}


def hadamard32_inverse(y: np.ndarray, mask: int) -> np.ndarray:
    y = _f32(y).reshape(32)
    x = np.empty(32, dtype=np.float32)
    _load().orc_hadamard32_inverse(_ptr(y), ctypes.c_uint32(int(mask) & 0xFFFFFFFF), _ptr(x))
    return x


def mxfp4_unrotate(y: np.ndarray, sign_masks: np.ndarray) -> np.ndarray:
    """Rotated-domain rows x cols values back to the original domain."""
    y = _f32(y)
    rows, cols = y.shape
    m = np.ascontiguousarray(sign_masks, dtype=np.uint32)
    x = np.empty((rows, cols), dtype=np.float32)
    _load().orc_mxfp4_unrotate(_ptr(y), rows, cols, _ptr(m), _ptr(x))
    return x


def focus_quant(fmt: int, x: np.ndarray, scales: np.ndarray, coeffs: np.ndarray, sub: int, S=1.0) -> dict:
    """FOCUS forward quantizer: codes of x / (S_dq * c_k) with the given block
    scales (fmt 0 NVFP4 E4M3 patterns + global S, 1 MXFP4 E8M0 bytes) and the
    per-sub-block coefficients `coeffs` (fp16 or fp32 values, one per `sub`
    elements); the reconstruction uses S_dq."""
    x = _f32(x)
    rows, cols = x.shape
    bs = NVFP4_BLOCK if fmt == 0 else MXFP4_BLOCK
    scales = np.ascontiguousarray(scales, dtype=np.uint8).reshape(-1)
    c = np.ascontiguousarray(np.asarray(coeffs).astype(np.float32)).reshape(-1)   # fp16 -> fp32 is exact
    assert scales.size == rows * cols // bs and c.size == rows * cols // sub
    codes = np.empty(rows * cols // 2, dtype=np.uint8)
    y = np.empty((rows, cols), dtype=np.float32)
    loss = np.empty(rows * cols // bs, dtype=np.float32)
    st = _load().orc_focus_quant(int(fmt), _ptr(x), rows, cols, _ptr(scales), float(np.float32(S)), _ptr(c),
                                 int(sub), _ptr(codes), _ptr(y), _ptr(loss))
    return {"status": st, "codes": codes.reshape(rows, cols // 2), "y": y, "loss": loss.reshape(rows, cols // bs)}


def scales_to_mma_layout(scales: np.ndarray) -> np.ndarray:
    """[rows][scols] block-scale bytes -> the 128 x 4 tiled layout (flat uint8)."""
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, scols = scales.shape
    out = np.empty(int(_load().orc_mma_scale_bytes(rows, scols)), dtype=np.uint8)
    _load().orc_scales_to_mma_layout(_ptr(scales), rows, scols, _ptr(out))
    return out


def max_threads() -> int:
    return _load().orc_max_threads()
