"""CPU checks of the C ABI library and the Python binding (no GPU needed).

The library must load, export every entry point declared in include/fp4q.h,
and the binding must refuse CPU tensors instead of falling back to the CPU.
No compute call is made here.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fq():
    from fp4_post_weight_grid_b200 import build
    build.build()
    import fp4_post_weight_grid_b200 as m
    m.load()
    return m


def _declared():
    text = open(os.path.join(ROOT, "include", "fp4q.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4q_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    names = _declared()
    for want in ("fp4q_global_absmax", "fp4q_nvfp4_sweepmse", "fp4q_nvfp4_sweepwmse",
                 "fp4q_mxfp4_quant", "fp4q_mxfp4_quant_hadamard", "fp4q_dequant"):
        assert want in names


def test_library_exports_every_declared_symbol(fq):
    lib = ctypes.CDLL(fq.library_path())
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(fq.EXPORTS) == _declared()


def test_version_and_status_strings(fq):
    lib = fq.load()
    assert lib.fp4q_version() >= 10000
    for s in range(8):
        assert lib.fp4q_status_string(s)
    assert b"unknown" in lib.fp4q_status_string(99)


def test_argument_errors_without_a_gpu(fq):
    """Argument checks run before any CUDA call, so they work on a CPU-only host."""
    lib = fq.load()
    buf = ctypes.create_string_buffer(256)
    p = ctypes.addressof(buf)
    p16 = p + (-p % 16)
    # bad dtype, bad shape, NULL pointers, misalignment
    assert lib.fp4q_nvfp4_sweepmse(p16, 7, 1, 16, p16, p16, p16, p16, None, None, p16, None) == fq.ERR_DTYPE
    assert lib.fp4q_nvfp4_sweepmse(p16, 1, 1, 17, p16, p16, p16, p16, None, None, p16, None) == fq.ERR_SHAPE
    assert lib.fp4q_nvfp4_sweepmse(p16, 1, -1, 16, p16, p16, p16, p16, None, None, p16, None) == fq.ERR_SHAPE
    assert lib.fp4q_nvfp4_sweepmse(None, 1, 1, 16, p16, p16, p16, p16, None, None, p16, None) == fq.ERR_NULL
    assert lib.fp4q_nvfp4_sweepmse(p16 + 2, 1, 1, 16, p16, p16, p16, p16, None, None, p16, None) == fq.ERR_ALIGN
    assert lib.fp4q_nvfp4_sweepwmse(p16, 1, 1, 16, p16, None, p16, p16, p16, None, None, p16, None) == fq.ERR_NULL
    assert lib.fp4q_mxfp4_quant(p16, 1, 1, 48, p16, p16, None, None, p16, None) == fq.ERR_SHAPE
    assert lib.fp4q_mxfp4_quant(p16, 1, 1, 32, p16 + 8, p16, None, None, p16, None) == fq.ERR_ALIGN
    assert lib.fp4q_mxfp4_quant_hadamard(p16, 1, 1, 32, None, p16, p16, None, None, p16, None) == fq.ERR_NULL
    assert lib.fp4q_dequant(5, p16, p16, p16, 1, 16, p16, 1, None) == fq.ERR_DTYPE
    assert lib.fp4q_dequant(0, p16, p16, None, 1, 16, p16, 1, None) == fq.ERR_NULL
    assert lib.fp4q_global_absmax(p16, 1, -5, p16, None, None) == fq.ERR_SHAPE
    assert lib.fp4q_global_absmax(p16 + 4, 1, 5, p16, None, None) == fq.ERR_ALIGN
    assert lib.fp4q_global_absmax(p16, 1, 5, p16, p16 + 2, None) == fq.ERR_ALIGN
    assert lib.fp4q_global_absmax(p16, 7, 5, p16, p16, None) == fq.ERR_DTYPE
    assert lib.fp4q_global_absmax(p16, 1, 5, None, p16, None) == fq.ERR_NULL
    # empty tensors are valid and touch nothing
    assert lib.fp4q_nvfp4_sweepmse(None, 1, 0, 16, None, None, None, None, None, None, None, None) == fq.OK
    assert lib.fp4q_mxfp4_quant(None, 0, 5, 0, None, None, None, None, None, None) == fq.OK
    assert lib.fp4q_dequant(1, None, None, None, 0, 32, None, 0, None) == fq.OK


def test_batch_argument_errors_without_a_gpu(fq):
    lib = fq.load()
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.addressof(buf)
    p16 = p + (-p % 16)
    ws = fq.fp4q_batch_workspace_bytes()
    assert ws >= 4 * (4 + 2 * fq.BATCH_MAX)

    def one(**kw):
        t = fq.BatchTensor()
        for f, _ in fq.BatchTensor._fields_:
            setattr(t, f, p16)
        t.rows, t.cols, t.importance, t.sign_masks = 2, 64, None, None
        t.nv_deq = t.nv_loss = t.mx_deq = t.mx_loss = None
        for k, v in kw.items():
            setattr(t, k, v)
        arr = (fq.BatchTensor * 1)(t)
        return lib.fp4q_quantize_batch(arr, 1, 1, p16, ws, p16, None)

    assert one(cols=48) == fq.ERR_SHAPE
    assert one(rows=-1) == fq.ERR_SHAPE
    assert one(w=None) == fq.ERR_NULL
    assert one(amax=None) == fq.ERR_NULL
    assert one(w=p16 + 2) == fq.ERR_ALIGN
    assert one(mx_codes=p16 + 8) == fq.ERR_ALIGN
    arr = (fq.BatchTensor * 1)()
    assert lib.fp4q_quantize_batch(arr, 1, 1, p16, ws - 1, p16, None) == fq.ERR_ARG
    assert lib.fp4q_quantize_batch(arr, 1, 9, p16, ws, p16, None) == fq.ERR_DTYPE
    assert lib.fp4q_quantize_batch(arr, -1, 1, p16, ws, p16, None) == fq.ERR_SHAPE
    assert lib.fp4q_quantize_batch(arr, 0, 1, None, 0, None, None) == fq.OK


def test_group_argument_errors_without_a_gpu(fq):
    lib = fq.load()
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.addressof(buf)
    p16 = p + (-p % 16)

    def one(fn, **kw):
        t = fq.BatchTensor()
        for f, _ in fq.BatchTensor._fields_:
            setattr(t, f, p16)
        t.rows, t.cols, t.importance, t.sign_masks = 2, 64, None, None
        t.nv_deq = t.nv_loss = t.mx_deq = t.mx_loss = None
        for k, v in kw.items():
            setattr(t, k, v)
        arr = (fq.BatchTensor * 1)(t)
        return getattr(lib, fn)(arr, 1, 1, p16, None)

    for fn in ("fp4q_mxfp4_quant_group", "fp4q_nvfp4_sweep_group"):
        assert one(fn, rows=-1) == fq.ERR_SHAPE
        assert one(fn, w=None) == fq.ERR_NULL
        assert one(fn, amax=None) == fq.ERR_NULL
        assert one(fn, w=p16 + 2) == fq.ERR_ALIGN
        assert one(fn, amax=p16 + 2) == fq.ERR_ALIGN
        arr = (fq.BatchTensor * 1)()
        assert getattr(lib, fn)(arr, 1, 9, p16, None) == fq.ERR_DTYPE
        assert getattr(lib, fn)(arr, -1, 1, p16, None) == fq.ERR_SHAPE
        assert getattr(lib, fn)(None, 1, 1, p16, None) == fq.ERR_NULL
        assert getattr(lib, fn)(arr, 1, 1, None, None) == fq.ERR_NULL
        assert getattr(lib, fn)(arr, 0, 1, None, None) == fq.OK
    # per-format block sizes and outputs
    assert one("fp4q_mxfp4_quant_group", cols=48) == fq.ERR_SHAPE
    assert one("fp4q_nvfp4_sweep_group", cols=48) != fq.ERR_SHAPE          # 48 % 16 == 0: shape is fine
    assert one("fp4q_mxfp4_quant_group", mx_codes=p16 + 8) == fq.ERR_ALIGN
    assert one("fp4q_nvfp4_sweep_group", nv_codes=p16 + 4) == fq.ERR_ALIGN
    assert one("fp4q_nvfp4_sweep_group", global_scale=None) == fq.ERR_NULL
    assert one("fp4q_nvfp4_sweep_group", importance=p16 + 4) == fq.ERR_ALIGN
    assert one("fp4q_mxfp4_quant_group", sign_masks=p16 + 2) == fq.ERR_ALIGN
    # a later bad descriptor stops the call before anything is enqueued
    good = fq.BatchTensor()
    for f, _ in fq.BatchTensor._fields_:
        setattr(good, f, p16)
    good.rows, good.cols = 0, 64
    bad = fq.BatchTensor()
    bad.rows, bad.cols = 1, 40
    arr = (fq.BatchTensor * 2)(good, bad)
    assert lib.fp4q_mxfp4_quant_group(arr, 2, 1, p16, None) == fq.ERR_SHAPE


def test_dynamic_argument_errors_without_a_gpu(fq):
    lib = fq.load()
    buf = ctypes.create_string_buffer(256)
    p = ctypes.addressof(buf)
    p16 = p + (-p % 16)
    ws = fq.fp4q_dynamic_workspace_bytes()
    assert ws >= 12

    def call(x=p16, dt=1, rows=1, cols=16, imp=None, amax=p16, wsp=p16, nbytes=ws):
        return lib.fp4q_nvfp4_sweep_dynamic(x, dt, rows, cols, imp, amax, p16, p16, p16, None, None,
                                            wsp, nbytes, p16, None)

    assert call(dt=7) == fq.ERR_DTYPE
    assert call(cols=24) == fq.ERR_SHAPE
    assert call(amax=None) == fq.ERR_NULL
    assert call(x=None) == fq.ERR_NULL
    assert call(wsp=None) == fq.ERR_NULL
    assert call(x=p16 + 2) == fq.ERR_ALIGN
    assert call(wsp=p16 + 4) == fq.ERR_ALIGN
    assert call(imp=p16 + 4) == fq.ERR_ALIGN
    assert call(nbytes=ws - 1) == fq.ERR_ARG


def test_widening_entries_argument_errors_without_a_gpu(fq):
    """FOCUS, the inverse rotation, GPTQ, the tiled scale layout and the copy
    probe check their arguments before any CUDA call."""
    lib = fq.load()
    buf = ctypes.create_string_buffer(512)
    p = ctypes.addressof(buf)
    q = p + (-p % 16)
    NV, MX = fq.NVFP4, fq.MXFP4
    # FOCUS: format, sub-block size, shape, pointers, alignment
    assert lib.fp4q_focus_quant(9, q, 1, 1, 16, q, q, q, 8, q, None, None, q, None) == fq.ERR_DTYPE
    assert lib.fp4q_focus_quant(NV, q, 1, 1, 16, q, q, q, 32, q, None, None, q, None) == fq.ERR_ARG
    assert lib.fp4q_focus_quant(NV, q, 1, 1, 16, q, q, q, 6, q, None, None, q, None) == fq.ERR_ARG
    assert lib.fp4q_focus_quant(MX, q, 1, 1, 48, q, None, q, 8, q, None, None, q, None) == fq.ERR_SHAPE
    assert lib.fp4q_focus_quant(NV, q, 1, 1, 16, q, None, q, 8, q, None, None, q, None) == fq.ERR_NULL
    assert lib.fp4q_focus_quant(NV, q, 1, 1, 16, q, q, None, 8, q, None, None, q, None) == fq.ERR_NULL
    assert lib.fp4q_focus_quant(NV, q, 1, 1, 16, q, q, q + 1, 8, q, None, None, q, None) == fq.ERR_ALIGN
    assert lib.fp4q_focus_quant(MX, q, 1, 0, 32, None, None, None, 32, None, None, None, None, None) == fq.OK
    # inverse rotation
    assert lib.fp4q_mxfp4_unrotate(q, 4, 1, 32, q, q, None) == fq.ERR_DTYPE
    assert lib.fp4q_mxfp4_unrotate(q, 1, 1, 16, q, q, None) == fq.ERR_SHAPE
    assert lib.fp4q_mxfp4_unrotate(q, 1, 1, 32, None, q, None) == fq.ERR_NULL
    assert lib.fp4q_mxfp4_unrotate(q, 1, 1, 32, q, q + 8, None) == fq.ERR_ALIGN
    assert lib.fp4q_mxfp4_unrotate(None, 1, 0, 32, None, None, None) == fq.OK
    # GPTQ: shape, pointers, workspace size
    ws = fq.fp4q_gptq_workspace_bytes(4)
    assert ws == 2 * 4 * 128 * 4 and fq.fp4q_gptq_workspace_bytes(0) == 0
    assert lib.fp4q_nvfp4_gptq(q, 4, 24, q, q, q, q, q, None, q, ws, q, None) == fq.ERR_SHAPE
    assert lib.fp4q_nvfp4_gptq(q, 4, 16, None, q, q, q, q, None, q, ws, q, None) == fq.ERR_NULL
    assert lib.fp4q_nvfp4_gptq(q, 4, 16, q, q, q, q, q, None, None, ws, q, None) == fq.ERR_NULL
    assert lib.fp4q_nvfp4_gptq(q, 4, 16, q, q, q, q, q, None, q + 4, ws, q, None) == fq.ERR_ALIGN
    assert lib.fp4q_nvfp4_gptq(q, 4, 16, q, q, q, q, q, None, q, ws - 16, q, None) == fq.ERR_ARG
    assert lib.fp4q_nvfp4_gptq(q, 4, (1 << 20) + 16, q, q, q, q, q, None, q, ws, q, None) == fq.ERR_SHAPE
    # tiled scale layout: size arithmetic and checks
    assert fq.fp4q_mma_scale_bytes(1, 1) == 512
    assert fq.fp4q_mma_scale_bytes(129, 5) == 2 * 2 * 512
    assert fq.fp4q_mma_scale_bytes(0, 7) == 0
    assert fq.fp4q_mma_scale_bytes(-1, 4) == -1 and fq.fp4q_mma_scale_bytes(1 << 62, 4) == -1
    assert lib.fp4q_scales_to_mma_layout(q, -1, 4, q, None) == fq.ERR_SHAPE
    assert lib.fp4q_scales_to_mma_layout(None, 4, 4, q, None) == fq.ERR_NULL
    assert lib.fp4q_scales_to_mma_layout(q, 4, 4, q + 4, None) == fq.ERR_ALIGN
    assert lib.fp4q_scales_to_mma_layout(None, 0, 4, None, None) == fq.OK
    # copy probe
    assert lib.fp4q_probe_copy(q, q + 256, 24, None) == fq.ERR_SHAPE
    assert lib.fp4q_probe_copy(q, q + 256, -16, None) == fq.ERR_SHAPE
    assert lib.fp4q_probe_copy(None, q, 16, None) == fq.ERR_NULL
    assert lib.fp4q_probe_copy(q + 8, q + 256, 16, None) == fq.ERR_ALIGN
    assert lib.fp4q_probe_copy(None, None, 0, None) == fq.OK


def test_binding_refuses_cpu_tensors(fq):
    w = torch.zeros((4, 32), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        fq.fp4q_global_absmax(w, torch.zeros(1))
    with pytest.raises(ValueError, match="CUDA"):
        fq.nvfp4_quantize(w)


def test_missing_library_fails_loudly(fq, monkeypatch, tmp_path):
    monkeypatch.setattr(fq, "_lib", None)
    monkeypatch.setattr(fq, "_LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fq.load()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "fp4_post_weight_grid_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower().replace("oracle-free", ""), f


def test_oracle_and_library_share_no_source():
    orc = open(os.path.join(ROOT, "oracle", "fp4q_oracle.c")).read()
    assert "#include \"" not in orc          # the oracle includes only system headers
    for f in os.listdir(os.path.join(ROOT, "fp4_post_weight_grid_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "fp4_post_weight_grid_b200", "csrc", f)).read()
