"""GPU tests of the fused entry points: fp4q_mxfp4_quant_absmax (MXFP4 that
also reduces max|w| for the NVFP4 global scale) and fp4q_quantize_dual
(both formats of one weight in two launches).  They must reproduce the
separate calls bit for bit, and the oracle on sampled rows."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _deq_bits, _np

pytestmark = pytest.mark.gpu


def _masks(cols, seed):
    return torch.from_numpy(synth.sign_masks(cols, seed=seed).view(np.int32)).to(DEV)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 288), (300, 1056), (1024, 4096)])
@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("rotate", [False, True])
def test_dual_equals_separate_calls(dtype, rows, cols, weighted, rotate):
    w = synth.q_proj(rows, cols, seed=rows + cols).to(dtype).to(DEV)
    imp = synth.importance_diag_xtx(cols=cols, tokens=64, seed=rows).to(DEV) if weighted else None
    masks = _masks(cols, rows) if rotate else None
    nv, mx = fq.quantize_dual(w, importance=imp, sign_masks=masks)
    nv_ref = fq.nvfp4_quantize(w, importance=imp)
    mx_ref = fq.mxfp4_quantize(w, masks)
    torch.cuda.synchronize()
    assert int(nv.status.item()) == 0
    for name, a, b in (("amax", nv.amax, nv_ref.amax), ("S", nv.global_scale, nv_ref.global_scale),
                       ("nv codes", nv.codes, nv_ref.codes), ("nv scales", nv.scales, nv_ref.scales),
                       ("nv deq", nv.deq, nv_ref.deq), ("nv loss", nv.block_loss, nv_ref.block_loss),
                       ("mx codes", mx.codes, mx_ref.codes), ("mx scales", mx.scales, mx_ref.scales),
                       ("mx deq", mx.deq, mx_ref.deq), ("mx loss", mx.block_loss, mx_ref.block_loss)):
        _assert_eq(name, _np(a), _np(b))


def test_dual_llama_tensor_against_oracle():
    shapes = synth.llama3_8b_shapes()
    name, rows, cols = shapes[6]          # down projection, 4096 x 14336
    w = synth.llama3_8b_tensor(6, rows, cols, device=DEV)
    nv, mx = fq.quantize_dual(w)
    torch.cuda.synchronize()
    x_full = w.float().cpu().numpy()
    gmax = oracle.global_absmax(x_full)
    assert _np(nv.amax)[0] == gmax
    idx = np.array([0, 1, 2047, rows - 1])
    x = np.ascontiguousarray(x_full[idx])
    o = oracle.nvfp4_quant(x, S=oracle.global_scale(gmax))
    _assert_eq("nv scales", _np(nv.scales)[idx], o["scales"])
    _assert_eq("nv codes", _np(nv.codes)[idx], o["codes"])
    _assert_eq("nv deq", _np(nv.deq)[idx], _deq_bits(o["y"], torch.bfloat16))
    om = oracle.mxfp4_quant(x)
    _assert_eq("mx scales", _np(mx.scales)[idx], om["scales"])
    _assert_eq("mx codes", _np(mx.codes)[idx], om["codes"])


def test_absmax_of_rotated_call_is_of_the_unrotated_weight():
    w = synth.q_proj(64, 256, seed=3).to(DEV)
    codes = torch.empty((64, 128), dtype=torch.uint8, device=DEV)
    scales = torch.empty((64, 8), dtype=torch.uint8, device=DEV)
    amax = torch.full((1,), 123.0, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    fq.fp4q_mxfp4_quant_absmax(w, _masks(256, 3), codes, scales, amax, d_status=st)
    torch.cuda.synchronize()
    assert _np(amax)[0] == w.float().abs().max().item()


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_dual_nonfinite(bad):
    w = synth.q_proj(8, 128, seed=5)
    w[3, 17] = bad
    nv, mx = fq.quantize_dual(w.to(DEV))
    torch.cuda.synchronize()
    assert int(nv.status.item()) == fq.FLAG_NONFINITE


def test_dual_empty():
    w = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    nv, mx = fq.quantize_dual(w)
    torch.cuda.synchronize()
    assert _np(nv.amax)[0] == 0.0
