"""GPU parity of the FOCUS forward quantizer (fp4q_focus_quant) and of the
inverse block Hadamard (fp4q_mxfp4_unrotate) against the oracle, bit for bit,
on ragged shapes in both dtypes and every sub-block size; plus the device
flags for invalid scales, coefficients and inputs."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _deq_bits, _np


def _coeffs(rows, n, seed):
    rng = np.random.default_rng(seed)
    return rng.uniform(0.7, 1.4, size=(rows, n)).astype(np.float16)


pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt,sub", [(fq.NVFP4, 4), (fq.NVFP4, 8), (fq.NVFP4, 16),
                                     (fq.MXFP4, 4), (fq.MXFP4, 8), (fq.MXFP4, 16), (fq.MXFP4, 32)])
@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 288), (300, 1056)])
def test_focus_equals_oracle(dtype, fmt, sub, rows, cols):
    w = synth.q_proj(rows, cols, seed=rows + cols + sub).to(dtype)
    x = w.float().numpy()
    if fmt == fq.NVFP4:
        S = oracle.global_scale(oracle.global_absmax(x))
        sc = oracle.nvfp4_quant(x, S=S)["scales"]
    else:
        S = np.float32(1.0)
        sc = oracle.mxfp4_quant(x)["scales"]
    c = _coeffs(rows, cols // sub, seed=sub + rows)
    o = oracle.focus_quant(0 if fmt == fq.NVFP4 else 1, x, sc, c, sub, S=S)
    assert o["status"] == 0
    r = fq.focus_quantize(w.to(DEV), fmt, torch.from_numpy(sc).to(DEV), torch.from_numpy(c).to(DEV), sub,
                          global_scale=torch.tensor([S], dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    assert int(r.status.item()) == 0
    _assert_eq("codes", _np(r.codes), o["codes"])
    _assert_eq("deq", _np(r.deq), _deq_bits(o["y"], dtype))
    _assert_eq("loss", _np(r.block_loss).view(np.uint32), o["loss"].view(np.uint32))


def test_focus_with_unit_coefficients_is_the_sweep_result():
    w = synth.q_proj(512, 4096, seed=31).to(DEV)
    nv = fq.nvfp4_quantize(w)
    ones = torch.ones((512, 4096 // 8), dtype=torch.float16, device=DEV)
    r = fq.focus_quantize(w, fq.NVFP4, nv.scales, ones, 8, global_scale=nv.global_scale)
    torch.cuda.synchronize()
    _assert_eq("codes", _np(r.codes), _np(nv.codes))
    _assert_eq("deq", _np(r.deq), _np(nv.deq))
    _assert_eq("loss", _np(r.block_loss), _np(nv.block_loss))


def test_focus_flags():
    w = synth.q_proj(4, 64, seed=2).to(DEV)
    sc = torch.full((4, 4), 0x38, dtype=torch.uint8, device=DEV)
    ones = torch.ones((4, 8), dtype=torch.float16, device=DEV)
    S = torch.ones(1, device=DEV)
    assert int(fq.focus_quantize(w, fq.NVFP4, sc, ones, 8, global_scale=S).status.item()) == 0
    bad = sc.clone(); bad[2, 1] = 0x7F
    assert int(fq.focus_quantize(w, fq.NVFP4, bad, ones, 8, global_scale=S).status.item()) == fq.FLAG_RANGE
    c = ones.clone(); c[1, 3] = 0.0
    assert int(fq.focus_quantize(w, fq.NVFP4, sc, c, 8, global_scale=S).status.item()) == fq.FLAG_RANGE
    c = ones.clone(); c[0, 0] = float("inf")
    assert int(fq.focus_quantize(w, fq.NVFP4, sc, c, 8, global_scale=S).status.item()) == fq.FLAG_RANGE
    w2 = w.clone(); w2[3, 5] = float("nan")
    assert int(fq.focus_quantize(w2, fq.NVFP4, sc, ones, 8, global_scale=S).status.item()) == fq.FLAG_NONFINITE
    with pytest.raises(fq.Fp4qError):
        fq.focus_quantize(w, fq.NVFP4, sc, torch.ones((4, 2), dtype=torch.float16, device=DEV), 32,
                          global_scale=S)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 288), (1000, 4096)])
def test_unrotate_equals_oracle_and_inverts_the_rotation(dtype, rows, cols):
    w = synth.q_proj(rows, cols, seed=rows * 3 + cols).to(dtype)
    masks = synth.sign_masks(cols, seed=rows)
    m = torch.from_numpy(masks.view(np.int32)).to(DEV)
    mx = fq.mxfp4_quantize(w.to(DEV), m)
    back = fq.mxfp4_unrotate(mx.deq, m)
    torch.cuda.synchronize()
    want = oracle.mxfp4_unrotate(mx.deq.float().cpu().numpy(), masks)
    _assert_eq("unrotated", _np(back), _deq_bits(want, dtype))
    # and the unrotated reconstruction is a reconstruction of w: per block, its
    # error equals the rotated-domain error up to rounding (the rotation is orthonormal)
    err_o = (back.double() - w.to(DEV).double()).pow(2).reshape(rows, -1, 32).sum(-1)
    rot = oracle.mxfp4_quant(w.float().numpy(), sign_masks=masks)
    err_r = torch.from_numpy(rot["loss"]).double().to(DEV)
    # the output is rounded to dt (relative u per element): |err_o - err_r| <=
    # 2 sqrt(err_r * E) u + E u^2 with E = sum of squares of the block, plus the
    # rounding of the two rotations (1e-3 relative is generous)
    E = w.to(DEV).double().pow(2).reshape(rows, -1, 32).sum(-1)
    u = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -22
    tol = 2 * (err_r * E).sqrt() * u + E * u * u + 1e-3 * err_r
    assert bool(((err_o - err_r).abs() <= tol + 1e-30).all())
