"""GPU tests of fp4q_quantize_batch: one persistent launch per 128 weights must
reproduce the single-weight calls (fp4q_quantize_dual) bit for bit, whatever
the mix of shapes, objectives (MSE / WMSE), rotations, dtypes, empty weights,
and lists longer than one launch."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import synth
from test_gpu_parity import DEV, _assert_eq, _np

pytestmark = pytest.mark.gpu


def _masks(cols, seed):
    return torch.from_numpy(synth.sign_masks(cols, seed=seed).view(np.int32)).to(DEV)


def _check_against_dual(weights, imps, masks):
    got = fq.quantize_batch(weights, imps, masks)
    torch.cuda.synchronize()
    assert int(got[0][0].status.item()) == 0 if got else True
    for k, w in enumerate(weights):
        nv_ref, mx_ref = fq.quantize_dual(w, imps[k] if imps else None, masks[k] if masks else None)
        torch.cuda.synchronize()
        nv, mx = got[k]
        if w.numel() == 0:          # the batch also writes S = 1 for an empty weight
            assert _np(nv.global_scale)[0] == 1.0 and _np(nv.amax)[0] == 0.0
            continue
        for name, a, b in (("amax", nv.amax, nv_ref.amax), ("S", nv.global_scale, nv_ref.global_scale),
                           ("nv codes", nv.codes, nv_ref.codes), ("nv scales", nv.scales, nv_ref.scales),
                           ("nv deq", nv.deq, nv_ref.deq), ("nv loss", nv.block_loss, nv_ref.block_loss),
                           ("mx codes", mx.codes, mx_ref.codes), ("mx scales", mx.scales, mx_ref.scales),
                           ("mx deq", mx.deq, mx_ref.deq), ("mx loss", mx.block_loss, mx_ref.block_loss)):
            _assert_eq(f"tensor {k} {name}", _np(a), _np(b))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_batch_mixed_shapes(dtype):
    shapes = [(1, 32), (37, 288), (300, 1056), (1024, 4096), (0, 64), (4096, 1024), (3, 96)]
    weights = [synth.q_proj(r, c, seed=r + c + 1).to(dtype).to(DEV) for r, c in shapes]
    _check_against_dual(weights, None, None)


def test_batch_wmse_and_rotation_mix():
    shapes = [(256, 512), (64, 2048), (1000, 320), (17, 4096)]
    weights = [synth.t_weight(r, c, seed=r * 3 + c).to(DEV) for r, c in shapes]
    imps = [synth.importance_diag_xtx(cols=c, tokens=64, seed=k).to(DEV) if k % 2 == 0 else None
            for k, (r, c) in enumerate(shapes)]
    masks = [_masks(c, k) if k % 3 != 1 else None for k, (r, c) in enumerate(shapes)]
    _check_against_dual(weights, imps, masks)


def test_batch_longer_than_one_launch():
    weights = [synth.q_proj(8 + (k % 5), 32 * (1 + k % 4), seed=k).to(DEV) for k in range(fq.BATCH_MAX + 7)]
    _check_against_dual(weights, None, None)


def test_batch_llama_layer():
    shapes = synth.llama3_8b_shapes()[:7]
    weights = [synth.llama3_8b_tensor(i, r, c, device=DEV) for i, (_, r, c) in enumerate(shapes)]
    _check_against_dual(weights, None, None)


def test_batch_nonfinite_flag_and_other_tensors_exact():
    a = synth.q_proj(64, 256, seed=1).to(DEV)
    b = synth.q_proj(64, 256, seed=2)
    b[5, 9] = float("nan")
    b = b.to(DEV)
    c = synth.q_proj(64, 256, seed=3).to(DEV)
    got = fq.quantize_batch([a, b, c])
    torch.cuda.synchronize()
    assert int(got[0][0].status.item()) & fq.FLAG_NONFINITE
    assert np.isnan(_np(got[1][0].amax)[0])
    for k, w in ((0, a), (2, c)):
        nv_ref, mx_ref = fq.quantize_dual(w)
        torch.cuda.synchronize()
        _assert_eq("codes", _np(got[k][0].codes), _np(nv_ref.codes))
        _assert_eq("mx codes", _np(got[k][1].codes), _np(mx_ref.codes))


def test_batch_graph_capture():
    weights = [synth.q_proj(512, 1024, seed=k).to(DEV) for k in range(3)]
    ref = fq.quantize_batch(weights)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(fq.fp4q_batch_workspace_bytes(), dtype=torch.uint8, device=DEV)
    outs = []
    items = []
    for w in weights:
        o = dict(w=w, amax=torch.empty(1, device=DEV), global_scale=torch.empty(1, device=DEV),
                 nv_codes=torch.empty((512, 512), dtype=torch.uint8, device=DEV),
                 nv_scales=torch.empty((512, 64), dtype=torch.uint8, device=DEV),
                 nv_deq=torch.empty_like(w),
                 mx_codes=torch.empty((512, 512), dtype=torch.uint8, device=DEV),
                 mx_scales=torch.empty((512, 32), dtype=torch.uint8, device=DEV))
        items.append(o)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fq.fp4q_quantize_batch(items, ws, status)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for k, o in enumerate(items):
        _assert_eq("graph nv codes", _np(o["nv_codes"]), _np(ref[k][0].codes))
        _assert_eq("graph nv deq", _np(o["nv_deq"]), _np(ref[k][0].deq))
        _assert_eq("graph mx codes", _np(o["mx_codes"]), _np(ref[k][1].codes))
        _assert_eq("graph S", _np(o["global_scale"]), _np(ref[k][0].global_scale))
