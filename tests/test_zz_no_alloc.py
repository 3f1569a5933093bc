"""The allocation-free batch entry point, fp4q_quantize_batch_static.

Some callers cannot allocate device memory when they quantize -- their device
memory belongs entirely to another allocator, they run under a fixed memory
budget, or they are on a path that must not call cudaMalloc -- so they cannot
provide the small workspace fp4q_quantize_batch needs.  The static entry point
uses a scratch array inside the library instead.  It must give exactly the
results of the workspace entry point, call after call: the scratch keeps the
previous call's counters, and each call has to start from zero.
"""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _items(weights, imps, masks):
    items = []
    for k, w in enumerate(weights):
        rows, cols = w.shape
        f32 = dict(dtype=torch.float32, device=DEV)
        u8 = dict(dtype=torch.uint8, device=DEV)
        items.append(dict(
            w=w, importance=imps[k], sign_masks=masks[k],
            amax=torch.empty(1, **f32), global_scale=torch.empty(1, **f32),
            nv_codes=torch.empty((rows, cols // 2), **u8), nv_scales=torch.empty((rows, cols // 16), **u8),
            nv_deq=torch.empty_like(w), nv_loss=torch.empty((rows, cols // 16), **f32),
            mx_codes=torch.empty((rows, cols // 2), **u8), mx_scales=torch.empty((rows, cols // 32), **u8),
            mx_deq=torch.empty_like(w), mx_loss=torch.empty((rows, cols // 32), **f32)))
    return items


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.numpy()


FIELDS = ("amax", "global_scale", "nv_codes", "nv_scales", "nv_deq", "nv_loss",
          "mx_codes", "mx_scales", "mx_deq", "mx_loss")


def test_static_scratch_matches_workspace_entry_on_two_calls():
    plans = [[(64, 512), (300, 1056), (1024, 4096), (8, 96)],
             [(4096, 1024), (37, 288), (512, 2048)]]
    ws = torch.empty(fq.fp4q_batch_workspace_bytes(), dtype=torch.uint8, device=DEV)
    for call, shapes in enumerate(plans):
        weights = [synth.q_proj(r, c, seed=100 * call + k).to(DEV) for k, (r, c) in enumerate(shapes)]
        imps = [synth.importance_diag_xtx(cols=c, tokens=64, seed=k).to(DEV) if k % 2 == 0 else None
                for k, (_, c) in enumerate(shapes)]
        masks = [torch.from_numpy(synth.sign_masks(c, seed=k).view(np.int32)).to(DEV) if k % 3 == 1 else None
                 for k, (_, c) in enumerate(shapes)]
        ref, got = _items(weights, imps, masks), _items(weights, imps, masks)
        st_ref = torch.zeros(1, dtype=torch.int32, device=DEV)
        st_got = torch.zeros(1, dtype=torch.int32, device=DEV)
        fq.fp4q_quantize_batch(ref, ws, st_ref)
        fq.fp4q_quantize_batch_static(got, st_got)
        torch.cuda.synchronize()
        assert int(st_ref.item()) == 0 and int(st_got.item()) == 0
        for k in range(len(shapes)):
            for f in FIELDS:
                a, b = _bits(got[k][f]), _bits(ref[k][f])
                assert np.array_equal(a, b), f"call {call}, weight {k}, {f}: {int(np.sum(a != b))} differ"


def test_static_scratch_rejects_more_than_one_launch():
    arr = (fq.BatchTensor * (fq.BATCH_MAX + 1))()
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert fq.load().fp4q_quantize_batch_static(arr, fq.BATCH_MAX + 1, 1, st.data_ptr(), None) == fq.ERR_ARG
