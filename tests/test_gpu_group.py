"""GPU parity of the grouped calls (fp4q_mxfp4_quant_group, fp4q_nvfp4_sweep_group).

A list of weights of mixed shapes (empty, one block, ragged, several thread
blocks, one large enough for several grid-stride rounds) goes through the
grouped calls and through the single-weight calls; every output must be
identical byte for byte: max|w|, S, codes, scale bytes, reconstructions and
block losses.  Plain and rotated MXFP4 weights and MSE and WMSE weights are
mixed in one list (they go to separate launches), and a list longer than
GROUP_MAX is split.  A few weights are also compared with the oracle.
"""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import _assert_eq, _np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

SHAPES = [(0, 64), (1, 32), (3, 96), (37, 288), (300, 1056), (1000, 64), (2048, 4096), (5, 0)]


def _weights(dtype, seed):
    out = []
    for k, (r, c) in enumerate(SHAPES):
        w = synth.q_proj(max(r, 1), max(c, 32), seed=seed + k)[:r, :c].contiguous().to(dtype)
        out.append(w.to(DEV))
    return out


def _outputs(w, with_loss=True):
    r, c = w.shape
    kw = dict(device=DEV)
    return dict(amax=torch.full((1,), -1.0, **kw), S=torch.full((1,), -1.0, **kw),
                nv_codes=torch.zeros((r, c // 2), dtype=torch.uint8, **kw),
                nv_scales=torch.zeros((r, c // 16), dtype=torch.uint8, **kw),
                nv_deq=torch.zeros((r, c), dtype=w.dtype, **kw),
                nv_loss=torch.zeros((r, c // 16), dtype=torch.float32, **kw) if with_loss else None,
                mx_codes=torch.zeros((r, c // 2), dtype=torch.uint8, **kw),
                mx_scales=torch.zeros((r, c // 32), dtype=torch.uint8, **kw),
                mx_deq=torch.zeros((r, c), dtype=w.dtype, **kw),
                mx_loss=torch.zeros((r, c // 32), dtype=torch.float32, **kw) if with_loss else None)


def _single(w, o, masks, imp, st):
    r, c = w.shape
    fq.fp4q_mxfp4_quant_absmax(w, masks, o["mx_codes"], o["mx_scales"], o["amax"], o["mx_deq"], o["mx_loss"], st)
    if r * c == 0:
        return
    if imp is None:
        fq.fp4q_nvfp4_sweepmse(w, o["amax"], o["nv_codes"], o["nv_scales"], o["S"], o["nv_deq"], o["nv_loss"], st)
    else:
        fq.fp4q_nvfp4_sweepwmse(w, o["amax"], imp, o["nv_codes"], o["nv_scales"], o["S"], o["nv_deq"],
                                o["nv_loss"], st)


def _grouped(ws, outs, masks, imps, st):
    mx = [dict(w=w, amax=o["amax"], sign_masks=m, mx_codes=o["mx_codes"], mx_scales=o["mx_scales"],
               mx_deq=o["mx_deq"], mx_loss=o["mx_loss"]) for w, o, m in zip(ws, outs, masks)]
    fq.fp4q_mxfp4_quant_group(mx, st)
    nv = [dict(w=w, amax=o["amax"], global_scale=o["S"], importance=i, nv_codes=o["nv_codes"],
               nv_scales=o["nv_scales"], nv_deq=o["nv_deq"], nv_loss=o["nv_loss"])
          for w, o, i in zip(ws, outs, imps)]
    fq.fp4q_nvfp4_sweep_group(nv, st)


def _compare(ws, masks, imps):
    st1 = torch.zeros(1, dtype=torch.int32, device=DEV)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    ref = [_outputs(w) for w in ws]
    got = [_outputs(w) for w in ws]
    for w, o, m, i in zip(ws, ref, masks, imps):
        _single(w, o, m, i, st1)
    _grouped(ws, got, masks, imps, st2)
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0
    for k, (a, b) in enumerate(zip(ref, got)):
        for name in a:
            if a[name] is not None:
                _assert_eq(f"weight {k} {tuple(ws[k].shape)} {name}", _np(b[name]), _np(a[name]))
    return got


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_groups_equal_single_calls_mixed_kinds(dtype):
    ws = _weights(dtype, seed=70)
    masks = [None if k % 2 else torch.from_numpy(synth.sign_masks(max(w.shape[1], 32), seed=71 + k)
                                                 [: w.shape[1] // 32].view(np.int32).copy()).to(DEV)
             for k, w in enumerate(ws)]
    imps = [None if k % 3 else synth.importance_diag_xtx(cols=max(w.shape[1], 16), tokens=64, seed=72 + k)
            [: w.shape[1]].contiguous().to(DEV) for k, w in enumerate(ws)]
    got = _compare(ws, masks, imps)
    # two of them against the oracle as well
    for k in (3, 4):
        x = ws[k].float().cpu().numpy()
        gmax = oracle.global_absmax(x)
        assert _np(got[k]["amax"])[0] == gmax
        S = oracle.global_scale(gmax)
        imp = None if imps[k] is None else imps[k].cpu().numpy()
        o = oracle.nvfp4_quant(x, S=S, importance=imp,
                               window=oracle.NVFP4_MSE_WINDOW if imp is None else oracle.NVFP4_WMSE_WINDOW)
        _assert_eq("oracle nv codes", _np(got[k]["nv_codes"]), o["codes"])
        _assert_eq("oracle nv scales", _np(got[k]["nv_scales"]), o["scales"])
        m = None if masks[k] is None else masks[k].cpu().numpy().view(np.uint32)
        om = oracle.mxfp4_quant(x, sign_masks=m)
        _assert_eq("oracle mx codes", _np(got[k]["mx_codes"]), om["codes"])
        _assert_eq("oracle mx scales", _np(got[k]["mx_scales"]), om["scales"])


def test_group_longer_than_group_max():
    n = fq.GROUP_MAX + 9
    ws = [synth.q_proj(4 + (k % 5), 64 * (1 + k % 3), seed=80 + k).to(DEV) for k in range(n)]
    _compare(ws, [None] * n, [None] * n)


def test_group_llama_layer_sampled_rows():
    """One Llama-3-8B-shaped layer (the benchmark's group), sampled rows against the oracle."""
    shapes = synth.llama3_8b_shapes()[:7]
    ws = [synth.llama3_8b_tensor(i, r, c, device=DEV) for i, (_, r, c) in enumerate(shapes)]
    outs = [_outputs(w, with_loss=False) for w in ws]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    _grouped(ws, outs, [None] * 7, [None] * 7, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rng = np.random.default_rng(81)
    for w, o in zip(ws, outs):
        r = w.shape[0]
        rows = np.unique(np.concatenate([[0, r - 1], rng.integers(0, r, size=6)]))
        x_full = w.float().cpu().numpy()
        gmax = oracle.global_absmax(x_full)
        assert _np(o["amax"])[0] == gmax
        S = oracle.global_scale(gmax)
        _assert_eq("S", _np(o["S"]), np.array([S], np.float32))
        x = np.ascontiguousarray(x_full[rows])
        on = oracle.nvfp4_quant(x, S=S)
        _assert_eq("nv codes", _np(o["nv_codes"])[rows], on["codes"])
        _assert_eq("nv deq", _np(o["nv_deq"])[rows], oracle.bf16_round(on["y"]))
        om = oracle.mxfp4_quant(x)
        _assert_eq("mx codes", _np(o["mx_codes"])[rows], om["codes"])
        _assert_eq("mx scales", _np(o["mx_scales"])[rows], om["scales"])


def test_group_flags_a_nonfinite_weight():
    ws = [synth.q_proj(64, 256, seed=90 + k).to(DEV) for k in range(3)]
    ws[1][10, 100] = float("nan")
    outs = [_outputs(w) for w in ws]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    _grouped(ws, outs, [None] * 3, [None] * 3, st)
    torch.cuda.synchronize()
    assert int(st.item()) == fq.FLAG_NONFINITE
    assert np.isnan(_np(outs[1]["amax"])[0])
