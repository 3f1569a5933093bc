"""GPU parity of the prefetching rotated-MXFP4 kernel, and of the other paths
at the same size.

For bf16 weights large enough that every thread handles two blocks or more,
MXFP4 with the block Hadamard (alone, and with the fused global max) runs a
kernel that loads the next block's bytes while the current block is
quantized.  The shape below gives three grid-stride rounds with a ragged last
one (threads whose next block lies past the end load nothing), so the first,
the middle and the last rounds are all compared with the oracle; the NVFP4
sweep and plain MXFP4 are compared on the same weight.  Non-finite inputs and
a rotation that overflows binary32 must still raise the status flag.
"""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import _assert_eq, _np, mxfp4_parity, nvfp4_parity

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
ROWS, COLS = 2465, 4096        # 315,520 MXFP4 and 631,040 NVFP4 blocks on 148 SMs: three rounds


def _rows():
    return np.unique(np.concatenate([np.arange(0, ROWS, 16), np.arange(ROWS - 24, ROWS)]))


@pytest.fixture(scope="module")
def weight():
    return synth.t_weight(ROWS, COLS, nu=4, scale=0.02, seed=61, device=DEV).cpu()


def test_prefetch_nvfp4_mse(weight):
    nvfp4_parity(weight, rows_sample=_rows())


def test_prefetch_mxfp4_plain_and_rotated(weight):
    mxfp4_parity(weight, rows_sample=_rows())
    mxfp4_parity(weight, synth.sign_masks(COLS, seed=61), rows_sample=_rows())


@pytest.mark.parametrize("rotated", [False, True])
def test_prefetch_dual_fused_max(weight, rotated):
    masks = synth.sign_masks(COLS, seed=62) if rotated else None
    md = None if masks is None else torch.from_numpy(masks.view(np.int32)).to(DEV)
    nv, mx = fq.quantize_dual(weight.to(DEV), sign_masks=md)
    torch.cuda.synchronize()
    assert fq.check_status(nv.status) == 0
    x = weight.float().numpy()
    gmax = oracle.global_absmax(x)
    assert _np(nv.amax)[0] == gmax
    S = oracle.global_scale(gmax)
    idx = _rows()
    o = oracle.nvfp4_quant(np.ascontiguousarray(x[idx]), S=S)
    _assert_eq("nv scales", _np(nv.scales)[idx], o["scales"])
    _assert_eq("nv codes", _np(nv.codes)[idx], o["codes"])
    m = oracle.mxfp4_quant(np.ascontiguousarray(x[idx]), sign_masks=masks)
    _assert_eq("mx scales", _np(mx.scales)[idx], m["scales"])
    _assert_eq("mx codes", _np(mx.codes)[idx], m["codes"])
    _assert_eq("mx deq", _np(mx.deq)[idx], oracle.bf16_round(m["y"]))


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_prefetch_nonfinite_flags(weight, bad):
    w = weight.clone()
    w[ROWS - 3, 1000] = bad                 # in the last, ragged round
    wd = w.to(DEV)
    md = torch.from_numpy(synth.sign_masks(COLS, seed=61).view(np.int32)).to(DEV)
    r = fq.nvfp4_quantize(wd)
    m = fq.mxfp4_quantize(wd)
    h = fq.mxfp4_quantize(wd, md)
    nv, mx = fq.quantize_dual(wd)
    torch.cuda.synchronize()
    for st in (r.status, m.status, h.status, nv.status):
        assert int(st.item()) == fq.FLAG_NONFINITE


def test_prefetch_rotation_overflow_flag(weight):
    """32 finite bf16 values of 2^127 with equal signs after the sign flips sum
    past the binary32 range in the rotation: the rotated block is not finite
    and the oracle flags it too."""
    w = weight.clone()
    masks = synth.sign_masks(COLS, seed=61)
    r, g = ROWS - 2, 37                     # one 32-column group in the last round
    m = int(masks[g])
    signs = np.array([-1.0 if (m >> j) & 1 else 1.0 for j in range(32)], np.float32)
    w[r, 32 * g:32 * g + 32] = torch.from_numpy(signs * np.float32(2.0 ** 127)).to(torch.bfloat16)
    o = oracle.mxfp4_quant(np.ascontiguousarray(w[r:r + 1].float().numpy()), sign_masks=masks)
    assert o["status"] == oracle.STATUS_NONFINITE
    h = fq.mxfp4_quantize(w.to(DEV), torch.from_numpy(masks.view(np.int32)).to(DEV))
    torch.cuda.synchronize()
    assert int(h.status.item()) == fq.FLAG_NONFINITE


def test_prefetch_rotated_wide_rows_without_the_sign_table():
    """More than 1024 column groups (33,024 columns): the rotated kernel reads
    each block's sign mask instead of a shared table of sign words; three
    rounds with a ragged last one."""
    rows, cols = 300, 33024
    w = synth.t_weight(rows, cols, nu=4, scale=0.02, seed=63, device=DEV).cpu()
    masks = synth.sign_masks(cols, seed=63)
    sample = np.unique(np.concatenate([np.arange(0, rows, 23), [rows - 2, rows - 1]]))
    mxfp4_parity(w, masks, rows_sample=sample)


def test_rotated_calls_with_changing_table_sizes():
    """The shared table of sign words grows with the column count (up to 64 KB,
    above the 48 KB default limit).  Calls of different widths in any order
    must all launch and stay bit-exact: a kernel's shared-memory limit is only
    ever raised, so a narrow call cannot break a later wider one."""
    for rows, cols in [(1200, 4096), (2400, 2048), (1200, 4096), (160, 32768), (2400, 2048), (160, 32768)]:
        w = synth.t_weight(rows, cols, nu=4, scale=0.02, seed=rows + cols, device=DEV).cpu()
        masks = synth.sign_masks(cols, seed=rows)
        mxfp4_parity(w, masks, rows_sample=[0, rows - 1])
        nv, mx = fq.quantize_dual(w.to(DEV), sign_masks=torch.from_numpy(masks.view(np.int32)).to(DEV))
        torch.cuda.synchronize()
        assert fq.check_status(nv.status) == 0
        m = oracle.mxfp4_quant(np.ascontiguousarray(w[-1:].float().numpy()), sign_masks=masks)
        _assert_eq("dual mx codes", _np(mx.codes)[-1:], m["codes"])
