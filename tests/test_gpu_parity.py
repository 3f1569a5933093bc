"""GPU parity: the CUDA library, called through the C ABI, against the CPU oracle.

Bit-exact on packed codes, scales, S, the bf16/fp32 reconstruction and the
per-block losses; aggregate reconstruction MSE (fp64) agrees to a relative
1e-6 (implied by bit-exactness, checked anyway).  Small cases span several
thread blocks and a ragged tail; the full-size workloads (4096x4096 MSE,
11008x4096 WMSE) are compared in full, the largest ones (28672x8192
MXFP4+Hadamard, the Llama-3-8B-shaped model) on sampled rows with the
oracle given the full tensor's global scale.
"""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
MSE_RTOL = 1e-6


def _np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _deq_bits(y32: np.ndarray, dtype) -> np.ndarray:
    return oracle.bf16_round(y32) if dtype == torch.bfloat16 else y32


def _assert_eq(name, got, want):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    bad = np.nonzero(got.reshape(-1) != want.reshape(-1))[0]
    assert bad.size == 0, f"{name}: {bad.size} mismatches, first at flat index {bad[0]}: " \
                          f"got {got.reshape(-1)[bad[0]]} want {want.reshape(-1)[bad[0]]}"


def _agg_mse(x, deq_bits, dtype):
    y = deq_bits.view(np.uint16).astype(np.uint32) << 16 if dtype == torch.bfloat16 else deq_bits
    y = np.asarray(y).view(np.float32) if dtype == torch.bfloat16 else y
    return float(np.mean((x.astype(np.float64) - y.astype(np.float64)) ** 2))


def nvfp4_parity(w: torch.Tensor, importance=None, rows_sample=None):
    """Quantize w on the GPU, compare (optionally a sample of rows) with the oracle."""
    wd = w.to(DEV)
    imp_d = None if importance is None else importance.to(DEV)
    r = fq.nvfp4_quantize(wd, importance=imp_d)
    torch.cuda.synchronize()
    assert fq.check_status(r.status) == 0
    x_full = w.float().numpy()
    gmax = oracle.global_absmax(x_full)
    assert _np(r.amax)[0] == gmax
    S = oracle.global_scale(gmax)
    _assert_eq("S", _np(r.global_scale), np.array([S], np.float32))
    idx = np.arange(x_full.shape[0]) if rows_sample is None else np.asarray(rows_sample)
    x = np.ascontiguousarray(x_full[idx])
    window = oracle.NVFP4_MSE_WINDOW if importance is None else oracle.NVFP4_WMSE_WINDOW
    o = oracle.nvfp4_quant(x, S=S, importance=None if importance is None else importance.numpy(),
                           window=window)
    _assert_eq("scales", _np(r.scales)[idx], o["scales"])
    _assert_eq("codes", _np(r.codes)[idx], o["codes"])
    _assert_eq("block_loss", _np(r.block_loss)[idx], o["loss"])
    deq = _np(r.deq)[idx]
    _assert_eq("deq", deq, _deq_bits(o["y"], w.dtype))
    m_gpu = _agg_mse(x, deq, w.dtype)
    m_orc = _agg_mse(x, _deq_bits(o["y"], w.dtype), w.dtype)
    assert abs(m_gpu - m_orc) <= MSE_RTOL * max(m_orc, 1e-300)
    # the decoder reproduces the reconstruction
    back = fq.dequantize(fq.NVFP4, r.codes, r.scales, r.global_scale, dtype=w.dtype)
    _assert_eq("dequant", _np(back), _np(r.deq))
    return r, o


def mxfp4_parity(w: torch.Tensor, masks=None, rows_sample=None):
    wd = w.to(DEV)
    md = None if masks is None else torch.from_numpy(masks.view(np.int32)).to(DEV)
    r = fq.mxfp4_quantize(wd, md)
    torch.cuda.synchronize()
    assert fq.check_status(r.status) == 0
    idx = np.arange(w.shape[0]) if rows_sample is None else np.asarray(rows_sample)
    x = np.ascontiguousarray(w[torch.as_tensor(idx)].float().numpy())
    o = oracle.mxfp4_quant(x, sign_masks=masks)
    assert o["status"] == 0
    _assert_eq("scales", _np(r.scales)[idx], o["scales"])
    _assert_eq("codes", _np(r.codes)[idx], o["codes"])
    _assert_eq("block_loss", _np(r.block_loss)[idx], o["loss"])
    deq = _np(r.deq)[idx]
    _assert_eq("deq", deq, _deq_bits(o["y"], w.dtype))
    ref = o["rotated"]
    m_gpu = _agg_mse(ref, deq, w.dtype)
    m_orc = _agg_mse(ref, _deq_bits(o["y"], w.dtype), w.dtype)
    assert abs(m_gpu - m_orc) <= MSE_RTOL * max(m_orc, 1e-300)
    back = fq.dequantize(fq.MXFP4, r.codes, r.scales, None, dtype=w.dtype)
    _assert_eq("dequant", _np(back), _np(r.deq))
    return r, o


# --------------------------------------------------------------------------- small, ragged

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (37, 272), (300, 1040), (1000, 64)])
def test_nvfp4_mse_small(dtype, rows, cols):
    w = synth.q_proj(rows, cols, seed=rows * 7 + cols).to(dtype)
    nvfp4_parity(w)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 16), (37, 272), (300, 1040)])
def test_nvfp4_wmse_small(dtype, rows, cols):
    w = synth.t_weight(rows, cols, seed=rows + cols).to(dtype)
    imp = synth.importance_diag_xtx(cols=cols, tokens=64, seed=rows)
    nvfp4_parity(w, importance=imp)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (37, 288), (300, 1056)])
@pytest.mark.parametrize("hadamard", [False, True])
def test_mxfp4_small(dtype, rows, cols, hadamard):
    w = synth.t_weight(rows, cols, nu=3, scale=0.015, seed=rows * 3 + cols).to(dtype)
    masks = synth.sign_masks(cols, seed=rows) if hadamard else None
    mxfp4_parity(w, masks)


# --------------------------------------------------------------------------- the five workloads

def test_cfg1_small_outliers_fp32_with_bruteforce():
    """128x256 fp32 N(0,0.02) + 2 outliers/row: bit-exact, and the GPU's window
    minimum equals the oracle's exhaustive minimum over all 126 E4M3 scales."""
    w = synth.small_outliers()
    r, o = nvfp4_parity(w)
    bf = oracle.nvfp4_bruteforce(w.numpy(), o["S"])
    _assert_eq("bruteforce loss", _np(r.block_loss), bf["loss"])


def test_cfg2_q_proj_4096_full():
    nvfp4_parity(synth.q_proj(4096, 4096, seed=2))


def test_cfg3_wmse_11008x4096_full():
    w = synth.t_weight(11008, 4096, nu=4, scale=0.02, seed=3)
    imp = synth.importance_diag_xtx(cols=4096, tokens=2048, seed=3)
    nvfp4_parity(w, importance=imp)


def test_cfg4_mxfp4_hadamard_28672x8192_sampled():
    w = synth.t_weight(28672, 8192, nu=3, scale=0.015, seed=4, device=DEV).cpu()
    masks = synth.sign_masks(8192, seed=4)
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, 1, 28671], rng.integers(0, 28672, size=96)]))
    mxfp4_parity(w, masks, rows_sample=rows)


def test_cfg5_llama3_8b_sampled_tensors():
    """A sample of the 224 tensors (one of each shape, two layers), both formats."""
    shapes = synth.llama3_8b_shapes()
    rng = np.random.default_rng(5)
    for index in [0, 1, 2, 3, 4, 5, 6, 7 * 31 + 6]:
        name, rows, cols = shapes[index]
        w = synth.llama3_8b_tensor(index, rows, cols, device=DEV).cpu()
        sample = np.unique(np.concatenate([[0, rows - 1], rng.integers(0, rows, size=24)]))
        nvfp4_parity(w, rows_sample=sample)
        mxfp4_parity(w, rows_sample=sample)
