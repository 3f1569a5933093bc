"""Pins for the oracle's NVFP4 ScaleSweep (CPU only).

Source: ScaleSweep technical summary (gist.science, arXiv 2606.07618),
"Metodologia: ScaleSweep": sec. 1 (MSE and importance-weighted MSE), sec. 2
(S = max|x| / (256*6); s_base = block max rounded to FP8; Lemma 4.1 upper
bound 12/7 s_base -> +7; Lemma 4.3 lower bound 4/5 s_base -> -3; WMSE
empirical lower bound 1/2 s_base -> -8; naive sweep over all 126 scales),
sec. 3 (sweep the window, keep the best candidate).
"""
import os

import numpy as np
import pytest
import torch

import synth
from fp64_check import block_losses, e4m3_values, unpack_nibbles

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL_SUM = 4e-6          # rounding of a 16-term binary32 sequential sum of squares


def _e4m3_f32(p):
    return e4m3_values()[np.asarray(p)].astype(np.float32)


def _window_candidates(base, lo, hi):
    k = np.arange(lo, hi + 1)
    return np.clip(base[..., None].astype(np.int64) + k, 1, 126)


# --------------------------------------------------------------------------- window offsets

def _normal_patterns():
    return np.arange(16, 119)     # keep p-8 .. p+8 inside the normal range


def test_upper_offset_is_first_pattern_reaching_12_over_7():
    v = e4m3_values()
    need = [next(k for k in range(1, 9) if v[p + k] >= 12 / 7 * v[p]) for p in _normal_patterns()]
    import oracle
    assert max(need) == 7 == oracle.NVFP4_MSE_WINDOW[1] == oracle.NVFP4_WMSE_WINDOW[1]
    assert min(need) == 6          # +6 is not enough for every mantissa


def test_lower_offsets_cover_4_over_5_and_one_half():
    v = e4m3_values()
    mse = [max(k for k in range(0, 12) if v[p - k] >= 0.8 * v[p]) for p in _normal_patterns()]
    wmse = [max(k for k in range(0, 12) if v[p - k] >= 0.5 * v[p]) for p in _normal_patterns()]
    import oracle
    assert max(mse) == 3 == -oracle.NVFP4_MSE_WINDOW[0]
    assert max(wmse) == 8 == -oracle.NVFP4_WMSE_WINDOW[0]
    assert all(v[p - 8] == v[p] / 2 for p in _normal_patterns())


# --------------------------------------------------------------------------- global scale

@pytest.mark.parametrize("k", [-20, -10, -1, 0, 3, 17])
def test_global_scale_closed_form(orc, k):
    gmax = np.float32(1536.0 * 2.0 ** k)
    assert orc.global_scale(gmax) == np.float32(2.0 ** k)


def test_global_scale_specials(orc):
    assert orc.global_scale(3.0) == np.float32(2.0 ** -9)
    assert orc.global_scale(0.0) == 1.0
    assert orc.gmax_status(np.inf) == orc.STATUS_NONFINITE
    assert orc.gmax_status(np.nan) == orc.STATUS_NONFINITE
    assert orc.gmax_status(2.0 ** -65) == orc.STATUS_RANGE
    assert orc.gmax_status(2.0 ** 65) == orc.STATUS_RANGE
    assert orc.gmax_status(0.0) == orc.STATUS_OK
    assert orc.gmax_status(2.0 ** -64) == orc.STATUS_OK


def test_global_absmax_and_nan(orc):
    x = np.array([0.5, -3.25, 1.0, -0.0], dtype=np.float32)
    assert orc.global_absmax(x) == np.float32(3.25)
    x[2] = np.nan
    assert np.isnan(orc.global_absmax(x))


def test_max_block_gets_s_base_256(orc):
    """The block holding max|x| has s_base = E4M3(256) = 0x78 (the 256 of S = max/(256*6))."""
    x = synth.small_outliers().numpy()
    out = orc.nvfp4_quant(x)
    a = np.abs(x).reshape(-1, 16).max(axis=1)
    top = a == a.max()
    assert np.all(out["base"].reshape(-1)[top] == 0x78)


# --------------------------------------------------------------------------- exact blocks

def _read_golden():
    blocks, cur = [], None
    with open(os.path.join(GOLDEN, "nvfp4_exact_blocks.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "block":
                cur = {}
                blocks.append(cur)
            elif key == "d":
                cur["d"] = float(vals[0])
            elif key == "scale":
                cur["scale"] = int(vals[0], 16)
            elif key == "x_over_d":
                cur["x_over_d"] = [float(v) for v in vals]
            elif key == "nibbles":
                cur["nibbles"] = [int(v, 16) for v in vals]
            elif key == "bytes":
                cur["bytes"] = [int(v, 16) for v in vals]
    return blocks


def test_hand_derived_exact_blocks(orc):
    blocks = _read_golden()
    x = np.concatenate([np.array(b["x_over_d"], dtype=np.float64) * b["d"] for b in blocks])
    x = x.astype(np.float32).reshape(1, -1)
    out = orc.nvfp4_quant(x)
    assert out["S"] == np.float32(2.0 ** -10)
    np.testing.assert_array_equal(out["scales"].reshape(-1), [b["scale"] for b in blocks])
    np.testing.assert_array_equal(out["codes"].reshape(-1), sum((b["bytes"] for b in blocks), []))
    np.testing.assert_array_equal(unpack_nibbles(out["codes"]), sum((b["nibbles"] for b in blocks), []))
    np.testing.assert_array_equal(out["loss"], 0.0)
    np.testing.assert_array_equal(out["y"], x)
    assert np.signbit(out["y"][0, 15]) and np.signbit(x[0, 15])


def test_all_zero_tensor(orc):
    x = np.zeros((2, 32), dtype=np.float32)
    out = orc.nvfp4_quant(x)
    assert out["S"] == 1.0
    np.testing.assert_array_equal(out["scales"], 1)      # first candidate max(1, 0-3)
    np.testing.assert_array_equal(out["codes"], 0)
    np.testing.assert_array_equal(out["loss"], 0.0)


def test_single_nonzero_block_closed_form(orc):
    """One value v in an otherwise zero tensor: S = v/1536, s_base = 0x78, and the
    best candidate's loss is (v - RN32(q*d))^2 for its own q (one term)."""
    for v in [0.02, 1.0, 3.7, 1e-5, 123.456]:
        x = np.zeros((1, 16), dtype=np.float32)
        x[0, 5] = np.float32(v)
        out = orc.nvfp4_quant(x)
        S = np.float32(np.float32(v) / np.float32(1536.0))
        assert out["S"] == S and out["base"][0, 0] == 0x78
        cands = np.arange(0x75, 0x7F)
        d = (_e4m3_f32(cands) * S).astype(np.float32)
        inv = (np.float32(1.0) / d).astype(np.float32)
        loss, _, y = block_losses(x.reshape(1, 16), d[None], inv[None])
        k = int(out["scales"][0, 0]) - 0x75
        assert loss[0, k] == loss[0].min()
        assert out["loss"][0, 0] == np.float32(loss[0, k])     # single term: exact
        np.testing.assert_array_equal(out["y"][0], y[0, k])


# --------------------------------------------------------------------------- fp64 recomputation

def _check_against_fp64(x, out, S, window, w=None):
    xb = x.reshape(-1, 16)
    base = out["base"].reshape(-1)
    cand = _window_candidates(base, *window)
    d = (_e4m3_f32(cand) * np.float32(S)).astype(np.float32)
    inv = (np.float32(1.0) / d).astype(np.float32)
    wb = None if w is None else np.broadcast_to(w.reshape(1, -1), x.shape).reshape(-1, 16)
    loss64, codes, y32 = block_losses(xb, d, inv, wb)
    chosen = out["scales"].reshape(-1)
    k = np.argmax(cand == chosen[:, None], axis=1)
    assert np.all(cand[np.arange(cand.shape[0]), k] == chosen)
    picked = loss64[np.arange(len(k)), k]
    best = loss64.min(axis=1)
    # the fp32 argmin is an fp64 minimiser up to the rounding of the sums
    assert np.all(picked <= best * (1 + 2 * RTOL_SUM) + 1e-37)
    # the reported fp32 loss is the fp64 loss of the chosen candidate
    np.testing.assert_allclose(out["loss"].reshape(-1), picked, rtol=RTOL_SUM, atol=1e-37)
    # codes and reconstruction are exactly those of the chosen candidate
    np.testing.assert_array_equal(unpack_nibbles(out["codes"]).reshape(-1, 16),
                                  codes[np.arange(len(k)), k])
    np.testing.assert_array_equal(out["y"].reshape(-1, 16), y32[np.arange(len(k)), k])
    # s_base: amax / RN(6 S) rounded to E4M3
    amax = np.abs(xb).max(axis=1)
    v = (amax / np.float32(np.float32(6.0) * np.float32(S))).astype(np.float32)
    np.testing.assert_array_equal(base, orc_encode_array(v))
    return picked, best


def orc_encode_array(v):
    import oracle
    return oracle.e4m3_encode_array(np.ascontiguousarray(v, dtype=np.float32))


def test_mse_sweep_against_fp64(orc):
    x = synth.small_outliers().numpy()
    out = orc.nvfp4_quant(x)
    S = orc.global_scale(orc.global_absmax(x))
    assert out["S"] == S
    _check_against_fp64(x, out, S, orc.NVFP4_MSE_WINDOW)


def test_wmse_sweep_against_fp64(orc):
    x = synth.t_weight(96, 512, seed=31).float().numpy()
    w = synth.importance_diag_xtx(cols=512, tokens=256, seed=31).numpy()
    out = orc.nvfp4_quant(x, importance=w, window=orc.NVFP4_WMSE_WINDOW)
    _check_against_fp64(x, out, out["S"], orc.NVFP4_WMSE_WINDOW, w=w)


def test_sweep_not_worse_than_absmax(orc):
    x = synth.q_proj(64, 512, seed=7).float().numpy()
    sweep = orc.nvfp4_quant(x)
    absmax = orc.nvfp4_quant(x, window=(0, 0))
    assert np.all(sweep["loss"] <= absmax["loss"])
    assert sweep["loss"].sum() < absmax["loss"].sum()
    np.testing.assert_array_equal(absmax["scales"], absmax["base"])


# --------------------------------------------------------------------------- brute force (Lemmas 4.1/4.3)

def test_window_reaches_bruteforce_optimum_mse(orc):
    """On the 128x256 outlier matrix the -3..+7 window attains the minimum over
    all 126 E4M3 scales in every block, bit for bit."""
    x = synth.small_outliers().numpy()
    out = orc.nvfp4_quant(x)
    bf = orc.nvfp4_bruteforce(x, out["S"])
    np.testing.assert_array_equal(out["loss"], bf["loss"])
    same = out["scales"] == bf["pattern"]
    # where the first minimiser differs, the window's pick is a tie of the optimum
    assert np.all(same | (bf["ties"] > 1))


def test_window_reaches_bruteforce_optimum_mse_heavy_tails(orc):
    x = synth.q_proj(64, 1024, seed=8).float().numpy()
    out = orc.nvfp4_quant(x)
    bf = orc.nvfp4_bruteforce(x, out["S"])
    np.testing.assert_array_equal(out["loss"], bf["loss"])


def test_wmse_window_is_a_subsearch(orc):
    x = synth.t_weight(64, 512, seed=9).float().numpy()
    w = synth.importance_diag_xtx(cols=512, tokens=256, seed=9).numpy()
    out = orc.nvfp4_quant(x, importance=w, window=orc.NVFP4_WMSE_WINDOW)
    bf = orc.nvfp4_bruteforce(x, out["S"], importance=w)
    assert np.all(out["loss"] >= bf["loss"])
    # the lower bound is empirical on the page; it holds for most blocks
    assert np.mean(out["loss"] == bf["loss"]) > 0.95


# --------------------------------------------------------------------------- dequant

def test_dequant_reproduces_reconstruction(orc):
    x = synth.q_proj(32, 256, seed=10).float().numpy()
    out = orc.nvfp4_quant(x)
    y = orc.nvfp4_dequant(out["codes"], out["scales"], out["S"], 32, 256)
    np.testing.assert_array_equal(y, out["y"])
    yb = orc.bf16_round(out["y"])
    want = torch.from_numpy(out["y"]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(yb, want)


def test_threads_do_not_change_results(orc):
    x = synth.q_proj(64, 256, seed=12).float().numpy()
    a = orc.nvfp4_quant(x, threads=1)
    b = orc.nvfp4_quant(x, threads=4)
    for k in ("codes", "scales", "y", "loss"):
        np.testing.assert_array_equal(a[k], b[k])
