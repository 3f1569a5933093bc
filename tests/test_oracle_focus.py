"""Pins of the oracle's FOCUS forward quantizer and of the inverse block
Hadamard ("FOCUS" summary, "Metodologia" 2-3: S_q = S_dq * c_k per sub-block,
codes Q(W_k / S_q), reconstruction with S_dq; MR-GPTQ summary sec. 2: the
random-sign block Hadamard, here undone).

Pinned against: the ScaleSweep and MXFP4 routines (c = 1 is the coupled
baseline the page starts from, so FOCUS must reproduce them exactly); the
exact power-of-two invariance of MXFP4 scales (c = 2 at exponent e quantizes
like c = 1 at e + 1); sub-block independence; the independent decoder; a
brute-force nearest-grid search in fp64; and, for the inverse rotation, the
dense Sylvester matrix (scipy) and the round trip, within their rounding
bounds."""
import numpy as np
import pytest
from scipy.linalg import hadamard

import synth
from fp64_check import unpack_nibbles

GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def _coeffs(rows, cols, sub, seed, lo=0.8, hi=1.25):
    rng = np.random.default_rng(seed)
    return rng.uniform(lo, hi, size=(rows, cols // sub)).astype(np.float16)


def test_nvfp4_c1_is_the_scalesweep_result(orc):
    x = synth.q_proj(64, 512, seed=3).float().numpy()
    S = orc.global_scale(orc.global_absmax(x))
    ss = orc.nvfp4_quant(x, S=S)
    ones = np.ones((64, 512 // 8), dtype=np.float16)
    f = orc.focus_quant(0, x, ss["scales"], ones, 8, S=S)
    assert f["status"] == 0
    assert np.array_equal(f["codes"], ss["codes"])
    assert np.array_equal(f["y"].view(np.uint32), ss["y"].view(np.uint32))
    assert np.array_equal(f["loss"].view(np.uint32), ss["loss"].view(np.uint32))


def test_mxfp4_c1_is_the_mxfp4_result(orc):
    x = synth.q_proj(32, 256, seed=4).float().numpy()
    mx = orc.mxfp4_quant(x)
    f = orc.focus_quant(1, x, mx["scales"], np.ones((32, 256 // 8), np.float16), 8)
    assert f["status"] == 0
    assert np.array_equal(f["codes"], mx["codes"])
    assert np.array_equal(f["y"].view(np.uint32), mx["y"].view(np.uint32))
    assert np.array_equal(f["loss"].view(np.uint32), mx["loss"].view(np.uint32))


def test_mxfp4_power_of_two_coefficient_shifts_the_exponent(orc):
    x = synth.q_proj(16, 256, seed=5).float().numpy()
    mx = orc.mxfp4_quant(x)
    twos = np.full((16, 256 // 8), 2.0, np.float16)
    a = orc.focus_quant(1, x, mx["scales"], twos, 8)
    b = orc.focus_quant(1, x, mx["scales"] + 1, np.ones_like(twos), 8)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["y"], b["y"] / 2)               # same codes, half the stored step


def test_sub_blocks_are_independent(orc):
    x = synth.q_proj(8, 128, seed=6).float().numpy()
    S = orc.global_scale(orc.global_absmax(x))
    sc = orc.nvfp4_quant(x, S=S)["scales"]
    c = _coeffs(8, 128, 8, seed=6)
    a = orc.focus_quant(0, x, sc, c, 8, S=S)
    c2 = c.copy()
    c2[3, 5] = np.float16(0.55)                              # elements 40..47 of row 3
    b = orc.focus_quant(0, x, sc, c2, 8, S=S)
    na, nb = unpack_nibbles(a["codes"]).reshape(8, 128), unpack_nibbles(b["codes"]).reshape(8, 128)
    diff = np.argwhere(na != nb)
    assert diff.size > 0
    assert all(r == 3 and 40 <= col < 48 for r, col in diff)


@pytest.mark.parametrize("fmt,sub", [(0, 8), (0, 16), (0, 4), (1, 8), (1, 32)])
def test_codes_are_nearest_grid_points_and_decode(orc, fmt, sub):
    rows, cols = 32, 256
    x = synth.q_proj(rows, cols, seed=7 + sub).float().numpy()
    if fmt == 0:
        S = orc.global_scale(orc.global_absmax(x))
        sc = orc.nvfp4_quant(x, S=S)["scales"]
        d = np.array([orc.e4m3_value(int(p)) for p in range(256) if p < 127] + [0] * 129, np.float32)[sc] \
            * np.float32(S)
        bs = 16
    else:
        S = 1.0
        sc = orc.mxfp4_quant(x)["scales"]
        d = np.ldexp(np.float32(1), sc.astype(np.int32) - 127).astype(np.float32)
        bs = 32
    c = _coeffs(rows, cols, sub, seed=sub)
    f = orc.focus_quant(fmt, x, sc, c, sub, S=S)
    assert f["status"] == 0
    # decode: the codes with the stored scales give y
    y_dec = orc.nvfp4_dequant(f["codes"], sc, S, rows, cols) if fmt == 0 else \
        orc.mxfp4_dequant(f["codes"], sc, rows, cols)
    assert np.array_equal(y_dec.view(np.uint32), f["y"].view(np.uint32))
    # codes: nearest grid point of x / (d * c) in fp64, wherever it is not a near tie
    dq = (np.repeat(d, bs, axis=1).astype(np.float32) * np.repeat(c.astype(np.float32), sub, axis=1)).astype(np.float64)
    r = np.abs(x.astype(np.float64) / dq)
    mag = unpack_nibbles(f["codes"]).reshape(rows, cols) & 7
    dist = np.abs(np.minimum(r, 6.0)[..., None] - GRID)
    best = np.argmin(dist, axis=-1)
    srt = np.sort(dist, axis=-1)
    clear = (srt[..., 1] - srt[..., 0]) > 1e-5 * np.maximum(r, 1.0)
    assert clear.mean() > 0.99
    assert np.array_equal(mag[clear], best[clear])


def test_invalid_scale_or_coefficient_flags_range(orc):
    x = synth.q_proj(2, 32, seed=8).float().numpy()
    sc = np.full((2, 2), 0x38, np.uint8)
    ones = np.ones((2, 4), np.float16)
    assert orc.focus_quant(0, x, sc, ones, 8)["status"] == 0
    bad = sc.copy(); bad[1, 1] = 0
    assert orc.focus_quant(0, x, bad, ones, 8)["status"] == orc.STATUS_RANGE
    c = ones.copy(); c[0, 2] = np.float16(-1.0)
    assert orc.focus_quant(0, x, sc, c, 8)["status"] == orc.STATUS_RANGE
    assert orc.focus_quant(1, x, np.full((2, 1), 255, np.uint8), ones, 8)["status"] == orc.STATUS_RANGE


def test_inverse_hadamard_matches_the_dense_matrix(orc):
    rng = np.random.default_rng(9)
    H = hadamard(32).astype(np.float64)
    c = float(orc.hadamard_scale())
    for _ in range(50):
        y = rng.standard_normal(32).astype(np.float32)
        mask = int(rng.integers(0, 2 ** 32))
        got = orc.hadamard32_inverse(y, mask).astype(np.float64)
        sig = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
        want = sig * (c * (H @ y.astype(np.float64)))
        bound = 8 * 2.0 ** -24 * (np.abs(H) @ np.abs(y.astype(np.float64))) * c + 1e-30
        assert np.all(np.abs(got - want) <= bound)


def test_unrotate_undoes_the_rotation(orc):
    x = synth.q_proj(16, 256, seed=10).float().numpy()
    masks = synth.sign_masks(256, seed=10)
    rot = orc.mxfp4_quant(x, sign_masks=masks)["rotated"]
    back = orc.mxfp4_unrotate(rot, masks).astype(np.float64)
    # forward and inverse: 2 x (5 rounded stages + 1 multiply), and c^2 * 32 = 1 + O(2^-24)
    err = np.abs(back - x.astype(np.float64))
    scale = np.abs(x).reshape(16, 8, 32).max(axis=2).repeat(32, axis=1) * np.sqrt(32)
    assert np.all(err <= 64 * 2.0 ** -24 * scale)
