"""CPU simulation of the kernels' screen-then-verify NVFP4 selection, checked
against the oracle's exact search: the screened losses are computed as the
kernels compute them (binary32: r = RN(x*inv), q = E2M1(r), et = RN(q - r),
L = RN(L + et*et) or RN(L + RN(w*et)*et), lam = RN(v^2 * L)), the survivor
threshold as survivor_threshold does (upper bound of the norm from the block
maximum for MSE), and the oracle's winner must be among the survivors of every
block -- on the q_proj-shaped weight, the outlier matrix, the WMSE workload
and adversarial blocks that the grid reproduces exactly (zero loss).  The
survivors per block stay close to one (the verification is rare)."""
import numpy as np
import pytest

import synth
from fp64_check import e2m1_nearest, e4m3_values
from test_screen_threshold import kernel_threshold

V = e4m3_values().astype(np.float32)


def _screen(orc, x, S, lo, hi, w=None):
    f = np.float32
    xb = x.reshape(-1, 16).astype(np.float32)
    a = np.abs(xb)
    amax = a.max(1)
    t6 = f(6.0) * f(S)
    p = orc.e4m3_encode_array((amax / t6).astype(np.float32)).astype(np.int64)
    cand = np.clip(p[:, None] + np.arange(lo, hi + 1), 1, 126)
    v = V[cand]
    d = (v * f(S)).astype(np.float32)
    inv = (f(1) / d).astype(np.float32)
    r = (a[:, None, :] * inv[:, :, None]).astype(np.float32)
    _, q = e2m1_nearest(r)
    et = (np.abs(q).astype(np.float32) - r).astype(np.float32)
    if w is None:
        terms = et.astype(np.float64) ** 2
    else:
        wb = np.broadcast_to(w.reshape(1, -1), x.shape).reshape(-1, 16).astype(np.float32)
        terms = (wb[:, None, :] * et).astype(np.float32).astype(np.float64) * et
    L = np.zeros(et.shape[:2], np.float32)
    for i in range(16):
        L = (L.astype(np.float64) + terms[:, :, i]).astype(np.float32)
    lam = (L * (v * v).astype(np.float32)).astype(np.float32)
    invS = np.float32(1) / np.float32(S)
    if w is None:
        alpha2 = 16.0 * (amax * invS).astype(np.float64) ** 2 * (1 + 2 ** -16)
        tau = np.full(len(amax), (2.0 ** -70 / float(S)) ** 2 + 2.0 ** -120)
    else:
        wb = np.broadcast_to(w.reshape(1, -1), x.shape).reshape(-1, 16)
        alpha2 = (wb * (a * invS).astype(np.float64) ** 2).sum(1) * (1 + 2 ** -16)
        tau = ((2.0 ** -70 / float(S)) ** 2 + 2.0 ** -120) * (1 + wb.max(1))
    M = lam.min(1)
    T = np.array([float(kernel_threshold(M[i], alpha2[i], tau[i])) for i in range(len(M))])
    return cand, lam <= T[:, None]


def _check(orc, x, lo, hi, w=None, max_mean=1.05):
    S = orc.global_scale(orc.global_absmax(x))
    o = orc.nvfp4_quant(x, S=S, importance=w, window=(lo, hi))
    cand, surv = _screen(orc, x, S, lo, hi, w)
    win = o["scales"].reshape(-1)
    kept = (surv & (cand == win[:, None])).any(1)
    assert kept.all(), f"{int((~kept).sum())} winners excluded"
    ns = np.array([len(set(cand[i][surv[i]])) for i in range(len(win))])
    assert ns.mean() <= max_mean, ns.mean()


def test_q_proj_blocks(orc):
    _check(orc, synth.q_proj(128, 4096, seed=2).float().numpy(), -3, 7)


def test_outlier_blocks(orc):
    _check(orc, synth.small_outliers().numpy(), -3, 7)


def test_wmse_blocks(orc):
    x = synth.t_weight(64, 4096, seed=3).float().numpy()
    w = synth.importance_diag_xtx(cols=4096, tokens=2048, seed=3).numpy()
    _check(orc, x, -8, 7, w=w)


def test_blocks_reproduced_exactly(orc):
    rng = np.random.default_rng(0)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    xb = (grid[rng.integers(0, 8, size=(2048, 16))] * np.where(rng.random((2048, 16)) < .5, -1, 1)).astype(np.float32)
    xb[:, 0] = 6.0
    xb *= (2.0 ** rng.integers(-8, 2, size=(2048, 1))).astype(np.float32)
    # exact reproductions tie at zero loss in several candidates: many survive, none is lost
    _check(orc, xb.reshape(128, 256), -3, 7, max_mean=12.0)
