"""Pins of the oracle's ScaleSweep-inside-GPTQ routine (ScaleSweep summary,
"Contribuicoes" 2: the sweep selects block scales in RTN and GPTQ pipelines;
GPTQ in its Cholesky form, U^T U = H^-1).

Pinned against: the ScaleSweep RTN routine when H has no cross terms (U the
identity or diagonal: GPTQ then spreads no error and must reproduce RTN bit
for bit); an independent fp64 implementation of the optimal-brain-surgeon
form (explicit inverse of the remaining columns' Gram matrix, downdated after
every column), which the Cholesky form equals in exact arithmetic; and the
purpose of the method: a smaller H-weighted error than RTN."""
import numpy as np
import pytest

import synth


def _hessian(cols, tokens, seed, damp=0.01):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((tokens, cols))
    X[:, rng.choice(cols, max(1, cols // 100), replace=False)] *= 50.0      # a few hot input columns
    H = X.T @ X
    H += damp * np.mean(np.diag(H)) * np.eye(cols)
    return H


def _chol_upper_of_inverse(H):
    Hinv = np.linalg.inv(H)
    return np.linalg.cholesky(Hinv).T.astype(np.float32)                    # U^T U = H^-1


def test_identity_hessian_gives_scalesweep_rtn(orc):
    x = synth.q_proj(32, 256, seed=21).float().numpy()
    S = orc.global_scale(orc.global_absmax(x))
    g = orc.nvfp4_gptq(x, np.eye(256, dtype=np.float32), S=S)
    r = orc.nvfp4_quant(x, S=S)
    assert np.array_equal(g["codes"], r["codes"])
    assert np.array_equal(g["scales"], r["scales"])
    assert np.array_equal(g["y"].view(np.uint32), r["y"].view(np.uint32))


def test_diagonal_hessian_gives_scalesweep_rtn(orc):
    x = synth.q_proj(16, 128, seed=22).float().numpy()
    rng = np.random.default_rng(22)
    U = np.diag(rng.uniform(0.1, 3.0, 128)).astype(np.float32)
    g = orc.nvfp4_gptq(x, U)
    r = orc.nvfp4_quant(x, S=g["S"])
    assert np.array_equal(g["codes"], r["codes"]) and np.array_equal(g["scales"], r["scales"])


def _obs_fp64(orc, w_row, H, S):
    """Optimal-brain-surgeon GPTQ of one row in fp64 with explicit inverse
    downdates; the block scale of each 16-column group is the ScaleSweep of
    the group's current values (rounded to fp32, as the oracle sees them)."""
    cols = w_row.size
    w = w_row.astype(np.float64).copy()
    Hinv = np.linalg.inv(H)
    codes, scales = [], []
    d = inv = None
    for j in range(cols):
        if j % 16 == 0:
            blk = w[j:j + 16].astype(np.float32).reshape(1, 16)
            p = int(orc.nvfp4_quant(blk, S=S)["scales"][0, 0])
            scales.append(p)
            d = np.float32(np.float32(orc.e4m3_value(p)) * np.float32(S))
            inv = np.float32(np.float32(1.0) / d)
        r = np.float32(np.float32(w[j]) * inv)
        c = orc.e2m1_encode(float(r))
        y = np.float32(np.float32(orc.e2m1_decode(c)) * d)
        codes.append(c)
        e = (w[j] - float(y)) / Hinv[j, j]
        w[j:] -= e * Hinv[j, j:]
        Hinv = Hinv - np.outer(Hinv[:, j], Hinv[j, :]) / Hinv[j, j]
    return np.array(codes), np.array(scales)


def test_cholesky_form_equals_the_obs_form(orc):
    from fp64_check import unpack_nibbles
    rows, cols = 8, 64
    x = synth.q_proj(rows, cols, seed=23).float().numpy()
    H = _hessian(cols, 256, seed=23)
    U = _chol_upper_of_inverse(H)
    g = orc.nvfp4_gptq(x, U)
    nib = unpack_nibbles(g["codes"]).reshape(rows, cols)
    for r in range(rows):
        c, s = _obs_fp64(orc, x[r], H, g["S"])
        assert np.array_equal(g["scales"][r], s), r
        assert np.array_equal(nib[r], c), r


def test_gptq_lowers_the_weighted_error(orc):
    # GPTQ exploits correlated inputs: activations of rank 16 plus a little noise
    rows, cols = 64, 256
    x = synth.q_proj(rows, cols, seed=24).float().numpy()
    rng = np.random.default_rng(24)
    X = rng.standard_normal((1024, 16)) @ rng.standard_normal((16, cols)) + 0.1 * rng.standard_normal((1024, cols))
    H = X.T @ X
    H += 0.01 * np.mean(np.diag(H)) * np.eye(cols)
    g = orc.nvfp4_gptq(x, _chol_upper_of_inverse(H))
    r = orc.nvfp4_quant(x, S=g["S"])

    def werr(y):
        E = (x - y).astype(np.float64)
        return float(np.einsum("ij,jk,ik->", E, H, E))
    assert werr(g["y"]) < 0.5 * werr(r["y"])
