"""Independent fp64 recomputation used to pin the oracle (numpy only).

Given the method's per-candidate step size d and reciprocal inv (defined as
binary32 RN(E4M3(p)*S) and RN(1/d), or 2^e for MXFP4), this recomputes the
element codes by a nearest-grid search and the block loss in fp64, without
touching the oracle's C code.  The oracle's fp32 loss must agree with the
fp64 loss of the same candidate to within the rounding of a 16- or 32-term
sum, and its chosen candidate must be an fp64 minimiser up to that bound.
"""
import numpy as np

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_values() -> np.ndarray:
    """Value of every pattern 0..126 from the format (bias 7, subnormals)."""
    v = np.zeros(127)
    for p in range(1, 127):
        e, m = p >> 3, p & 7
        v[p] = m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10)
    return v


def e2m1_nearest(r: np.ndarray):
    """Magnitude code and signed value of the nearest E2M1 point (ties to even)."""
    a = np.minimum(np.abs(r.astype(np.float64)), 24.0)
    d = np.abs(a[..., None] - E2M1_GRID)
    dmin = d.min(axis=-1, keepdims=True)
    hit = d == dmin
    idx = np.argmax(hit, axis=-1)
    tie = hit.sum(axis=-1) > 1
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)
    sign = np.signbit(r)
    val = np.where(sign, -E2M1_GRID[idx], E2M1_GRID[idx])
    return idx | (sign.astype(np.int64) << 3), val


def block_losses(xb: np.ndarray, d32: np.ndarray, inv32: np.ndarray, w=None):
    """fp64 loss of each block under each candidate.

    xb: (nblocks, bs) float32; d32, inv32: (nblocks, ncand) float32;
    w: (nblocks, bs) float or None.  Returns (loss64 (nblocks, ncand),
    codes (nblocks, ncand, bs), y32 (nblocks, ncand, bs) = RN32(q*d)).
    """
    r = (xb[:, None, :] * inv32[:, :, None]).astype(np.float32)   # binary32 RN product
    codes, q = e2m1_nearest(r)
    y64 = q * d32[:, :, None].astype(np.float64)                   # exact in fp64
    y32 = y64.astype(np.float32)
    err = xb[:, None, :].astype(np.float64) - y32.astype(np.float64)
    e2 = err * err
    if w is not None:
        e2 = e2 * np.asarray(w, dtype=np.float64)[:, None, :]
    return e2.sum(axis=-1), codes, y32


def unpack_nibbles(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(c.size * 2, dtype=np.uint8)
    out[0::2] = c & 15
    out[1::2] = c >> 4
    return out
