"""Pins for the oracle's number-format codecs (CPU only).

The E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6} with ties to even and saturation,
the E4M3 format with exactly 126 positive finite values (ScaleSweep summary,
"Limites Teoricos para Varredura Eficiente") and the E8M0 power-of-two scale
(MR-GPTQ summary, section 1) are checked against brute-force nearest-value
search written here in numpy fp64, independently of the oracle's C code.
"""
import numpy as np
import pytest
import torch

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _nearest_even(values: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest table entry to each value; ties to the even index.

    Values beyond 4x the largest entry are clipped there first (their nearest
    entry is the largest one either way), so every fp64 distance is exact.
    """
    out = np.empty(values.shape, dtype=np.int64)
    cap = 4.0 * float(table[-1])
    for s in range(0, values.size, 1 << 20):
        v = np.minimum(values[s:s + (1 << 20)].astype(np.float64), cap)
        d = np.abs(v[:, None] - table[None, :])
        dmin = d.min(axis=1, keepdims=True)
        hit = d == dmin
        idx = np.argmax(hit, axis=1)
        # a tie has exactly two nearest entries, adjacent: take the even one
        tie = hit.sum(axis=1) > 1
        idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)
        out[s:s + (1 << 20)] = idx
    return out


def _around(points, ulps, lo=0.0):
    pts = np.asarray(points, dtype=np.float32)
    bits = pts.view(np.uint32).astype(np.int64)
    offs = np.arange(-ulps, ulps + 1, dtype=np.int64)
    b = (bits[:, None] + offs[None, :]).reshape(-1)
    b = b[(b >= 0) & (b < 0x7F800000)]
    v = b.astype(np.uint32).view(np.float32)
    return v[v >= lo]


def _random_finite(rng, n):
    b = rng.integers(0, 0x7F800000, size=n, dtype=np.int64).astype(np.uint32)
    return b.view(np.float32)


# --------------------------------------------------------------------------- E2M1

def test_e2m1_decode_is_the_format_grid(orc):
    mags = [orc.e2m1_decode(c) for c in range(8)]
    assert mags == list(E2M1_GRID)
    for c in range(8):
        neg = orc.e2m1_decode(8 | c)
        assert neg == -E2M1_GRID[c] and np.signbit(neg)


@pytest.mark.parametrize("r,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    (0.0, 0), (0.5, 1), (6.0, 7), (7.0, 7), (1e30, 7), (0.2499999, 0), (0.2500001, 1),
    (4.9999995, 6), (5.0000005, 7),
])
def test_e2m1_tie_table(orc, r, code):
    assert orc.e2m1_encode(r) == code
    assert orc.e2m1_encode(-r) == 8 | code


def test_e2m1_negative_zero_keeps_sign(orc):
    assert orc.e2m1_encode(-0.1) == 0x8
    assert orc.e2m1_encode(-0.0) == 0x8
    assert orc.e2m1_encode(0.0) == 0x0


def test_e2m1_encode_matches_nearest_search(orc):
    rng = np.random.default_rng(11)
    mids = (E2M1_GRID[:-1] + E2M1_GRID[1:]) / 2
    near = np.concatenate([_around(mids, 4096), _around(E2M1_GRID[1:], 4096)])
    rnd = np.concatenate([_random_finite(rng, 1 << 20),
                          rng.uniform(0, 8, size=1 << 20).astype(np.float32)])
    v = np.concatenate([near, rnd]).astype(np.float32)
    v = np.concatenate([v, -v])
    got = orc.e2m1_encode_array(v)
    want = _nearest_even(np.abs(v), E2M1_GRID) | (np.signbit(v).astype(np.int64) << 3)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first r={v[bad[0]]!r} got {got[bad[0]]} want {want[bad[0]]}"


# --------------------------------------------------------------------------- E4M3

def _e4m3_value_set():
    """Positive finite E4M3 values from the format: subnormal m*2^-9, normal (8+m)*2^(e-10)."""
    vals = [m * 2.0 ** -9 for m in range(1, 8)]
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue            # the NaN pattern
            vals.append((8 + m) * 2.0 ** (e - 10))
    return np.array(sorted(vals))


def test_e4m3_has_126_positive_finite_values(orc):
    ref = _e4m3_value_set()
    assert ref.size == 126              # the count the ScaleSweep summary states
    got = np.array([orc.e4m3_value(p) for p in range(1, 127)])
    np.testing.assert_array_equal(got, ref)    # monotone in the bit pattern
    assert orc.e4m3_value(0) == 0.0
    assert np.isnan(orc.e4m3_value(0x7F))
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(1) == 2.0 ** -9
    assert orc.e4m3_value(0x80 | 0x38) == -1.0


def test_e4m3_encode_matches_nearest_search(orc):
    rng = np.random.default_rng(12)
    table = np.concatenate([[0.0], _e4m3_value_set()])
    mids = (table[:-1] + table[1:]) / 2
    v = np.concatenate([
        _around(mids, 512), _around(table[1:], 512),
        np.exp2(rng.uniform(-14, 10, size=1 << 20)).astype(np.float32),
        _random_finite(rng, 1 << 18),
        np.array([0.0, 448.0, 449.0, 464.0, 480.0, 1e30, 2.0 ** -10, 2.0 ** -11], np.float32),
    ]).astype(np.float32)
    got = orc.e4m3_encode_array(v)
    want = _nearest_even(v, table)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first v={v[bad[0]]!r} got {got[bad[0]]} want {want[bad[0]]}"


def test_e4m3_roundtrip(orc):
    for p in range(127):
        assert orc.e4m3_encode(orc.e4m3_value(p)) == p


# --------------------------------------------------------------------------- E8M0, bf16

def test_e8m0_is_power_of_two(orc):
    for b in range(255):
        assert orc.e8m0_value(b) == 2.0 ** (b - 127)
    assert np.isnan(orc.e8m0_value(255))


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(13)
    x = np.concatenate([_random_finite(rng, 1 << 18), -_random_finite(rng, 1 << 18),
                        (np.arange(1 << 16, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    x = x[np.isfinite(x)]
    got = orc.bf16_round(x)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)
