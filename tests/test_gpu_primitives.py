"""GPU check of the device rounding primitives against the oracle's codecs.

The quantizer kernels round with the sm_100a conversions (E2M1 pairs and
E4M3); these probes run the same device helpers over dense sets of inputs --
every value within thousands of ulps of each rounding midpoint and grid point,
plus millions of random bit patterns -- and compare with the CPU codecs.  The
exhaustive tests then cover every finite binary32 input: all 2^32 - 2^24 bit
patterns for E2M1 (both signs) and all non-negative ones for E4M3 (the scale
argument amax / (6 S) is never negative).
"""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _around(points, ulps):
    bits = np.asarray(points, dtype=np.float32).view(np.uint32).astype(np.int64)
    b = (bits[:, None] + np.arange(-ulps, ulps + 1)[None, :]).reshape(-1)
    b = b[(b >= 0) & (b < 0x7F800000)]
    return b.astype(np.uint32).view(np.float32)


def _probe(fn, v: np.ndarray) -> np.ndarray:
    vd = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(DEV)
    out = torch.empty(v.size, dtype=torch.uint8, device=DEV)
    fn(vd, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_e2m1_conversion_matches_oracle():
    rng = np.random.default_rng(1)
    grid = np.array([0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    v = np.concatenate([
        _around(mids, 1 << 14), _around(grid, 1 << 12),
        rng.integers(0, 0x7F800000, size=1 << 23, dtype=np.int64).astype(np.uint32).view(np.float32),
        rng.uniform(0, 8, size=1 << 22).astype(np.float32),
        np.array([0.0, 1e-45, 1e38, 3.4e38], dtype=np.float32),
    ])
    v = np.concatenate([v, -v])
    got = _probe(fq.fp4q_probe_e2m1, v)
    want = oracle.e2m1_encode_array(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches; first r={v[bad[0]]!r} gpu={got[bad[0]]} oracle={want[bad[0]]}"


def test_e2m1_pair_order_and_odd_length():
    v = np.array([6.0, -0.5, 1.0, 3.0, -2.0], dtype=np.float32)
    got = _probe(fq.fp4q_probe_e2m1, v)
    np.testing.assert_array_equal(got, [0x7, 0x9, 0x2, 0x5, 0xC])


def test_e4m3_conversion_matches_oracle():
    rng = np.random.default_rng(2)
    vals = np.array([oracle.e4m3_value(p) for p in range(127)], dtype=np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    v = np.concatenate([
        _around(mids, 1 << 12), _around(vals[1:].astype(np.float32), 1 << 10),
        np.exp2(rng.uniform(-16, 12, size=1 << 22)).astype(np.float32),
        rng.integers(0, 0x7F800000, size=1 << 21, dtype=np.int64).astype(np.uint32).view(np.float32),
        np.array([0.0, 448.0, 449.0, 464.0, 465.0, 1e30, 2.0 ** -10, 2.0 ** -11], dtype=np.float32),
    ])
    got = _probe(fq.fp4q_probe_e4m3, v)
    want = oracle.e4m3_encode_array(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches; first v={v[bad[0]]!r} gpu={got[bad[0]]} oracle={want[bad[0]]}"


CHUNK = 1 << 26
FINITE_END = 0x7F800000          # first non-finite magnitude pattern (+Inf)


def _exhaustive(probe, encode, negative: bool):
    """Every finite pattern of one sign, CHUNK at a time: the inputs are made
    on the device (an int32 range viewed as binary32) and on the host (the same
    range as uint32), probed there, encoded by the oracle here, compared."""
    out = torch.empty(CHUNK, dtype=torch.uint8, device=DEV)
    base = 0x80000000 if negative else 0
    signed_base = -(1 << 31) if negative else 0
    for lo in range(0, FINITE_END, CHUNK):
        hi = min(lo + CHUNK, FINITE_END)
        vd = torch.arange(signed_base + lo, signed_base + hi, dtype=torch.int32, device=DEV).view(torch.float32)
        probe(vd, out[:hi - lo])
        got = out[:hi - lo].cpu().numpy()
        v = np.arange(base + lo, base + hi, dtype=np.uint32).view(np.float32)
        want = encode(v)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (f"{bad.size} mismatches in [{base + lo:#x}, {base + hi:#x}); first "
                               f"bits={int(v[bad[0]:bad[0] + 1].view(np.uint32)[0]):#x} gpu={got[bad[0]]} "
                               f"oracle={want[bad[0]]}")


@pytest.mark.parametrize("negative", [False, True])
def test_e2m1_conversion_every_finite_input(negative):
    _exhaustive(fq.fp4q_probe_e2m1, oracle.e2m1_encode_array, negative)


def test_e4m3_conversion_every_nonnegative_finite_input():
    _exhaustive(fq.fp4q_probe_e4m3, oracle.e4m3_encode_array, False)
