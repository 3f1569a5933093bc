"""Pins for the oracle's MXFP4 path and block Hadamard (CPU only).

Sources: "Bridging the Gap Between Promise and Performance for Microscaling
FP4 Quantization" (gist.science, arXiv 2509.23202), technical summary sec. 1
(MXFP4: 32-element groups, power-of-two E8M0 scales) and sec. 2 (MSE-optimised
grid; fused block Hadamard micro-rotation, orthogonal); TORQ summary (arXiv
2605.19561) sec. 2.B (S-step maps the block maximum onto the largest code).
The e0-1..e0+1 window itself has no optimality statement on the pages: beyond
the defined computation it is parity unpinned; an fp64 brute force over twelve
exponents finds the window's choice optimal in every block of two heavy-tailed
synthetic weights (an observation, not a claim of the pages).
"""
import numpy as np
import pytest
from scipy.linalg import hadamard

import synth
from fp64_check import block_losses, unpack_nibbles

RTOL_SUM32 = 6e-6        # rounding of a 32-term binary32 sequential sum of squares


def test_hadamard_scale_is_rn_inverse_sqrt32(orc):
    c = np.float32(1.0 / np.sqrt(np.float64(32.0)))
    assert np.float32(orc.hadamard_scale()) == c
    assert np.float32(orc.hadamard_scale()).view(np.uint32) == 0x3E3504F3


@pytest.mark.parametrize("j", [0, 1, 5, 16, 31])
@pytest.mark.parametrize("mask", [0, 0xFFFFFFFF, 0xA5A5A5A5])
def test_hadamard_basis_vectors_closed_form(orc, j, mask):
    x = np.zeros(32, dtype=np.float32)
    x[j] = 1.0
    y = orc.hadamard32(x, mask)
    c = np.float32(orc.hadamard_scale())
    sigma = -1.0 if (mask >> j) & 1 else 1.0
    want = np.array([sigma * (-1) ** bin(i & j).count("1") for i in range(32)], dtype=np.float32) * c
    np.testing.assert_array_equal(y, want)


def test_hadamard_matches_sylvester_matrix(orc):
    rng = np.random.default_rng(3)
    H = hadamard(32).astype(np.float64)          # natural (Sylvester) order
    for _ in range(50):
        x = (rng.standard_t(3, size=32) * 0.02).astype(np.float32)
        mask = int(rng.integers(0, 2 ** 32))
        sig = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(32)])
        want = H @ (sig * x.astype(np.float64)) / np.sqrt(32.0)
        got = orc.hadamard32(x, mask).astype(np.float64)
        # 5 stages of rounded adds plus one rounded multiply
        bound = 8 * 2.0 ** -24 * np.sqrt(32.0) * np.abs(x).max() * 6
        assert np.max(np.abs(got - want)) <= bound


def test_hadamard_is_orthogonal(orc):
    rng = np.random.default_rng(4)
    x = rng.standard_normal(32).astype(np.float32)
    y = orc.hadamard32(x, 0)
    z = orc.hadamard32(y, 0)
    np.testing.assert_allclose(z, x, rtol=0, atol=1e-5 * np.abs(x).max())
    assert abs(np.sum(y.astype(np.float64) ** 2) / np.sum(x.astype(np.float64) ** 2) - 1) < 1e-6


@pytest.mark.parametrize("amax,e0", [(0.0, -127), (6.0, 0), (6.0000005, 1), (3.0, -1), (4.0, 0),
                                     (1.5, -2), (1.5000001, -1), (2.0 ** -130, -127),
                                     (3.0e38, 126)])
def test_centre_exponent_cases(orc, amax, e0):
    assert orc.mx_centre_exponent(amax) == e0


def test_centre_exponent_property(orc):
    rng = np.random.default_rng(5)
    a = np.exp2(rng.uniform(-120, 120, size=20000)).astype(np.float32)
    for v in a:
        e = orc.mx_centre_exponent(v)
        assert 6.0 * 2.0 ** e >= v and 6.0 * 2.0 ** (e - 1) < v


def test_grid_exact_blocks(orc):
    rng = np.random.default_rng(6)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    rows = []
    ks = [-10, -3, 0, 4]
    for k in ks:
        g = grid[rng.integers(0, 8, size=32)] * np.where(rng.random(32) < 0.5, -1, 1)
        g[3] = 6.0
        rows.append(g * 2.0 ** k)
    x = np.array(rows, dtype=np.float32).reshape(len(ks), 32)
    out = orc.mxfp4_quant(x)
    assert out["status"] == 0
    np.testing.assert_array_equal(out["scales"].reshape(-1), np.array(ks) + 127)
    np.testing.assert_array_equal(out["loss"], 0.0)
    np.testing.assert_array_equal(out["y"], x)


def _check_mx_against_fp64(v, out):
    vb = v.reshape(-1, 32)
    amax = np.abs(vb).max(axis=1)
    import oracle
    e0 = np.array([oracle.mx_centre_exponent(a) for a in amax])
    cand = np.clip(e0[:, None] + np.arange(-1, 2), -127, 127)
    d = np.exp2(cand.astype(np.float64)).astype(np.float32)
    inv = np.exp2(-cand.astype(np.float64)).astype(np.float32)
    loss64, codes, y32 = block_losses(vb, d, inv)
    chosen = out["scales"].reshape(-1).astype(np.int64) - 127
    k = np.argmax(cand == chosen[:, None], axis=1)
    assert np.all(cand[np.arange(len(k)), k] == chosen)
    picked = loss64[np.arange(len(k)), k]
    assert np.all(picked <= loss64.min(axis=1) * (1 + 2 * RTOL_SUM32) + 1e-37)
    np.testing.assert_allclose(out["loss"].reshape(-1), picked, rtol=RTOL_SUM32, atol=1e-37)
    np.testing.assert_array_equal(unpack_nibbles(out["codes"]).reshape(-1, 32), codes[np.arange(len(k)), k])
    np.testing.assert_array_equal(out["y"].reshape(-1, 32), y32[np.arange(len(k)), k])


def test_mxfp4_plain_against_fp64(orc):
    x = synth.t_weight(64, 512, nu=3, scale=0.015, seed=21).float().numpy()
    out = orc.mxfp4_quant(x)
    assert out["status"] == 0
    np.testing.assert_array_equal(out["rotated"], x)
    _check_mx_against_fp64(x, out)


def test_mxfp4_hadamard_against_fp64(orc):
    x = synth.t_weight(64, 512, nu=3, scale=0.015, seed=22).float().numpy()
    masks = synth.sign_masks(512, seed=22)
    out = orc.mxfp4_quant(x, sign_masks=masks)
    assert out["status"] == 0
    rot = np.stack([np.concatenate([orc.hadamard32(x[r, 32 * g:32 * g + 32], masks[g])
                                    for g in range(16)]) for r in range(64)])
    np.testing.assert_array_equal(out["rotated"], rot)
    _check_mx_against_fp64(rot, out)


def test_mxfp4_sweep_not_worse_than_centre(orc):
    """Loss at the chosen exponent never exceeds the loss at e0 (fp64 check)."""
    x = synth.t_weight(32, 1024, nu=3, scale=0.015, seed=23).float().numpy()
    out = orc.mxfp4_quant(x)
    xb = x.reshape(-1, 32)
    import oracle
    e0 = np.array([oracle.mx_centre_exponent(a) for a in np.abs(xb).max(axis=1)])
    d = np.exp2(e0.astype(np.float64)).astype(np.float32)[:, None]
    inv = np.exp2(-e0.astype(np.float64)).astype(np.float32)[:, None]
    l0, _, _ = block_losses(xb, d, inv)
    assert np.all(out["loss"].reshape(-1) <= l0[:, 0] * (1 + 2 * RTOL_SUM32))


@pytest.mark.parametrize("nu,scale,seed", [(4, 0.02, 31), (3, 0.015, 32)])
def test_mxfp4_choice_is_the_best_of_all_exponents(orc, nu, scale, seed):
    """fp64 brute force over twelve exponents around floor(log2 amax) (found here
    with frexp, not with the oracle's centre rule): on heavy-tailed weights the
    oracle's exponent attains the least loss of all of them in every block, so
    the e0-1..e0+1 window and its centre are where the optimum lies."""
    x = synth.t_weight(256, 1024, nu=nu, scale=scale, seed=seed).float().numpy()
    out = orc.mxfp4_quant(x)
    xb = x.reshape(-1, 32)
    _, ex = np.frexp(np.abs(xb).max(axis=1).astype(np.float64))      # amax = m * 2^ex, m in [0.5, 1)
    cand = (ex - 1)[:, None] + np.arange(-8, 4)[None, :]
    d = np.exp2(cand.astype(np.float64)).astype(np.float32)
    inv = np.exp2(-cand.astype(np.float64)).astype(np.float32)
    loss64, _, _ = block_losses(xb, d, inv)
    chosen = out["scales"].reshape(-1).astype(np.int64) - 127
    assert np.all((chosen[:, None] == cand).any(axis=1))              # inside the brute-force range
    k = np.argmax(cand == chosen[:, None], axis=1)
    picked = loss64[np.arange(len(k)), k]
    assert np.all(picked <= loss64.min(axis=1) * (1 + 2 * RTOL_SUM32) + 1e-37)


def test_mxfp4_nonfinite_status(orc):
    x = np.ones((2, 64), dtype=np.float32)
    x[1, 40] = np.inf
    assert orc.mxfp4_quant(x)["status"] == orc.STATUS_NONFINITE
    x[1, 40] = np.nan
    assert orc.mxfp4_quant(x)["status"] == orc.STATUS_NONFINITE


def test_mxfp4_dequant_reproduces_reconstruction(orc):
    x = synth.t_weight(16, 256, nu=3, scale=0.015, seed=24).float().numpy()
    out = orc.mxfp4_quant(x, sign_masks=synth.sign_masks(256, seed=1))
    y = orc.mxfp4_dequant(out["codes"], out["scales"], 16, 256)
    np.testing.assert_array_equal(y, out["y"])


# ---------------------------------------------------------------- tiled scale layout
# The layout is a hardware interface the pages do not describe.  Two pins: its
# size, that every input byte lands exactly once and that the padding is zero
# (here), and the position of every byte against the layout as CUTLASS defines
# it (below, from its hierarchical shape/stride description); a library GEMM
# reading it pins it once more on the GPU.

@pytest.mark.parametrize("rows,scols", [(1, 1), (128, 4), (130, 6), (300, 257), (4096, 256)])
def test_mma_layout_size_coverage_and_padding(orc, rows, scols):
    rng = np.random.default_rng(rows * 1000 + scols)
    s = rng.integers(1, 256, size=(rows, scols), dtype=np.uint8)     # no zero bytes in the input
    out = orc.scales_to_mma_layout(s)
    rt, ct = -(-rows // 128), -(-scols // 4)
    assert out.size == rt * ct * 512
    assert np.count_nonzero(out) == rows * scols                      # padding is zero
    assert sorted(out[out != 0].tolist()) == sorted(s.reshape(-1).tolist())


# CUTLASS, include/cutlass/detail/sm100_blockscaled_layout.hpp: the scale-factor
# atom of a K-major operand (Sm1xxBlockScaledBasicChunk::SfKMajorAtom) covers
# 128 rows x 4 scales.  Its row mode has shape (32, 4) with strides (16, 4); its
# K mode has shape (SFVecSize elements, 4 scales) with strides (0, 1) -- every
# element of one scale's vector maps to the same byte.  tile_atom_to_shape_SFA
# tiles the atom over (M, K) with Step<_2,_1>: atoms along K are adjacent.
SF_ATOM = {"shape": ((32, 4), (16, 4)), "stride": ((16, 4), (0, 1))}   # SFVecSize = 16 (NVFP4)


def _size(shape):
    return int(np.prod([_size(s) for s in shape])) if isinstance(shape, tuple) else shape


def _crd2idx(c, shape, stride):
    """CuTe's coordinate -> index map: an integer coordinate of a tuple mode is
    split colexicographically (first sub-mode fastest), then each part is mapped
    by its sub-mode."""
    if not isinstance(shape, tuple):
        return c * stride
    if isinstance(c, tuple):
        return sum(_crd2idx(ci, si, di) for ci, si, di in zip(c, shape, stride))
    idx = 0
    for si, di in zip(shape, stride):
        n = _size(si)
        idx += _crd2idx(c % n, si, di)
        c //= n
    return idx


def _cosize(shape, stride):
    """One past the largest index the layout produces."""
    last = tuple(_size(s) - 1 for s in shape)
    return _crd2idx(last, shape, stride) + 1


def _tile_to_shape(atom, target, order):
    """Tile `atom` over `target` (each mode rounded up to whole atoms); the tile
    counts of the modes are laid out one after another in the given order
    (smallest step fastest), each tile cosize(atom) apart."""
    a_shape, a_stride = atom["shape"], atom["stride"]
    counts = [-(-t // _size(s)) for t, s in zip(target, a_shape)]
    step = _cosize(a_shape, a_stride)
    tile_stride = [0] * len(counts)
    for m in sorted(range(len(counts)), key=lambda i: order[i]):
        tile_stride[m] = step
        step *= counts[m]
    shape = tuple((a_shape[i], counts[i]) for i in range(len(counts)))
    stride = tuple((a_stride[i], tile_stride[i]) for i in range(len(counts)))
    return shape, stride, step


@pytest.mark.parametrize("rows,scols", [(1, 1), (128, 4), (130, 6), (300, 37), (513, 65)])
def test_mma_layout_matches_the_cutlass_layout_algebra(orc, rows, scols):
    vec = 16
    shape, stride, total = _tile_to_shape(SF_ATOM, (rows, scols * vec), order=(2, 1))
    rng = np.random.default_rng(rows + 7 * scols)
    s = rng.integers(1, 256, size=(rows, scols), dtype=np.uint8)
    out = orc.scales_to_mma_layout(s)
    assert out.size == total
    want = np.zeros(total, dtype=np.uint8)
    for r in range(rows):
        for c in range(scols):
            # every element k of scale c's vector addresses the same byte
            offs = {_crd2idx((r, c * vec + j), shape, stride) for j in (0, vec // 2, vec - 1)}
            assert len(offs) == 1
            want[offs.pop()] = s[r, c]
    np.testing.assert_array_equal(out, want)


def test_cutlass_atom_constants_match_the_header():
    """The atom numbers above against the CUTLASS header shipped in this image, when
    one is there (a source file read as text)."""
    import glob
    import re
    import site
    paths = []
    for root in site.getsitepackages():
        paths += glob.glob(f"{root}/*/data/cutlass/include/cutlass/detail/sm100_blockscaled_layout.hpp")
        paths += glob.glob(f"{root}/*/3rdparty/cutlass/include/cutlass/detail/sm100_blockscaled_layout.hpp")
    if not paths:
        pytest.skip("no CUTLASS header in this image")
    text = re.sub(r"\s+", "", open(paths[0]).read())
    assert "usingSfKMajorAtom=Layout<Shape<Shape<_32,_4>,Shape<Int<SFVecSize>,_4>>," in text
    assert "Stride<Stride<_16,_4>,Stride<_0,_1>>>;" in text
    assert "tile_to_shape(SfAtom{},make_shape(M,K),Step<_2,_1>{})" in text


def _centre(xb):
    import oracle
    return np.array([oracle.mx_centre_exponent(a) for a in np.abs(xb).max(axis=1)])


@pytest.mark.parametrize("kind", ["t3", "t4", "uniform", "ties", "huge", "tiny", "rotated"])
def test_mxfp4_never_picks_the_exponent_above_the_centre(orc, kind):
    """E8M0 steps are powers of two and e0 is the smallest exponent whose grid
    covers the block maximum, so the grid of e0+1 restricted to the block's
    range is a subset of the grid of e0: every element's error at e0+1 is at
    least its error at e0, every product and quotient is exact in binary32
    (powers of two), and each rounding step of the loss is monotone, so the
    loss at e0+1 is never below the loss at e0 and the first minimum is never
    e0+1 (the kernels skip screening it).  Checked on the oracle's choice over
    heavy-tailed, uniform, tie-only, near-overflow, subnormal and rotated
    blocks, and in fp64 against the e0 loss."""
    rng = np.random.default_rng(40 + len(kind))
    masks = None
    if kind in ("t3", "t4"):
        x = synth.t_weight(64, 1024, nu=int(kind[1]), scale=0.02, seed=41).float().numpy()
    elif kind == "uniform":
        x = rng.uniform(-1, 1, size=(64, 1024)).astype(np.float32)
    elif kind == "ties":
        # every element on a midpoint of the e0 grid (the equal-loss edge), plus the block maximum 6 * 2^k
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        g = mids[rng.integers(0, len(mids), size=(2048, 32))] * np.where(rng.random((2048, 32)) < .5, -1, 1)
        g[:, 7] = 6.0
        x = (g * 2.0 ** rng.integers(-20, 20, size=(2048, 1))).astype(np.float32).reshape(64, 1024)
    elif kind == "huge":
        x = (rng.uniform(-1, 1, size=(64, 1024)) * 3.0e38).astype(np.float32)
    elif kind == "tiny":
        x = (rng.uniform(-1, 1, size=(64, 1024)) * 2.0 ** -126).astype(np.float32)
    else:
        x = synth.t_weight(64, 1024, nu=3, scale=0.015, seed=42).float().numpy()
        masks = synth.sign_masks(1024, seed=42)
    out = orc.mxfp4_quant(x, sign_masks=masks)
    if kind != "huge":
        assert out["status"] == 0
    vb = (out["rotated"] if masks is not None else x).reshape(-1, 32)
    e0 = _centre(vb)
    chosen = out["scales"].reshape(-1).astype(np.int64) - 127
    above = np.minimum(e0 + 1, 127)
    assert np.all((chosen != above) | (above == e0)), "e0+1 chosen"
    if kind not in ("huge", "tiny"):
        d = np.exp2(np.stack([e0, e0 + 1], 1).astype(np.float64)).astype(np.float32)
        inv = np.exp2(-np.stack([e0, e0 + 1], 1).astype(np.float64)).astype(np.float32)
        loss64, _, _ = block_losses(vb, d, inv)
        assert np.all(loss64[:, 1] >= loss64[:, 0])


@pytest.mark.parametrize("e0", [-127, -126, -100, -3, 0, 5, 100, 126])
def test_mxfp4_element_error_is_never_smaller_above_the_centre(e0):
    """The lemma behind skipping e0+1, element by element and exhaustively:
    for every positive finite bf16 value x (the sign is symmetric) with
    x <= 6 * 2^e0, the definition's binary32 error term RN(RN(x - y)^2),
    y = RN(q * 2^e), q the E2M1 point nearest to RN(x * 2^-e) (fp64 search,
    ties to the even code), is at least as large at e = e0+1 as at e = e0."""
    from fp64_check import e2m1_nearest
    x = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        lim = np.float32(6.0) * np.float32(2.0 ** e0)
        x = x[x <= lim]

        def term(e):
            d = np.float32(2.0 ** e)
            inv = np.float32(2.0 ** -e)
            r = (x * inv).astype(np.float32)
            _, q = e2m1_nearest(r)
            y = (q * np.float64(d)).astype(np.float32)
            err = (x - y).astype(np.float32)
            return (err * err).astype(np.float32)

        t0, t1 = term(e0), term(e0 + 1)
    assert x.size >= 300                       # 320 bf16 values even at the subnormal end
    assert np.all(t1 >= t0)
