"""GPU edge cases: empty and degenerate tensors, status flags, argument errors,
streams and graph capture, determinism, and a tensor above 2^31 elements."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _np, mxfp4_parity, nvfp4_parity

pytestmark = pytest.mark.gpu


def test_empty_tensors():
    for dt in (torch.bfloat16, torch.float32):
        w = torch.empty((0, 64), dtype=dt, device=DEV)
        r = fq.nvfp4_quantize(w)
        m = fq.mxfp4_quantize(w)
        torch.cuda.synchronize()
        assert r.codes.numel() == 0 and m.codes.numel() == 0
        assert _np(r.amax)[0] == 0.0


def test_all_zero_and_negative_zero():
    w = torch.zeros((8, 64), dtype=torch.bfloat16)
    w[3, 5] = -0.0
    w[4] = -0.0
    nvfp4_parity(w)
    mxfp4_parity(w)
    mxfp4_parity(w, synth.sign_masks(64, seed=9))


def test_subnormal_and_tiny_values():
    w = synth.q_proj(16, 256, seed=41).float()
    w[2, :16] = torch.tensor(np.float32(1e-40)) * torch.arange(16)    # fp32 subnormals
    w[5, 32:48] = 1e-30
    nvfp4_parity(w)
    mxfp4_parity(w)
    wb = torch.full((4, 64), 2.0 ** -130, dtype=torch.float32)        # MXFP4: e clamps at -127
    mxfp4_parity(wb)


@pytest.mark.parametrize("gmax,flag", [(2.0 ** -70, fq.FLAG_RANGE), (2.0 ** 65, fq.FLAG_RANGE),
                                       (2.0 ** -64, 0), (2.0 ** 64, 0)])
def test_global_scale_range(gmax, flag):
    w = synth.q_proj(8, 64, seed=42)
    w = (w.float() / w.float().abs().max() * gmax).to(torch.bfloat16)
    w[0, 0] = gmax
    if flag == 0:
        nvfp4_parity(w)
    else:
        r = fq.nvfp4_quantize(w.to(DEV))
        torch.cuda.synchronize()
        assert int(r.status.item()) == flag
        with pytest.raises(fq.Fp4qError):
            fq.check_status(r.status)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_nonfinite_flags(bad):
    w = synth.q_proj(8, 128, seed=43)
    w[6, 77] = bad
    wd = w.to(DEV)
    r = fq.nvfp4_quantize(wd)
    m = fq.mxfp4_quantize(wd)
    h = fq.mxfp4_quantize(wd, torch.from_numpy(synth.sign_masks(128).view(np.int32)).to(DEV))
    torch.cuda.synchronize()
    assert int(r.status.item()) == fq.FLAG_NONFINITE
    assert int(m.status.item()) == fq.FLAG_NONFINITE
    assert int(h.status.item()) == fq.FLAG_NONFINITE
    if bad != bad:
        assert np.isnan(_np(r.amax)[0])
    else:
        assert _np(r.amax)[0] == np.inf


def test_argument_errors_on_device():
    w = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    bad = w.view(-1)[1:1 + 64].view(1, 64)                             # 2-byte offset
    with pytest.raises(fq.Fp4qError, match="aligned"):
        fq.nvfp4_quantize(bad)
    with pytest.raises(fq.Fp4qError, match="shape"):
        fq.mxfp4_quantize(torch.zeros((2, 48), dtype=torch.bfloat16, device=DEV))
    with pytest.raises(TypeError):
        fq.nvfp4_quantize(torch.zeros((2, 32), dtype=torch.float16, device=DEV))


def test_absmax_tails_and_dtypes():
    rng = np.random.default_rng(44)
    for n in [1, 3, 7, 8, 9, 1000, 4097, 1 << 20, (1 << 20) + 5]:
        for dt in (torch.bfloat16, torch.float32):
            x = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).to(dt)
            x[rng.integers(0, n)] = -7.25
            a = torch.empty(1, dtype=torch.float32, device=DEV)
            fq.fp4q_global_absmax(x.to(DEV), a)
            torch.cuda.synchronize()
            assert _np(a)[0] == oracle.global_absmax(x.float().numpy())


def test_absmax_status_word_flags_unusable_maxima():
    """fp4q_global_absmax alone reports, through its status word, a maximum that
    cannot give a global scale (ScaleSweep summary, "Metodologia" sec. 2:
    S = max|x| / 1536): NaN/Inf, or nonzero outside [2^-64, 2^64]."""
    cases = [
        (np.array([1.0, np.nan, 2.0] + [0.5] * 13, np.float32), fq.FLAG_NONFINITE),
        (np.array([1.0, -np.inf] + [0.5] * 14, np.float32), fq.FLAG_NONFINITE),
        (np.array([3.0 * 2.0 ** 70] + [1.0] * 15, np.float32), fq.FLAG_RANGE),
        (np.array([2.0 ** -70] * 16, np.float32), fq.FLAG_RANGE),
        (np.zeros(16, np.float32), 0),
        (np.array([2.0 ** -64] + [0.0] * 15, np.float32), 0),
        (np.array([2.0 ** 64] + [0.0] * 15, np.float32), 0),
        (np.array([0.75] * 16, np.float32), 0),
    ]
    for x, want in cases:
        for dt in (torch.float32, torch.bfloat16):
            xt = torch.from_numpy(x).to(dt)      # every value above is exact in bf16
            a = torch.empty(1, dtype=torch.float32, device=DEV)
            st = torch.zeros(1, dtype=torch.int32, device=DEV)
            fq.fp4q_global_absmax(xt.to(DEV), a, st)
            torch.cuda.synchronize()
            assert int(st.item()) == want, (x[:3], dt, int(st.item()))
            got = _np(a)[0]
            ref = oracle.global_absmax(xt.float().numpy())
            assert (np.isnan(got) and np.isnan(ref)) or got == ref
    # NULL status word: no flag anywhere, the maximum is still written
    a = torch.empty(1, dtype=torch.float32, device=DEV)
    fq.fp4q_global_absmax(torch.from_numpy(cases[0][0]).to(DEV), a)
    torch.cuda.synchronize()
    assert np.isnan(_np(a)[0])


def test_stream_and_graph_capture_reproduce_eager():
    w = synth.q_proj(512, 1024, seed=45).to(DEV)
    eager = fq.nvfp4_quantize(w)
    eager_mx = fq.mxfp4_quantize(w)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    amax = torch.empty(1, dtype=torch.float32, device=DEV)
    S = torch.empty(1, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    codes = torch.empty_like(eager.codes)
    scales = torch.empty_like(eager.scales)
    deq = torch.empty_like(w)
    loss = torch.empty_like(eager.block_loss)
    mcodes = torch.empty_like(eager_mx.codes)
    mscales = torch.empty_like(eager_mx.scales)
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fq.fp4q_global_absmax(w, amax)
            fq.fp4q_nvfp4_sweepmse(w, amax, codes, scales, S, deq, loss, st)
            fq.fp4q_mxfp4_quant(w, mcodes, mscales, None, None, st)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for a, b in ((codes, eager.codes), (scales, eager.scales), (deq, eager.deq), (loss, eager.block_loss),
                 (S, eager.global_scale), (mcodes, eager_mx.codes), (mscales, eager_mx.scales)):
        _assert_eq("graph", _np(a), _np(b))
    assert int(st.item()) == 0


def test_deterministic_across_runs():
    w = synth.t_weight(333, 2048, seed=46).to(DEV)
    imp = synth.importance_diag_xtx(cols=2048, tokens=64, seed=46).to(DEV)
    a = fq.nvfp4_quantize(w, importance=imp)
    b = fq.nvfp4_quantize(w, importance=imp)
    torch.cuda.synchronize()
    for x, y in zip(a[:5], b[:5]):
        _assert_eq("rerun", _np(x), _np(y))


def test_above_2_31_elements():
    """65600 x 32768 bf16 (2.15e9 elements): 64-bit indexing in every kernel."""
    rows, cols = 65600, 32768
    assert rows * cols > 2 ** 31
    g = torch.Generator(device=DEV)
    g.manual_seed(47)
    w = (torch.randn((rows, cols), generator=g, device=DEV, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    w[rows - 1, cols - 3] = 0.75                        # the max sits in the last row
    r = fq.nvfp4_quantize(w, with_loss=False)
    m = fq.mxfp4_quantize(w, with_loss=False)
    torch.cuda.synchronize()
    assert _np(r.amax)[0] == np.float32(0.75)
    sample = np.array([0, 65535, 65536, rows - 2, rows - 1])
    x = w[torch.as_tensor(sample, device=DEV)].float().cpu().numpy()
    S = oracle.global_scale(np.float32(0.75))
    o = oracle.nvfp4_quant(x, S=S)
    _assert_eq("big scales", _np(r.scales[torch.as_tensor(sample, device=DEV)]), o["scales"])
    _assert_eq("big codes", _np(r.codes[torch.as_tensor(sample, device=DEV)]), o["codes"])
    _assert_eq("big deq", _np(r.deq[torch.as_tensor(sample, device=DEV)]), oracle.bf16_round(o["y"]))
    om = oracle.mxfp4_quant(x)
    _assert_eq("big mx scales", _np(m.scales[torch.as_tensor(sample, device=DEV)]), om["scales"])
    _assert_eq("big mx codes", _np(m.codes[torch.as_tensor(sample, device=DEV)]), om["codes"])
    del w, r, m
    torch.cuda.empty_cache()
