"""GPU tests of fp4q_nvfp4_sweep_dynamic: the global max and the NVFP4
ScaleSweep in one launch (one thread-block cluster for small tensors, a
cooperative launch with a grid-wide barrier for larger ones).  It must write
exactly the bytes of fp4q_global_absmax followed by
fp4q_nvfp4_sweep{mse,wmse}, leave its workspace zeroed, and agree with the
oracle on sampled rows."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _deq_bits, _np

pytestmark = pytest.mark.gpu

# decode-sized activations (1 and 16 tokens), a ragged case, prefill-sized and
# Llama-3-8B down-projection-sized tensors
SHAPES = [(1, 16), (1, 4096), (16, 4096), (37, 1056), (256, 14336), (4096, 4096)]


def _ws():
    return torch.zeros(fq.fp4q_dynamic_workspace_bytes() // 4, dtype=torch.int32, device=DEV)


def _compare(a, b):
    for name in ("amax", "global_scale", "codes", "scales", "deq", "block_loss"):
        _assert_eq(name, _np(getattr(a, name)), _np(getattr(b, name)))
    assert int(a.status.item()) == int(b.status.item())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("weighted", [False, True])
def test_dynamic_equals_two_launches(dtype, rows, cols, weighted):
    x = synth.q_proj(rows, cols, seed=rows * 7 + cols).to(dtype).to(DEV)
    imp = synth.importance_diag_xtx(cols=cols, tokens=64, seed=rows).to(DEV) if weighted else None
    ws = _ws()
    got = fq.nvfp4_quantize_dynamic(x, importance=imp, workspace=ws)
    ref = fq.nvfp4_quantize(x, importance=imp)
    torch.cuda.synchronize()
    assert int(got.status.item()) == 0
    _compare(got, ref)
    assert int(ws.abs().sum().item()) == 0          # the call leaves its workspace zeroed


def test_workspace_reused_across_calls_and_sizes():
    ws = _ws()
    xs = [synth.q_proj(r, c, seed=r + c).to(DEV) for r, c in [(16, 4096), (1, 4096), (512, 2048), (16, 4096)]]
    outs = [fq.nvfp4_quantize_dynamic(x, workspace=ws) for x in xs]
    refs = [fq.nvfp4_quantize(x) for x in xs]
    torch.cuda.synchronize()
    for a, b in zip(outs, refs):
        _compare(a, b)
    _compare(outs[0], outs[3])
    assert int(ws.abs().sum().item()) == 0


def test_dynamic_against_oracle_sampled_rows():
    rows, cols = 2048, 4096
    x = synth.q_proj(rows, cols, seed=2).to(DEV)
    got = fq.nvfp4_quantize_dynamic(x)
    torch.cuda.synchronize()
    x_full = x.float().cpu().numpy()
    gmax = oracle.global_absmax(x_full)
    assert _np(got.amax)[0] == gmax
    idx = np.array([0, 1, 777, rows - 1])
    o = oracle.nvfp4_quant(np.ascontiguousarray(x_full[idx]), S=oracle.global_scale(gmax))
    _assert_eq("scales", _np(got.scales)[idx], o["scales"])
    _assert_eq("codes", _np(got.codes)[idx], o["codes"])
    _assert_eq("deq", _np(got.deq)[idx], _deq_bits(o["y"], torch.bfloat16))
    _assert_eq("loss", _np(got.block_loss)[idx], o["loss"])


def test_dynamic_in_a_cuda_graph():
    x = synth.q_proj(16, 4096, seed=9).to(DEV)
    ws = _ws()
    amax = torch.empty(1, device=DEV)
    S = torch.empty(1, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    codes = torch.empty((16, 2048), dtype=torch.uint8, device=DEV)
    scales = torch.empty((16, 256), dtype=torch.uint8, device=DEV)
    deq = torch.empty_like(x)
    stream = torch.cuda.Stream()
    fq.fp4q_nvfp4_sweep_dynamic(x, None, amax, codes, scales, S, deq, None, ws, st, stream)   # warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fq.fp4q_nvfp4_sweep_dynamic(x, None, amax, codes, scales, S, deq, None, ws, st, stream)
    for _ in range(3):
        codes.zero_()
        g.replay()
    torch.cuda.synchronize()
    ref = fq.nvfp4_quantize(x, with_loss=False)
    torch.cuda.synchronize()
    _assert_eq("codes", _np(codes), _np(ref.codes))
    _assert_eq("scales", _np(scales), _np(ref.scales))
    _assert_eq("deq", _np(deq), _np(ref.deq))
    assert int(st.item()) == 0 and int(ws.abs().sum().item()) == 0


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_dynamic_nonfinite(bad):
    x = synth.q_proj(8, 256, seed=5)
    x[3, 17] = bad
    ws = _ws()
    got = fq.nvfp4_quantize_dynamic(x.to(DEV), workspace=ws)
    torch.cuda.synchronize()
    assert int(got.status.item()) == fq.FLAG_NONFINITE
    assert int(ws.abs().sum().item()) == 0


def test_dynamic_range_flag_and_zero_tensor():
    x = torch.full((4, 64), 2.0 ** 70, dtype=torch.float32, device=DEV)
    got = fq.nvfp4_quantize_dynamic(x)
    torch.cuda.synchronize()
    assert int(got.status.item()) == fq.FLAG_RANGE
    z = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    got = fq.nvfp4_quantize_dynamic(z)
    ref = fq.nvfp4_quantize(z)
    torch.cuda.synchronize()
    _compare(got, ref)
    assert _np(got.global_scale)[0] == 1.0


def test_dynamic_empty_and_small_workspace():
    amax = torch.full((1,), 5.0, device=DEV)
    e = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    fq.fp4q_nvfp4_sweep_dynamic(e, None, amax, torch.empty(0, dtype=torch.uint8, device=DEV),
                                torch.empty(0, dtype=torch.uint8, device=DEV), torch.empty(1, device=DEV),
                                None, None, _ws(), torch.zeros(1, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert _np(amax)[0] == 0.0
    x = synth.q_proj(4, 64, seed=1).to(DEV)
    with pytest.raises(fq.Fp4qError) as ei:
        fq.nvfp4_quantize_dynamic(x, workspace=torch.zeros(2, dtype=torch.int32, device=DEV))
    assert ei.value.status == fq.ERR_ARG


def test_small_tensors_use_the_cluster_kernel_large_ones_the_grid_barrier():
    from torch.profiler import ProfilerActivity, profile
    small = synth.q_proj(16, 4096, seed=21).to(DEV)          # 4096 blocks: one cluster of 16
    large = synth.q_proj(512, 4096, seed=22).to(DEV)         # 131072 blocks: cooperative launch
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fq.nvfp4_quantize_dynamic(small)
        fq.nvfp4_quantize_dynamic(large)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events()]
    assert any("nvfp4_cluster_kernel" in n for n in names), names
    assert any("nvfp4_dynamic_kernel" in n for n in names), names
