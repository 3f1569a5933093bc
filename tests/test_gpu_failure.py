"""Failure detection and memory-safety checks on the GPU, with no fault:

* the library's bounded spin-wait (the one the batch kernel and the one-launch
  sweep use to wait for other thread blocks) run on a flag that nothing sets
  gives up within its bound, raises FP4Q_FLAG_TIMEOUT, and leaves the context
  usable;
* canary guard bytes before and after every output buffer of every entry
  point stay untouched, on odd small shapes (a single row, one block,
  ragged row counts)."""
import time

import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _np

pytestmark = pytest.mark.gpu

GUARD = 64          # guard elements on each side (a multiple of 16 bytes for every dtype used)
PATTERN = 0xA5


def _guarded(shape, dtype):
    n = int(np.prod(shape)) if len(shape) else 1
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device=DEV)
    buf.view(torch.uint8).fill_(PATTERN)
    view = buf[GUARD:GUARD + n].view(shape)
    return buf, view


def _intact(name, buf, n):
    raw = buf.view(torch.uint8).cpu().numpy()
    isz = buf.element_size()
    head, tail = raw[:GUARD * isz], raw[(GUARD + n) * isz:]
    assert (head == PATTERN).all() and (tail == PATTERN).all(), f"{name}: guard bytes overwritten"


def test_bounded_wait_runs_out_and_the_context_survives():
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fq.fp4q_probe_wait(flag, 1, 1 << 16, st)          # nothing ever sets the flag
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == fq.FLAG_TIMEOUT
    assert dt < 5.0                                     # 2^16 polls of ~128 ns, far below
    flag.fill_(3)
    st.zero_()
    fq.fp4q_probe_wait(flag, 1, 1 << 16, st)            # already satisfied: no flag
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    with pytest.raises(fq.Fp4qError):
        fq.fp4q_probe_wait(flag, 1, (1 << 24) + 1, st)
    # the context is healthy: a quantization still matches the oracle
    w = synth.q_proj(8, 256, seed=77)
    r = fq.nvfp4_quantize(w.to(DEV))
    torch.cuda.synchronize()
    o = oracle.nvfp4_quant(w.float().numpy())
    _assert_eq("codes", _np(r.codes), o["codes"])


@pytest.mark.parametrize("nbytes", [0, 16, 48, 4096 + 16, 3 * 65536 + 208])
def test_copy_probe_is_exact_and_stays_in_bounds(nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).to(DEV)
    buf, dst = _guarded((nbytes,), torch.uint8)
    fq.fp4q_probe_copy(src, dst)
    torch.cuda.synchronize()
    assert torch.equal(dst, src)
    _intact("copy", buf, nbytes)
    if nbytes >= 16:
        with pytest.raises(fq.Fp4qError):           # not a multiple of 16 bytes
            fq.fp4q_probe_copy(src[:8], dst[:8])


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (37, 288)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_guard_bytes_of_every_output(rows, cols, dtype):
    w = synth.q_proj(rows, cols, seed=rows * 11 + cols).to(dtype).to(DEV)
    n = rows * cols
    masks = torch.from_numpy(synth.sign_masks(cols, seed=rows).view(np.int32)).to(DEV)
    imp = synth.importance_diag_xtx(cols=cols, tokens=32, seed=rows).to(DEV)
    outs = {}

    def g(name, shape, dt):
        outs[name] = _guarded(shape, dt)
        return outs[name][1]

    amax, S, st = g("amax", (1,), torch.float32), g("S", (1,), torch.float32), g("st", (1,), torch.int32)
    st.zero_()
    fq.fp4q_global_absmax(w, amax)
    fq.fp4q_nvfp4_sweepmse(w, amax, g("nv_codes", (rows, cols // 2), torch.uint8),
                           g("nv_scales", (rows, cols // 16), torch.uint8), S, g("nv_deq", (rows, cols), dtype),
                           g("nv_loss", (rows, cols // 16), torch.float32), st)
    fq.fp4q_nvfp4_sweepwmse(w, amax, imp, g("wm_codes", (rows, cols // 2), torch.uint8),
                            g("wm_scales", (rows, cols // 16), torch.uint8), S, g("wm_deq", (rows, cols), dtype),
                            g("wm_loss", (rows, cols // 16), torch.float32), st)
    fq.fp4q_mxfp4_quant_hadamard(w, masks, g("mx_codes", (rows, cols // 2), torch.uint8),
                                 g("mx_scales", (rows, cols // 32), torch.uint8), g("mx_deq", (rows, cols), dtype),
                                 g("mx_loss", (rows, cols // 32), torch.float32), st)
    fq.fp4q_mxfp4_quant_absmax(w, None, g("mxa_codes", (rows, cols // 2), torch.uint8),
                               g("mxa_scales", (rows, cols // 32), torch.uint8), g("amax2", (1,), torch.float32),
                               g("mxa_deq", (rows, cols), dtype), g("mxa_loss", (rows, cols // 32), torch.float32),
                               st)
    ws = g("dyn_ws", (4,), torch.int32)
    ws.zero_()
    fq.fp4q_nvfp4_sweep_dynamic(w, None, g("dyn_amax", (1,), torch.float32),
                                g("dyn_codes", (rows, cols // 2), torch.uint8),
                                g("dyn_scales", (rows, cols // 16), torch.uint8), g("dyn_S", (1,), torch.float32),
                                g("dyn_deq", (rows, cols), dtype), g("dyn_loss", (rows, cols // 16), torch.float32),
                                ws, st)
    coeffs = torch.ones((rows, cols // 8), dtype=torch.float16, device=DEV)
    fq.fp4q_focus_quant(fq.NVFP4, w, outs["nv_scales"][1], S, coeffs, 8,
                        g("fo_codes", (rows, cols // 2), torch.uint8), g("fo_deq", (rows, cols), dtype),
                        g("fo_loss", (rows, cols // 16), torch.float32), st)
    fq.fp4q_mxfp4_unrotate(outs["mx_deq"][1], masks, g("unrot", (rows, cols), dtype))
    fq.fp4q_scales_to_mma_layout(outs["nv_scales"][1],
                                 g("tiled", (fq.fp4q_mma_scale_bytes(rows, cols // 16),), torch.uint8))
    fq.fp4q_dequant(fq.NVFP4, outs["nv_codes"][1], outs["nv_scales"][1], S, rows, cols,
                    g("dq", (rows, cols), dtype))
    if dtype == torch.float32:
        wc = g("gptq_w", (rows, cols), torch.float32)
        wc.copy_(w)
        U = torch.eye(cols, device=DEV)
        fq.fp4q_nvfp4_gptq(wc, U, amax, g("gq_codes", (rows, cols // 2), torch.uint8),
                           g("gq_scales", (rows, cols // 16), torch.uint8), g("gq_S", (1,), torch.float32),
                           g("gq_deq", (rows, cols), torch.float32),
                           g("gq_ws", (fq.fp4q_gptq_workspace_bytes(rows),), torch.uint8), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for name, (buf, view) in outs.items():
        _intact(name, buf, view.numel())
