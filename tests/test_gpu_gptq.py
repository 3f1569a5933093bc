"""GPU parity of the ScaleSweep inside GPTQ (fp4q_nvfp4_gptq) with the
oracle's sequential definition, bit for bit: codes, scales, global scale and
reconstruction -- on small matrices in full (several 128-column blocks and a
narrower last block) and, at the size of the WMSE workload (11008 x 4096 with
the Gram matrix of 2048 x 4096 synthetic activations), on sampled rows (rows
are independent in GPTQ)."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _np

pytestmark = pytest.mark.gpu


def _U_from_X(X: torch.Tensor, damp=0.01) -> torch.Tensor:
    """Upper Cholesky factor of the inverse dampened Gram matrix, computed in
    fp64 on the GPU and rounded to fp32 (U^T U = H^-1)."""
    X = X.to(DEV, torch.float64)
    H = X.T @ X
    H += damp * H.diagonal().mean() * torch.eye(H.shape[0], dtype=torch.float64, device=DEV)
    Hinv = torch.cholesky_inverse(torch.linalg.cholesky(H))
    return torch.linalg.cholesky(Hinv).mT.contiguous().float()


def _correlated_X(tokens, cols, seed, rank=16):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(tokens, rank, generator=g, dtype=torch.float64) @
            torch.randn(rank, cols, generator=g, dtype=torch.float64) +
            0.1 * torch.randn(tokens, cols, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("rows,cols", [(37, 256), (64, 304), (300, 1024)])
def test_gptq_equals_oracle(rows, cols):
    w = synth.q_proj(rows, cols, seed=rows + cols).float()
    U = _U_from_X(_correlated_X(512, cols, seed=cols), damp=0.01)
    g = fq.nvfp4_gptq(w.to(DEV), U)
    torch.cuda.synchronize()
    assert int(g.status.item()) == 0
    o = oracle.nvfp4_gptq(w.numpy(), U.cpu().numpy())
    _assert_eq("S", _np(g.global_scale), np.array([o["S"]], np.float32))
    _assert_eq("scales", _np(g.scales), o["scales"])
    _assert_eq("codes", _np(g.codes), o["codes"])
    _assert_eq("deq", _np(g.deq).view(np.uint32), o["y"].view(np.uint32))


def test_gptq_with_identity_hessian_is_the_sweep():
    w = synth.q_proj(128, 512, seed=5).float().to(DEV)
    g = fq.nvfp4_gptq(w, torch.eye(512, device=DEV))
    r = fq.nvfp4_quantize(w)
    torch.cuda.synchronize()
    _assert_eq("codes", _np(g.codes), _np(r.codes))
    _assert_eq("scales", _np(g.scales), _np(r.scales))


def test_gptq_wmse_workload_sampled_rows():
    rows, cols = 11008, 4096
    w = synth.t_weight(rows, cols, nu=4, scale=0.02, seed=3, device=DEV).float()
    # the WMSE workload's activations: 2048 x 4096 bf16 N(0,1), 41 columns (1%) x50
    g0 = torch.Generator(device="cpu").manual_seed(3)
    Xa = torch.randn(2048, cols, generator=g0, dtype=torch.float32)
    Xa[:, torch.randperm(cols, generator=g0)[:41]] *= 50.0
    U = _U_from_X(Xa.to(torch.bfloat16).double())
    g = fq.nvfp4_gptq(w, U)
    torch.cuda.synchronize()
    assert int(g.status.item()) == 0
    S = float(g.global_scale.item())
    idx = np.array([0, 1, 5000, rows - 1])
    o = oracle.nvfp4_gptq(w.cpu().numpy()[idx], U.cpu().numpy(), S=S)
    _assert_eq("scales", _np(g.scales)[idx], o["scales"])
    _assert_eq("codes", _np(g.codes)[idx], o["codes"])
    _assert_eq("deq", _np(g.deq)[idx].view(np.uint32), o["y"].view(np.uint32))
