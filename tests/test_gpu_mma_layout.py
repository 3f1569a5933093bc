"""GPU tests of fp4q_scales_to_mma_layout: block scales in the 128 x 4 tiled
layout that Blackwell block-scaled FP4 GEMMs read.

The layout kernel must reproduce the oracle byte for byte; and a library
block-scaled NVFP4 GEMM (torch._scaled_mm on cuBLASLt) fed with our packed
codes and the tiled scales, of the kernel and of the oracle, must reproduce
the GEMM of our dequantized matrices -- which pins both the layout and the
code packing to an independent consumer.  MXFP4 operands go through the same
GEMM with each E8M0 scale rewritten as an E4M3 power of two."""
import numpy as np
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import oracle
import synth
from test_gpu_parity import DEV, _assert_eq, _np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,scols", [(1, 1), (128, 4), (130, 6), (300, 257), (4096, 256), (16384, 512)])
def test_layout_kernel_equals_oracle(rows, scols):
    rng = np.random.default_rng(rows + 7 * scols)
    s = rng.integers(0, 256, size=(rows, scols), dtype=np.uint8)
    out = fq.mma_scales(torch.from_numpy(s).to(DEV))
    torch.cuda.synchronize()
    _assert_eq("layout", _np(out), oracle.scales_to_mma_layout(s))


def test_layout_unaligned_source_and_empty():
    base = torch.zeros(1 + 64 * 24, dtype=torch.uint8, device=DEV)
    view = base[1:].view(64, 24)                   # scale bytes starting at an odd address
    view.copy_(torch.randint(0, 256, (64, 24), dtype=torch.uint8, device=DEV))
    out = fq.mma_scales(view)
    torch.cuda.synchronize()
    _assert_eq("layout", _np(out), oracle.scales_to_mma_layout(_np(view)))
    assert fq.fp4q_mma_scale_bytes(0, 5) == 0


def _scaled_mm(codes_a, sa_tiled, codes_b, sb_tiled):
    """cuBLASLt block-scaled NVFP4 GEMM A @ B^T, both operands K-major, fp32
    output when the library offers it, else bf16 (returned with its rounding
    unit).  The library wants M and N to be multiples of 16, not of 128, so
    partial row tiles of the scale layout are read too."""
    a4 = codes_a.view(torch.float4_e2m1fn_x2)
    b4 = codes_b.view(torch.float4_e2m1fn_x2)
    sa = sa_tiled.view(torch.float8_e4m3fn)
    sb = sb_tiled.view(torch.float8_e4m3fn)
    try:
        return torch._scaled_mm(a4, b4.t(), sa, sb, out_dtype=torch.float32).double(), 2.0 ** -22
    except RuntimeError:
        return torch._scaled_mm(a4, b4.t(), sa, sb, out_dtype=torch.bfloat16).double(), 2.0 ** -8


def _check_gemm(got, unit, ref, absref, K):
    # fp32 accumulation of K products in any order (at most K roundings of
    # 2^-24 relative to the running sum of magnitudes) plus the output rounding;
    # a wrong scale, a wrong nibble order or a misplaced tile is off by O(1)
    tol = unit * ref.abs() + K * 2.0 ** -23 * absref
    bad = (got - ref).abs() > tol
    assert not bool(bad.any()), f"{int(bad.sum())} of {bad.numel()} outputs off, worst " \
                                f"{float(((got - ref).abs() - tol).max())}"


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (272, 208, 1088), (512, 384, 4096)])
def test_nvfp4_gemm_reads_our_codes_and_tiled_scales(M, N, K):
    a = synth.q_proj(M, K, seed=M).float().to(DEV)              # fp32: deq is RN(q*d) in fp32
    b = synth.q_proj(N, K, seed=N + 1).float().to(DEV)
    qa, qb = fq.nvfp4_quantize(a), fq.nvfp4_quantize(b)
    torch.cuda.synchronize()
    assert int(qa.status.item()) == 0 and int(qb.status.item()) == 0
    sa, sb = fq.mma_scales(qa.scales), fq.mma_scales(qb.scales)
    got, unit = _scaled_mm(qa.codes, sa, qb.codes, sb)
    got = got * (float(qa.global_scale.item()) * float(qb.global_scale.item()))
    A, B = qa.deq.double(), qb.deq.double()
    ref = A @ B.t()
    absref = A.abs() @ B.abs().t()
    _check_gemm(got, unit, ref, absref, K)
    # the oracle's layout of the same scales gives the same GEMM, bit for bit
    sa_o = torch.from_numpy(oracle.scales_to_mma_layout(_np(qa.scales))).to(DEV)
    sb_o = torch.from_numpy(oracle.scales_to_mma_layout(_np(qb.scales))).to(DEV)
    got_o, _ = _scaled_mm(qa.codes, sa_o, qb.codes, sb_o)
    got_o = got_o * (float(qa.global_scale.item()) * float(qb.global_scale.item()))
    assert torch.equal(got, got_o)


def _mx_as_nv_scales(e8m0: torch.Tensor):
    """E8M0 bytes [rows][cols/32] -> E4M3 bytes [rows][cols/16] holding
    2^(e - ref) (each 32-block split into two 16-blocks) and 2^ref."""
    e = e8m0.long() - 127
    ref = int(e.max().item()) - 8
    k = e - ref
    assert int(k.min().item()) >= -9, "scale range wider than E4M3 powers of two"
    p = torch.where(k >= -6, (k + 7) << 3, torch.bitwise_left_shift(torch.ones_like(k), k + 9))
    return p.to(torch.uint8).repeat_interleave(2, dim=1).contiguous(), ref


def test_mxfp4_codes_through_the_block_scaled_gemm():
    M, N, K = 256, 256, 2048
    a = synth.q_proj(M, K, seed=41).float().to(DEV)             # fp32: deq is exactly q*2^e
    b = synth.q_proj(N, K, seed=42).float().to(DEV)
    qa, qb = fq.mxfp4_quantize(a), fq.mxfp4_quantize(b)
    torch.cuda.synchronize()
    sa, ra = _mx_as_nv_scales(qa.scales)
    sb, rb = _mx_as_nv_scales(qb.scales)
    got, unit = _scaled_mm(qa.codes, fq.mma_scales(sa), qb.codes, fq.mma_scales(sb))
    got = got * 2.0 ** (ra + rb)
    A, B = qa.deq.double(), qb.deq.double()
    _check_gemm(got, unit, A @ B.t(), A.abs() @ B.abs().t(), K)
