"""The two-part bf16 representation behind the router backward's tensor-core path.

With N' and d multiples of 64 and T >= max(256, 2 N'), dsmoe_backward_router splits the
fp32 logit gradient into hi = bf16(v) and lo = bf16(v - hi) (round to nearest even, as
__float2bfloat16_rn does) and runs dW_router = hi^T x + lo^T x and dx = [hi | lo] W
as bf16 products summed in fp32. bf16 keeps 8 significant bits, so each rounding is
within 2^-8 of its argument: |v - hi| <= 2^-8 |v| and |v - hi - lo| <= 2^-8 |v - hi|
<= 2^-16 |v|, for |v| below the largest finite bf16 (about 3.39e38; above it hi rounds to
infinity). These checks pin that bound on the CPU with torch's bf16 rounding, and the
element-wise bound it gives for a contraction against bf16 operands (which the tensor
cores multiply exactly): |err_ij| <= 2^-16 sum_i |dl_i| |W_ij|. The GPU test's tolerance
on dx and dW_router, 1e-4 of the RMS, sits above what these rounding residuals (of
random sign) give at the tested shapes, here and measured on the GPU (1e-5 to 4e-5);
one bf16 part alone would not meet it.
"""
import numpy as np
import torch


def _split(v: torch.Tensor):
    hi = v.to(torch.bfloat16)
    lo = (v - hi.float()).to(torch.bfloat16)
    return hi, lo


def test_two_part_split_is_within_two_to_the_minus_16():
    g = torch.Generator().manual_seed(7)
    parts = [torch.randn(1 << 16, generator=g) * s for s in (1e-30, 1e-6, 1.0, 3e4, 1e30)]
    edge = torch.tensor([0.0, -0.0, 1.0, -1.0, 1.0 + 2.0 ** -8, 1.0 + 2.0 ** -9, 1.0 + 3 * 2.0 ** -9,
                         3.3e38, -3.3e38, float(np.finfo(np.float32).tiny), 2.0 ** -100 * 3.0])
    v = torch.cat(parts + [edge]).float()
    hi, lo = _split(v)
    v64 = v.double()
    rest = (v64 - hi.double() - lo.double()).abs()
    assert bool(torch.isfinite(hi.float()).all()) and bool(torch.isfinite(lo.float()).all())
    assert bool((rest <= 2.0 ** -16 * v64.abs()).all())
    # hi alone is a plain bf16 rounding: within 2^-8, and lo carries what it dropped
    assert bool(((v64 - hi.double()).abs() <= 2.0 ** -8 * v64.abs()).all())
    # values with at most 16 significant bits split exactly
    exact = torch.tensor([1.0 + 2.0 ** -15, 3.0 + 2.0 ** -12, -(2.0 ** 20 + 2.0 ** 6)], dtype=torch.float32)
    h2, l2 = _split(exact)
    assert torch.equal(h2.double() + l2.double(), exact.double())
    # the domain limit: fp32 values above the largest finite bf16 round to infinity
    assert bool(torch.isinf(torch.tensor([float(np.finfo(np.float32).max)]).to(torch.bfloat16).float()).all())


def test_split_contraction_error_bound():
    """dx = dl W with dl = hi + lo + rest: |dx - (hi W + lo W)| <= 2^-16 sum_i |dl_i| |W_ij|
    when the products are exact (bf16 x bf16 in a wide accumulator); float64 stands in for
    the tensor cores' exact products here."""
    g = torch.Generator().manual_seed(11)
    T, N, d = 64, 256, 96
    dl = torch.randn(T, N, generator=g) * torch.exp(torch.randn(T, N, generator=g))
    W = (torch.randn(N, d, generator=g) * 0.05).to(torch.bfloat16)
    hi, lo = _split(dl)
    W64 = W.double()
    exact = dl.double() @ W64
    two_part = hi.double() @ W64 + lo.double() @ W64
    bound = 2.0 ** -16 * (dl.double().abs() @ W64.abs())
    assert bool(((exact - two_part).abs() <= bound).all())
    # and one bf16 part alone would not meet the GPU test's 1e-4 of the RMS
    one_part = hi.double() @ W64
    rms = exact.pow(2).mean().sqrt()
    assert float((exact - one_part).abs().max() / rms) > 1e-4
    assert float((exact - two_part).abs().max() / rms) < 1e-4
