"""Host checks of the arithmetic behind the wide kernel's E4M3 operand splits.

The tensor-core kernel for 128 query heads runs QK^T and PV in E4M3:
  * each bf16 query row, scaled by a power of two to a maximum in [128, 256),
    becomes hi = E4M3(q) and lo = E4M3(q - hi); the claim is that hi + lo == q
    exactly for every element of magnitude at least 2^-2 (a bf16 value has 8
    significant bits, hi keeps 4 and the residual fits in lo), and that smaller
    elements are off by at most half the E4M3 subnormal step, 2^-10;
  * each probability (token scale and a power of two folded in, largest value of
    a block in [128, 256) when the power is chosen, at most 448) becomes three
    terms t0 = E4M3(v), t1 = E4M3(v - t0), t2 = E4M3(v - t0 - t1): relative
    error at most 2^-12 from v = 4 up, absolute error at most 2^-10 below (the
    terms that fall under the E4M3 normal range are lost); two terms keep only
    about 2^-9, which the wide parity test on peaky scores showed to be too
    coarse for the 2e-3 bound.
E4M3 here is torch's float8_e4m3fn cast (round to nearest even), the rounding
of the kernel's cvt.rn.satfinite for values inside the E4M3 range.
"""
import numpy as np
import torch


def e4m3(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float8_e4m3fn).to(torch.float64)


def all_bf16_values() -> torch.Tensor:
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    v = bits.view(torch.bfloat16).to(torch.float64)
    return v[torch.isfinite(v)]


def test_query_two_terms_are_exact_from_a_quarter_up():
    v = all_bf16_values()
    v = v[(v.abs() >= 0.25) & (v.abs() < 256.0)]
    hi = e4m3(v.float())
    lo = e4m3((v - hi).float())
    assert torch.equal(hi + lo, v)


def test_query_two_terms_below_a_quarter_err_at_most_2_pow_minus_10():
    v = all_bf16_values()
    v = v[(v.abs() < 0.25)]
    hi = e4m3(v.float())
    lo = e4m3((v - hi).float())
    err = (hi + lo - v).abs().max().item()
    assert err <= 2.0 ** -10
    # and the bound is reached: the small elements are rounded, not kept
    assert err > 2.0 ** -11


def split_terms(a: torch.Tensor, terms: int):
    rest = a.clone()
    total = torch.zeros_like(a)
    for _ in range(terms):
        t = e4m3(rest.float())
        total += t
        rest = a - total
    return total


def _uniform_log2(lo, hi, n, seed):
    g = torch.Generator().manual_seed(seed)
    a = torch.exp2(torch.empty(n, dtype=torch.float64).uniform_(lo, hi, generator=g))
    return a.float().to(torch.float64)                   # the kernel holds v in fp32


def test_probability_three_terms_keep_twelve_bits_from_4_up():
    # every term is a normal E4M3 value once v >= 4 (residuals 2^-4 and 2^-8 of v)
    a = _uniform_log2(2.0, np.log2(448.0), 1 << 20, 5)
    rel3 = ((split_terms(a, 3) - a).abs() / a).max().item()
    assert rel3 <= 2.0 ** -12 * 1.001


def test_probability_three_terms_below_4_err_at_most_2_pow_minus_10():
    # smaller values lose the terms that fall under the E4M3 normal range: the
    # error is at most half the subnormal step, against a block maximum >= 128
    a = _uniform_log2(-20.0, 2.0, 1 << 20, 6)
    err = (split_terms(a, 3) - a).abs().max().item()
    assert err <= 2.0 ** -10


def test_probability_two_terms_keep_only_about_eight_bits():
    a = _uniform_log2(0.0, np.log2(448.0), 1 << 20, 7)
    rel2 = ((split_terms(a, 2) - a).abs() / a).max().item()
    assert 2.0 ** -10 < rel2 <= 2.0 ** -9 * 1.001


def test_probability_terms_of_a_block_bound_in_range():
    # the power of two puts a block's largest value in [128, 256); values up to
    # 448 (the E4M3 maximum) are split without saturation
    a = torch.tensor([128.0, 200.0, 255.9, 300.0, 447.9, 448.0], dtype=torch.float64)
    assert torch.all((split_terms(a, 3) - a).abs() / a <= 2.0 ** -12 * 1.001)
