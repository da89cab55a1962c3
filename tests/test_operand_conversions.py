"""Host checks of the exactness claims behind the 8-head kernel's f16 MMA operands.

The FP8 path of the 8-head decode kernel converts cached E4M3 codes to f16
(cvt e4m3x2 -> f16x2) and bf16 queries to f16, then multiplies on the f16
tensor path with FP32 accumulation.  The claims: every E4M3 value is an f16
value (no rounding in the conversion), and a bf16 value converts to f16
exactly when its magnitude lies in f16's normal range [2^-14, 65504]
(bf16 keeps 8 significant bits, f16 11).
"""
import torch


def test_every_e4m3_code_is_an_f16_value():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    v = codes.to(torch.float64)
    finite = torch.isfinite(v)
    via_f16 = codes.to(torch.float16).to(torch.float64)
    assert torch.equal(via_f16[finite], v[finite])
    assert torch.isnan(via_f16[~finite]).all()            # 0x7F / 0xFF stay NaN


def test_bf16_in_the_f16_normal_range_converts_exactly():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    v = bits.view(torch.bfloat16)
    d = v.to(torch.float64)
    inside = torch.isfinite(d) & (d.abs() >= 2.0 ** -14) & (d.abs() <= 65504.0)
    assert torch.equal(v[inside].to(torch.float16).to(torch.float64), d[inside])
    # and outside it the conversion is not exact for some values (the bound is tight)
    below = torch.isfinite(d) & (d.abs() > 0) & (d.abs() < 2.0 ** -14)
    assert not torch.equal(v[below].to(torch.float16).to(torch.float64), d[below])


def test_products_of_e4m3_and_f16_operands_are_exact_in_fp32():
    # 4 significant bits x 11 significant bits = at most 15: every single product of
    # an E4M3 value and an f16 value is an FP32 value
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    e = codes.to(torch.float64)
    e = e[torch.isfinite(e)]
    g = torch.Generator().manual_seed(9)
    q = torch.randn(4096, generator=g).to(torch.float16).to(torch.float64)
    prod = e[:, None] * q[None, :]
    assert torch.equal(prod.to(torch.float32).to(torch.float64), prod)
