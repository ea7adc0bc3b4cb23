"""CPU checks of how the bf16 output bound is applied (no GPU).

The forward's bf16 bound is: relative Frobenius error <= 5e-3 and max abs
error <= 2e-2 * rms(y).  Rounding the exact y to bf16 already moves an
element by up to half a bf16 spacing, 2^-8 |y| in the worst case, so an
element with |y| >= 2^e > 5.12 rms(y) near a rounding midpoint breaks the
literal max-abs bound with no computation error at all.  The tests apply the
max-abs bound to the error beyond the output's own final rounding
(helpers.max_abs_beyond_rounding).  These tests pin that reading: the
exactly rounded result always passes, the literal bound can fail on it, and
a real computation error of the bound's size still fails.
"""
import torch

from helpers import (MAX_ABS_BF16, assert_bf16_close, bf16_half_ulp, max_abs_beyond_rounding,
                     max_abs_over_rms)


def test_half_ulp_values():
    v = torch.tensor([1.0, 1.99, 2.0, 0.75, -3.0, 4.0, 7.99, 2.0 ** -126, 0.0, 2.0 ** -130])
    want = torch.tensor([2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -9, 2.0 ** -7, 2.0 ** -6, 2.0 ** -6,
                         2.0 ** -134, 2.0 ** -134, 2.0 ** -134], dtype=torch.float64)
    assert torch.equal(bf16_half_ulp(v), want)


def test_exactly_rounded_result_always_passes():
    """For any fp32 y (the kernels round their fp32 result once),
    |bf16(y) - y| <= half_ulp(bf16(y)): the exactly rounded output has zero
    error beyond its rounding (round to nearest even, every binade, signs,
    values that round up into the next binade).  (torch converts float64 to
    bf16 through fp32, a double rounding, so y is drawn in fp32.)"""
    g = torch.Generator().manual_seed(0)
    y = (torch.randn(200000, generator=g, dtype=torch.float64) * torch.exp2(
        torch.randint(-30, 30, (200000,), generator=g).double())).float()
    # values just below a power of two round up into the next binade
    y[:64] = (torch.exp2(torch.arange(64).double() - 32) * (1 - 2.0 ** -12)).float()
    got = y.to(torch.bfloat16)
    y = y.double()
    assert ((got.double() - y).abs() <= bf16_half_ulp(got)).all()
    assert max_abs_beyond_rounding(got, y) == 0.0


def test_literal_bound_fails_on_exact_rounding_and_the_reading_does_not():
    """rms(y) = 0.7 and one element on the rounding midpoint 4 + 2^-6 (bf16
    spacing in [4, 8) is 2^-5): the exactly rounded output is 2^-6 = 0.0223
    rms away, above the literal 2e-2 bound."""
    y = torch.full((10000,), 0.7, dtype=torch.float64)
    y[17] = 4.0 + 2.0 ** -6
    got = y.float().to(torch.bfloat16)
    assert got[17].item() == 4.0                         # ties to even
    assert max_abs_over_rms(got, y) > MAX_ABS_BF16
    assert max_abs_beyond_rounding(got, y) == 0.0
    assert_bf16_close(got, y, "exactly rounded")


def test_computation_error_of_the_bound_size_still_fails():
    """An element off by 0.03 (0.06 rms) before rounding fails the bound
    after rounding too."""
    y = torch.full((10000,), 0.5, dtype=torch.float64)
    y[3] = 1.0
    computed = y.clone()
    computed[3] += 0.03
    got = computed.float().to(torch.bfloat16)
    beyond = max_abs_beyond_rounding(got, y)
    assert beyond > MAX_ABS_BF16
    # exactly: |1.03125 - 1| - 2^-8 over rms 0.5 (the rms barely moves)
    rms = torch.sqrt((y * y).mean()).item()
    assert abs(beyond - (0.03125 - 2.0 ** -8) / rms) < 1e-12


def test_wider_outputs_get_no_allowance():
    """fp32 results (the grouped GEMM's slot outputs) are checked literally."""
    y = torch.full((100,), 1.0, dtype=torch.float64)
    got = y.float().clone()
    got[0] += 0.015
    assert abs(max_abs_beyond_rounding(got, y) - max_abs_over_rms(got, y)) < 1e-15
