"""The FP8 decode widens each stored code to an fp16 operand as (E4M3 value)
times the token's power-of-two scale.  These CPU checks pin the numeric facts
that step relies on, against torch's own float8 and float16 conversions
(library routines), not against the kernel:

* every finite E4M3 value is an fp16 value (the conversion is exact);
* for every finite code and every scale 2^k the header allows, the product
  rounded once to fp16 equals the exact product whenever its magnitude lies
  in fp16's normal range [2^-14, 65504), and is within half of fp16's
  subnormal step (2^-25) of it below that;
* the largest product the append can produce for a latent row of
  magnitude below 65504 stays below 65504 (no overflow)."""
import numpy as np
import torch


def _e4m3_values():
    codes = torch.arange(256, dtype=torch.uint8)
    v = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v[np.isfinite(v)]


def test_every_e4m3_value_is_an_fp16_value():
    v = _e4m3_values()
    as_f16 = torch.from_numpy(v).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(as_f16, v)


def test_scaled_codes_in_fp16_exact_in_normal_range():
    v = _e4m3_values()
    for k in range(-24, 16):
        exact = v * 2.0 ** k
        rounded = torch.from_numpy(exact).to(torch.float16).to(torch.float64).numpy()
        mag = np.abs(exact)
        normal = (mag >= 2.0 ** -14) & (mag < 65504.0)
        assert np.array_equal(rounded[normal], exact[normal]), k
        small = mag < 2.0 ** -14
        assert np.all(np.abs(rounded[small] - exact[small]) <= 2.0 ** -25), k


def test_append_scales_keep_products_in_range():
    # The append picks the smallest 2^k with max|c| / 2^k <= 448, so every
    # stored code times 2^k is at most 448 * 2^k < 2 max|c|, and for
    # max|c| < 2^15 that is below 65504.
    for amax in [1e-6, 0.01, 1.0, 3.7, 448.0, 1000.0, 2.0 ** 15 - 1]:
        k = int(np.ceil(np.log2(amax / 448.0)))
        assert amax / 2.0 ** k <= 448.0 and amax / 2.0 ** (k - 1) > 448.0
        assert 448.0 * 2.0 ** k < 65504.0 or amax >= 2.0 ** 15
