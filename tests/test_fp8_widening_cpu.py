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


# ---------------------------------------------------------------------------
# Why the decode widens the codes instead of multiplying them as FP8 operands:
# a float64 model of both designs against the attention over the same
# dequantised rows (the oracle's E4M3 codec and row quantiser), at the
# decode's shapes (d_c = 512, d_r = 64, softmax scale 1/sqrt(192)).
# ---------------------------------------------------------------------------
def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).double().numpy()


def _f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def _pow2_scale(amax):
    amax = np.where(amax > 0, amax, 448.0)
    return np.exp2(np.ceil(np.log2(amax / 448.0)))


def _e4m3(x):
    from oracle import mla_oracle as O
    return O.e4m3_decode(O.e4m3_encode(x))


def _fp8_operand_errors(H, L, q_gain, seed=7, d_c=512, d_r=64, tile=64):
    """Max over heads of ||o - o_ref|| / ||o_ref|| for: the fp16 widening
    (query, widened rows and P in fp16), an E4M3 query (per-head power-of-two
    scale) against the E4M3 codes, and P times the token scale rounded to
    E4M3 per 64-key tile against the codes."""
    from oracle import mla_oracle as O
    rng = np.random.default_rng(seed)
    c = O.rms_norm(rng.standard_normal((L, d_c)))
    codes, scale = O.quantize_latent_rows(_bf16(c))
    ct, e = O.dequantize_latent_rows(codes, scale), O.e4m3_decode(codes)
    kr = _bf16(rng.standard_normal((L, d_r)))
    q = _bf16(q_gain * 0.226 * rng.standard_normal((H, d_c + d_r)))
    sm = 1.0 / np.sqrt(192.0)
    S = sm * (q @ np.concatenate([ct, kr], 1).T)
    S16 = sm * (_f16(q) @ np.concatenate([_f16(ct), _f16(kr)], 1).T)
    qn = q[:, :d_c]
    sq = _pow2_scale(np.abs(qn).max(axis=1))[:, None]
    S8 = sm * (((_e4m3(qn / sq) * sq) @ e.T) * scale[None, :] + q[:, d_c:] @ kr.T)
    err = {"fp16": [], "e4m3_query": [], "e4m3_p": []}
    for i in range(H):
        p = np.exp(S[i] - S[i].max())
        ref = p @ ct / p.sum()
        p16 = _f16(np.exp(S16[i] - S16[i].max()))
        p8q = np.exp(S8[i] - S8[i].max())
        acc, l = np.zeros(d_c), 0.0
        for t0 in range(0, L, tile):
            pp = p[t0:t0 + tile] * scale[t0:t0 + tile]
            sp = _pow2_scale(np.abs(pp).max())
            p8 = _e4m3(pp / sp) * sp
            acc += p8 @ e[t0:t0 + tile]
            l += (p8 / scale[t0:t0 + tile]).sum()
        for k, o in (("fp16", p16 @ _f16(ct) / p16.sum()), ("e4m3_query", p8q @ ct / p8q.sum()),
                     ("e4m3_p", acc / l)):
            err[k].append(np.linalg.norm(o - ref) / np.linalg.norm(ref))
    return {k: max(v) for k, v in err.items()}


def test_fp8_operands_would_miss_the_parity_bar():
    """The fp16 widening stays two orders of magnitude inside the 1e-2 bar;
    rounding either the query or P to E4M3 (what FP8-operand MMAs need)
    misses it on its own, with flat and with peaked attention alike."""
    for q_gain in (1.0, 10.0):
        err = _fp8_operand_errors(H=8, L=2048, q_gain=q_gain)
        assert err["fp16"] < 1e-3, err
        assert err["e4m3_query"] > 1e-2, err
        assert err["e4m3_p"] > 1e-2, err
