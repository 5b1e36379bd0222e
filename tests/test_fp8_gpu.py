"""GPU parity of the FP8 latent cache ([abeam] KV-cache quantisation; [yuuk]
"未解決の問い" FP8 for MLA) against the float64 oracle.

The cache is drawn in its stored format (E4M3 codes, power-of-two scales,
bf16 RoPE keys), so the decode is compared with the oracle's attention over
the exactly dequantised rows at the bf16 tolerance (dequantisation adds no
rounding), and with the bf16 decode over the same rows written as bf16, at
the same tolerance (the FP8 path multiplies fp16 operands: unscaled codes,
the query, the RoPE keys over the token's scale and P times it).  The append is compared code by code with the
oracle's quantisation of its own float64 latent; a code may differ by one
step only where the oracle's value lies within float32 accumulation error of
a rounding midpoint (the GPU forms the latent in fp32, in another order)."""
import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import inputs
from oracle import mla_oracle as O

from helpers import dev, dims_of, f64, rel_l2, rounded, tol

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    mla.load_library()
    torch.cuda.set_device(0)


def _fp8_cache(w, lens, cap, fill=0xFF):
    rb = mla.cache_fp8_row_bytes(w.d_c, w.d_r)
    cache = torch.empty(w.B, cap, rb, dtype=torch.uint8, device="cuda")
    scales = torch.empty(w.B, cap, dtype=torch.float32, device="cuda")
    inputs.fill_fp8_cache(w, cache, scales, lens, fill_rest_byte=fill)
    return cache, scales


def _oracle_rows(w, lens):
    """Float64 rows [c~ || k^R] of every sequence (c~ dequantised exactly)."""
    rows = {}
    for b in range(w.B):
        L = int(lens[b])
        codes, k, rope = inputs.fp8_cache_rows(w, b, L)
        c = O.dequantize_latent_rows(codes, np.ldexp(1.0, k))
        rows[b] = np.concatenate([c, rounded(rope, w)], axis=1)
    return rows


FP8_CASES = [
    ("H128", W["v3_bf16"].scaled(B=3, N=600), [600, 129, 1], 0, 1.0),
    ("H128-edges", W["v3_bf16"].scaled(B=8, N=200), [1, 63, 64, 65, 127, 128, 200, 0], 0, 1.0),
    ("H128-W7-peaked", W["v3_bf16"].scaled(B=2, N=900), [900, 77], 7, 10.0),
    ("H64", W["ragged_append_bf16"].scaled(B=5, N=700), [700, 1, 333, 64, 0], 0, 1.0),
    ("H16", W["v2lite_bf16"].scaled(B=4, N=300), [300, 65, 5, 64], 3, 1.0),
]


@pytest.mark.parametrize("name,w,lens,nsplit,boost", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_decode_fp8(name, w, lens, nsplit, boost):
    lens = np.array(lens, dtype=np.int32)
    cap = int(lens.max()) + 3
    d = dims_of(w, capacity=cap)
    cache, scales = _fp8_cache(w, lens, cap)
    seq = torch.from_numpy(lens).cuda()
    q_cat = inputs.normal((w.B, w.H, w.R), 0.5, 31, len(lens))
    scale = w.softmax_scale * boost
    Wn = nsplit or mla.decode_default_splits(d)
    ws = torch.full((mla.decode_workspace_bytes(d, Wn) // 4,), float("nan"), device="cuda")
    used = mla.decode_fp8(d, dev(q_cat, w), cache, scales, seq, scale, ws, Wn)
    o_lat = torch.empty(w.B, w.H, w.d_c, device="cuda")
    lse = torch.empty(w.B, w.H, device="cuda")
    mla.combine(d, seq, ws, used, o_lat, lse)
    assert mla.get_device_status() == 0
    rows = _oracle_rows(w, lens)
    ref_cache = np.zeros((w.B, cap, w.R))
    for b, r in rows.items():
        ref_cache[b, :len(r)] = r
    ref_o, ref_l = O.latent_attention(rounded(q_cat, w), ref_cache, lens, scale, w.d_c)
    nz = lens > 0
    got_o, got_l = f64(o_lat), f64(lse)
    assert rel_l2(got_o[nz], ref_o[nz]) < tol(w)
    assert np.all(got_o[~nz] == 0)
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(ref_l))
    assert np.max(np.abs(got_l[fin] - ref_l[fin])) < tol(w)
    # The same rows in a bf16 cache (exact: code x 2^k has 4 significant
    # bits): the bf16 decode agrees within the bf16 bar.
    bf = torch.zeros(w.B, cap, w.R, dtype=torch.bfloat16, device="cuda")
    for b, r in rows.items():
        if len(r):
            bf[b, :len(r)] = torch.from_numpy(r).to(torch.bfloat16).cuda()
    assert torch.equal(bf.float().cpu()[:, :, :w.d_c].double(),
                       torch.from_numpy(ref_cache[:, :, :w.d_c]))
    ws2 = torch.full_like(ws, float("nan"))
    used2 = mla.decode(d, dev(q_cat, w), bf, seq, scale, ws2, Wn)
    o2 = torch.empty_like(o_lat)
    l2 = torch.empty_like(lse)
    mla.combine(d, seq, ws2, used2, o2, l2)
    assert rel_l2(f64(o2)[nz], got_o[nz]) < tol(w)
    assert np.max(np.abs(f64(l2)[fin] - got_l[fin])) < tol(w)


def test_decode_fp8_small_scales():
    """Scales of 2^-20 .. 2^-17: most dequantised values fall below fp16's
    normal range and keep its subnormal step (2^-24) in the fp16 operands;
    the output stays within the bf16 bar of the oracle over the same rows."""
    w = W["v3_bf16"].scaled(B=3, N=500)
    lens = np.array([500, 129, 64], dtype=np.int32)
    cap = 503
    d = dims_of(w, capacity=cap)
    cache, scales = _fp8_cache(w, lens, cap)
    scales.mul_(2.0 ** -11)                     # k in [-20, -17]
    seq = torch.from_numpy(lens).cuda()
    q_cat = inputs.normal((w.B, w.H, w.R), 0.5, 31, 3)
    ws = torch.full((mla.decode_workspace_bytes(d, 0) // 4,), float("nan"), device="cuda")
    used = mla.decode_fp8(d, dev(q_cat, w), cache, scales, seq, w.softmax_scale, ws)
    o_lat = torch.empty(w.B, w.H, w.d_c, device="cuda")
    lse = torch.empty(w.B, w.H, device="cuda")
    mla.combine(d, seq, ws, used, o_lat, lse)
    assert mla.get_device_status() == 0
    ref_cache = np.zeros((w.B, cap, w.R))
    for b in range(w.B):
        L = int(lens[b])
        codes, k, rope = inputs.fp8_cache_rows(w, b, L)
        c = O.dequantize_latent_rows(codes, np.ldexp(1.0, k - 11))
        ref_cache[b, :L] = np.concatenate([c, rounded(rope, w)], axis=1)
    ref_o, ref_l = O.latent_attention(rounded(q_cat, w), ref_cache, lens, w.softmax_scale, w.d_c)
    assert rel_l2(f64(o_lat), ref_o) < tol(w)
    assert np.max(np.abs(f64(lse) - ref_l)) < tol(w)


def _near_midpoint(x, rel=2e-5):
    """True where x lies within `rel` (relative) of a rounding midpoint of the
    E4M3 grid, i.e. where fp32 accumulation error may flip the rounding."""
    a = np.abs(x)
    lo = O.e4m3_decode(O.e4m3_encode(a))
    # neighbours on the grid: the values one code below and above
    codes = O.e4m3_encode(a).astype(np.int64)
    up = O.e4m3_decode(np.clip(codes + 1, 0, 0x7E).astype(np.uint8))
    dn = O.e4m3_decode(np.clip(codes - 1, 0, 0x7E).astype(np.uint8))
    mids = np.stack([(lo + up) / 2, (lo + dn) / 2])
    return np.any(np.abs(mids - a) <= rel * np.maximum(a, 2.0 ** -9), axis=0)


@pytest.mark.parametrize("w", [W["ragged_append_bf16"].scaled(B=9, N=300, hidden=512),
                               W["ragged_append_bf16"]],
                         ids=lambda w: f"B{w.B}-hidden{w.hidden}")
def test_cache_append_fp8(w):
    lens = inputs.seqlens(w)
    cap = int(lens.max()) + 1
    d = dims_of(w, capacity=cap)
    h, Wdkv = inputs.append_inputs(w)
    gamma = 1.0 + inputs.normal((w.d_c,), 0.1, 77, 1)
    rb = mla.cache_fp8_row_bytes(w.d_c, w.d_r)
    cache = torch.full((w.B, cap, rb), 0xA5, dtype=torch.uint8, device="cuda")
    scales = torch.full((w.B, cap), -3.0, dtype=torch.float32, device="cuda")
    before, sbefore = cache.clone(), scales.clone()
    seq = torch.from_numpy(lens).cuda()
    ws = torch.empty(mla.cache_append_workspace_bytes(d, w.hidden) // 4, device="cuda")
    mla.cache_append_fp8(d, dev(h, w), dev(Wdkv, w), torch.from_numpy(gamma).cuda(), cache,
                         scales, seq, ws, eps=w.eps)
    assert mla.get_device_status() == 0
    np.testing.assert_array_equal(seq.cpu().numpy(), lens + 1)
    # Indexing bit-exact: only row L_b (and scale L_b) of each sequence changed.
    idx = torch.from_numpy(lens).long().cuda()
    mask = torch.zeros(w.B, cap, dtype=torch.bool, device="cuda")
    mask[torch.arange(w.B), idx] = True
    assert torch.equal(cache[~mask], before[~mask])
    assert torch.equal(scales[~mask], sbefore[~mask])
    # Values against the oracle's append, quantised by the oracle.
    zero = np.zeros((w.B, cap, w.R))
    _, _, rows_ref = O.cache_append(zero, lens, rounded(h, w), rounded(Wdkv, w), w.d_c,
                                    gamma=gamma.astype(np.float64), eps=w.eps)
    c_ref = rows_ref[:, :w.d_c]
    codes_ref, scale_ref = O.quantize_latent_rows(c_ref)
    got_rows = cache[torch.arange(w.B), idx].cpu()
    got_codes = got_rows[:, :w.d_c].numpy()
    got_scale = scales[torch.arange(w.B), idx].cpu().numpy().astype(np.float64)
    # Scales: exact, except where the row maximum sits at a binade edge.
    ratio = np.max(np.abs(c_ref), axis=1) / scale_ref       # in (224, 448]
    edge = (np.abs(ratio - 448.0) < 448.0 * 2e-5) | (np.abs(ratio - 224.0) < 224.0 * 2e-5)
    assert np.all((got_scale == scale_ref) | edge)
    same = got_scale == scale_ref
    diff = got_codes[same] != codes_ref[same]
    x = c_ref[same] / scale_ref[same][:, None]
    assert not np.any(diff & ~_near_midpoint(x)), int(np.sum(diff & ~_near_midpoint(x)))
    assert np.mean(diff) < 1e-3
    # RoPE keys in bf16 within the bf16 tolerance.
    rope = got_rows[:, w.d_c:].contiguous().view(torch.bfloat16).double().numpy()
    assert rel_l2(rope, rows_ref[:, w.d_c:]) < tol(w)
    # And the dequantised latent within E4M3's relative step (2^-4) of the oracle.
    deq = O.dequantize_latent_rows(got_codes, got_scale)
    assert rel_l2(deq, c_ref) < 2.0 ** -4
