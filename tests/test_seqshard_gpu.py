"""Sequence-sharded decode on one GPU.  The ranks are emulated one after the
other in one process (no kernel waits on another): each decodes and combines
its token range of every sequence from ``token_ranges``; the library's
log-sum-exp merge of their per-range results is compared with the float64
oracle over whole sequences.  ``sequence_sharded_attend`` with one rank must
give the unsharded step's output."""
import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import dist as mdist
from mla_latent_kv_nope_b200 import inputs
from oracle import mla_oracle as O

from helpers import dev, device_cache, dims_of, f64, host_cache, rel_l2, rounded, tol

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    mla.load_library()
    torch.cuda.set_device(0)


def _range_results(w, lens, cache, q_cat, ranges):
    """Each emulated rank's (o_lat, lse) over its token ranges, stacked."""
    world = ranges.shape[0]
    o_parts = torch.empty(world, w.B, w.H, w.d_c, dtype=torch.float32, device="cuda")
    l_parts = torch.empty(world, w.B, w.H, dtype=torch.float32, device="cuda")
    for k in range(world):
        n = (ranges[k, :, 1] - ranges[k, :, 0]).astype(np.int32)
        cap = max(int(n.max()), 1)
        local = torch.full((w.B, cap, w.R), float("nan"), dtype=cache.dtype, device="cuda")
        for b in range(w.B):
            lo, hi = int(ranges[k, b, 0]), int(ranges[k, b, 1])
            local[b, :hi - lo] = cache[b, lo:hi]
        d = dims_of(w, capacity=cap)
        seq = torch.from_numpy(n).cuda()
        ws = torch.empty(mla.decode_workspace_bytes(d) // 4, dtype=torch.float32, device="cuda")
        used = mla.decode(d, q_cat, local, seq, w.softmax_scale, ws)
        mla.combine(d, seq, ws, used, o_parts[k], l_parts[k])
    return o_parts, l_parts


CASES = [
    ("tiny_f32-3", W["tiny_f32"].scaled(B=4), [64, 1, 0, 300], 3),
    ("bf16-H16-4", W["v2lite_bf16"].scaled(B=3, N=700), [700, 65, 130], 4),
    ("bf16-H128-2", W["v3_bf16"].scaled(B=2, N=1000), [1000, 129], 2),
    ("bf16-H64-8", W["ragged_append_bf16"].scaled(B=3, N=900), [900, 1, 400], 8),
]


@pytest.mark.parametrize("name,w,lens,world", CASES, ids=[c[0] for c in CASES])
def test_merge_of_token_ranges_matches_oracle(name, w, lens, world):
    lens = np.array(lens, dtype=np.int32)
    cap = int(lens.max())
    cache = device_cache(w, lens, capacity=cap)
    q_np = inputs.normal((w.B, w.H, w.R), 0.5, 41, world)
    ranges = mdist.token_ranges(lens, world)
    o_parts, l_parts = _range_results(w, lens, cache, dev(q_np, w), ranges)
    d = dims_of(w, capacity=cap)
    o_lat = torch.empty(w.B, w.H, w.d_c, dtype=torch.float32, device="cuda")
    lse = torch.empty(w.B, w.H, dtype=torch.float32, device="cuda")
    mla.merge_partials(d, o_parts, l_parts, o_lat, lse)
    assert mla.get_device_status() == 0
    rows = host_cache(w, lens)
    full = np.zeros((w.B, cap, w.R))
    for b, r in rows.items():
        full[b, :len(r)] = r
    ref_o, ref_l = O.latent_attention(rounded(q_np, w), full, lens, w.softmax_scale, w.d_c)
    got_o, got_l = f64(o_lat), f64(lse)
    nz = lens > 0
    assert rel_l2(got_o[nz], ref_o[nz]) < tol(w)
    assert np.all(got_o[~nz] == 0) and np.all(np.isneginf(got_l[~nz]))
    assert np.max(np.abs(got_l[nz] - ref_l[nz])) < tol(w)


def test_merge_skips_empty_ranges():
    """A range result with lse = -inf is not read (its o_lat may be NaN); all
    empty gives zeros and -inf."""
    w = W["tiny_f32"].scaled(B=2, H=4)
    d = dims_of(w, capacity=64)
    rng = np.random.default_rng(3)
    o = rng.normal(size=(3, 2, 4, w.d_c))
    lse = rng.normal(size=(3, 2, 4))
    lse[1] = -np.inf
    o[1] = np.nan
    lse[:, 1, 2] = -np.inf
    o_t = torch.from_numpy(o).float().cuda()
    l_t = torch.from_numpy(lse).float().cuda()
    o_lat = torch.empty(2, 4, w.d_c, device="cuda")
    l_out = torch.empty(2, 4, device="cuda")
    mla.merge_partials(d, o_t, l_t, o_lat, l_out)
    ref_o, ref_l = O.combine_partials(np.moveaxis(f64(o_t), 0, 2), np.moveaxis(f64(l_t), 0, 2))
    got_o, got_l = f64(o_lat), f64(l_out)
    assert not np.isnan(got_o).any()
    np.testing.assert_allclose(got_o, ref_o, rtol=1e-5, atol=1e-6)
    assert np.isneginf(got_l[1, 2]) and np.all(got_o[1, 2] == 0)
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(got_l[fin], ref_l[fin], atol=1e-5)


def test_sequence_sharded_attend_one_rank_equals_step():
    w = W["v3_bf16"].scaled(B=2, N=300)
    lens = np.array([300, 77], dtype=np.int32)
    cap = int(lens.max())
    d = dims_of(w, capacity=cap)
    cache = device_cache(w, lens, capacity=cap)
    seq = torch.from_numpy(lens).cuda()
    qn, qp = inputs.query(w)
    Wuk, Wuv = inputs.weights(w)
    q_nope, q_pe, W_UK, W_UV = dev(qn, w), dev(qp, w), dev(Wuk, w), dev(Wuv, w)
    q_pos = seq - 1
    step = mla.DecodeStep(d, W_UK, W_UV, overlap=False)
    ref = step.attend(q_nope, q_pe, q_pos, cache, seq).clone()
    got = mdist.sequence_sharded_attend(step, q_nope, q_pe, q_pos, cache, seq, world=1)
    torch.cuda.synchronize()
    assert mla.get_device_status() == 0
    assert torch.equal(got, ref)
