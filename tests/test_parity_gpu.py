"""GPU parity: every entry point of the C ABI against the float64 CPU oracle on
the same seeded inputs.  Tolerances (from the target statement): max over
(sequence, head) of the relative L2 error <= 1e-2 for bf16 inputs with fp32
accumulation and <= 1e-5 for the fp32 path; lse by absolute error with the
same bounds; cache-append indexing bit-exact."""
import math

import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import inputs
from oracle import mla_oracle as O

from helpers import (dev, device_cache, dims_of, f64, host_cache, rel_l2, rounded, tol,
                     torch_dtype)

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS
SMALL_BF16 = W["v2lite_bf16"].scaled(B=3, N=200)


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    mla.load_library()
    torch.cuda.set_device(0)


def _lse_err(got, ref):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    return float(np.max(np.abs(got[fin] - ref[fin]))) if fin.any() else 0.0


# ---------------------------------------------------------------------------
# absorb_q
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [W["tiny_f32"], SMALL_BF16, W["v3_bf16"],
                               W["ragged_append_bf16"].scaled(B=17)],
                         ids=lambda w: f"{w.name}-B{w.B}-H{w.H}")
def test_absorb_q(w):
    qn, qp = inputs.query(w)
    Wuk, _ = inputs.weights(w)
    pos = np.arange(w.B, dtype=np.int32) * 977 + 5
    d = dims_of(w)
    q_cat = torch.empty(w.B, w.H, w.R, dtype=torch_dtype(w), device="cuda")
    mla.absorb_q(d, dev(qn, w), dev(qp, w), dev(Wuk, w), torch.from_numpy(pos).cuda(), q_cat)
    ref = O.absorb_q(rounded(qn, w), rounded(qp, w), rounded(Wuk, w), pos)
    got = f64(q_cat)
    assert rel_l2(got[..., :w.d_c], ref[..., :w.d_c]) < tol(w)
    assert rel_l2(got[..., w.d_c:], ref[..., w.d_c:]) < tol(w)
    # q_pos = NULL: the RoPE block is copied unchanged.
    mla.absorb_q(d, dev(qn, w), dev(qp, w), dev(Wuk, w), None, q_cat)
    np.testing.assert_array_equal(f64(q_cat)[..., w.d_c:], rounded(qp, w))


# ---------------------------------------------------------------------------
# out_proj
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [W["tiny_f32"], SMALL_BF16, W["v3_bf16"]],
                         ids=lambda w: w.name)
def test_out_proj(w):
    _, Wuv = inputs.weights(w)
    o_lat = inputs.normal((w.B, w.H, w.d_c), 0.05, 123, 1)
    out = torch.empty(w.B, w.H, w.d_v, dtype=torch_dtype(w), device="cuda")
    mla.out_proj(dims_of(w), dev(o_lat, w, torch.float32), dev(Wuv, w), out)
    ref = O.out_proj(o_lat.astype(np.float64), rounded(Wuv, w))
    assert rel_l2(f64(out), ref) < tol(w)


# ---------------------------------------------------------------------------
# cache append: values within tolerance, indexing bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [W["tiny_f32"].scaled(B=3, hidden=64),
                               W["ragged_append_bf16"].scaled(B=9, N=300),
                               W["ragged_append_bf16"]],
                         ids=lambda w: f"{w.name}-B{w.B}")
def test_cache_append(w):
    lens = inputs.seqlens(w) if w.ragged else np.array([0, 1, 63][:w.B] + [5] * max(0, w.B - 3),
                                                       dtype=np.int32)
    h, Wdkv = inputs.append_inputs(w)
    gamma = 1.0 + inputs.normal((w.d_c,), 0.1, 77, 1)
    d = dims_of(w)
    dt = torch_dtype(w)
    # Sentinel-filled cache: every element a fixed non-trivial pattern.
    cache = torch.full((w.B, w.capacity, w.R), -3.25, dtype=dt, device="cuda")
    before = cache.clone()
    seq = torch.from_numpy(lens).cuda()
    ws = torch.empty(mla.cache_append_workspace_bytes(d, h.shape[1]) // 4, dtype=torch.float32,
                     device="cuda")
    mla.cache_append(d, dev(h, w), dev(Wdkv, w), torch.from_numpy(gamma).cuda(), cache, seq, ws,
                     eps=w.eps)
    assert mla.get_device_status() == 0
    np.testing.assert_array_equal(seq.cpu().numpy(), lens + 1)
    # Bit-exact: only row L_b of each sequence changed.
    mask = torch.zeros(w.B, w.capacity, dtype=torch.bool, device="cuda")
    mask[torch.arange(w.B), torch.from_numpy(lens).long().cuda()] = True
    raw = lambda t: t.view(torch.int16) if dt == torch.bfloat16 else t.view(torch.int32)  # noqa
    assert torch.equal(raw(cache)[~mask], raw(before)[~mask])
    rows_got = f64(cache[torch.arange(w.B), torch.from_numpy(lens).long().cuda()])
    zero = np.zeros((w.B, w.capacity, w.R))
    _, _, rows_ref = O.cache_append(zero, lens, rounded(h, w), rounded(Wdkv, w), w.d_c,
                                    gamma=gamma.astype(np.float64), eps=w.eps)
    assert rel_l2(rows_got[:, :w.d_c], rows_ref[:, :w.d_c]) < tol(w)
    assert rel_l2(rows_got[:, w.d_c:], rows_ref[:, w.d_c:]) < tol(w)


def test_cache_append_capacity_is_reported():
    w = W["ragged_append_bf16"].scaled(B=3, N=10, hidden=64)
    d = dims_of(w, capacity=10)
    lens = np.array([3, 10, 9], dtype=np.int32)  # sequence 1 is full
    h, Wdkv = inputs.append_inputs(w)
    cache = torch.zeros(w.B, 10, w.R, dtype=torch.bfloat16, device="cuda")
    seq = torch.from_numpy(lens).cuda()
    ws = torch.empty(mla.cache_append_workspace_bytes(d, h.shape[1]) // 4, dtype=torch.float32, device="cuda")
    mla.get_device_status()
    mla.cache_append(d, dev(h, w), dev(Wdkv, w), None, cache, seq, ws)
    assert mla.get_device_status() == 7  # MLA_ERR_BOUNDS
    assert mla.get_device_status() == 0  # cleared by the read
    np.testing.assert_array_equal(seq.cpu().numpy(), [4, 10, 10])
    assert torch.count_nonzero(cache[1]) == 0
    assert torch.count_nonzero(cache[0, 3]) > 0 and torch.count_nonzero(cache[2, 9]) > 0


# ---------------------------------------------------------------------------
# decode + combine against the latent-attention definition
# ---------------------------------------------------------------------------
def _run_decode(w, lens, q_cat_np, scale, num_splits=0, capacity=None, fill_rest=float("nan")):
    cap = capacity if capacity is not None else max(int(lens.max()), 1)
    d = dims_of(w, capacity=cap)
    cache = device_cache(w, lens, capacity=cap, fill_rest=fill_rest)
    seq = torch.from_numpy(lens.astype(np.int32)).cuda()
    W_ = num_splits or mla.decode_default_splits(d)
    ws = torch.empty(mla.decode_workspace_bytes(d, W_) // 4, dtype=torch.float32, device="cuda")
    ws.fill_(float("nan"))  # nothing may depend on unwritten workspace
    used = mla.decode(d, dev(q_cat_np, w), cache, seq, scale, ws, W_)
    assert used == W_
    o_lat = torch.empty(w.B, w.H, w.d_c, dtype=torch.float32, device="cuda")
    lse = torch.empty(w.B, w.H, dtype=torch.float32, device="cuda")
    mla.combine(d, seq, ws, used, o_lat, lse)
    assert mla.get_device_status() == 0
    return f64(o_lat), f64(lse)


def _oracle_latent(w, lens, q_cat_np, scale):
    rows = host_cache(w, lens)
    cap = max(int(lens.max()), 1)
    cache = np.zeros((w.B, cap, w.R))
    for b, r in rows.items():
        cache[b, :len(r)] = r
    return O.latent_attention(rounded(q_cat_np, w), cache, lens, scale, w.d_c)


DECODE_CASES = [
    ("tiny_f32", W["tiny_f32"], [64], 0, 1.0),
    ("tiny_f32-ragged", W["tiny_f32"].scaled(B=5), [64, 1, 0, 130, 65], 3, 1.0),
    ("bf16-H16-edges", SMALL_BF16.scaled(B=8), [1, 63, 64, 65, 127, 128, 200, 0], 0, 1.0),
    ("bf16-H16-W1", SMALL_BF16.scaled(B=4), [200, 5, 64, 1], 1, 1.0),
    ("bf16-H16-Wbig", SMALL_BF16.scaled(B=4), [200, 5, 64, 1], 1000, 1.0),
    ("bf16-H64", W["ragged_append_bf16"].scaled(B=5, N=700), [700, 1, 333, 64, 0], 0, 1.0),
    ("bf16-H128", W["v3_bf16"].scaled(B=3, N=600), [600, 129, 1], 0, 1.0),
    ("bf16-H128-W7", W["v3_bf16"].scaled(B=3, N=600), [600, 129, 1], 7, 1.0),
    ("bf16-H128-peaked", W["v3_bf16"].scaled(B=2, N=400), [400, 77], 0, 10.0),
    ("bf16-H16-peaked", SMALL_BF16.scaled(B=2), [190, 64], 0, 10.0),
    # more than 64 heads: CTA pairs, 128 heads per pair
    ("bf16-H128-edges", W["v3_bf16"].scaled(B=8, N=200), [1, 63, 64, 65, 127, 128, 200, 0], 0, 1.0),
    ("bf16-H128-W1", W["v3_bf16"].scaled(B=3, N=300), [300, 1, 100], 1, 1.0),
    ("bf16-H128-Wbig", W["v3_bf16"].scaled(B=2, N=2000), [2000, 3], 300, 1.0),
    ("bf16-H128-peaked-long", W["v3_bf16"].scaled(B=1, N=3000), [3000], 2, 10.0),
    # Many partials per sequence with a peaked softmax: the combine's running
    # maximum jumps between rounds of partials (one sequence over 74 workers,
    # some of them with empty ranges; one long sequence among 31 short ones)
    ("bf16-H128-peaked-manysplits", W["v3_bf16"].scaled(B=1, N=3000), [3000], 0, 10.0),
    ("bf16-H128-one-long-many-short", W["v3_bf16"].scaled(B=25, N=4000),
     [4000] + [64] * 23 + [1], 0, 10.0),
    ("bf16-H100", W["v3_bf16"].scaled(B=3, H=100, N=300), [300, 65, 0], 0, 1.0),
    ("bf16-H192", W["v3_bf16"].scaled(B=2, H=192, N=200), [200, 64], 0, 1.0),
    # NoPE ([yuuk] 横断的知見: MLA layers without RoPE): d_r = 0, rows are c^KV alone
    ("bf16-nope-H128", W["v3_bf16"].scaled(B=3, N=600, d_r=0), [600, 129, 1], 0, 1.0),
    ("bf16-nope-H64", W["ragged_append_bf16"].scaled(B=4, N=300, d_r=0), [300, 64, 1, 0], 0,
     1.0),
    ("bf16-nope-H16-peaked", SMALL_BF16.scaled(B=2, d_r=0), [190, 64], 0, 10.0),
]


@pytest.mark.parametrize("name,w,lens,nsplit,boost", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_combine(name, w, lens, nsplit, boost):
    lens = np.array(lens, dtype=np.int32)
    q_cat = inputs.normal((w.B, w.H, w.R), 0.5, 31, len(lens))
    scale = w.softmax_scale * boost
    got_o, got_l = _run_decode(w, lens, q_cat, scale, nsplit)
    ref_o, ref_l = _oracle_latent(w, lens, q_cat, scale)
    nz = lens > 0
    assert rel_l2(got_o[nz], ref_o[nz]) < tol(w)
    assert np.all(got_o[~nz] == 0)
    assert _lse_err(got_l, ref_l) < tol(w)


@pytest.mark.parametrize("w", [SMALL_BF16.scaled(B=1100, N=40),
                               W["v3_bf16"].scaled(B=1030, N=24)],
                         ids=["H16-B1100", "H128-B1030"])
def test_decode_more_sequences_than_the_shared_prefix(w):
    """More than 1024 sequences: the decode kernels walk the length array in
    global memory instead of their shared-memory tile prefix.  Short ragged
    lengths (0 included); every sequence is checked against the oracle."""
    lens = np.random.default_rng(5).integers(0, w.N + 1, size=w.B).astype(np.int32)
    q_cat = inputs.normal((w.B, w.H, w.R), 0.5, 31, w.B)
    got_o, got_l = _run_decode(w, lens, q_cat, w.softmax_scale)
    ref_o, ref_l = _oracle_latent(w, lens, q_cat, w.softmax_scale)
    nz = lens > 0
    assert rel_l2(got_o[nz], ref_o[nz]) < tol(w)
    assert np.all(got_o[~nz] == 0)
    assert _lse_err(got_l, ref_l) < tol(w)


def _paged_copy(cache, seed=7, spare=5):
    """The contiguous cache [B, cap, R] (cap a multiple of 64) as a shuffled
    pool of 64-row pages with spare pages, and its block table."""
    B, cap, R = cache.shape
    nb = cap // mla.PAGE_ROWS
    n_pages = B * nb + spare
    perm = torch.from_numpy(np.random.default_rng(seed).permutation(n_pages)[:B * nb]).cuda()
    pool = torch.full((n_pages, mla.PAGE_ROWS, R), float("nan"), dtype=cache.dtype,
                      device="cuda")
    pool[perm] = cache.reshape(B * nb, mla.PAGE_ROWS, R)
    table = perm.to(torch.int32).reshape(B, nb).contiguous()
    return pool, table


PAGED_CASES = [
    ("bf16-H128", W["v3_bf16"].scaled(B=3, N=600), [600, 129, 1], 0),
    ("bf16-H64-W7", W["ragged_append_bf16"].scaled(B=5, N=700), [700, 1, 333, 64, 0], 7),
    ("f32-tiny", W["tiny_f32"].scaled(B=3), [64, 1, 130], 3),
]


@pytest.mark.parametrize("name,w,lens,nsplit", PAGED_CASES, ids=[c[0] for c in PAGED_CASES])
def test_paged_decode_matches_contiguous(name, w, lens, nsplit):
    """The paged decode reads the same rows through the block table: its
    partials, merged, are bit-identical to the contiguous decode's, and both
    match the oracle."""
    lens = np.array(lens, dtype=np.int32)
    cap = (int(lens.max()) + 63) // 64 * 64
    d = dims_of(w, capacity=cap)
    cache = device_cache(w, lens, capacity=cap, fill_rest=float("nan"))
    pool, table = _paged_copy(cache)
    seq = torch.from_numpy(lens).cuda()
    q_cat = inputs.normal((w.B, w.H, w.R), 0.5, 31, len(lens))
    qd = dev(q_cat, w)
    Wn = nsplit or mla.decode_default_splits(d)
    outs = []
    for paged in (False, True):
        ws = torch.full((mla.decode_workspace_bytes(d, Wn) // 4,), float("nan"), device="cuda")
        if paged:
            used = mla.decode_paged(d, qd, pool, table, seq, w.softmax_scale, ws, Wn)
        else:
            used = mla.decode(d, qd, cache, seq, w.softmax_scale, ws, Wn)
        o_lat = torch.empty(w.B, w.H, w.d_c, device="cuda")
        lse = torch.empty(w.B, w.H, device="cuda")
        mla.combine(d, seq, ws, used, o_lat, lse)
        assert mla.get_device_status() == 0
        outs.append((o_lat, lse))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ref_o, ref_l = _oracle_latent(w, lens, q_cat, w.softmax_scale)
    nz = lens > 0
    assert rel_l2(f64(outs[1][0])[nz], ref_o[nz]) < tol(w)
    assert _lse_err(f64(outs[1][1]), ref_l) < tol(w)


@pytest.mark.parametrize("w", [W["ragged_append_bf16"].scaled(B=5, N=300, hidden=512),
                               W["tiny_f32"].scaled(B=3, hidden=64)], ids=["bf16", "f32"])
def test_paged_append_matches_contiguous(w):
    """Appending through the block table writes the same bytes into the page
    that holds row L_b, and nothing else; lengths advance the same way."""
    lens = inputs.seqlens(w)
    cap = (int(lens.max()) + 1 + 63) // 64 * 64
    d = dims_of(w, capacity=cap)
    cache = device_cache(w, lens, capacity=cap, fill_rest=float("nan"))
    pool, table = _paged_copy(cache)
    h, Wdkv = inputs.append_inputs(w)
    hd, Wd = dev(h, w), dev(Wdkv, w)
    ws = torch.empty(mla.cache_append_workspace_bytes(d, w.hidden) // 4, device="cuda")
    seq_a = torch.from_numpy(lens).cuda()
    seq_b = seq_a.clone()
    mla.cache_append(d, hd, Wd, None, cache, seq_a, ws)
    pool_before = pool.clone()
    mla.cache_append_paged(d, hd, Wd, None, pool, table, seq_b, ws)
    assert mla.get_device_status() == 0
    assert torch.equal(seq_a, seq_b)
    gathered = pool[table.long().reshape(-1)].reshape(w.B, cap, w.R)
    assert torch.equal(gathered.view(torch.int16 if w.dtype == "bf16" else torch.int32),
                       cache.view(torch.int16 if w.dtype == "bf16" else torch.int32))
    # the spare pages are untouched
    used_pages = set(table.reshape(-1).tolist())
    spare = [p for p in range(pool.shape[0]) if p not in used_pages]
    assert torch.equal(pool[spare].isnan(), pool_before[spare].isnan())


def test_paged_bad_page_is_reported():
    """A page id outside the pool is never dereferenced: the decode reads zeros
    for it and the status word reports MLA_ERR_BOUNDS."""
    w = W["v3_bf16"].scaled(B=2, N=128)
    lens = np.array([128, 64], dtype=np.int32)
    d = dims_of(w, capacity=128)
    cache = device_cache(w, lens, capacity=128)
    pool, table = _paged_copy(cache)
    table[0, 1] = pool.shape[0] + 3           # outside the pool
    seq = torch.from_numpy(lens).cuda()
    ws = torch.empty(mla.decode_workspace_bytes(d, 4) // 4, device="cuda")
    mla.decode_paged(d, dev(inputs.normal((2, w.H, w.R), 0.5, 1, 1), w), pool, table, seq,
                     w.softmax_scale, ws, 4)
    assert mla.get_device_status() == 7      # MLA_ERR_BOUNDS
    assert mla.get_device_status() == 0


COMBINE_CASES = [
    ("few-partials", 6, [300, 0, 64, 1000, 1], 0.0),
    # 2 sequences over 100 workers (59 work units: some workers empty): the
    # kernel whose warps split the partials, rounds of four per warp
    ("many-partials-split-warps", 100, [3000, 200], 0.0),
    # one long sequence among short ones: the per-column kernel with about
    # 25 partials (7 rounds), a fifth of them empty (lse = -inf)
    ("many-partials-rounds-with-empties", 60, [4000] + [64] * 19, 0.2),
]


@pytest.mark.parametrize("name,Wn,lens,empty", COMBINE_CASES, ids=[c[0] for c in COMBINE_CASES])
def test_combine_alone(name, Wn, lens, empty):
    """Synthetic partials (lse spread with std 3, so the running maximum moves
    between rounds) placed in the documented workspace slots; the merge must
    equal the log-sum-exp combination of exactly those partials."""
    lens = np.array(lens, dtype=np.int32)
    B, H, d_c = len(lens), 16, 512
    w = SMALL_BF16.scaled(B=B)
    d = dims_of(w, capacity=int(lens.max()))
    # The documented deal: each non-empty sequence takes 4 start-up units,
    # then one unit per 64-key tile; worker w takes units [wT/W, (w+1)T/W).
    nt = [(L + 63) // 64 for L in lens]
    units = [n + 4 if n else 0 for n in nt]
    T = sum(units)
    pre = np.concatenate([[0], np.cumsum(units)])
    slots = B + Wn - 1
    o_all, l_all = inputs.partials(1, H, slots, d_c, seed=3, empty_frac=empty)
    ws = torch.full((mla.decode_workspace_bytes(d, Wn) // 4,), float("nan"), device="cuda")
    # documented partial layout: o_part[slot][d_c / 4][H][4]
    o_ws = o_all[0].reshape(H, slots, d_c // 4, 4).transpose(1, 2, 0, 3)
    ws[:slots * H * d_c] = torch.from_numpy(np.ascontiguousarray(o_ws).reshape(-1)).cuda()
    lse_off = ((slots * H * d_c * 4 + 255) // 256 * 256) // 4
    ws[lse_off:lse_off + slots * H] = torch.from_numpy(l_all[0].T.reshape(-1)).cuda()
    o_lat = torch.empty(B, H, d_c, device="cuda")
    lse = torch.empty(B, H, device="cuda")
    mla.combine(d, torch.from_numpy(lens).cuda(), ws, Wn, o_lat, lse)
    torch.cuda.synchronize()
    for b in range(B):
        if nt[b] == 0:
            assert torch.all(o_lat[b] == 0) and torch.all(torch.isneginf(lse[b]))
            continue
        ws_ = sorted({w_ for t in range(pre[b] + 4, pre[b + 1]) for w_ in range(Wn)
                      if w_ * T // Wn <= t < (w_ + 1) * T // Wn})
        sl = [b + w_ for w_ in ws_]
        ref_o, ref_l = O.combine_partials(o_all[0][:, sl].astype(np.float64),
                                          l_all[0][:, sl].astype(np.float64))
        assert rel_l2(f64(o_lat[b]), ref_o) < 1e-5
        assert _lse_err(f64(lse[b]), ref_l) < 1e-5


# ---------------------------------------------------------------------------
# Whole step (append, absorb, decode, combine, out_proj) against the
# materialised-MHA oracle.
# ---------------------------------------------------------------------------
def _full_step(w, sample_pairs=None, num_splits=0):
    lens = inputs.seqlens(w)
    d = dims_of(w)
    cache = device_cache(w, lens)
    seq = torch.from_numpy(lens).cuda()
    qn, qp = inputs.query(w)
    Wuk, Wuv = inputs.weights(w)
    step_kw = {}
    h = Wdkv = None
    if w.append:
        h, Wdkv = inputs.append_inputs(w)
        step_kw["h"] = dev(h, w)
        q_pos = lens.copy()              # the new token's position
    else:
        q_pos = lens - 1                 # the query is the newest cached token
    step = mla.DecodeStep(d, dev(Wuk, w), dev(Wuv, w), dev(Wdkv, w) if w.append else None,
                          num_splits=num_splits)
    out = step(dev(qn, w), dev(qp, w), torch.from_numpy(q_pos.astype(np.int32)).cuda(), cache,
               seq, **step_kw)
    torch.cuda.synchronize()
    assert mla.get_device_status() == 0
    got, got_lat, got_lse = f64(out), f64(step.o_lat), f64(step.lse)

    if sample_pairs is None:
        sample_pairs = [(b, i) for b in range(w.B) for i in range(w.H)]
    seqs = sorted({b for b, _ in sample_pairs})
    rows = host_cache(w, lens, seqs)
    rq_n, rq_p, rWuk, rWuv = (rounded(a, w) for a in (qn, qp, Wuk, Wuv))
    worst = worst_lat = worst_lse = 0.0
    for b in seqs:
        L = int(lens[b])
        cache_b = np.zeros((1, L + 1, w.R))
        cache_b[0, :L] = rows[b]
        Lb = np.array([L])
        if w.append:
            cache_b, Lb, _ = O.cache_append(cache_b, Lb, rounded(h, w)[b:b + 1],
                                            rounded(Wdkv, w), w.d_c, eps=w.eps)
        heads = [i for bb, i in sample_pairs if bb == b]
        o, ol, ls = O.mla_decode_materialised(
            rq_n[b:b + 1, heads], rq_p[b:b + 1, heads], q_pos[b:b + 1], rWuk[heads],
            rWuv[heads], cache_b, Lb, w.softmax_scale)
        worst = max(worst, rel_l2(got[b, heads], o[0]))
        worst_lat = max(worst_lat, rel_l2(got_lat[b, heads], ol[0]))
        worst_lse = max(worst_lse, float(np.max(np.abs(got_lse[b, heads] - ls[0]))))
    if w.append:
        np.testing.assert_array_equal(seq.cpu().numpy(), lens + 1)
    return worst, worst_lat, worst_lse


SMALL_STEPS = [
    W["tiny_f32"],
    W["v2lite_bf16"].scaled(B=2, N=300),
    W["v3_bf16"].scaled(B=2, N=260),
    W["ragged_append_bf16"].scaled(B=6, N=500, hidden=512),
    # NoPE ([yuuk] 横断的知見: MLA layers without RoPE): d_r = 0, so the cache
    # row is c^KV alone and the query has no decoupled part (fp32 path).
    W["tiny_f32"].scaled(name="tiny_f32_nope", B=3, N=150, d_r=0, ragged=True, append=True,
                         hidden=64),
    # NoPE on the bf16 tensor-core path at the production latent width (d_c = 512):
    # 128 heads (CTA pairs) and 64 heads, with the append
    W["v3_bf16"].scaled(name="v3_bf16_nope", B=3, N=300, d_r=0, ragged=True, append=True,
                        hidden=512),
    W["ragged_append_bf16"].scaled(name="ragged_bf16_nope", B=5, N=400, d_r=0, hidden=512),
]


@pytest.mark.parametrize("w", SMALL_STEPS, ids=lambda w: f"{w.name}-small")
def test_full_step_small(w):
    e, el, els = _full_step(w)
    assert e < tol(w) and el < tol(w) and els < tol(w), (e, el, els)


@pytest.mark.parametrize("w", [W["ragged_append_bf16"].scaled(B=6, N=500, hidden=512),
                               W["v3_bf16"].scaled(B=3, N=300, append=True, hidden=512)],
                         ids=["ragged-append", "v3-append"])
def test_decode_step_streams_and_graph(w):
    """DecodeStep with absorb_q on a forked stream, and the same step replayed
    from a CUDA graph, give bit-identical outputs to the single-stream step
    (same kernels, same inputs, deterministic reductions)."""
    lens = inputs.seqlens(w)
    d = dims_of(w)
    qn, qp = inputs.query(w)
    Wuk, Wuv = inputs.weights(w)
    h, Wdkv = inputs.append_inputs(w)
    args = [dev(qn, w), dev(qp, w), torch.from_numpy(lens.astype(np.int32)).cuda()]
    hd = dev(h, w)

    def run(step, cache, seq, graph=False):
        seq0 = seq.clone()
        if graph:
            g = step.capture(*args, cache, seq, h=hd, after=lambda: seq.copy_(seq0))
            for _ in range(2):
                g.replay()
        else:
            step(*args, cache, seq, h=hd)
            seq.copy_(seq0)
        torch.cuda.synchronize()
        assert mla.get_device_status() == 0
        return step.out.clone(), step.lse.clone()

    outs = []
    for overlap, graph in [(False, False), (True, False), (True, True)]:
        cache = device_cache(w, lens)
        seq = torch.from_numpy(lens).cuda()
        step = mla.DecodeStep(d, dev(Wuk, w), dev(Wuv, w), dev(Wdkv, w), overlap=overlap)
        outs.append(run(step, cache, seq, graph))
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0])
        assert torch.equal(l, outs[0][1])


def test_host_pipeline_matches_step():
    """DecodeStep.host_pipeline (inputs from pinned host memory, copies
    overlapped with the previous step) returns, in host memory, exactly the
    output of the plain step on the same inputs, for runs of 1, 2 and 5
    steps (both graphs, and the prologue and epilogue copies)."""
    w = W["v3_bf16"].scaled(B=3, N=300, append=True, hidden=512)
    lens = inputs.seqlens(w)
    d = dims_of(w)
    qn, qp = inputs.query(w)
    Wuk, Wuv = inputs.weights(w)
    h, Wdkv = inputs.append_inputs(w)
    cache = device_cache(w, lens)
    seq0 = torch.from_numpy(lens).cuda()
    seq = seq0.clone()
    step = mla.DecodeStep(d, dev(Wuk, w), dev(Wuv, w), dev(Wdkv, w))
    pos = torch.from_numpy(lens.astype(np.int32))
    host = [dev(qn, w).cpu().pin_memory(), dev(qp, w).cpu().pin_memory(), pos.pin_memory(),
            dev(h, w).cpu().pin_memory()]
    step(*[t.cuda() for t in host[:3]], cache, seq, h=host[3].cuda())
    seq.copy_(seq0)
    torch.cuda.synchronize()
    ref = step.out.cpu()
    out = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    pipe = step.host_pipeline(host, out, cache, seq, after=lambda: seq.copy_(seq0))
    for n in (1, 2, 5):
        out.zero_()
        pipe.run(n)
        torch.cuda.synchronize()
        assert mla.get_device_status() == 0
        assert torch.equal(out, ref)
    assert pipe.bytes_per_step() == (sum(t.numel() * t.element_size() for t in host),
                                     out.numel() * out.element_size())


def _sample(w, n_seq, heads, seed=0):
    r = np.random.default_rng(seed)
    seqs = sorted(set([0, w.B - 1] + list(r.choice(w.B, size=min(n_seq, w.B), replace=False))))
    return [(int(b), int(i)) for b in seqs for i in heads]


@pytest.mark.parametrize("name", ["tiny_f32", "v2lite_bf16", "v3_bf16", "longctx_bf16",
                                  "ragged_append_bf16"])
def test_full_step_full_size(name):
    """Each configuration at its full size in the launch configuration the
    bench times (default splits), checked on sampled (sequence, head) pairs
    that the oracle recomputes from scratch."""
    w = W[name]
    heads = sorted({0, w.H - 1, w.H // 2, 1 % w.H})
    n_seq = {"tiny_f32": 1, "v2lite_bf16": 4, "v3_bf16": 6, "longctx_bf16": 2,
             "ragged_append_bf16": 6}[name]
    e, el, els = _full_step(w, _sample(w, n_seq, heads))
    assert e < tol(w) and el < tol(w) and els < tol(w), (e, el, els)
