"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments with the documented status before launching anything.
No GPU is needed: validation runs first, and fake (never dereferenced)
pointers are enough to exercise it."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_nope_b200 import binding as bd
from mla_latent_kv_nope_b200 import build as bld

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUP, ALIGN, WS, CUDA = 0, 1, 2, 3, 4, 5


@pytest.fixture(scope="module")
def lib():
    bld.build()
    return bd.load_library()


def _dims(**kw):
    base = dict(B=4, H=16, d_c=512, d_r=64, d_nope=128, d_v=128, cache_capacity=4097,
                dtype=bd.MLA_BF16)
    base.update(kw)
    return bd.CDims(**base)


P = ctypes.c_void_p
GOOD = P(0x10000)      # 16-byte aligned, never dereferenced
GOOD2 = P(0x20000)
BAD = P(0x10008)       # misaligned


def test_header_symbols_all_exported(lib):
    hdr = open(os.path.join(ROOT, "include", "mla.h")).read()
    declared = set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", hdr))
    assert declared == set(bd.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(bd, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        bd.load_library(str(tmp_path / "nope.so"))


def test_row_elems_and_status_strings(lib):
    assert lib.mla_cache_row_elems(512, 64) == 576
    assert lib.mla_cache_row_elems(32, 16) == 48
    assert lib.mla_status_string(0) == b"ok"
    assert lib.mla_status_string(4) == b"workspace missing or too small"
    assert lib.mla_status_string(99) == b"unknown status"


def test_workspace_layout_formula(lib):
    for B, H, W, d_r in [(4, 16, 148, 64), (32, 128, 74, 64), (64, 64, 148, 64), (1, 4, 3, 64),
                         (3, 192, 37, 64), (4, 16, 74, 0)]:
        d = _dims(B=B, H=H, d_r=d_r)
        slots = B + W - 1
        r256 = lambda v: (v + 255) // 256 * 256  # noqa: E731
        expect = r256(slots * H * 512 * 4) + r256(slots * H * 4)
        assert lib.mla_decode_workspace_bytes(ctypes.byref(d), W) == expect
    d = _dims(B=64, d_c=512, d_r=64)
    # bf16 standard dims: one fp32 partial per 256-wide slice of the hidden dim
    assert lib.mla_cache_append_workspace_bytes(ctypes.byref(d), 7168) == 28 * 64 * 576 * 4
    f = _dims(B=3, d_c=32, d_r=16, d_nope=16, d_v=16, dtype=bd.MLA_F32)
    assert lib.mla_cache_append_workspace_bytes(ctypes.byref(f), 64) == 256 * 3  # 3*48*4 -> 576, rounded to 768
    assert lib.mla_decode_workspace_bytes(ctypes.byref(d), 2000) == 0  # > 1024 splits


def test_dims_validation(lib):
    cases = [
        (None, INVALID),
        (_dims(B=0), INVALID), (_dims(H=-1), INVALID), (_dims(d_c=0), INVALID),
        (_dims(cache_capacity=0), INVALID), (_dims(dtype=7), INVALID),
        (_dims(d_c=500), UNSUP),                    # bf16 needs multiples of 8
        (_dims(dtype=bd.MLA_F32, d_c=30), UNSUP),   # f32 needs multiples of 4
        (_dims(dtype=bd.MLA_F32, d_c=2048), UNSUP),
    ]
    for d, want in cases:
        ref = ctypes.byref(d) if d is not None else None
        st = lib.mla_absorb_q(ref, GOOD, GOOD, GOOD, None, 10000.0, GOOD2, None)
        assert st == want, (d and d.d_c, st, want)


def test_decode_argument_errors(lib):
    d = _dims()
    ws_need = lib.mla_decode_workspace_bytes(ctypes.byref(d), 8)
    used = ctypes.c_int(-1)
    call = lambda dd, q=GOOD, c=GOOD, s=GOOD, scale=0.07, W=8, ws=GOOD2, wsb=ws_need: \
        lib.mla_decode(ctypes.byref(dd), q, c, s, scale, W, ws, wsb, ctypes.byref(used), None)  # noqa: E731
    assert call(_dims(d_c=256)) == UNSUP            # bf16 decode tile is 512 + 64
    assert call(_dims(d_r=32)) == UNSUP
    # 2^31 contiguous rows are past the 32-bit tensor-copy row coordinate.
    big = _dims(B=1 << 15, cache_capacity=1 << 16)
    big_ws = lib.mla_decode_workspace_bytes(ctypes.byref(big), 8)
    assert lib.mla_decode(ctypes.byref(big), GOOD, GOOD, GOOD, 0.07, 8, GOOD2, big_ws,
                          ctypes.byref(used), None) == UNSUP
    assert lib.mla_decode_noalloc(ctypes.byref(big), GOOD, GOOD, GOOD, 0.07, GOOD2, None,
                                  None) == UNSUP
    assert call(d, q=None) == INVALID
    assert call(d, scale=-0.5) == INVALID
    assert call(d, scale=float("inf")) == INVALID
    assert call(d, scale=float("nan")) == INVALID
    assert call(d, W=-1) == INVALID
    assert call(d, W=5000) == INVALID
    assert call(d, c=BAD) == ALIGN
    assert call(d, ws=BAD) == ALIGN
    assert call(d, wsb=ws_need - 1) == WS
    assert call(d, ws=None) == WS
    assert used.value == -1  # nothing reported before a successful launch


def test_other_entry_point_errors(lib):
    d = _dims()
    # combine
    need = lib.mla_decode_workspace_bytes(ctypes.byref(d), 8)
    assert lib.mla_combine(ctypes.byref(d), GOOD, GOOD2, need, 0, GOOD, None, None) == INVALID
    assert lib.mla_combine(ctypes.byref(d), GOOD, GOOD2, need - 4, 8, GOOD, None, None) == WS
    assert lib.mla_combine(ctypes.byref(d), GOOD, BAD, need, 8, GOOD, None, None) == ALIGN
    # merge of per-range results (sequence sharding)
    mg = lambda n=2, o=GOOD, l=GOOD, out=GOOD2, ls=None: lib.mla_merge_partials(  # noqa: E731
        ctypes.byref(d), n, o, l, out, ls, None)
    assert mg(n=0) == INVALID
    assert mg(n=1025) == INVALID
    assert mg(o=None) == INVALID
    assert mg(l=None) == INVALID
    assert mg(out=None) == INVALID
    assert mg(o=BAD) == ALIGN
    assert mg(ls=BAD) == ALIGN
    # out_proj
    assert lib.mla_out_proj(ctypes.byref(d), None, GOOD, GOOD2, None) == INVALID
    assert lib.mla_out_proj(ctypes.byref(d), GOOD, BAD, GOOD2, None) == ALIGN
    # absorb_q
    assert lib.mla_absorb_q(ctypes.byref(d), GOOD, None, GOOD, None, 1e4, GOOD2, None) == INVALID
    assert lib.mla_absorb_q(ctypes.byref(d), GOOD, GOOD, GOOD, GOOD, -1.0, GOOD2, None) == INVALID
    assert lib.mla_absorb_q(ctypes.byref(d), GOOD, GOOD, GOOD, BAD, 1e4, GOOD2, None) == ALIGN
    # cache append
    wsb = lib.mla_cache_append_workspace_bytes(ctypes.byref(d), 7168)
    ap = lambda hidden=7168, h=GOOD, eps=1e-6, base=1e4, ws=GOOD2, n=wsb: lib.mla_cache_append(  # noqa: E731
        ctypes.byref(d), hidden, h, GOOD, None, eps, base, GOOD, GOOD, ws, n, None)
    assert ap(hidden=0) == INVALID
    assert ap(h=None) == INVALID
    assert ap(eps=-1.0) == INVALID
    assert ap(base=0.0) == INVALID
    assert ap(hidden=7161) == UNSUP
    assert ap(h=BAD) == ALIGN
    assert ap(n=wsb - 1) == WS
    assert ap(ws=None) == WS


def test_prefill_entry_point_errors(lib):
    d = _dims(H=8)
    need = lib.mla_prefill_workspace_bytes(ctypes.byref(d), 100, 300)
    # K^C and V [H, L, 128] + k^R [L, 64], 16-bit, and the queries' RoPE
    # angles [T, 32] (cos, sin) in fp32, each rounded up to 1 KB.
    r1k = lambda x: (x + 1023) // 1024 * 1024  # noqa: E731
    assert need == 2 * r1k(8 * 300 * 128 * 2) + r1k(300 * 64 * 2) + r1k(100 * 32 * 8)
    pf = lambda T=100, L=300, qn=GOOD, qpe=GOOD, pos=GOOD, scale=0.0, base=1e4, out=GOOD2, \
        ws=GOOD2, n=need, dims=d: lib.mla_prefill(  # noqa: E731
            ctypes.byref(dims), T, L, qn, qpe, pos, GOOD, GOOD, GOOD, scale, base, out, None,
            ws, n, None)
    assert pf(T=0) == OK                     # nothing to do, nothing launched
    assert pf(T=-1) == INVALID
    assert pf(L=0) == INVALID
    assert pf(qn=None) == INVALID
    assert pf(pos=None) == INVALID
    assert pf(qpe=None) == INVALID           # d_r = 64 needs q_pe
    assert pf(scale=-0.1) == INVALID
    assert pf(base=0.0) == INVALID
    assert pf(out=BAD) == ALIGN
    assert pf(n=need - 1) == WS
    assert pf(ws=None) == WS
    for bad in (dict(dtype=bd.MLA_F32), dict(d_c=256), dict(d_r=32), dict(d_v=64)):
        dd = _dims(H=8, **bad)
        assert pf(dims=dd) == UNSUP
        assert lib.mla_prefill_workspace_bytes(ctypes.byref(dd), 100, 300) == 0
    assert pf(L=1 << 28) == UNSUP            # H * L beyond a 32-bit TMA row coordinate
    d0 = _dims(H=8, d_r=0)
    need0 = lib.mla_prefill_workspace_bytes(ctypes.byref(d0), 100, 300)
    assert need0 == 2 * r1k(8 * 300 * 128 * 2)
    assert pf(dims=d0, qpe=None, n=need0 - 1) == WS   # NoPE: q_pe may be NULL


def test_fold_entry_point_errors(lib):
    d = _dims(B=32, H=8)
    fw = lambda dm=300, wo=GOOD, dims=d: lib.mla_fold_output_weights(  # noqa: E731
        ctypes.byref(dims), dm, wo, GOOD, GOOD2, None)
    assert fw(dm=0) == INVALID
    assert fw(wo=None) == INVALID
    assert fw(wo=BAD) == ALIGN
    assert fw(dims=_dims(B=32, H=8, dtype=bd.MLA_F32)) == UNSUP
    assert fw(dims=_dims(B=32, H=8, d_v=64)) == UNSUP
    need = lib.mla_out_proj_folded_workspace_bytes(ctypes.byref(d), 300)
    assert need > 0
    fp = lambda dims=d, ws=GOOD2, n=need, x=GOOD: lib.mla_out_proj_folded(  # noqa: E731
        ctypes.byref(dims), 300, x, GOOD, GOOD, ws, n, None)
    assert fp(x=None) == INVALID
    assert fp(x=BAD) == ALIGN
    assert fp(n=need - 1) == WS
    assert fp(ws=None) == WS
    big = _dims(B=65, H=8)
    assert lib.mla_out_proj_folded_workspace_bytes(ctypes.byref(big), 300) == 0
    assert fp(dims=big) == UNSUP


def test_paged_entry_point_errors(lib):
    d = _dims(cache_capacity=4096)          # 64 pages of 64 rows per sequence at most
    need = lib.mla_decode_workspace_bytes(ctypes.byref(d), 8)
    used = ctypes.c_int(-1)
    dp = lambda pool=GOOD, npages=100, table=GOOD2, mb=64, ws=GOOD2, n=need: lib.mla_decode_paged(  # noqa: E731
        ctypes.byref(d), GOOD, pool, npages, table, mb, GOOD, 0.07, 8, ws, n, ctypes.byref(used),
        None)
    assert dp(table=None) == INVALID
    assert dp(npages=0) == INVALID
    assert dp(mb=63) == INVALID              # 63 pages cannot hold 4096 rows
    assert dp(table=BAD) == ALIGN
    assert dp(pool=BAD) == ALIGN
    assert dp(npages=1 << 26) == UNSUP       # rows of the pool beyond a 32-bit TMA coordinate
    assert dp(n=need - 1) == WS
    wsb = lib.mla_cache_append_workspace_bytes(ctypes.byref(d), 7168)
    ap = lambda table=GOOD2, mb=64: lib.mla_cache_append_paged(  # noqa: E731
        ctypes.byref(d), 7168, GOOD, GOOD, None, 1e-6, 1e4, GOOD, 100, table, mb, GOOD, GOOD2,
        wsb, None)
    assert ap(table=None) == INVALID
    assert ap(mb=10) == INVALID
    assert used.value == -1


SWITCH_UNITS = 4   # start-up units ahead of each sequence's tiles in the deal


def _deal(lens, W, tile=64):
    """Host restatement of the documented split-KV dealing: each sequence with
    tiles takes SWITCH_UNITS units and then one unit per tile, in batch order
    (T units); worker w takes units [w*T//W, (w+1)*T//W).  Returns T, the
    owner of each unit, and the (worker, sequence) pairs that share tiles."""
    nt = [(L + tile - 1) // tile if L > 0 else 0 for L in lens]
    units = [n + SWITCH_UNITS if n else 0 for n in nt]
    T = sum(units)
    pre = [sum(units[:b]) for b in range(len(lens))]
    owner = {}
    for w in range(W):
        for t in range(w * T // W, (w + 1) * T // W):
            owner[t] = w
    pairs = set()
    for b, (p, n) in enumerate(zip(pre, nt)):
        for t in range(p + SWITCH_UNITS, p + SWITCH_UNITS + n):
            pairs.add((owner[t], b))
    return T, owner, pairs


@pytest.mark.parametrize("lens,W", [([8192] * 32, 74), ([1, 2, 64, 65, 0, 300], 7),
                                    ([5, 0, 0, 7], 16), ([131072] * 4, 148),
                                    ([0, 0], 3)])
def test_split_dealing_slots_unique(lens, W):
    """Every work unit has exactly one worker; the partial slots b + w of the
    (worker, sequence) pairs are distinct and below B + W - 1; the owner of
    unit t is ((t+1)*W - 1) // T, the closed form the kernels use."""
    T, owner, pairs = _deal(lens, W)
    assert len(owner) == T
    slots = [b + w for (w, b) in pairs]
    assert len(slots) == len(set(slots))
    assert all(s < len(lens) + W - 1 for s in slots)
    for t, w in owner.items():
        assert ((t + 1) * W - 1) // T == w
