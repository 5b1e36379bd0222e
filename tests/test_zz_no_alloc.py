"""The allocation-free decode entry point, mla_decode_noalloc, gives the same
result as mla_decode + mla_combine with a caller workspace.

It exists for callers that cannot allocate device memory (for example a
plugin that only receives fixed buffers from its host framework, or a
runtime whose device memory belongs to another allocator): its split-KV
partials live in a fixed array inside the library.  The test calls it through the C ABI twice in a row
on different inputs -- the shared array keeps the first call's contents, which
must not leak into the second -- and compares each result with the workspace
path, within the parity tolerances used elsewhere.  It builds and loads the
library itself, so it passes alone in a fresh process or after other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import binding as bd
from mla_latent_kv_nope_b200 import inputs

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS


@pytest.fixture(scope="module")
def lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    torch.cuda.set_device(0)
    return bd.load_library()


def _case(w, lens, seed):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    cap = int(max(lens))
    dims = mla.Dims(w.B, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, cap, w.dtype)
    cache = torch.empty(w.B, cap, w.R, dtype=dt, device="cuda")
    inputs.fill_cache(w.scaled(seed=seed), cache, lens, fill_rest=float("nan"))
    q_cat = torch.from_numpy(inputs.normal((w.B, w.H, w.R), 0.5, seed, 99)).to("cuda", dt)
    seq = torch.from_numpy(np.asarray(lens, dtype=np.int32)).cuda()
    return dims, cache, q_cat, seq


def _reference(dims, cache, q_cat, seq, scale):
    ws = torch.empty(mla.decode_workspace_bytes(dims) // 4, dtype=torch.float32, device="cuda")
    used = mla.decode(dims, q_cat, cache, seq, scale, ws)
    o = torch.empty(dims.B, dims.H, dims.d_c, device="cuda")
    lse = torch.empty(dims.B, dims.H, device="cuda")
    mla.combine(dims, seq, ws, used, o, lse)
    return o, lse


def _noalloc(lib, dims, cache, q_cat, seq, scale):
    o = torch.full((dims.B, dims.H, dims.d_c), float("nan"), device="cuda")
    lse = torch.full((dims.B, dims.H), float("nan"), device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = lib.mla_decode_noalloc(ctypes.byref(dims.c()), p(q_cat), p(cache), p(seq), scale,
                                p(o), p(lse),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, bd.STATUS.get(st, st)
    return o, lse


def _rel(a, b):
    a, b = a.double().cpu(), b.double().cpu()
    num = (a - b).norm(dim=-1)
    den = b.norm(dim=-1).clamp_min(1e-30)
    return float((num / den).max())


CASES = [
    (W["v3_bf16"].scaled(B=3), [700, 65, 1], [300, 300, 2], 1e-2),
    (W["ragged_append_bf16"].scaled(B=4), [1000, 64, 0, 129], [5, 900, 64, 17], 1e-2),
    (W["tiny_f32"].scaled(B=2), [64, 33], [10, 64], 1e-5),
]


@pytest.mark.parametrize("w,lens1,lens2,tol", CASES, ids=["bf16-H128", "bf16-H64", "f32"])
def test_noalloc_matches_workspace_path_twice(lib, w, lens1, lens2, tol):
    for call, (lens, seed) in enumerate([(lens1, 1), (lens2, 2)]):
        dims, cache, q_cat, seq = _case(w, lens, seed)
        ref_o, ref_l = _reference(dims, cache, q_cat, seq, w.softmax_scale)
        got_o, got_l = _noalloc(lib, dims, cache, q_cat, seq, w.softmax_scale)
        torch.cuda.synchronize()
        assert mla.get_device_status() == 0
        nz = torch.from_numpy(np.asarray(lens) > 0).cuda()
        assert _rel(got_o[nz], ref_o[nz]) < tol, f"call {call}"
        assert torch.all(got_o[~nz] == 0) and torch.all(torch.isneginf(got_l[~nz]))
        fin = torch.isfinite(ref_l)
        assert torch.equal(torch.isneginf(got_l), torch.isneginf(ref_l))
        assert float((got_l[fin] - ref_l[fin]).abs().max()) < tol, f"call {call}"


def test_noalloc_rejects_sizes_beyond_the_array(lib):
    # B * H * (d_c + 1) * 4 bytes above the fixed scratch: refused, nothing launched.
    too_big = bd.CDims(B=200, H=128, d_c=512, d_r=64, d_nope=128, d_v=128, cache_capacity=64,
                       dtype=bd.MLA_BF16)
    x = torch.empty(16, device="cuda")
    p = ctypes.c_void_p(x.data_ptr())
    st = lib.mla_decode_noalloc(ctypes.byref(too_big), p, p, p, 0.07, p, p, None)
    assert st == 4  # MLA_ERR_WORKSPACE
