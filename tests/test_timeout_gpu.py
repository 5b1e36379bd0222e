"""Failure detection without a fault: every wait inside the tensor-core
decode is bounded.  The library's test hook makes the decode wait on a
barrier that nothing ever arrives on, with a short limit; the
kernel must give up, drain its own copies and products, record
MLA_ERR_DEVICE_TIMEOUT in the status word and return, leaving the context
usable: the next decode (hook off) is correct and reports no error."""
import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import inputs
from oracle import mla_oracle as O

from helpers import dev, device_cache, dims_of, f64, host_cache, rel_l2, rounded, tol

pytestmark = pytest.mark.gpu

TIMEOUT = 6


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    mla.load_library()
    torch.cuda.set_device(0)


def _decode(w, lens, q_cat, d):
    cache = device_cache(w, lens, capacity=d.cache_capacity)
    seq = torch.from_numpy(lens).cuda()
    Wn = mla.decode_default_splits(d)
    ws = torch.empty(mla.decode_workspace_bytes(d, Wn) // 4, dtype=torch.float32, device="cuda")
    used = mla.decode(d, dev(q_cat, w), cache, seq, w.softmax_scale, ws, Wn)
    o_lat = torch.zeros(w.B, w.H, w.d_c, dtype=torch.float32, device="cuda")
    lse = torch.zeros(w.B, w.H, dtype=torch.float32, device="cuda")
    mla.combine(d, seq, ws, used, o_lat, lse)
    return o_lat, lse


@pytest.mark.parametrize("d_r", [64, 0], ids=["rope", "nope"])
def test_injected_wait_gives_up_and_context_survives(d_r):
    w = inputs.WORKLOADS["v3_bf16"].scaled(B=3, N=700, d_r=d_r)
    lens = np.array([700, 65, 1], dtype=np.int32)
    d = dims_of(w, capacity=700)
    q_cat = inputs.normal((w.B, w.H, w.R), 0.5, 31, 3)
    assert mla.get_device_status() == 0
    try:
        mla.debug_inject_wait(200_000)      # ~0.1 ms of SM cycles, then give up
        _decode(w, lens, q_cat, d)
        status = mla.get_device_status()    # synchronises: the kernel returned
    finally:
        mla.debug_inject_wait(0)
    assert status == TIMEOUT
    # The context is intact: the same decode now completes and is correct.
    o_lat, lse = _decode(w, lens, q_cat, d)
    assert mla.get_device_status() == 0
    rows = host_cache(w, lens)
    cache = np.zeros((w.B, 700, w.R))
    for b, r in rows.items():
        cache[b, :len(r)] = r
    ref_o, ref_l = O.latent_attention(rounded(q_cat, w), cache, lens, w.softmax_scale, w.d_c)
    assert rel_l2(f64(o_lat), ref_o) < tol(w)
    assert np.max(np.abs(f64(lse) - ref_l)) < tol(w)
