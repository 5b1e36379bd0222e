"""GPU parity of the materialised prefill ([MLA-とは] "実装上のトレードオフ":
prefill forms k^C = W^UK c and v^C = W^UV c and runs ordinary causal
attention) against the float64 oracle's prefill_materialised, element by
element: out per (query, head) by relative L2 error, lse by absolute error,
both within the bf16 bar of 1e-2.  Cases: one token, a tile minus/plus one,
several ragged query and key tiles, a cached prefix before the prompt,
unordered positions (some past the last row), NoPE, a peaked softmax (the
lazy rescale of O), the full 128 heads, and a long prompt."""
import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import inputs
from oracle import mla_oracle as O

from helpers import dev, f64, rel_l2, rounded

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS
BASE = W["v3_bf16"]


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    mla.load_library()
    torch.cuda.set_device(0)


def _case(H, T, L, d_r=64, seed=0):
    w = BASE.scaled(B=1, H=H, d_r=d_r, N=L, seed=seed)
    qn = inputs.normal((T, H, w.d_nope), 1.0, seed, 61, T)
    qp = inputs.normal((T, H, max(d_r, 1)), 1.0, seed, 62, T)[:, :, :d_r]
    Wuk, Wuv = inputs.weights(w)
    rows = inputs.cache_rows(w, 0, L)
    return w, qn, np.ascontiguousarray(qp), Wuk, Wuv, rows


def _run(w, qn, qp, q_pos, Wuk, Wuv, rows, scale=0.0, ws_fill=None):
    T, L = qn.shape[0], rows.shape[0]
    d = mla.Dims(1, w.H, w.d_c, w.d_r, w.d_nope, w.d_v, 1, "bf16")
    out = torch.full((T, w.H, w.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, w.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(mla.prefill_workspace_bytes(d, T, L), dtype=torch.uint8, device="cuda")
    if ws_fill is not None:
        ws.fill_(ws_fill)
    mla.prefill(d, dev(qn, w), dev(qp, w) if w.d_r else None,
                torch.from_numpy(np.asarray(q_pos, np.int32)).cuda(), dev(Wuk, w), dev(Wuv, w),
                dev(rows, w), out, ws, lse=lse, softmax_scale=scale)
    assert mla.get_device_status() == 0
    return f64(out), f64(lse)


def _oracle(w, qn, qp, q_pos, Wuk, Wuv, rows, scale):
    return O.prefill_materialised(rounded(qn, w), rounded(qp, w), np.asarray(q_pos),
                                  rounded(Wuk, w), rounded(Wuv, w), rounded(rows, w), w.d_c,
                                  scale)


def _check(got, ref):
    out, lse = got
    r_out, r_lse = ref
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    assert rel_l2(out, r_out) < 1e-2
    assert np.max(np.abs(lse - r_lse)) < 1e-2


@pytest.mark.parametrize("H,T,L,prefix,d_r", [
    (4, 1, 1, 0, 64),
    (4, 63, 63, 0, 64),
    (4, 64, 64, 0, 64),
    (4, 129, 129, 0, 64),
    (4, 300, 300, 0, 64),
    (4, 130, 230, 100, 64),       # a cached prefix of 100 rows before the prompt
    (4, 200, 200, 0, 0),          # NoPE
    (16, 257, 390, 133, 0),
], ids=["T1", "T63", "T64", "T129", "T300", "prefix100", "nope-T200", "nope-prefix133"])
def test_prefill_causal(H, T, L, prefix, d_r):
    w, qn, qp, Wuk, Wuv, rows = _case(H, T, L, d_r)
    q_pos = prefix + np.arange(T)
    scale = 1.0 / np.sqrt(w.d_nope + d_r)
    _check(_run(w, qn, qp, q_pos, Wuk, Wuv, rows, ws_fill=0xFF),
           _oracle(w, qn, qp, q_pos, Wuk, Wuv, rows, scale))


def test_prefill_unordered_positions():
    """Positions in any order, repeated, and past the last row (which then
    sees every row, rotated at its own position)."""
    w, qn, qp, Wuk, Wuv, rows = _case(4, 150, 170)
    q_pos = np.random.default_rng(3).integers(0, 200, size=150)
    scale = 1.0 / np.sqrt(192)
    _check(_run(w, qn, qp, q_pos, Wuk, Wuv, rows, scale=scale),
           _oracle(w, qn, qp, q_pos, Wuk, Wuv, rows, scale))


def test_prefill_negative_position_sees_nothing():
    w, qn, qp, Wuk, Wuv, rows = _case(4, 70, 90)
    q_pos = np.arange(70)
    q_pos[[0, 33, 69]] = -1
    out, lse = _run(w, qn, qp, q_pos, Wuk, Wuv, rows)
    neg = q_pos < 0
    assert np.all(out[neg] == 0) and np.all(lse[neg] == -np.inf)
    ref = _oracle(w, qn, qp, np.where(neg, 0, q_pos), Wuk, Wuv, rows, 1.0 / np.sqrt(192))
    assert rel_l2(out[~neg], ref[0][~neg]) < 1e-2
    assert np.max(np.abs(lse[~neg] - ref[1][~neg])) < 1e-2


def test_prefill_peaked_softmax():
    """A 10x scale: logits with std ~7, so the running maximum jumps by more
    than 2^8 between key tiles and O is rescaled in tensor memory."""
    w, qn, qp, Wuk, Wuv, rows = _case(4, 384, 384)
    q_pos = np.arange(384)
    scale = 10.0 / np.sqrt(192)
    _check(_run(w, qn, qp, q_pos, Wuk, Wuv, rows, scale=scale),
           _oracle(w, qn, qp, q_pos, Wuk, Wuv, rows, scale))


def test_prefill_all_heads():
    w, qn, qp, Wuk, Wuv, rows = _case(128, 200, 200)
    q_pos = np.arange(200)
    _check(_run(w, qn, qp, q_pos, Wuk, Wuv, rows),
           _oracle(w, qn, qp, q_pos, Wuk, Wuv, rows, 1.0 / np.sqrt(192)))


def test_prefill_long_prompt_sampled():
    """T = L = 2048 at 8 heads (16 query tiles, up to 16 key tiles each); the
    oracle runs on every fourth query token of every head."""
    w, qn, qp, Wuk, Wuv, rows = _case(8, 2048, 2048)
    q_pos = np.arange(2048)
    out, lse = _run(w, qn, qp, q_pos, Wuk, Wuv, rows)
    sel = np.arange(0, 2048, 4)
    ref_out, ref_lse = _oracle(w, qn[sel], qp[sel], q_pos[sel], Wuk, Wuv, rows,
                               1.0 / np.sqrt(192))
    assert rel_l2(out[sel], ref_out) < 1e-2
    assert np.max(np.abs(lse[sel] - ref_lse)) < 1e-2


def test_prefill_deterministic():
    w, qn, qp, Wuk, Wuv, rows = _case(4, 200, 260)
    q_pos = 60 + np.arange(200)
    a = _run(w, qn, qp, q_pos, Wuk, Wuv, rows)
    b = _run(w, qn, qp, q_pos, Wuk, Wuv, rows, ws_fill=0x7F)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
