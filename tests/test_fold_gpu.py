"""GPU parity of W^O folded into the value side ([MLA-とは] "Value側の吸収":
B_i = W^O_i W^UV_i, u = sum_i B_i o_lat_i) against the float64 oracle: the
folded weights against the oracle's fold, and the folded projection against
the unfolded definition u = sum_i W^O_i (W^UV_i o_lat_i)."""
import numpy as np
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import inputs
from oracle import mla_oracle as O

from helpers import dev, dims_of, f64, rel_l2, rounded

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from mla_latent_kv_nope_b200 import build
    build.build()
    mla.load_library()
    torch.cuda.set_device(0)


def _w_o(w, d_model):
    return inputs.normal((d_model, w.H * w.d_v), 0.02, 41, d_model)


@pytest.mark.parametrize("w,d_model", [(W["v2lite_bf16"].scaled(B=4, H=4), 300),
                                       (W["v3_bf16"], 7168)], ids=["H4-d300", "v3-d7168"])
def test_fold_output_weights(w, d_model):
    d = dims_of(w)
    _, Wuv = inputs.weights(w)
    Wo = _w_o(w, d_model)
    W_fold = torch.empty(d_model, w.H * w.d_c, dtype=torch.bfloat16, device="cuda")
    mla.fold_output_weights(d, dev(Wo, w), dev(Wuv, w), W_fold)
    assert mla.get_device_status() == 0
    got = W_fold.view(d_model, w.H, w.d_c)
    # Sampled heads (all at the small size), every row of those heads.
    heads = range(w.H) if w.H <= 8 else [0, 1, w.H // 2, w.H - 1]
    for i in heads:
        ref = O.fold_output_weights(rounded(Wo[:, i * w.d_v:(i + 1) * w.d_v], w),
                                    rounded(Wuv[i:i + 1], w))[0]
        assert rel_l2(f64(got[:, i]), ref) < 1e-2


@pytest.mark.parametrize("B,H,d_model", [(4, 4, 300), (32, 128, 1024), (64, 16, 2048)],
                         ids=["B4-H4-d300", "B32-H128-d1024", "B64-H16-d2048"])
def test_out_proj_folded(B, H, d_model):
    w = W["v3_bf16"].scaled(B=B, H=H)
    d = dims_of(w)
    _, Wuv = inputs.weights(w)
    Wo = _w_o(w, d_model)
    o_lat = inputs.normal((B, H, w.d_c), 0.05, 123, 1)
    W_fold = torch.empty(d_model, H * w.d_c, dtype=torch.bfloat16, device="cuda")
    mla.fold_output_weights(d, dev(Wo, w), dev(Wuv, w), W_fold)
    u = torch.empty(B, d_model, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(mla.out_proj_folded_workspace_bytes(d, d_model), dtype=torch.uint8,
                     device="cuda")
    for _ in range(2):   # a second call on the same workspace gives the same bits
        mla.out_proj_folded(d, dev(o_lat, w, torch.float32), W_fold, u, ws)
        first = u.clone() if _ == 0 else first
    assert mla.get_device_status() == 0
    assert torch.equal(u, first)
    # The unfolded definition, in float64 from the same rounded weights.
    ref = O.output_projection(O.out_proj(o_lat.astype(np.float64), rounded(Wuv, w)),
                              rounded(Wo, w))
    assert rel_l2(f64(u), ref) < 1e-2
    if H * d_model * w.d_c <= 1 << 22:   # the folded form too, where it is small
        B_fold = O.fold_output_weights(rounded(Wo, w), rounded(Wuv, w))
        assert rel_l2(f64(u), O.folded_output(o_lat, B_fold)) < 1e-2


def test_out_proj_folded_rejects_large_batches():
    w = W["v3_bf16"].scaled(B=65, H=4)
    assert mla.out_proj_folded_workspace_bytes(dims_of(w), 256) == 0
