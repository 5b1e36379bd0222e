"""The Python binding marshals arguments only: host (CPU) tensors are refused
with an error before anything reaches the library, so no call can run on the
CPU or hand a host address to a kernel.  Runs without a GPU."""
import pytest
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import binding as bd

B, H, d_c, d_r, d_n, d_v, cap, hid = 2, 4, 32, 16, 16, 16, 128, 64
D = mla.Dims(B, H, d_c, d_r, d_n, d_v, cap, "f32")
R = d_c + d_r


def f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


CALLS = {
    "cache_append": lambda: mla.cache_append(D, f32(B, hid), f32(R, hid), None, f32(B, cap, R),
                                             i32(B), f32(1024)),
    "cache_append_paged": lambda: mla.cache_append_paged(D, f32(B, hid), f32(R, hid), None,
                                                         f32(4, 64, R), i32(B, 2), i32(B),
                                                         f32(1024)),
    "absorb_q": lambda: mla.absorb_q(D, f32(B, H, d_n), f32(B, H, d_r), f32(H, d_n, d_c),
                                     i32(B), f32(B, H, R)),
    "decode": lambda: mla.decode(D, f32(B, H, R), f32(B, cap, R), i32(B), 0.2, f32(1024), 4),
    "decode_paged": lambda: mla.decode_paged(D, f32(B, H, R), f32(4, 64, R), i32(B, 2), i32(B),
                                             0.2, f32(1024), 4),
    "combine": lambda: mla.combine(D, i32(B), f32(1024), 4, f32(B, H, d_c), f32(B, H)),
    "out_proj": lambda: mla.out_proj(D, f32(B, H, d_c), f32(H, d_v, d_c), f32(B, H, d_v)),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name, monkeypatch):
    # Any call that got past validation would reach the library: make that fail
    # the test rather than run.
    def no_lib(*a, **k):
        raise AssertionError("the library was reached with host tensors")
    monkeypatch.setattr(bd, "load_library", no_lib)
    with pytest.raises(ValueError, match="CUDA"):
        CALLS[name]()


def test_workspace_must_be_device_memory():
    with pytest.raises(ValueError, match="workspace"):
        bd._need_ws(torch.zeros(16))
    with pytest.raises(ValueError, match="workspace"):
        bd._need_ws(None)
