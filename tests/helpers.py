"""Test-side helpers: put seeded generator values on the device in the
workload's dtype, and give the oracle the exact same (rounded) values."""
import numpy as np
import torch

import mla_latent_kv_nope_b200 as mla
from mla_latent_kv_nope_b200 import inputs


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def rounded(a: np.ndarray, w) -> np.ndarray:
    """The float64 value of a float32 array after rounding to the workload
    dtype (what the device sees)."""
    t = torch.from_numpy(np.ascontiguousarray(a)).to(torch_dtype(w))
    return t.float().numpy().astype(np.float64)


def dev(a: np.ndarray, w, dtype=None):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype or torch_dtype(w))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def dims_of(w, capacity=None) -> mla.Dims:
    return mla.Dims(w.B, w.H, w.d_c, w.d_r, w.d_nope, w.d_v,
                    capacity if capacity is not None else w.capacity, w.dtype)


def host_cache(w, lens, seqs=None, capacity=None) -> dict:
    """Rounded float64 rows [0, L_b) of the requested sequences."""
    seqs = range(w.B) if seqs is None else seqs
    return {b: rounded(inputs.cache_rows(w, b, int(lens[b])), w) for b in seqs}


def device_cache(w, lens, capacity=None, fill_rest=float("nan")):
    cap = capacity if capacity is not None else w.capacity
    c = torch.empty(w.B, cap, w.R, dtype=torch_dtype(w), device="cuda")
    inputs.fill_cache(w, c, lens, fill_rest=fill_rest)
    return c


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    """max over leading index of ||got - ref||_2 / ||ref||_2 along the last axis."""
    got = got.reshape(-1, got.shape[-1])
    ref = ref.reshape(-1, ref.shape[-1])
    num = np.linalg.norm(got - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return float(np.max(num / np.where(den > 0, den, 1.0)))


def tol(w) -> float:
    return 1e-2 if w.dtype == "bf16" else 1e-5
