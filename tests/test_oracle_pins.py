"""Pins for the CPU oracle: it is checked against values the pages print,
closed forms, invariants and brute force -- never against itself.

Each test names the passage it pins.  Page keys:
  [MLA-とは]  disassemble-channel.com "Multi-head Latent Attention（MLA）とは？"
  [variants] youngju.dev "model internals: attention variants"
  [yuuk]     notes.yuuk.io wiki "Multi-Head Latent Attention"
  [abeam]    abeam.tech "Multi-Head Latent Attention" (DeepSeek-V2 reading)
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import mla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# The pages' own float64 numpy checks, rebuilt from their seeded inputs.
# The draw order and shapes are fixed by the page; the arithmetic below goes
# through the oracle's functions.
# ---------------------------------------------------------------------------
# The seeded inputs of [MLA-とは] "数値検証" and its RoPE follow-ups, as data:
# (name, kind, shape, fan-in divisor) in the order the page draws them from
# default_rng(0).  "normal" draws are scaled by 1/sqrt(fan-in); "attn" is a
# uniform draw normalised over the key axis.  The order is an interface (it
# decides every printed value); the arithmetic after it goes through the
# oracle.
_PAGE_DIMS = dict(d=256, d_c=64, d_cq=96, d_h=32, n_h=4, T=6, d_r=16)
_PAGE_DRAWS = (
    ("hid", "normal", ("T", "d"), None),
    ("w_dkv", "normal", ("d", "d_c"), "d"),
    ("w_uk", "normal", ("d_c", "n_h*d_h"), "d_c"),
    ("w_dq", "normal", ("d", "d_cq"), "d"),
    ("w_uq", "normal", ("d_cq", "n_h*d_h"), "d_cq"),
    ("w_uv", "normal", ("d_c", "n_h*d_h"), "d_c"),
    ("w_o", "normal", ("n_h*d_h", "d"), "n_h*d_h"),
    ("attn", "attn", ("T", "T", "n_h"), None),
    ("w_qr", "normal", ("d_cq", "n_h*d_r"), "d_cq"),
    ("w_kr", "normal", ("d", "d_r"), "d"),
)


def _size(expr):
    out = 1
    for f in expr.split("*"):
        out *= _PAGE_DIMS[f]
    return out


def _pages_inputs():
    g = np.random.default_rng(0)
    x = {}
    for name, kind, shape, fan_in in _PAGE_DRAWS:
        dims = tuple(_size(e) for e in shape)
        if kind == "attn":
            a = g.random(dims)
            x[name] = a / a.sum(axis=1, keepdims=True)
        else:
            a = g.normal(size=dims)
            x[name] = a / np.sqrt(_size(fan_in)) if fan_in else a
    d, d_c, d_cq, d_h, n_h, T, d_r = (_PAGE_DIMS[k]
                                      for k in ("d", "d_c", "d_cq", "d_h", "n_h", "T", "d_r"))
    x["dims"] = (d, d_c, d_cq, d_h, n_h, T, d_r)
    # Row-vector weights of the page's checks -> the oracle's column convention.
    x["W_UK"] = x["w_uk"].reshape(d_c, n_h, d_h).transpose(1, 2, 0)
    x["W_UV"] = x["w_uv"].reshape(d_c, n_h, d_h).transpose(1, 2, 0)
    x["c_kv"] = O.down_project(x["hid"], x["w_dkv"].T)
    c_q = x["hid"] @ x["w_dq"]  # query latent: input preparation only
    x["Q"] = (c_q @ x["w_uq"]).reshape(T, n_h, d_h)
    x["QR"] = (c_q @ x["w_qr"]).reshape(T, n_h, d_r)
    x["KR"] = O.down_project(x["hid"], x["w_kr"].T)  # pre-rotation k^R
    return x


@pytest.fixture(scope="module")
def pages():
    return _pages_inputs()


@pytest.fixture(scope="module")
def gold():
    return _load("pages_numpy_checks.json")


def _naive_scores(x):
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    S = np.zeros((T, T, n_h))
    for t in range(T):
        for i in range(n_h):
            S[t, :, i] = O.head_logits(x["Q"][t, i], np.zeros(0), t,
                                       x["W_UK"][i], x["c_kv"],
                                       np.zeros((T, 0)))
    return S


def test_key_side_score_value_and_absorption(pages, gold):
    """[MLA-とは] 数値検証: S_naive[3,1,0] and the absorbed-vs-naive error."""
    x = pages
    S = _naive_scores(x)
    assert abs(S[3, 1, 0] - gold["S_naive_3_1_0"]) < 1e-9
    # Absorbed through the oracle's q~ = W^UK_i^T q: q~ . c_j.
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    S_abs = np.zeros_like(S)
    for t in range(T):
        qc = O.absorb_q(x["Q"][t][None], np.zeros((1, n_h, 0)), x["W_UK"],
                        None)[0]  # [n_h, d_c]
        S_abs[t] = (qc @ x["c_kv"].T).T
    assert np.abs(S - S_abs).max() < 1e-9
    assert abs(S_abs[3, 1, 0] - gold["S_absorb_3_1_0"]) < 1e-9


def test_absorbed_matrix_rank_is_head_dim(pages, gold):
    """[MLA-とは] 数値検証: A_i = W^UQ_i^T W^UK_i has shape (n_h, d_cq, d_c)
    and rank d_h (=32) -- pins the per-head block layout of W^UK."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    W_UQ = x["w_uq"].reshape(d_cq, n_h, d_h).transpose(1, 2, 0)  # [n_h,d_h,d_cq]
    A = np.stack([W_UQ[i].T @ x["W_UK"][i] for i in range(n_h)])
    assert list(A.shape) == gold["A_shape"]
    assert np.linalg.matrix_rank(A[0]) == gold["A0_rank"]


def test_rope_on_content_breaks_absorption(pages, gold):
    """[MLA-とは] RoPEが吸収を壊す: with RoPE on the content dims the true
    score at [3,1,0] is -2.7349..., and a position-free absorbed matrix is off
    by 11.69 at worst.  Pins the rotation's pairing, sign and frequencies."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    S_true = np.zeros((T, T, n_h))
    for i in range(n_h):
        K = x["c_kv"] @ x["W_UK"][i].T  # [T, d_h] materialised keys
        Kr = np.stack([O.rope(K[j], j) for j in range(T)])
        for t in range(T):
            # rope on the whole content vector: treat it as the "rope" block
            S_true[t, :, i] = O.head_logits(np.zeros(0), x["Q"][t, i], t,
                                            np.zeros((0, d_c)), x["c_kv"], Kr)
    assert abs(S_true[3, 1, 0] - gold["S_rope_true_3_1_0"]) < 1e-9
    S_const = _naive_scores(x)
    assert abs(S_const[3, 1, 0] - gold["S_rope_constant_A_3_1_0"]) < 1e-9
    assert abs(np.abs(S_true - S_const).max() - gold["rope_max_abs_err"]) < 1e-9


def test_decoupled_rope_restores_absorption(pages, gold):
    """[MLA-とは] Decoupled RoPE: content part absorbed, shared rotated k^R
    added; absorbed and materialised scores agree to float64 rounding."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    k_pe = np.stack([O.rope(x["KR"][j], j) for j in range(T)])
    S_mat = np.zeros((T, T, n_h))
    S_abs = np.zeros((T, T, n_h))
    rows = np.concatenate([x["c_kv"], k_pe], axis=1)
    for t in range(T):
        for i in range(n_h):
            S_mat[t, :, i] = O.head_logits(x["Q"][t, i], x["QR"][t, i], t,
                                           x["W_UK"][i], x["c_kv"], k_pe)
        qcat = O.absorb_q(x["Q"][t][None], x["QR"][t][None], x["W_UK"],
                          np.array([t]))[0]
        S_abs[t] = (qcat @ rows.T).T
    err = np.abs(S_mat - S_abs).max()
    assert err < 1e-9 and err >= 0.0
    # The rope block must actually contribute (guards a dropped term).
    assert np.abs(S_mat - _naive_scores(x)).max() > 0.5


def test_cache_append_rope_position_matches_pages(pages):
    """[MLA-とは] Decoupled RoPE: k^R_j = R_j W^KR h_j with position j.  Appending
    tokens 0..T-1 in order must store exactly those rotated keys; the content
    part is the RMS-normalised W^DKV h_j ([MLA-とは] 正規化の扱い)."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    W = np.concatenate([x["w_dkv"].T, x["w_kr"].T], axis=0)
    cache = np.full((1, T + 2, d_c + d_r), np.nan)
    L = np.array([0])
    for j in range(T):
        cache, L, _ = O.cache_append(cache, L, x["hid"][j][None], W, d_c)
    k_expect = np.stack([O.rope(x["KR"][j], j) for j in range(T)])
    assert np.abs(cache[0, :T, d_c:] - k_expect).max() < 1e-12
    c = x["c_kv"]
    c_expect = c / np.sqrt(np.mean(c * c, axis=1, keepdims=True) + 1e-6)
    assert np.abs(cache[0, :T, :d_c] - c_expect).max() < 1e-12
    assert L[0] == T and np.isnan(cache[0, T:]).all()


def test_value_side_absorption(pages, gold):
    """[MLA-とは] 数値検証 (Value側): weighting materialised V then W^O equals
    weighting the latents then W^UV once (and W^O); pages report 1.1e-15."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    P = x["attn"]
    u_mat = np.zeros((T, d))
    u_abs = np.zeros((T, d))
    for t in range(T):
        for i in range(n_h):
            W_O_i = x["w_o"][i * d_h:(i + 1) * d_h, :].T  # [d, d_h]
            o_m = O.materialised_values(P[t, :, i], x["c_kv"], x["W_UV"][i])
            o_lat = P[t, :, i] @ x["c_kv"]
            o_a = O.out_proj(o_lat[None, None], x["W_UV"][i][None])[0, 0]
            u_mat[t] += W_O_i @ o_m
            u_abs[t] += W_O_i @ o_a
    # Independent form of the page's naive path: V reshaped, weighted, @ W_O.
    V = (x["c_kv"] @ x["w_uv"]).reshape(T, n_h, d_h)
    u_page = np.einsum("tji,jih->tih", P, V).reshape(T, n_h * d_h) @ x["w_o"]
    assert np.abs(u_mat - u_page).max() < 1e-12
    assert np.abs(u_mat - u_abs).max() < 1e-12


# ---------------------------------------------------------------------------
# RoPE and RMSNorm invariants and closed forms
# ---------------------------------------------------------------------------
def test_rope_closed_forms_and_invariants():
    rng = np.random.default_rng(1)
    # d = 2: a plain rotation by angle pos (theta_0 = pos / base^0).
    v = np.array([0.3, -1.7])
    for pos in [0, 1, 5, 1000]:
        c, s = math.cos(pos), math.sin(pos)
        np.testing.assert_allclose(O.rope(v, pos),
                                   [v[0] * c - v[1] * s, v[0] * s + v[1] * c],
                                   rtol=0, atol=1e-14)
    # d = 4: second pair rotates by pos / base^(2/4) = pos / 100, pairs (0,2),(1,3)
    v = np.array([1.0, 2.0, 3.0, 4.0])
    pos = 7
    a0, a1 = pos, pos / 100.0
    exp = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
           1 * math.sin(a0) + 3 * math.cos(a0), 2 * math.sin(a1) + 4 * math.cos(a1)]
    np.testing.assert_allclose(O.rope(v, pos), exp, rtol=0, atol=1e-13)
    x = rng.normal(size=64)
    y = rng.normal(size=64)
    np.testing.assert_array_equal(O.rope(x, 0), x)  # identity at pos 0
    assert abs(np.linalg.norm(O.rope(x, 123)) - np.linalg.norm(x)) < 1e-12
    # R_t^T R_j = R_{j-t}: the dot product depends only on j - t.
    d1 = O.rope(x, 17) @ O.rope(y, 40)
    d2 = O.rope(x, 117) @ O.rope(y, 140)
    d3 = x @ O.rope(y, 23)
    assert abs(d1 - d2) < 1e-10 and abs(d1 - d3) < 1e-10


def test_rms_norm_properties():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 512)) * 3.0
    y = O.rms_norm(x, None, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, atol=1e-12)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, None, 0.0), y, atol=1e-12)
    g = rng.normal(size=512)
    np.testing.assert_allclose(O.rms_norm(x, g, 0.0), y * g, atol=1e-12)
    # eps enters under the root: x = [a, a] gives a / sqrt(a^2 + eps).
    a, eps = 0.01, 1e-4
    np.testing.assert_allclose(O.rms_norm(np.array([a, a]), None, eps),
                               [a / math.sqrt(a * a + eps)] * 2, atol=1e-15)


# ---------------------------------------------------------------------------
# Brute force on tiny shapes and special cases
# ---------------------------------------------------------------------------
def _rand_problem(rng, B, H, d_c, d_r, d_n, d_v, cap, lens):
    return dict(
        q_nope=rng.normal(size=(B, H, d_n)),
        q_pe=rng.normal(size=(B, H, d_r)),
        q_pos=rng.integers(0, 50, size=B),
        W_UK=rng.normal(size=(H, d_n, d_c)) * 0.3,
        W_UV=rng.normal(size=(H, d_v, d_c)) * 0.3,
        cache=rng.normal(size=(B, cap, d_c + d_r)),
        seqlens=np.array(lens),
    )


def test_single_token_closed_form():
    """L = 1: the softmax weight is exactly 1, so out = W^UV_i c_0 and
    lse = s_0 = scale * ([q^C; R q^R] . [W^UK_i c_0; k^R_0])."""
    rng = np.random.default_rng(3)
    p = _rand_problem(rng, 1, 1, 6, 4, 3, 5, 3, [1])
    out, o_lat, lse = O.mla_decode_materialised(
        p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"], p["cache"],
        p["seqlens"], 0.5)
    c0 = p["cache"][0, 0, :6]
    kpe = p["cache"][0, 0, 6:]
    np.testing.assert_allclose(out[0, 0], p["W_UV"][0] @ c0, atol=1e-12)
    np.testing.assert_allclose(o_lat[0, 0], c0, atol=1e-12)
    # Rotate q_pe by hand (d_r = 4: pairs (0,2) at angle pos, (1,3) at pos/100).
    pos = int(p["q_pos"][0])
    q = p["q_pe"][0, 0]
    a0, a1 = pos, pos / 100.0
    qr = np.array([q[0] * math.cos(a0) - q[2] * math.sin(a0),
                   q[1] * math.cos(a1) - q[3] * math.sin(a1),
                   q[0] * math.sin(a0) + q[2] * math.cos(a0),
                   q[1] * math.sin(a1) + q[3] * math.cos(a1)])
    s0 = 0.5 * (p["q_nope"][0, 0] @ (p["W_UK"][0] @ c0) + qr @ kpe)
    assert abs(lse[0, 0] - s0) < 1e-12


def test_two_token_sigmoid_closed_form():
    """L = 2: p_0 = sigma(s_0 - s_1) and lse = log(e^{s_0} + e^{s_1})."""
    rng = np.random.default_rng(4)
    p = _rand_problem(rng, 1, 2, 8, 2, 4, 3, 2, [2])
    scale = 0.37
    out, o_lat, lse = O.mla_decode_materialised(
        p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"], p["cache"],
        p["seqlens"], scale)
    for i in range(2):
        s = [scale * O.head_logits(p["q_nope"][0, i], p["q_pe"][0, i],
                                   p["q_pos"][0], p["W_UK"][i],
                                   p["cache"][0, :, :8], p["cache"][0, :, 8:])[j]
             for j in range(2)]
        p0 = 1.0 / (1.0 + math.exp(-(s[0] - s[1])))
        v = [p["W_UV"][i] @ p["cache"][0, j, :8] for j in range(2)]
        np.testing.assert_allclose(out[0, i], p0 * v[0] + (1 - p0) * v[1], atol=1e-12)
        assert abs(lse[0, i] - math.log(math.exp(s[0]) + math.exp(s[1]))) < 1e-12


def test_zero_query_gives_mean_of_values():
    """All-zero query: every logit is 0, the softmax is uniform and the output
    is the mean of the materialised values (identical keys)."""
    rng = np.random.default_rng(5)
    p = _rand_problem(rng, 2, 3, 8, 4, 4, 5, 7, [7, 3])
    p["q_nope"][:] = 0.0
    p["q_pe"][:] = 0.0
    out, o_lat, lse = O.mla_decode_materialised(
        p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"], p["cache"],
        p["seqlens"], 1.0)
    for b, L in enumerate([7, 3]):
        for i in range(3):
            v = (p["cache"][b, :L, :8] @ p["W_UV"][i].T).mean(axis=0)
            np.testing.assert_allclose(out[b, i], v, atol=1e-12)
            assert abs(lse[b, i] - math.log(L)) < 1e-12


def test_brute_force_formula_by_formula():
    """Exhaustive small shapes (B<=2, H<=3, L<=5): every quantity evaluated
    one scalar at a time with Python loops, against the oracle."""
    rng = np.random.default_rng(6)
    for B, H, L in [(1, 1, 1), (2, 3, 5), (1, 2, 4), (2, 1, 3)]:
        d_c, d_r, d_n, d_v = 4, 2, 3, 2
        lens = [L] * B
        if B == 2:
            lens[1] = max(1, L - 2)
        p = _rand_problem(rng, B, H, d_c, d_r, d_n, d_v, 6, lens)
        scale = 0.8
        out, o_lat, lse = O.mla_decode_materialised(
            p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"],
            p["cache"], p["seqlens"], scale)
        for b in range(B):
            pos = int(p["q_pos"][b])
            for i in range(H):
                qp = p["q_pe"][b, i]
                th = pos  # d_r = 2: one pair, angle pos
                qr = [qp[0] * math.cos(th) - qp[1] * math.sin(th),
                      qp[0] * math.sin(th) + qp[1] * math.cos(th)]
                s = []
                for j in range(lens[b]):
                    row = p["cache"][b, j]
                    acc = 0.0
                    for r in range(d_n):
                        k = sum(p["W_UK"][i, r, a] * row[a] for a in range(d_c))
                        acc += p["q_nope"][b, i, r] * k
                    acc += qr[0] * row[d_c] + qr[1] * row[d_c + 1]
                    s.append(scale * acc)
                m = max(s)
                z = sum(math.exp(v - m) for v in s)
                w = [math.exp(v - m) / z for v in s]
                for vv in range(d_v):
                    o = 0.0
                    for j in range(lens[b]):
                        o += w[j] * sum(p["W_UV"][i, vv, a] * p["cache"][b, j, a]
                                        for a in range(d_c))
                    assert abs(out[b, i, vv] - o) < 1e-12
                assert abs(lse[b, i] - (m + math.log(z))) < 1e-12


def test_absorbed_equals_materialised_independent():
    """[MLA-とは] 行列吸収 / Value側の吸収: an independently written absorbed
    computation (q~ by explicit sums, latent attention, one W^UV at the end)
    equals the materialised oracle to ~1e-12 relative."""
    rng = np.random.default_rng(7)
    B, H, d_c, d_r, d_n, d_v = 2, 4, 32, 8, 16, 12
    lens = [37, 5]
    p = _rand_problem(rng, B, H, d_c, d_r, d_n, d_v, 40, lens)
    scale = 1.0 / math.sqrt(d_n + d_r)
    out, o_lat, lse = O.mla_decode_materialised(
        p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"], p["cache"],
        p["seqlens"], scale)
    for b in range(B):
        pos = p["q_pos"][b]
        half = d_r // 2
        for i in range(H):
            qt = np.zeros(d_c)
            for r in range(d_n):
                qt += p["q_nope"][b, i, r] * p["W_UK"][i, r, :]
            qp = p["q_pe"][b, i]
            ang = pos * np.power(10000.0, -np.arange(half) * 2.0 / d_r)
            qr = np.concatenate([qp[:half] * np.cos(ang) - qp[half:] * np.sin(ang),
                                 qp[:half] * np.sin(ang) + qp[half:] * np.cos(ang)])
            rows = p["cache"][b, :lens[b]]
            s = scale * (rows[:, :d_c] @ qt + rows[:, d_c:] @ qr)
            w = np.exp(s - s.max())
            w /= w.sum()
            ol = w @ rows[:, :d_c]
            o = np.array([p["W_UV"][i, v] @ ol for v in range(d_v)])
            assert np.linalg.norm(o - out[b, i]) <= 1e-12 * np.linalg.norm(o)
            assert np.linalg.norm(ol - o_lat[b, i]) <= 1e-12 * np.linalg.norm(ol)


def test_latent_attention_and_out_proj_match_materialised():
    """The absorbed-path oracle functions (absorb_q -> latent_attention ->
    out_proj) reproduce the materialised decode."""
    rng = np.random.default_rng(8)
    B, H, d_c, d_r, d_n, d_v = 3, 2, 16, 8, 8, 8
    lens = [9, 1, 0]
    p = _rand_problem(rng, B, H, d_c, d_r, d_n, d_v, 12, lens)
    scale = 0.3
    out, o_lat, lse = O.mla_decode_materialised(
        p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"], p["cache"],
        p["seqlens"], scale)
    qcat = O.absorb_q(p["q_nope"], p["q_pe"], p["W_UK"], p["q_pos"])
    ol2, lse2 = O.latent_attention(qcat, p["cache"], p["seqlens"], scale, d_c)
    out2 = O.out_proj(ol2, p["W_UV"])
    np.testing.assert_allclose(ol2, o_lat, atol=1e-12)
    np.testing.assert_allclose(out2, out, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(lse2), np.isinf(lse))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse2[fin], lse[fin], atol=1e-12)
    # Empty sequence: zeros and -inf, never NaN.
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))


def test_mqa_special_case():
    """[yuuk] 横断的知見: pure MQA is MLA whose compressed dim equals one head's
    dim.  With d_c = d_n = d_v and W^UK_i = W^UV_i = I the MLA decode equals a
    textbook MQA with shared key [c; k^R] and shared value c (rope on the
    query's decoupled part).  Also d_r = 0 (NoPE)."""
    rng = np.random.default_rng(9)
    for d_r in (4, 0):
        B, H, d = 2, 3, 6
        lens = [5, 2]
        p = _rand_problem(rng, B, H, d, d_r, d, d, 6, lens)
        p["W_UK"] = np.stack([np.eye(d)] * H)
        p["W_UV"] = np.stack([np.eye(d)] * H)
        scale = 0.7
        out, _, _ = O.mla_decode_materialised(
            p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"],
            p["cache"], p["seqlens"], scale)
        for b in range(B):
            qr = O.rope(p["q_pe"][b], p["q_pos"][b]) if d_r else np.zeros((H, 0))
            for i in range(H):
                q = list(p["q_nope"][b, i]) + list(qr[i])
                logits = []
                for j in range(lens[b]):
                    key = list(p["cache"][b, j])
                    logits.append(scale * sum(a * k for a, k in zip(q, key)))
                m = max(logits)
                e = [math.exp(v - m) for v in logits]
                z = sum(e)
                ref = [sum(e[j] / z * p["cache"][b, j, a] for j in range(lens[b]))
                       for a in range(d)]
                np.testing.assert_allclose(out[b, i], ref, atol=1e-12)


def test_combine_equals_unsplit_attention():
    """Chunked softmax merged by log-sum-exp equals the unchunked one;
    empty chunks (lse = -inf) contribute nothing."""
    rng = np.random.default_rng(10)
    B, H, d_c, d_r = 2, 3, 8, 4
    cache = rng.normal(size=(B, 30, d_c + d_r))
    qcat = rng.normal(size=(B, H, d_c + d_r))
    lens = np.array([29, 7])
    o_ref, lse_ref = O.latent_attention(qcat, cache, lens, 0.4, d_c)
    bounds = [0, 4, 4, 15, 30]  # includes an empty chunk [4, 4)
    parts_o, parts_l = [], []
    for s in range(len(bounds) - 1):
        kr = [(min(bounds[s], L), min(bounds[s + 1], L)) for L in lens]
        o, l = O.latent_attention(qcat, cache, lens, 0.4, d_c, key_range=kr)
        parts_o.append(o)
        parts_l.append(l)
    o_parts = np.stack(parts_o, axis=2)  # [B,H,S,d_c]
    l_parts = np.stack(parts_l, axis=2)
    assert np.isneginf(l_parts[1, :, 3]).all()  # chunk beyond L_1 is empty
    o, l = O.combine_partials(o_parts, l_parts)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(l, lse_ref, atol=1e-12)
    o0, l0 = O.combine_partials(np.full((1, 3, 4), 7.0), np.full((1, 3), -np.inf))
    assert np.all(o0 == 0) and np.all(np.isneginf(l0))


def test_cache_append_indexing_and_capacity():
    """Append writes exactly row L_b of each sequence and increments L_b; a
    full sequence raises and writes nothing."""
    rng = np.random.default_rng(11)
    B, cap, d_c, d_r, hid = 3, 5, 4, 2, 7
    cache = np.full((B, cap, d_c + d_r), 9.0)
    L = np.array([0, 2, 4])
    h = rng.normal(size=(B, hid))
    W = rng.normal(size=(d_c + d_r, hid))
    g = rng.normal(size=d_c)
    new, L2, rows = O.cache_append(cache, L, h, W, d_c, gamma=g, eps=1e-6,
                                   rope_base=10000.0)
    np.testing.assert_array_equal(L2, L + 1)
    for b in range(B):
        for j in range(cap):
            if j == L[b]:
                x = W @ h[b]
                c = x[:d_c] / math.sqrt(np.mean(x[:d_c] ** 2) + 1e-6) * g
                th = L[b]  # d_r = 2: one pair at angle pos
                k = [x[d_c] * math.cos(th) - x[d_c + 1] * math.sin(th),
                     x[d_c] * math.sin(th) + x[d_c + 1] * math.cos(th)]
                np.testing.assert_allclose(new[b, j], list(c) + k, atol=1e-12)
            else:
                assert np.all(new[b, j] == 9.0)
    with pytest.raises(IndexError):
        O.cache_append(new, np.array([0, 0, cap]), h, W, d_c)


# ---------------------------------------------------------------------------
# Closed forms printed on the pages
# ---------------------------------------------------------------------------
def test_cache_size_closed_forms():
    g = _load("cache_size_closed_forms.json")
    v2 = g["deepseek_v2"]
    kw = dict(layers=v2["layers"], n_h=v2["n_h"], d_h=v2["d_h"], n_g=v2["n_g"],
              d_c=v2["d_c"], d_r=v2["d_r"])
    mha = O.cache_elems_per_token("MHA", **kw)
    gqa = O.cache_elems_per_token("GQA", **kw)
    mqa = O.cache_elems_per_token("MQA", **kw)
    mla = O.cache_elems_per_token("MLA", **kw)
    assert (mha, gqa, mqa, mla) == (v2["MHA"], v2["GQA"], v2["MQA"], v2["MLA"])
    for k, e in [("MHA", mha), ("GQA", gqa), ("MQA", mqa), ("MLA", mla)]:
        assert round(e * 2 / 1e6, 3) == v2[f"{k}_fp16_MB"]
    assert round(mha / mla, 1) == v2["MHA_over_MLA"]
    assert round(gqa / mla, 2) == v2["GQA_over_MLA"]
    assert round(mqa / mla, 2) == v2["MQA_over_MLA"]
    assert (v2["d_c"] + v2["d_r"]) / (2 * v2["d_h"]) == v2["n_g_equiv"]
    assert round(mha * 2 * 8192 / 1e9) == v2["MHA_fp16_8192_ctx_GB"]
    v3 = g["deepseek_v3"]
    kw3 = dict(layers=v3["layers"], n_h=v3["n_h"], d_h=v3["d_h"], d_c=v3["d_c"],
               d_r=v3["d_r"])
    assert O.cache_elems_per_token("MLA", **kw3) == v3["MLA"]
    assert O.cache_elems_per_token("MHA", **kw3) == v3["MHA"]
    assert round(v3["MHA"] / v3["MLA"], 1) == v3["MHA_over_MLA"]
    assert round(v3["MLA"] * 32768 * 2 / 2 ** 30, 2) == v3["cache_32k_fp16_GiB"]
    k2 = g["kimi_k2"]
    kwk = dict(layers=k2["layers"], n_h=k2["n_h"], d_h=k2["d_h"], d_c=k2["d_c"],
               d_r=k2["d_r"])
    mla_k = O.cache_elems_per_token("MLA", **kwk)
    assert mla_k == k2["MLA"]
    assert round(O.cache_elems_per_token("MHA", **kwk) / mla_k, 1) == k2["MHA_over_MLA"]
    m = g["mults_per_cached_token"]
    n = O.mults_per_cached_token("naive", m["n_h"], m["d_h"], m["d_c"])
    a = O.mults_per_cached_token("absorbed", m["n_h"], m["d_h"], m["d_c"])
    h = O.mults_per_cached_token("MHA", m["n_h"], m["d_h"], m["d_c"])
    assert (n, a, h) == (m["naive"], m["absorbed"], m["MHA"])
    assert a // h == m["absorbed_over_MHA"] and n // a == m["naive_over_absorbed"]


# ---------------------------------------------------------------------------
# W^O fold: B_i = W^O_i W^UV_i ([MLA-とは] "Value側の吸収")
# ---------------------------------------------------------------------------
def test_output_fold_matches_pages_value_side(pages, gold):
    """[MLA-とは] 数値検証 (Value側): projecting the materialised per-head
    outputs through W^O equals pushing the latent sums through the folded
    B_i; the page prints a float64 gap of about 1.1e-15."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    P = x["attn"]
    W_O = x["w_o"].T  # snippet's row-vector [n_h*d_h, d] -> column [d, n_h*d_h]
    out = np.zeros((T, n_h, d_h))
    o_lat = np.zeros((T, n_h, d_c))
    for t in range(T):
        for i in range(n_h):
            out[t, i] = O.materialised_values(P[t, :, i], x["c_kv"], x["W_UV"][i])
            o_lat[t, i] = P[t, :, i] @ x["c_kv"]
    u_unfolded = O.output_projection(out, W_O)
    Bf = O.fold_output_weights(W_O, x["W_UV"])
    assert Bf.shape == (n_h, d, d_c)  # B_i in R^{d x d_c}, as the page states
    u_folded = O.folded_output(o_lat, Bf)
    # The page's own naive path, written independently of the oracle.
    V = (x["c_kv"] @ x["w_uv"]).reshape(T, n_h, d_h)
    u_page = np.einsum("tji,jih->tih", P, V).reshape(T, n_h * d_h) @ x["w_o"]
    assert np.abs(u_unfolded - u_page).max() < 1e-12
    err = np.abs(u_folded - u_page).max()
    assert err < 1e-12
    assert gold["value_side_max_abs_err"] < 1e-12


def test_output_fold_special_cases():
    """W^UV_i = I (d_v = d_c) leaves W^O's head blocks unchanged; a W^O that
    selects one head's output returns that head's W^UV; the fold's rank is at
    most d_v (it factors through a d_v-dimensional space)."""
    rng = np.random.default_rng(21)
    H, d, d_c = 3, 7, 5
    W_O = rng.normal(size=(d, H * d_c))
    Bf = O.fold_output_weights(W_O, np.stack([np.eye(d_c)] * H))
    for i in range(H):
        np.testing.assert_array_equal(Bf[i], W_O[:, i * d_c:(i + 1) * d_c])
    d_v = 2
    W_UV = rng.normal(size=(H, d_v, d_c))
    sel = np.zeros((d_v, H * d_v))
    sel[:, d_v:2 * d_v] = np.eye(d_v)  # picks head 1
    Bs = O.fold_output_weights(sel, W_UV)
    np.testing.assert_array_equal(Bs[1], W_UV[1])
    assert np.all(Bs[0] == 0) and np.all(Bs[2] == 0)
    Bg = O.fold_output_weights(rng.normal(size=(d, H * d_v)), W_UV)
    assert all(np.linalg.matrix_rank(Bg[i]) <= d_v for i in range(H))
    # Brute force: u = sum_i sum_a sum_c W_O[:, i*d_v + a] W_UV[i, a, c] o[i, c].
    o = rng.normal(size=(1, H, d_c))
    W_O2 = rng.normal(size=(d, H * d_v))
    u = O.folded_output(o, O.fold_output_weights(W_O2, W_UV))[0]
    ref = [sum(W_O2[r, i * d_v + a] * W_UV[i, a, c] * o[0, i, c]
               for i in range(H) for a in range(d_v) for c in range(d_c))
           for r in range(d)]
    np.testing.assert_allclose(u, ref, atol=1e-12)


# ---------------------------------------------------------------------------
# FP8 latent cache: E4M3 codes with a power-of-two scale per token.  The pages
# name KV quantisation ([abeam] "モデル全体でも推論効率が大きく改善した") and
# FP8 for MLA ([yuuk] "未解決の問い") but no format; the format is a reading,
# and these pins fix the oracle to the E4M3 definition it states.
# ---------------------------------------------------------------------------
def test_e4m3_decode_table():
    """Every byte against the format's closed-form values and against torch's
    float8_e4m3fn (a library routine)."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(v)
    np.testing.assert_array_equal(nan, np.isnan(lib))
    np.testing.assert_array_equal(v[~nan], lib[~nan].astype(np.float64))
    assert list(np.flatnonzero(nan)) == [0x7F, 0xFF]
    spot = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
            0x38: 1.0, 0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0,
            0xFE: -448.0, 0x80: 0.0}
    for c, val in spot.items():
        assert v[c] == val, hex(c)
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)  # the positive codes are ordered
    np.testing.assert_array_equal(v[0x80:0xFF], -v[:0x7F])


def test_e4m3_encode_rounding_and_saturation():
    """Round-trip of every finite code; ties to even at each midpoint; one
    float32 ulp either side of a midpoint goes to the nearer code; agreement
    with torch's conversion wherever it does not overflow (|x| <= 464);
    saturation to +-448 beyond."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes)
    fin = ~np.isnan(v) & (codes != 0x80)
    np.testing.assert_array_equal(O.e4m3_encode(v[fin]), codes[fin])
    pos = v[:0x7F]
    mid = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)  # exact in float32
    got = O.e4m3_encode(mid)
    even = np.where(np.arange(0x7E) % 2 == 0, np.arange(0x7E), np.arange(1, 0x7F))
    np.testing.assert_array_equal(got, even.astype(np.uint8))
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(0))
    np.testing.assert_array_equal(O.e4m3_encode(up), np.arange(1, 0x7F, dtype=np.uint8))
    np.testing.assert_array_equal(O.e4m3_encode(dn), np.arange(0, 0x7E, dtype=np.uint8))
    rng = np.random.default_rng(22)
    mag = np.exp2(rng.uniform(-12, np.log2(464), size=20000))
    x = (mag * rng.choice([-1, 1], size=mag.size)).astype(np.float32)
    x = np.concatenate([x, mid, -mid, up, dn]).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x), lib)
    sat = np.array([465.0, 1e6, np.inf, -500.0, -np.inf, np.nan, -0.0, -1e-9])
    np.testing.assert_array_equal(O.e4m3_encode(sat),
                                  [0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x80, 0x80])


def test_latent_row_scale_and_quantisation_bounds():
    """The scale is the smallest power of two that brings the row's largest
    |c| under 448 (so that element lands in [224, 448]); each element is then
    within half a step of its binade: |c~ - c| <= 2^-4 |c| in the normal range
    and <= 2^-10 scale in the subnormal one; c~ re-encodes to the same codes."""
    rng = np.random.default_rng(23)
    c = rng.normal(size=(64, 96)) * np.exp2(rng.integers(-20, 20, size=(64, 1)))
    c[3] = 0.0
    c[5, :] = 1e-3
    c[5, 7] = 448.0 * 2.0 ** -5          # exactly on a binade edge
    c[6, :] = 0.5
    c[6, 0] = 448.0 * 2.0 ** 3 * (1 + 2.0 ** -30)  # just above one
    codes, scale = O.quantize_latent_rows(c)
    k = np.log2(scale)
    assert np.all(k == np.round(k))
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    assert scale[5] == 2.0 ** -5 and scale[6] == 2.0 ** 4
    amax = np.abs(c).max(axis=1)
    nz = amax > 0
    r = amax[nz] / scale[nz]
    assert np.all(r <= 448) and np.all(r > 224)
    deq = O.dequantize_latent_rows(codes, scale)
    y = np.abs(c / scale[:, None])
    normal = y >= 2.0 ** -6
    err = np.abs(deq - c)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(c)[normal] * (1 + 1e-12))
    sub_bound = (2.0 ** -10 * scale[:, None] * np.ones_like(c))[~normal]
    assert np.all(err[~normal] <= sub_bound * (1 + 1e-12))
    np.testing.assert_array_equal(O.e4m3_encode(deq / scale[:, None]), codes)
    # The row maximum keeps its sign and stays the largest magnitude.
    j = np.abs(c).argmax(axis=1)
    assert np.all(np.sign(deq[np.arange(64), j]) == np.sign(c[np.arange(64), j]))


def test_decode_over_lossless_fp8_cache_equals_unquantised():
    """When every latent is already an E4M3 value times a power of two, the
    quantised cache holds the same numbers, and decode over its dequantised
    rows equals decode over the original cache exactly."""
    rng = np.random.default_rng(24)
    B, H, d_c, d_r, d_n, d_v, cap = 2, 3, 8, 4, 5, 6, 7
    lens = [7, 3]
    p = _rand_problem(rng, B, H, d_c, d_r, d_n, d_v, cap, lens)
    codes = rng.integers(0, 0x7E, size=(B, cap, d_c)).astype(np.uint8)
    codes[..., 0] = 0x7E  # the row maximum is 448 * scale
    codes |= (rng.integers(0, 2, size=codes.shape) * 0x80).astype(np.uint8)
    sc = np.exp2(rng.integers(-12, -4, size=(B, cap)).astype(np.float64))
    c = O.dequantize_latent_rows(codes, sc)
    p["cache"][..., :d_c] = c
    q_codes, q_sc = O.quantize_latent_rows(c)
    np.testing.assert_array_equal(q_sc, sc)
    np.testing.assert_array_equal(O.e4m3_decode(q_codes), O.e4m3_decode(codes))
    deq_cache = p["cache"].copy()
    deq_cache[..., :d_c] = O.dequantize_latent_rows(q_codes, q_sc)
    args = (p["q_nope"], p["q_pe"], p["q_pos"], p["W_UK"], p["W_UV"])
    a = O.mla_decode_materialised(*args, p["cache"], p["seqlens"], 0.3)
    b = O.mla_decode_materialised(*args, deq_cache, p["seqlens"], 0.3)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ---------------------------------------------------------------------------
# Prefill in materialised form ([MLA-とは] "実装上のトレードオフ")
# ---------------------------------------------------------------------------
def test_prefill_scores_match_pages_key_side(pages, gold):
    """[MLA-とは] 数値検証: the page's T x T content scores (no RoPE) from its
    seeded inputs; entry [3, 1, 0] is printed.  The causal mask keeps it
    (key 1 is before query 3) and hides every key after the query."""
    x = pages
    d, d_c, d_cq, d_h, n_h, T, d_r = x["dims"]
    pos = np.arange(T)
    S0 = O.prefill_scores(x["Q"][:, 0], np.zeros((T, 0)), pos, x["W_UK"][0], x["c_kv"],
                          np.zeros((T, 0)))
    assert abs(S0[3, 1] - gold["S_naive_3_1_0"]) < 1e-9
    K = (x["c_kv"] @ x["w_uk"]).reshape(T, n_h, d_h)        # the page's naive K
    S_page = np.einsum("th,jh->tj", x["Q"][:, 0], K[:, 0])
    lower = np.tril(np.ones((T, T), dtype=bool))
    np.testing.assert_allclose(S0[lower], S_page[lower], atol=1e-12)
    assert np.all(np.isneginf(S0[~lower]))


def test_prefill_rows_equal_single_token_decode():
    """Every prefill row is the single-token decode of its query over the rows
    it may see (the decode oracle is pinned independently above); the last
    row is the plain decode; a key after a query never changes that row."""
    rng = np.random.default_rng(25)
    H, d_c, d_r, d_n, d_v, L, T = 3, 8, 4, 5, 6, 9, 4
    W_UK = rng.normal(size=(H, d_n, d_c))
    W_UV = rng.normal(size=(H, d_v, d_c))
    rows = rng.normal(size=(L, d_c + d_r))
    q_nope = rng.normal(size=(T, H, d_n))
    q_pe = rng.normal(size=(T, H, d_r))
    q_pos = np.array([L - 4, L - 3, L - 2, L - 1])
    scale = 0.37
    out, lse = O.prefill_materialised(q_nope, q_pe, q_pos, W_UK, W_UV, rows, d_c, scale)
    for t in range(T):
        n = q_pos[t] + 1
        cache = rows[None, :n].copy()
        o_d, _, l_d = O.mla_decode_materialised(q_nope[t][None], q_pe[t][None], [q_pos[t]],
                                                W_UK, W_UV, cache, [n], scale)
        np.testing.assert_allclose(out[t], o_d[0], atol=1e-12)
        np.testing.assert_allclose(lse[t], l_d[0], atol=1e-12)
    # Causality: perturbing the last row changes only the query that sees it.
    rows2 = rows.copy()
    rows2[L - 1] += 5.0
    out2, _ = O.prefill_materialised(q_nope, q_pe, q_pos, W_UK, W_UV, rows2, d_c, scale)
    np.testing.assert_array_equal(out2[:T - 1], out[:T - 1])
    assert np.abs(out2[T - 1] - out[T - 1]).max() > 1e-6


def test_two_level_merge_equals_one_level():
    """The log-sum-exp merge composes: merging the partials of each group
    (one rank's split-KV partials) and then merging the groups' results (the
    ranks) equals one merge of all partials, and both equal attention over the
    union of the key sets.  Sequence sharding relies on exactly this."""
    rng = np.random.default_rng(26)
    B, H, d_c, d_r = 2, 3, 6, 2
    L = 23
    rows = rng.normal(size=(B, L, d_c + d_r))
    q = rng.normal(size=(B, H, d_c + d_r))
    cuts = [0, 4, 9, 9, 15, 23]            # six chunks, one of them empty
    parts = [O.latent_attention(q, rows, None, 0.8, d_c,
                                key_range=[(cuts[k], cuts[k + 1])] * B)
             for k in range(len(cuts) - 1)]
    o_all = np.stack([p[0] for p in parts], axis=2)
    l_all = np.stack([p[1] for p in parts], axis=2)
    one_o, one_l = O.combine_partials(o_all, l_all)
    groups = [[0, 1], [2, 3], [4]]         # ranks holding consecutive chunks
    g = [O.combine_partials(o_all[:, :, idx], l_all[:, :, idx]) for idx in groups]
    two_o, two_l = O.combine_partials(np.stack([x[0] for x in g], axis=2),
                                      np.stack([x[1] for x in g], axis=2))
    ref_o, ref_l = O.latent_attention(q, rows, [L] * B, 0.8, d_c)
    for o, lse in ((one_o, one_l), (two_o, two_l)):
        np.testing.assert_allclose(o, ref_o, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, atol=1e-12)


def test_rope_rotations_compose():
    """RoPE at position a then at b equals RoPE at a + b (each pair is a plane
    rotation by an angle linear in the position), and rotating back by -a
    restores the input."""
    rng = np.random.default_rng(27)
    x = rng.normal(size=(5, 16))
    for a, b in [(3, 4), (1000, 17), (0, 9)]:
        np.testing.assert_allclose(O.rope(O.rope(x, a), b), O.rope(x, a + b), atol=1e-9)
        np.testing.assert_allclose(O.rope(O.rope(x, a), -a), x, atol=1e-9)
