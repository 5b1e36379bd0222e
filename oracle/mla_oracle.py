"""Plain CPU oracle for single-token MLA decode over the latent KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs call it.  It shares no code, table or constant with the CUDA
library under ``mla_latent_kv_nope_b200/``; the only thing the two sides share is
the seeded input generator, which holds none of the method's arithmetic.

Everything is float64 numpy.  bf16 inputs are upcast exactly before use; the
oracle never rounds intermediate values.  Matrix products use numpy's matmul as
a library primitive; nothing is blocked, fused or reordered beyond what each
definition states, so every function can be read against the equation it cites.

Sources (cited by page title and section, as the pages name them):

* [MLA-とは] "Multi-head Latent Attention（MLA）とは？KVキャッシュを圧縮する
  DeepSeekの注意機構を完全解説" (disassemble-channel.com), sections
  "MLAの発想", "行列吸収", "Value側の吸収", "RoPEが吸収を壊す",
  "Decoupled RoPE", "KVキャッシュ容量の比較", "実装上のトレードオフ".
* [attention-variants] youngju.dev "model internals: attention variants",
  sections "MLA: キャッシュする対象そのものを変える" and "一つの表で比べる".
* [yuuk-wiki] notes.yuuk.io wiki "Multi-Head Latent Attention", sections
  "横断的知見" (MQA as the special case of MLA) and "未解決の問い" (FP8/FP4).
* [abeam] abeam.tech "Multi-Head Latent Attention" (DeepSeek-V2 reading),
  section "モデル全体でも推論効率が大きく改善した" (KV-cache quantisation).

Conventions (column vectors, y = W x, as [MLA-とは] states in its preamble):

* ``W_UK[i]`` and ``W_UV[i]`` are the per-head blocks W^UK_i, W^UV_i in
  R^{d_h x d_c}, stored as arrays of shape [H, d_h, d_c] ([MLA-とは] "MLAの発想",
  the equation k^C = W^UK c^KV and the row-block definition after it).
* A latent cache row is [c^KV (d_c) || k^R (d_r)]; k^R is stored already
  rotated ([MLA-とは] "Decoupled RoPE", the two-part cache figure text).
* ``W_DKV`` is the vertical concatenation [W^DKV ; W^KR] of shape
  [d_c + d_r, hidden]: rows [0, d_c) give c^KV, rows [d_c, d_c + d_r) give
  the pre-rotation k^R (both are applied to h, [MLA-とは] "Decoupled RoPE",
  equation for k^R_j).

Every function here has at least one independent pin in
``tests/test_oracle_pins.py``; none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "rope",
    "rms_norm",
    "down_project",
    "cache_append",
    "absorb_q",
    "head_logits",
    "softmax_lse",
    "materialised_values",
    "mla_decode_materialised",
    "latent_attention",
    "combine_partials",
    "out_proj",
    "prefill_scores",
    "prefill_materialised",
    "output_projection",
    "fold_output_weights",
    "folded_output",
    "E4M3_MAX",
    "e4m3_decode",
    "e4m3_encode",
    "latent_row_scale",
    "quantize_latent_rows",
    "dequantize_latent_rows",
    "cache_elems_per_token",
    "mults_per_cached_token",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# RoPE and RMSNorm
# ---------------------------------------------------------------------------
def rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding with half-split pairing, [MLA-とは] "RoPEが吸収を壊す".

    The page defines the rotation used throughout its checks: for a vector of
    even length d, with half = d/2 and angle theta_k = pos / base^(2k/d) for
    k < half, the pair (x[k], x[k+half]) is rotated by theta_k:

        y[k]        = x[k] cos(theta_k) - x[k+half] sin(theta_k)
        y[k+half]   = x[k] sin(theta_k) + x[k+half] cos(theta_k)

    ``x`` may carry leading batch axes; ``pos`` is a scalar or broadcasts
    against those axes.  Angles and trigonometry are evaluated in float64.
    """
    x = _f64(x)
    d = x.shape[-1]
    if d == 0:
        return x.copy()
    if d % 2:
        raise ValueError("rope needs an even last dimension")
    half = d // 2
    k = np.arange(half, dtype=np.float64)
    inv_freq = 1.0 / (float(base) ** (2.0 * k / d))
    pos = _f64(pos)
    theta = pos[..., None] * inv_freq  # broadcasts over leading axes
    c, s = np.cos(theta), np.sin(theta)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rms_norm(x, gamma=None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm of the latent before it is cached, [MLA-とは] "実装上のトレードオフ"
    (正規化の扱い): a per-token scalar division by the root mean square,
    followed by the learned diagonal gain.

        y = x / sqrt(mean(x^2) + eps) * gamma

    ``eps`` is not given by the pages; the library's default is 1e-6.
    """
    x = _f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + float(eps))
    if gamma is not None:
        y = y * _f64(gamma)
    return y


# ---------------------------------------------------------------------------
# Cache append: down-projection, latent RMSNorm, decoupled RoPE key
# ---------------------------------------------------------------------------
def down_project(h, W_DKV) -> np.ndarray:
    """x = [W^DKV ; W^KR] h for each row of ``h`` ([MLA-とは] "MLAの発想",
    c^KV_t = W^DKV h_t, and "Decoupled RoPE", k^R_j = R_j W^KR h_j before R_j).

    h: [B, hidden]; W_DKV: [d_c + d_r, hidden] -> [B, d_c + d_r].
    """
    return _f64(h) @ _f64(W_DKV).T


def cache_append(cache, seqlens, h, W_DKV, d_c: int, gamma=None,
                 eps: float = 1e-6, rope_base: float = 10000.0):
    """Append one token per sequence to the latent cache.

    For each sequence b with current length L_b (the new token's position):
      x = W_DKV h_b                                   (down-projection)
      c = RMSNorm(x[0:d_c]) * gamma                    (latent RMSNorm)
      k = RoPE(x[d_c:], pos = L_b)                     (decoupled key, rotated)
      cache[b, L_b, :] = [c || k];  L_b += 1
    ([MLA-とは] "MLAの発想" eq. c^KV; "Decoupled RoPE" eq. k^R_j = R_j W^KR h_j
    and the statement that the cache holds the already-rotated k^R;
    "実装上のトレードオフ" 正規化の扱い for caching the normalised latent.)

    Returns (new_cache float64 copy, new_seqlens int64 copy, rows [B, R] float64).
    Raises IndexError if a sequence is already at capacity (nothing written).
    """
    cache = _f64(cache).copy()
    seqlens = np.asarray(seqlens, dtype=np.int64).copy()
    B, cap, R = cache.shape
    x = down_project(h, W_DKV)
    if x.shape != (B, R):
        raise ValueError("W_DKV rows must equal the cache row width")
    c = rms_norm(x[:, :d_c], gamma, eps)
    rows = np.empty((B, R), dtype=np.float64)
    for b in range(B):
        L = int(seqlens[b])
        if L >= cap:
            raise IndexError(f"sequence {b} is at capacity {cap}")
        k = rope(x[b, d_c:], L, rope_base)
        rows[b] = np.concatenate([c[b], k])
        cache[b, L] = rows[b]
        seqlens[b] = L + 1
    return cache, seqlens, rows


# ---------------------------------------------------------------------------
# Materialised MHA decode (the plain definition the absorbed form must equal)
# ---------------------------------------------------------------------------
def head_logits(q_nope_i, q_pe_i, q_pos, W_UK_i, c, k_pe,
                rope_base: float = 10000.0) -> np.ndarray:
    """Raw (unscaled) attention logits of one head against L cached tokens,
    with K materialised.

    q = [q^C ; RoPE(q^R, q_pos)]       ([MLA-とは] "Decoupled RoPE", q_{t,i})
    k_j = [W^UK_i c_j ; k^R_j]          (k^C = W^UK c^KV, "MLAの発想";
                                         k^R_j shared by all heads, stored rotated)
    logit_j = q . k_j                   ("Decoupled RoPE", the split dot product)

    q_nope_i: [d_h]; q_pe_i: [d_r]; W_UK_i: [d_h, d_c]; c: [L, d_c];
    k_pe: [L, d_r].  Returns [L].
    """
    q = np.concatenate([_f64(q_nope_i), rope(q_pe_i, q_pos, rope_base)])
    kC = _f64(c) @ _f64(W_UK_i).T  # [L, d_h]: rows are k^C_j = W^UK_i c_j
    K = np.concatenate([kC, _f64(k_pe)], axis=1)  # [L, d_h + d_r]
    return K @ q


def softmax_lse(s):
    """Softmax of a logit vector with max subtraction, and its log-sum-exp.

    An empty vector gives (empty weights, -inf)."""
    s = _f64(s)
    if s.size == 0:
        return s.copy(), -math.inf
    m = np.max(s)
    e = np.exp(s - m)
    z = np.sum(e)
    return e / z, float(m + math.log(z))


def materialised_values(p, c, W_UV_i) -> np.ndarray:
    """o = sum_j p_j v_j with v_j = W^UV_i c_j materialised per cached token
    ([MLA-とは] "Value側の吸収", first equation for o_{t,i}).

    p: [L]; c: [L, d_c]; W_UV_i: [d_v, d_c] -> [d_v]."""
    V = _f64(c) @ _f64(W_UV_i).T  # [L, d_v]: rows are v^C_j
    return _f64(p) @ V


def mla_decode_materialised(q_nope, q_pe, q_pos, W_UK, W_UV, cache, seqlens,
                            softmax_scale: float, rope_base: float = 10000.0):
    """Single-token decode as plain multi-head attention with K and V
    materialised from the latent cache (what the absorbed kernel must equal).

    For every sequence b and head i:
      s_j = scale * (q . k_j)  for j < L_b                  (head_logits)
      p = softmax(s); lse = log sum_j exp(s_j)
      out[b,i]   = sum_j p_j W^UV_i c_j                     ("Value側の吸収")
      o_lat[b,i] = sum_j p_j c_j                            (latent-space sum)
    scale is 1/sqrt(d_h + d_r) in the configs ([MLA-とは] "Decoupled RoPE",
    softmax scaling by the concatenated dimension).

    q_nope: [B,H,d_h]; q_pe: [B,H,d_r]; q_pos: [B] ints; W_UK: [H,d_h,d_c];
    W_UV: [H,d_v,d_c]; cache: [B,cap,d_c+d_r]; seqlens: [B].
    Returns out [B,H,d_v], o_lat [B,H,d_c], lse [B,H] (float64).
    An empty sequence gives out = 0, o_lat = 0, lse = -inf.
    """
    q_nope, q_pe = _f64(q_nope), _f64(q_pe)
    W_UK, W_UV, cache = _f64(W_UK), _f64(W_UV), _f64(cache)
    B, H, _ = q_nope.shape
    d_c = W_UK.shape[2]
    d_v = W_UV.shape[1]
    out = np.zeros((B, H, d_v))
    o_lat = np.zeros((B, H, d_c))
    lse = np.full((B, H), -math.inf)
    for b in range(B):
        L = int(seqlens[b])
        if L == 0:
            continue
        c = cache[b, :L, :d_c]
        k_pe = cache[b, :L, d_c:]
        for i in range(H):
            s = softmax_scale * head_logits(q_nope[b, i], q_pe[b, i],
                                            q_pos[b], W_UK[i], c, k_pe,
                                            rope_base)
            p, lse[b, i] = softmax_lse(s)
            out[b, i] = materialised_values(p, c, W_UV[i])
            o_lat[b, i] = p @ c
    return out, o_lat, lse


# ---------------------------------------------------------------------------
# The absorbed quantities, each by its own plain definition
# ---------------------------------------------------------------------------
def absorb_q(q_nope, q_pe, W_UK, q_pos, rope_base: float = 10000.0):
    """q_cat[b,i] = [ W^UK_i^T q^C_{b,i} ; RoPE(q^R_{b,i}, q_pos[b]) ].

    The first block is q~ := W^UK_i^T q_{t,i} in R^{d_c} ([MLA-とは] "行列吸収",
    the per-step equation for q~); the second is the rotated decoupled query
    ("Decoupled RoPE", q^R = R_t W^QR c^Q).  If ``q_pos`` is None the q_pe
    input is taken as already rotated.
    Returns [B, H, d_c + d_r] float64.
    """
    q_nope, q_pe, W_UK = _f64(q_nope), _f64(q_pe), _f64(W_UK)
    q_tilde = np.einsum("bir,ird->bid", q_nope, W_UK)
    if q_pos is None:
        q_rot = q_pe.copy()
    else:
        q_rot = rope(q_pe, _f64(q_pos)[:, None], rope_base)
    return np.concatenate([q_tilde, q_rot], axis=-1)


def latent_attention(q_cat, cache, seqlens, softmax_scale: float,
                     d_c: int, key_range=None):
    """Attention of the absorbed query over the latent rows, i.e. MQA whose
    one shared key is the whole row [c || k^R] and whose shared value is c
    ([MLA-とは] "実装上のトレードオフ": the absorbed form is MQA with head dim
    d_c + d_r; "Value側の吸収": the weighted sum is taken in latent space).

      s_j = scale * (q_cat[b,i] . row_j)   for j in the key range
      o_lat[b,i] = sum_j softmax(s)_j c_j,  lse[b,i] = log sum_j exp(s_j)

    ``key_range`` (optional) is a (start, stop) pair per sequence, used to
    produce split-KV partials; by default it is [0, L_b).
    Returns o_lat [B,H,d_c], lse [B,H] (float64).  Empty ranges give 0 / -inf.
    """
    q_cat, cache = _f64(q_cat), _f64(cache)
    B, H, _ = q_cat.shape
    o_lat = np.zeros((B, H, d_c))
    lse = np.full((B, H), -math.inf)
    for b in range(B):
        lo, hi = (0, int(seqlens[b])) if key_range is None else key_range[b]
        if hi <= lo:
            continue
        rows = cache[b, lo:hi]  # [n, R]
        S = softmax_scale * (q_cat[b] @ rows.T)  # [H, n]
        for i in range(H):
            p, lse[b, i] = softmax_lse(S[i])
            o_lat[b, i] = p @ rows[:, :d_c]
    return o_lat, lse


def combine_partials(o_parts, lse_parts):
    """Merge split-KV partial results by their log-sum-exp.

    Each partial s holds o_s = softmax over its key chunk applied to the values
    and lse_s = log of its chunk's exp-sum.  The whole-sequence result is
        lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) o_s,
    with partials whose lse_s = -inf (empty chunks) contributing nothing and
    an all-empty set giving o = 0, lse = -inf.  (Split-KV is not described on
    the pages; this is the plain identity that makes chunked softmax equal the
    unchunked one, pinned in the tests against unsplit attention.)

    o_parts: [..., S, D]; lse_parts: [..., S] -> o [..., D], lse [...].
    """
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    m = np.max(lse_parts, axis=-1, keepdims=True)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe), 0.0)
    z = np.sum(w, axis=-1, keepdims=True)
    z_safe = np.where(z > 0, z, 1.0)
    o = np.einsum("...s,...sd->...d", w / z_safe, np.where(
        np.isfinite(lse_parts)[..., None], o_parts, 0.0))
    lse = np.where(finite[..., 0], m_safe[..., 0] + np.log(z_safe[..., 0]),
                   -math.inf)
    return o, lse


def out_proj(o_lat, W_UV) -> np.ndarray:
    """out[b,i] = W^UV_i o_lat[b,i]: the value up-projection applied once,
    after the latent-space weighted sum ([MLA-とは] "Value側の吸収", second
    equation for o_{t,i}).  o_lat: [B,H,d_c]; W_UV: [H,d_v,d_c] -> [B,H,d_v]."""
    return np.einsum("ivd,bid->biv", _f64(W_UV), _f64(o_lat))


# ---------------------------------------------------------------------------
# Prefill: many query tokens of one sequence, K and V materialised
# ---------------------------------------------------------------------------
def prefill_scores(q_nope, q_pe, q_pos, W_UK_i, c, k_pe, rope_base: float = 10000.0):
    """Raw logits of head i for T query tokens against L cached rows, with the
    causal mask: query t (at position q_pos[t]) sees rows j <= q_pos[t], and
    the others get -inf.  Each unmasked entry is head_logits' dot product
    [q^C ; RoPE(q^R, q_pos[t])] . [W^UK_i c_j ; k^R_j].

    q_nope: [T, d_h]; q_pe: [T, d_r]; q_pos: [T]; W_UK_i: [d_h, d_c];
    c: [L, d_c]; k_pe: [L, d_r] (stored rotated).  Returns [T, L]."""
    q_nope, q_pe = _f64(q_nope), _f64(q_pe)
    T, L = q_nope.shape[0], _f64(c).shape[0]
    K = np.concatenate([_f64(c) @ _f64(W_UK_i).T, _f64(k_pe)], axis=1)   # [L, d_h + d_r]
    Q = np.concatenate([q_nope, rope(q_pe, _f64(q_pos), rope_base)], axis=1)
    S = Q @ K.T
    j = np.arange(L)[None, :]
    return np.where(j <= np.asarray(q_pos)[:, None], S, -math.inf)


def prefill_materialised(q_nope, q_pe, q_pos, W_UK, W_UV, rows, d_c: int,
                         softmax_scale: float, rope_base: float = 10000.0):
    """Prefill of one sequence in the materialised form the pages recommend
    when the step is compute-bound ([MLA-とは] "実装上のトレードオフ",
    プリフィルとデコードで最適な形が違う): k^C = W^UK c and v^C = W^UV c are
    formed for every cached row and the heads run ordinary causal attention.

    q_nope: [T, H, d_h]; q_pe: [T, H, d_r]; q_pos: [T] positions (query t sees
    rows j <= q_pos[t]); rows: [L, d_c + d_r] latent cache rows (the prompt's
    own rows included).  Returns out [T, H, d_v] and lse [T, H] (float64)."""
    q_nope, q_pe, W_UK, W_UV, rows = map(_f64, (q_nope, q_pe, W_UK, W_UV, rows))
    T, H, _ = q_nope.shape
    c, k_pe = rows[:, :d_c], rows[:, d_c:]
    out = np.zeros((T, H, W_UV.shape[1]))
    lse = np.full((T, H), -math.inf)
    for i in range(H):
        S = softmax_scale * prefill_scores(q_nope[:, i], q_pe[:, i], q_pos, W_UK[i], c, k_pe,
                                           rope_base)
        V = c @ W_UV[i].T                                                   # [L, d_v]
        for t in range(T):
            n = min(int(q_pos[t]) + 1, rows.shape[0])   # rows query t may see
            p, lse[t, i] = softmax_lse(S[t, :n])
            out[t, i] = p @ V[:n]
    return out, lse


# ---------------------------------------------------------------------------
# Output projection W^O, and its fold with W^UV
# ---------------------------------------------------------------------------
def output_projection(out, W_O) -> np.ndarray:
    """u[b] = sum_i W^O_i out[b,i], where W^O_i in R^{d x d_v} is the column
    block of W^O that belongs to head i ([MLA-とは] "Value側の吸収", the
    equation for u_t, left-hand form).

    out: [B, H, d_v]; W_O: [d, H*d_v] (column convention, u = W^O o with the
    heads' outputs concatenated) -> u [B, d]."""
    out, W_O = _f64(out), _f64(W_O)
    B, H, d_v = out.shape
    u = np.zeros((B, W_O.shape[0]))
    for i in range(H):
        u += out[:, i, :] @ W_O[:, i * d_v:(i + 1) * d_v].T
    return u


def fold_output_weights(W_O, W_UV) -> np.ndarray:
    """B_i = W^O_i W^UV_i in R^{d x d_c}: W^UV absorbed into the output
    projection once, at load time ([MLA-とは] "Value側の吸収", the
    definition of B_i under the equation for u_t).

    W_O: [d, H*d_v]; W_UV: [H, d_v, d_c] -> B [H, d, d_c]."""
    W_O, W_UV = _f64(W_O), _f64(W_UV)
    H, d_v, _ = W_UV.shape
    return np.stack([W_O[:, i * d_v:(i + 1) * d_v] @ W_UV[i]
                     for i in range(H)])


def folded_output(o_lat, B_fold) -> np.ndarray:
    """u[b] = sum_i B_i o_lat[b,i]: the latent-space weighted sums go straight
    through the folded weights ([MLA-とは] "Value側の吸収", the right-hand form
    of the equation for u_t).  o_lat: [B, H, d_c]; B_fold: [H, d, d_c] -> [B, d]."""
    return np.einsum("idc,bic->bd", _f64(B_fold), _f64(o_lat))


# ---------------------------------------------------------------------------
# FP8 latent cache: E4M3 codes for c^KV with one power-of-two scale per token
#
# The pages name KV-cache quantisation ([abeam] "モデル全体でも推論効率が大きく
# 改善した") and FP8 for MLA as an open question ([yuuk-wiki] "未解決の問い")
# without fixing a format.  The reading taken here: c^KV is stored as OCP FP8
# E4M3 codes (the finite-only variant, largest magnitude 448), each cached
# token carries one scale 2^k chosen so that its largest |c| fits under 448,
# and the decoupled key k^R stays in the 16-bit cache type.  A per-token
# scale keeps an append a purely local write; a power-of-two scale makes
# code * scale exact in bf16, so the only rounding is the E4M3 one.
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 byte, from the format's definition: bit 7 the sign,
    bits 6..3 the exponent field e (bias 7), bits 2..0 the mantissa m.
    e = 0 is subnormal, m/8 * 2^-6; otherwise (1 + m/8) * 2^(e-7); the one
    pattern e = 15, m = 7 is NaN (there are no infinities)."""
    code = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(code & 0x80, -1.0, 1.0)
    e = (code >> 3) & 0xF
    m = (code & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6,
                   (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & (code & 0x7 == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code of each value, rounded to nearest with ties to even and
    saturated to +-448 (finite inputs above 448, and infinities, give the
    largest code of their sign; NaN gives 0x7F).  The sign bit follows the
    input's sign, so a negative value that rounds to zero gives 0x80.

    The magnitude is rounded on the grid of its binade: spacing 2^(E-3) for
    2^E <= |x| < 2^(E+1) with E >= -6, and 2^-9 below 2^-6 (subnormals)."""
    x = _f64(x)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)          # saturate (inf included)
    nan = np.isnan(x)
    a = np.where(nan, 0.0, a)
    _, k = np.frexp(a)                            # a = f 2^k, f in [0.5, 1)
    E = np.maximum(k - 1, -6)
    quantum = np.exp2((E - 3).astype(np.float64))
    r = np.round(a / quantum) * quantum           # numpy rounds ties to even
    # Back to the bit pattern of r (r <= 448 is always representable).
    _, k2 = np.frexp(r)
    E2 = k2 - 1
    sub = r < 2.0 ** -6
    mant_sub = np.round(r / 2.0 ** -9).astype(np.int64)
    field = np.where(sub, 0, E2 + 7).astype(np.int64)
    mant_norm = np.round((r / np.exp2(E2.astype(np.float64)) - 1.0) * 8.0)
    mant = np.where(sub, mant_sub, mant_norm.astype(np.int64))
    code = (field << 3) | mant
    code = np.where(neg, code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def latent_row_scale(c) -> np.ndarray:
    """Per-token scale 2^k with k the smallest integer such that
    max_j |c_j| / 2^k <= 448; a row of zeros gets scale 1.
    c: [..., d_c] -> [...] float64 (exact powers of two)."""
    c = _f64(c)
    amax = np.max(np.abs(c), axis=-1)
    safe = np.where(amax > 0, amax, E4M3_MAX)
    k = np.ceil(np.log2(safe / E4M3_MAX))
    # Guard the log2 rounding at exact binade edges: settle k by comparison.
    k = np.where(safe / np.exp2(k) > E4M3_MAX, k + 1, k)
    k = np.where(safe / np.exp2(k - 1) <= E4M3_MAX, k - 1, k)
    return np.exp2(k)


def quantize_latent_rows(c):
    """(codes, scale) of each cached latent: scale = latent_row_scale(c) and
    codes = E4M3(c / scale).  Division by a power of two is exact, so each
    code is the E4M3 rounding of the latent value itself.
    c: [..., d_c] -> codes uint8 [..., d_c], scale float64 [...]."""
    c = _f64(c)
    scale = latent_row_scale(c)
    return e4m3_encode(c / scale[..., None]), scale


def dequantize_latent_rows(codes, scale) -> np.ndarray:
    """c~ = E4M3 value of each code times its token's scale (float64, exact)."""
    return e4m3_decode(codes) * _f64(scale)[..., None]


# ---------------------------------------------------------------------------
# Closed forms: cache size and multiply counts
# ---------------------------------------------------------------------------
def cache_elems_per_token(kind: str, layers: int, n_h: int = 0, d_h: int = 0,
                          n_g: int = 0, d_c: int = 0, d_r: int = 0) -> int:
    """KV-cache elements per token over all layers.

    MHA 2 n_h d_h l; GQA 2 n_g d_h l; MQA 2 d_h l; MLA (d_c + d_h^R) l
    ([MLA-とは] "KVキャッシュはなぜ推論の急所なのか" and "KVキャッシュ容量の比較";
    [attention-variants] "MLA: キャッシュする対象そのものを変える").
    """
    if kind == "MHA":
        return 2 * n_h * d_h * layers
    if kind == "GQA":
        return 2 * n_g * d_h * layers
    if kind == "MQA":
        return 2 * d_h * layers
    if kind == "MLA":
        return (d_c + d_r) * layers
    raise ValueError(kind)


def mults_per_cached_token(form: str, n_h: int, d_h: int, d_c: int) -> int:
    """Multiplies per cached token per layer for the key side.

    naive: n_h d_h d_c (re-projecting every cached latent); absorbed: n_h d_c
    (one d_c-long dot product per head); MHA: n_h d_h
    ([MLA-とは] "行列吸収" closing paragraph and "実装上のトレードオフ", FLOPは増える).
    """
    if form == "naive":
        return n_h * d_h * d_c
    if form == "absorbed":
        return n_h * d_c
    if form == "MHA":
        return n_h * d_h
    raise ValueError(form)
