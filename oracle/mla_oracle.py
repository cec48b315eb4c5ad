"""CPU fp64 oracle for Multi-Head Latent Attention (MLA) decode.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module.  It shares no code with the CUDA path and does NOT
use weight absorption: per head it rebuilds the full key K = [c_KV W_UK^T | k_R] and value
V = c_KV W_UV^T from the cached latent rows and then runs textbook causal softmax attention.

Sources (web pages on MLA; cited by title and section):
  [LP]  linuxpro.com.br, "Como a DeepSeek reescreveu o Transformer (MLA)"
        - "Classic attention and the cost of the KV cache": Attention(Q,K,V) =
          softmax(Q K^T / sqrt(d_k) + M) V with M the causal mask; decode computes one new
          query row and reads the whole cache; MHA cache bytes formula.
        - "MLA: compress the pair, not the heads": latent c^KV (512) plus decoupled RoPE key
          k^R (64) cached, 576 numbers per token per layer; absorption by associativity.
  [TN]  technova-ai.online, "DeepSeek AI efficiency architecture benchmarks",
        section "Architectural Innovations: Multi-Head Latent Attention (MLA)":
        c_KV = W_DKV h_t,  K_t = W_UK c_KV,  V_t = W_UV c_KV  (column-vector form).
  [MD]  Medium mirror, "How Transformers Become Faster And Smarter: From KV Cache to MLA",
        section "KV Cache": causal mask by an upper-triangular fill inside the softmax; rows
        of K and V for past tokens do not change as the sequence grows.
  [IA]  ia.com.br, "Como a MLA da DeepSeek cortou 93% da memoria ...", sections
        "Um resumo no lugar de 128 copias" and "A conta feita fora da DeepSeek".

Readings where the pages are silent:
  * Query path: plain q = W_Q h_t, per head 128 non-rotary then 64 rotary rows.
  * Score scale 1/sqrt(d_k) with d_k = d_nope + d_R = 192.
  * RoPE: original interleaved-pair form, base theta (10000), frequencies
    theta^(-2i/d_R) for pair i, rotation angle = position * frequency.  The same rotation is
    applied to k_R (shared by all heads) and to each head's q_rope at the new token's position.
  * The new token attends to itself: with a cache of n rows the query sits at position n-1.
  * FP8 weights ([IA] "De onde vem o 93%" names FP8 without a format): E4M3 (bias 7, 3
    mantissa bits, subnormals, max 448), one fp32 scale per row, round to nearest even.

All arithmetic here is float64; inputs are upcast from whatever dtype the caller holds.
"""
from __future__ import annotations

import math

import numpy as np

PAGE = 64


def f64(x) -> np.ndarray:
    """Upcast a numpy array or torch tensor (any float dtype, incl. bfloat16) to float64."""
    if hasattr(x, "detach"):
        import torch  # local: the oracle itself only needs numpy
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------------------------
# Cache-size arithmetic ([LP] "Classic attention and the cost of the KV cache", "MQA and GQA",
# "MLA: compress the pair, not the heads"; [IA] "A conta feita fora da DeepSeek")
# ---------------------------------------------------------------------------------------------

def mha_cache_bytes_per_token(d_h: int, n_heads: int, n_layers: int, bytes_per_elem: int) -> int:
    """MHA stores a key and a value of width d_h per head per layer for every token."""
    return 2 * d_h * n_heads * n_layers * bytes_per_elem


def grouped_cache_bytes_per_token(d_h: int, n_kv_groups: float, n_layers: int,
                                  bytes_per_elem: int) -> float:
    """GQA/MQA store one key/value pair per group of heads (MQA: one group)."""
    return 2 * d_h * n_kv_groups * n_layers * bytes_per_elem


def mla_cache_bytes_per_token(d_c: int, d_rope: int, n_layers: int, bytes_per_elem: int) -> int:
    """MLA stores only the latent c^KV and the decoupled RoPE key k^R per token per layer,
    independent of the number of heads."""
    return (d_c + d_rope) * n_layers * bytes_per_elem


# ---------------------------------------------------------------------------------------------
# RoPE (decoupled rotary part; [LP] "MLA: compress the pair ...", [IA] "Um resumo ...")
# ---------------------------------------------------------------------------------------------

def rope(x, pos: int, theta: float = 10000.0) -> np.ndarray:
    """Rotate consecutive pairs (x[2i], x[2i+1]) by the angle pos * theta^(-2i/d)."""
    x = f64(x)
    d = x.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    ang = float(pos) * np.power(float(theta), -2.0 * i / d)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ---------------------------------------------------------------------------------------------
# Projections ([TN] MLA equations; [LP] Q = X W_Q)
# ---------------------------------------------------------------------------------------------

def latent_row(h, w_dkv, w_kr, pos: int, theta: float = 10000.0):
    """The numbers the new token adds to the cache: c_KV = W_DKV h_t and k_R = RoPE(W_KR h_t).

    Returns (c_kv [d_c], k_r [d_R]) in float64 (the caller rounds to the cache dtype).
    """
    h = f64(h)
    c_kv = f64(w_dkv) @ h
    k_r = rope(f64(w_kr) @ h, pos, theta)
    return c_kv, k_r


def query_heads(h, w_q, n_heads: int, d_nope: int, d_rope: int, pos: int,
                theta: float = 10000.0):
    """q = W_Q h_t split per head into (q_nope [H, d_nope], RoPE(q_rope) [H, d_R])."""
    q = (f64(w_q) @ f64(h)).reshape(n_heads, d_nope + d_rope)
    return q[:, :d_nope].copy(), rope(q[:, d_nope:], pos, theta)


# ---------------------------------------------------------------------------------------------
# Paged cache access
# ---------------------------------------------------------------------------------------------

def gather_rows(pool, page_table_row, n_rows: int, page_size: int = PAGE) -> np.ndarray:
    """Rows 0..n_rows-1 of one sequence: row j lives in page page_table_row[j // page_size],
    slot j % page_size."""
    pt = np.asarray(page_table_row, dtype=np.int64)
    n_pages = -(-n_rows // page_size)
    if n_pages == 0:
        return np.zeros((0, pool.shape[-1]), dtype=np.float64)
    if hasattr(pool, "detach"):
        import torch
        pages = f64(pool[torch.from_numpy(pt[:n_pages])])
    else:
        pages = f64(np.asarray(pool)[pt[:n_pages]])
    # pages[i][k] is row i * page_size + k
    return pages.reshape(n_pages * page_size, -1)[:n_rows].copy()


# ---------------------------------------------------------------------------------------------
# Attention ([LP] softmax(QK^T/sqrt(d_k) + M) V; [MD] triu causal mask)
# ---------------------------------------------------------------------------------------------

def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    """Max-subtracted softmax; -inf entries get weight 0."""
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def causal_attention(q, k, v, scale: float) -> np.ndarray:
    """Full textbook causal attention for T query rows against T keys/values:
    row t attends to positions 0..t (the strictly upper triangle is masked)."""
    q, k, v = f64(q), f64(k), f64(v)
    t = q.shape[0]
    s = (q @ k.T) * scale
    s[np.triu(np.ones((t, t), dtype=bool), k=1)] = -np.inf
    return softmax(s, axis=-1) @ v


def head_keys_values(c_kv, k_r, w_uk, w_uv, head: int, d_nope: int, d_v: int):
    """Per-head full key and value rebuilt from the latent cache (no absorption):
    K_h[j] = [W_UK_h c_j | k_R,j] and V_h[j] = W_UV_h c_j, with W_UK_h = rows
    head*d_nope .. of W_UK and W_UV_h = rows head*d_v .. of W_UV."""
    c_kv, k_r = f64(c_kv), f64(k_r)
    w_uk_h = f64(w_uk)[head * d_nope:(head + 1) * d_nope]   # [d_nope, d_c]
    w_uv_h = f64(w_uv)[head * d_v:(head + 1) * d_v]         # [d_v, d_c]
    k_h = np.concatenate([c_kv @ w_uk_h.T, k_r], axis=1)    # [n, d_nope + d_R]
    v_h = c_kv @ w_uv_h.T                                   # [n, d_v]
    return k_h, v_h


def decode_attention(q_nope, q_rope, c_kv, k_r, w_uk, w_uv, scale: float | None = None,
                     heads=None):
    """One new query per head attending to all n cached rows (it sits at position n-1, so the
    causal mask admits every row).  Returns dict with
      o_heads [len(heads), d_v]   attention output per head in value space,
      o_lat   [len(heads), d_c]   sum_j p_j c_j (diagnostic; W_UV_h o_lat_h = o_heads),
      lse     [len(heads)]        natural-log sum of exp(score), scores already scaled.
    """
    q_nope, q_rope = f64(q_nope), f64(q_rope)
    c_kv, k_r = f64(c_kv), f64(k_r)
    n_heads, d_nope = q_nope.shape
    d_rope = q_rope.shape[1]
    d_v = f64(w_uv).shape[0] // n_heads
    if scale is None:
        scale = 1.0 / math.sqrt(d_nope + d_rope)
    if heads is None:
        heads = range(n_heads)
    heads = list(heads)
    n = c_kv.shape[0]
    o_heads = np.zeros((len(heads), d_v))
    o_lat = np.zeros((len(heads), c_kv.shape[1]))
    lse = np.full(len(heads), -np.inf)
    if n == 0:
        return {"o_heads": o_heads, "o_lat": o_lat, "lse": lse}
    for i, h in enumerate(heads):
        k_h, v_h = head_keys_values(c_kv, k_r, w_uk, w_uv, h, d_nope, d_v)
        q_h = np.concatenate([q_nope[h], q_rope[h]])
        s = (k_h @ q_h) * scale
        m = np.max(s)
        lse[i] = m + math.log(np.sum(np.exp(s - m)))
        p = softmax(s)
        o_heads[i] = p @ v_h
        o_lat[i] = p @ c_kv
    return {"o_heads": o_heads, "o_lat": o_lat, "lse": lse}


def latent_attention(q_lat, q_rope, c_kv, k_r, scale: float | None = None):
    """Diagnostic for the attention step alone, stated in latent space: scores
    s_j = scale * (q_lat . c_j + q_rope . k_R,j), p = softmax(s), o_lat = sum_j p_j c_j.
    The end-to-end reference is decode_attention (no absorption); this form equals it by the
    associativity the pages state ([LP] "MLA: compress the pair, not the heads") and is
    pinned against it.  q_lat [H, d_c], q_rope [H, d_R]; returns o_lat [H, d_c], lse [H]."""
    q_lat, q_rope = f64(q_lat), f64(q_rope)
    c_kv, k_r = f64(c_kv), f64(k_r)
    H = q_lat.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(128 + q_rope.shape[1])
    if c_kv.shape[0] == 0:
        return np.zeros((H, c_kv.shape[1])), np.full(H, -np.inf)
    s = (q_lat @ c_kv.T + q_rope @ k_r.T) * scale          # [H, n]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    tot = e.sum(axis=1, keepdims=True)
    return (e / tot) @ c_kv, (m + np.log(tot))[:, 0]


def output_projection(o_heads, w_o) -> np.ndarray:
    """out = W_O concat_h(o_h)."""
    return f64(w_o) @ f64(o_heads).reshape(-1)


# ---------------------------------------------------------------------------------------------
# FP8 (E4M3) storage of weights
# ---------------------------------------------------------------------------------------------
# [IA] "De onde vem o 93%": the pages' one throughput figure was measured with the weights
# converted to FP8.  The pages do not define the 8-bit format; this reads it as the common
# "E4M3" float: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at
# exponent field 0, no infinities, S.1111.111 = NaN, largest finite magnitude 448.  A weight
# row is stored as codes of w / s with one fp32 scale s per row (so the row's largest
# magnitude maps to 448).

def e4m3_decode(codes) -> np.ndarray:
    """The value of each E4M3 byte, in float64 (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return np.where((c & 0x7F) == 0x7F, np.nan, sign * mag)


def e4m3_quantize(x) -> np.ndarray:
    """The E4M3 byte of each value: the nearest finite E4M3 value, a tie going to the code whose
    last mantissa bit is 0, magnitudes above 448 saturating to 448; the sign is kept (also on
    zero)."""
    x = np.asarray(x, dtype=np.float64)
    grid = e4m3_decode(np.arange(0x7F))  # codes 0x00 .. 0x7E: 0 .. 448, increasing
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(grid, a), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    code = np.where((d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0)), hi, lo)
    code = np.where(grid[hi] == a, hi, code)
    return (code | (np.signbit(x).astype(np.int64) << 7)).astype(np.uint8)


def quantize_rows_e4m3(w):
    """Per-row E4M3 storage of a weight matrix [rows, cols]: s_r = max_j |w_rj| / 448 in fp32
    (1 for a zero row) and the codes of w_rj / s_r, the division in fp32 -- the precision in
    which the GPU takes the same decision.  Returns (codes uint8 [rows, cols], s float32
    [rows])."""
    w32 = np.asarray(w, dtype=np.float32)
    amax = np.abs(w32).max(axis=1)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    y = (w32 / s[:, None]).astype(np.float32)
    return e4m3_quantize(y.astype(np.float64)), s


def dequantize_rows_e4m3(codes, s) -> np.ndarray:
    """The weights an E4M3-stored matrix stands for: decode(code) * s_r, in float64."""
    return e4m3_decode(codes) * np.asarray(s, dtype=np.float64)[:, None]


# ---------------------------------------------------------------------------------------------
# One whole decode step for one sequence of one layer
# ---------------------------------------------------------------------------------------------

def decode_step(h, w, history_rows, pos: int, n_heads: int, theta: float = 10000.0,
                round_row=None, heads=None, with_out: bool = True,
                d_c: int = 512, d_rope: int = 64, d_nope: int = 128):
    """Append the new token's latent row at ``pos`` (= number of history rows), then attend.

    ``w`` has attributes w_dkv, w_kr, w_q, w_uk, w_uv, w_o.  ``history_rows`` [pos, d_c+d_R]
    are the cached rows before this step.  ``round_row`` (optional) maps the float64 appended
    row to the value actually stored in the cache (e.g. rounding to bfloat16), because the
    cache stores the row in its own dtype before any later read of it.
    """
    hist = f64(history_rows)
    assert hist.shape[0] == pos
    c_new, k_new = latent_row(h, w.w_dkv, w.w_kr, pos, theta)
    row = np.concatenate([c_new, k_new])
    if round_row is not None:
        row = f64(round_row(row))
    rows = np.concatenate([hist, row[None, :]], axis=0)
    q_nope, q_rope = query_heads(h, w.w_q, n_heads, d_nope, d_rope, pos, theta)
    res = decode_attention(q_nope, q_rope, rows[:, :d_c], rows[:, d_c:], w.w_uk, w.w_uv,
                           heads=heads)
    res["row"] = row
    res["q_nope"] = q_nope
    res["q_rope"] = q_rope
    if with_out and heads is None and f64(w.w_o).size:
        res["out"] = output_projection(res["o_heads"], w.w_o)
    return res
