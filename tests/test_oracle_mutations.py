"""Plants plausible mistakes in the oracle (CPU only, via monkeypatch) and checks that the pins
in test_oracle_pins catch every one of them."""
import math

import numpy as np
import pytest

from oracle import mla_oracle as O
from tests import test_oracle_pins as P

PINS = [getattr(P, n) for n in dir(P) if n.startswith("test_") and callable(getattr(P, n))]


def _rope_sign_flip(x, pos, theta=10000.0):
    x = O.f64(x)
    d = x.shape[-1]
    i = np.arange(d // 2)
    ang = pos * theta ** (-2.0 * i / d)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * np.cos(ang) + x[..., 1::2] * np.sin(ang)
    out[..., 1::2] = -x[..., 0::2] * np.sin(ang) + x[..., 1::2] * np.cos(ang)
    return out


def _rope_half_split(x, pos, theta=10000.0):
    # rotate (x[i], x[i + d/2]) instead of interleaved pairs
    x = O.f64(x)
    d = x.shape[-1]
    i = np.arange(d // 2)
    ang = pos * theta ** (-2.0 * i / d)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)],
                          axis=-1)


def _rope_wrong_freq(x, pos, theta=10000.0):
    x = O.f64(x)
    d = x.shape[-1]
    i = np.arange(d // 2)
    ang = pos * theta ** (-1.0 * i / d)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * np.cos(ang) - x[..., 1::2] * np.sin(ang)
    out[..., 1::2] = x[..., 0::2] * np.sin(ang) + x[..., 1::2] * np.cos(ang)
    return out


_real_decode = O.decode_attention
_real_hkv = O.head_keys_values


def _decode_wrong_scale(q_nope, q_rope, c_kv, k_r, w_uk, w_uv, scale=None, heads=None):
    if scale is None:
        scale = 1.0 / math.sqrt(O.f64(q_nope).shape[1])  # d_nope only, rope width forgotten
    return _real_decode(q_nope, q_rope, c_kv, k_r, w_uk, w_uv, scale, heads)


def _decode_no_rope(q_nope, q_rope, c_kv, k_r, w_uk, w_uv, scale=None, heads=None):
    if scale is None:
        scale = 1.0 / math.sqrt(192)
    return _real_decode(q_nope, np.zeros_like(O.f64(q_rope)), c_kv, k_r, w_uk, w_uv, scale, heads)


def _hkv_transposed_uk(c_kv, k_r, w_uk, w_uv, head, d_nope, d_v):
    # slice W_UK by columns of its transpose: a head's rows taken with the wrong stride
    w_uk = O.f64(w_uk)
    H = w_uk.shape[0] // d_nope
    w_uk_perm = w_uk.reshape(d_nope, H, -1).transpose(1, 0, 2).reshape(H * d_nope, -1)
    return _real_hkv(c_kv, k_r, w_uk_perm, w_uv, head, d_nope, d_v)


def _hkv_values_from_uk(c_kv, k_r, w_uk, w_uv, head, d_nope, d_v):
    return _real_hkv(c_kv, k_r, w_uk, w_uk, head, d_nope, d_v)


def _causal_no_mask(q, k, v, scale):
    q, k, v = O.f64(q), O.f64(k), O.f64(v)
    return O.softmax((q @ k.T) * scale, axis=-1) @ v


_real_gather = O.gather_rows


def _gather_slot_order_reversed(pool, page_table_row, n_rows, page_size=64):
    pool = O.f64(pool)[:, ::-1]  # slot j read as page_size-1-j
    return _real_gather(pool, page_table_row, n_rows, page_size)


def _latent_row_no_rope(h, w_dkv, w_kr, pos, theta=10000.0):
    h = O.f64(h)
    return O.f64(w_dkv) @ h, O.f64(w_kr) @ h


def _query_heads_swapped(h, w_q, n_heads, d_nope, d_rope, pos, theta=10000.0):
    q = (O.f64(w_q) @ O.f64(h)).reshape(n_heads, d_nope + d_rope)
    return q[:, d_rope:].copy(), O.rope(q[:, :d_rope], pos, theta)


def _mla_bytes_with_heads(d_c, d_rope, n_layers, bytes_per_elem):
    return (d_c + 2 * d_rope) * n_layers * bytes_per_elem


_real_e4m3_decode = O.e4m3_decode
_real_e4m3_quantize = O.e4m3_quantize


def _e4m3_bias_8(codes):
    # exponent bias 8 instead of 7: every normal value halved
    v = _real_e4m3_decode(codes)
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    return np.where((c >> 3) & 0xF, v / 2.0, v)


def _e4m3_no_subnormals(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    return np.where(((c >> 3) & 0xF) == 0, 0.0, _real_e4m3_decode(codes))


def _e4m3_ties_up(x):
    # ties resolved away from zero instead of to the even code
    x = np.asarray(x, dtype=np.float64)
    grid = _real_e4m3_decode(np.arange(0x7F))
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(grid, a), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    code = np.where(grid[hi] - a <= a - grid[lo], hi, lo)
    return (code | (np.signbit(x).astype(np.int64) << 7)).astype(np.uint8)


def _e4m3_truncate(x):
    # rounding toward zero instead of to nearest
    x = np.asarray(x, dtype=np.float64)
    grid = _real_e4m3_decode(np.arange(0x7F))
    a = np.minimum(np.abs(x), 448.0)
    code = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, 0x7E)
    return (code | (np.signbit(x).astype(np.int64) << 7)).astype(np.uint8)


MUTATIONS = {
    "E4M3 exponent bias 8": ("e4m3_decode", _e4m3_bias_8),
    "E4M3 subnormals read as zero": ("e4m3_decode", _e4m3_no_subnormals),
    "E4M3 ties away from zero": ("e4m3_quantize", _e4m3_ties_up),
    "E4M3 rounding toward zero": ("e4m3_quantize", _e4m3_truncate),
    "rope sign flipped": ("rope", _rope_sign_flip),
    "rope half-split pairs": ("rope", _rope_half_split),
    "rope wrong frequencies": ("rope", _rope_wrong_freq),
    "score scale 1/sqrt(d_nope)": ("decode_attention", _decode_wrong_scale),
    "rope term dropped from score": ("decode_attention", _decode_no_rope),
    "W_UK head slice wrong": ("head_keys_values", _hkv_transposed_uk),
    "V built from W_UK": ("head_keys_values", _hkv_values_from_uk),
    "causal mask missing": ("causal_attention", _causal_no_mask),
    "RoPE missing on k_R": ("latent_row", _latent_row_no_rope),
    "query nope/rope split swapped": ("query_heads", _query_heads_swapped),
    "cache bytes count RoPE twice": ("mla_cache_bytes_per_token", _mla_bytes_with_heads),
    "page slots read in reverse": ("gather_rows", _gather_slot_order_reversed),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in PINS:
        try:
            if "pos" in pin.__code__.co_varnames[: pin.__code__.co_argcount]:
                pin(7)
            else:
                pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught: {name}"
