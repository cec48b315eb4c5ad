"""Pins for the fp64 oracle: each test checks the oracle against something other than itself
(figures the MLA pages print, closed forms, special cases, invariants the pages state, brute
force on tiny inputs).  CPU only."""
import math
import os

import numpy as np
import pytest

from oracle import mla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_sizes.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, value, how = line.split()[:3]
            out[name] = (float(value), how)
    return out


def _check(value, printed, how):
    if how == "exact":
        assert value == printed, (value, printed)
    elif how.startswith("round:"):
        k = int(how.split(":")[1])
        assert round(value, k) == printed, (value, printed)
    elif how.startswith("approx:"):
        r = float(how.split(":")[1])
        assert abs(value - printed) <= r * abs(printed), (value, printed)
    else:
        raise AssertionError(how)


# ---------------------------------------------------------------------------------------------
# Figures printed on the pages
# ---------------------------------------------------------------------------------------------

def test_cache_sizes_match_printed_figures():
    g = _golden()
    mha = O.mha_cache_bytes_per_token(d_h=128, n_heads=128, n_layers=61, bytes_per_elem=2)
    mla = O.mla_cache_bytes_per_token(d_c=512, d_rope=64, n_layers=61, bytes_per_elem=2)
    mqa = O.grouped_cache_bytes_per_token(d_h=128, n_kv_groups=1, n_layers=61, bytes_per_elem=2)
    gqa8 = O.grouped_cache_bytes_per_token(d_h=128, n_kv_groups=128 // 8, n_layers=61,
                                           bytes_per_elem=2)
    values = {
        "mha_bytes_per_token": mha,
        "mla_bytes_per_token": mla,
        "mla_numbers_per_token": O.mla_cache_bytes_per_token(512, 64, 1, 1),
        "mla_vs_mha_factor": mha / mla,
        "mqa_kb_per_token": mqa / 1000.0,
        "gqa8_kb_per_token": gqa8 / 1000.0,
        "mla_gib_at_32k": mla * 32768 / 2 ** 30,
        "mla_gb_at_128k": mla * 131072 / 1e9,
        "mha_gb_read_at_100k": mha * 100_000 / 1e9,
        "low_rank_full_cost": 100 * 100,
        "low_rank_factored_cost": 100 * 20 + 100 * 20,
    }
    # MLA's cache equals GQA's with g groups where 2 * d_h * g = 576 -> g = 2.25
    g_equiv = O.mla_cache_bytes_per_token(512, 64, 61, 2) / O.grouped_cache_bytes_per_token(
        128, 1, 61, 2)
    values["gqa_groups_equal_to_mla"] = g_equiv
    assert set(values) == set(g), set(values) ^ set(g)
    for name, (printed, how) in g.items():
        _check(values[name], printed, how)


def test_mla_cache_independent_of_heads():
    a = O.mla_cache_bytes_per_token(512, 64, 61, 2)
    # the MHA figure grows with the head count, the MLA figure does not take it at all
    assert O.mha_cache_bytes_per_token(128, 64, 61, 2) * 2 == O.mha_cache_bytes_per_token(
        128, 128, 61, 2)
    assert a == 576 * 61 * 2


# ---------------------------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------------------------

def _rope_complex(x, pos, theta):
    """Independent formulation: pair (x0, x1) as the complex number x0 + i x1, rotated by
    multiplying with exp(i * pos * theta^(-2k/d))."""
    d = x.shape[-1]
    z = x[..., 0::2] + 1j * x[..., 1::2]
    k = np.arange(d // 2)
    z = z * np.exp(1j * pos * theta ** (-2.0 * k / d))
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


@pytest.mark.parametrize("pos", [0, 1, 7, 4095, 131071])
def test_rope_equals_complex_rotation(pos):
    rng = np.random.default_rng(pos)
    x = rng.standard_normal((3, 64))
    np.testing.assert_allclose(O.rope(x, pos), _rope_complex(x, pos, 10000.0), rtol=0,
                               atol=1e-12)


def test_rope_identity_at_position_zero():
    x = np.random.default_rng(1).standard_normal(64)
    assert np.array_equal(O.rope(x, 0), x)


def test_rope_preserves_norm():
    x = np.random.default_rng(2).standard_normal((5, 64))
    for pos in (1, 100, 99999):
        np.testing.assert_allclose(np.linalg.norm(O.rope(x, pos), axis=-1),
                                   np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    a = O.rope(q, 50) @ O.rope(k, 20)
    b = O.rope(q, 1030) @ O.rope(k, 1000)
    np.testing.assert_allclose(a, b, rtol=1e-10)


def test_rope_first_pair_rotates_by_position_radians():
    # pair 0 has frequency theta^0 = 1: a unit vector along x0 turns by exactly pos radians
    x = np.zeros(64)
    x[0] = 1.0
    y = O.rope(x, 3)
    assert y[0] == pytest.approx(math.cos(3.0), abs=1e-15)
    assert y[1] == pytest.approx(math.sin(3.0), abs=1e-15)


# ---------------------------------------------------------------------------------------------
# Projections and layouts (special inputs that reduce a product to reading one column)
# ---------------------------------------------------------------------------------------------

class _W:
    pass


def _tiny_weights(rng, H, D, d_c=512, d_r=64, d_nope=128, d_v=128, w_o=True):
    w = _W()
    w.w_dkv = rng.standard_normal((d_c, D))
    w.w_kr = rng.standard_normal((d_r, D))
    w.w_q = rng.standard_normal((H * (d_nope + d_r), D))
    w.w_uk = rng.standard_normal((H * d_nope, d_c))
    w.w_uv = rng.standard_normal((H * d_v, d_c))
    w.w_o = rng.standard_normal((D, H * d_v)) if w_o else np.zeros(0)
    return w


def test_latent_row_of_unit_input_is_a_weight_column():
    rng = np.random.default_rng(4)
    w = _tiny_weights(rng, 2, 16)
    e = np.zeros(16)
    e[5] = 1.0
    c, k = O.latent_row(e, w.w_dkv, w.w_kr, pos=9)
    assert np.array_equal(c, w.w_dkv[:, 5])
    np.testing.assert_allclose(k, _rope_complex(w.w_kr[:, 5], 9, 10000.0), atol=1e-13)


def test_query_heads_layout():
    rng = np.random.default_rng(5)
    H, D = 3, 8
    w = _tiny_weights(rng, H, D)
    e = np.zeros(D)
    e[2] = 1.0
    qn, qr = O.query_heads(e, w.w_q, H, 128, 64, pos=0)
    for h in range(H):
        assert np.array_equal(qn[h], w.w_q[h * 192:h * 192 + 128, 2])
        assert np.array_equal(qr[h], w.w_q[h * 192 + 128:(h + 1) * 192, 2])


def test_output_projection_of_one_hot_is_a_column():
    rng = np.random.default_rng(6)
    w_o = rng.standard_normal((16, 2 * 128))
    o = np.zeros((2, 128))
    o[1, 7] = 1.0
    assert np.array_equal(O.output_projection(o, w_o), w_o[:, 128 + 7])


# ---------------------------------------------------------------------------------------------
# Attention: special cases with closed forms
# ---------------------------------------------------------------------------------------------

def test_single_row_output_is_its_value():
    rng = np.random.default_rng(7)
    H = 2
    w = _tiny_weights(rng, H, 8)
    c = rng.standard_normal((1, 512))
    kr = rng.standard_normal((1, 64))
    qn, qr = rng.standard_normal((H, 128)), rng.standard_normal((H, 64))
    r = O.decode_attention(qn, qr, c, kr, w.w_uk, w.w_uv)
    for h in range(H):
        # softmax over one element is 1, so the output is V_h[0] = W_UV_h c_0
        np.testing.assert_allclose(r["o_heads"][h], w.w_uv[h * 128:(h + 1) * 128] @ c[0],
                                   rtol=1e-12)
        np.testing.assert_allclose(r["o_lat"][h], c[0], rtol=0, atol=0)


def test_zero_query_gives_mean_of_rows_and_log_n():
    rng = np.random.default_rng(8)
    w = _tiny_weights(rng, 2, 8)
    n = 37
    c, kr = rng.standard_normal((n, 512)), rng.standard_normal((n, 64))
    r = O.decode_attention(np.zeros((2, 128)), np.zeros((2, 64)), c, kr, w.w_uk, w.w_uv)
    np.testing.assert_allclose(r["o_lat"], np.broadcast_to(c.mean(0), (2, 512)), atol=1e-13)
    np.testing.assert_allclose(r["lse"], math.log(n), rtol=1e-14)


def test_two_rows_weights_follow_the_logistic_function():
    # only the first RoPE coordinate of the query is non-zero, so the scores are
    # a * b_j / sqrt(192) and the two softmax weights are logistic in their difference
    rng = np.random.default_rng(9)
    w = _tiny_weights(rng, 1, 8)
    a, b0, b1 = 2.0, 0.3, -1.1
    qn, qr = np.zeros((1, 128)), np.zeros((1, 64))
    qr[0, 0] = a
    c = rng.standard_normal((2, 512))
    kr = np.zeros((2, 64))
    kr[0, 0], kr[1, 0] = b0, b1
    r = O.decode_attention(qn, qr, c, kr, w.w_uk, w.w_uv)
    s0, s1 = a * b0 / math.sqrt(192), a * b1 / math.sqrt(192)
    p0 = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(r["o_lat"][0], p0 * c[0] + (1 - p0) * c[1], rtol=1e-12)
    np.testing.assert_allclose(r["lse"][0], math.log(math.exp(s0) + math.exp(s1)), rtol=1e-13)


def test_softmax_weights_sum_to_one_through_a_constant_latent_column():
    rng = np.random.default_rng(10)
    w = _tiny_weights(rng, 3, 8)
    c = rng.standard_normal((300, 512)) * 3
    c[:, 511] = 1.0
    kr = rng.standard_normal((300, 64)) * 3
    r = O.decode_attention(rng.standard_normal((3, 128)) * 3, rng.standard_normal((3, 64)) * 3,
                           c, kr, w.w_uk, w.w_uv)
    np.testing.assert_allclose(r["o_lat"][:, 511], 1.0, rtol=1e-13)


def test_one_dominant_key_selects_its_row():
    rng = np.random.default_rng(11)
    w = _tiny_weights(rng, 1, 8)
    c = rng.standard_normal((50, 512))
    kr = rng.standard_normal((50, 64)) * 0.01
    qn, qr = np.zeros((1, 128)), np.zeros((1, 64))
    qr[0] = 1.0
    kr[17] = 400.0  # score 400 * 64 / sqrt(192) ~ 1850 above the rest
    r = O.decode_attention(qn, qr, c, kr, w.w_uk, w.w_uv)
    np.testing.assert_allclose(r["o_lat"][0], c[17], rtol=1e-12)


# ---------------------------------------------------------------------------------------------
# Invariants the pages state
# ---------------------------------------------------------------------------------------------

def test_absorbed_form_equals_reconstructed_form():
    """QK^T = Q (c W_UK)^T = (Q W_UK^T) c^T, and W_UV applied after the weighted sum of latent
    rows ([LP] "MLA: compress the pair, not the heads", associativity)."""
    rng = np.random.default_rng(12)
    H, n = 4, 91
    w = _tiny_weights(rng, H, 8)
    w.w_uk /= math.sqrt(512)
    w.w_uv /= math.sqrt(512)
    c, kr = rng.standard_normal((n, 512)), rng.standard_normal((n, 64))
    qn, qr = rng.standard_normal((H, 128)), rng.standard_normal((H, 64))
    r = O.decode_attention(qn, qr, c, kr, w.w_uk, w.w_uv)
    for h in range(H):
        w_uk_h = w.w_uk[h * 128:(h + 1) * 128]
        q_lat = qn[h] @ w_uk_h                          # absorbed query, 512 wide
        s = (c @ q_lat + kr @ qr[h]) / math.sqrt(192)
        p = np.exp(s - s.max())
        p /= p.sum()
        o_lat = p @ c
        np.testing.assert_allclose(r["o_lat"][h], o_lat, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(r["o_heads"][h], w.w_uv[h * 128:(h + 1) * 128] @ o_lat,
                                   rtol=1e-11, atol=1e-12)


def test_latent_attention_equals_reconstructed_form():
    rng = np.random.default_rng(18)
    H, n = 3, 70
    w = _tiny_weights(rng, H, 8)
    w.w_uk /= math.sqrt(512)
    c, kr = rng.standard_normal((n, 512)), rng.standard_normal((n, 64))
    qn, qr = rng.standard_normal((H, 128)), rng.standard_normal((H, 64))
    naive = O.decode_attention(qn, qr, c, kr, w.w_uk, w.w_uv)
    q_lat = np.stack([w.w_uk[h * 128:(h + 1) * 128].T @ qn[h] for h in range(H)])
    o_lat, lse = O.latent_attention(q_lat, qr, c, kr)
    np.testing.assert_allclose(o_lat, naive["o_lat"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, naive["lse"], rtol=1e-12)
    z, zl = O.latent_attention(q_lat, qr, np.zeros((0, 512)), np.zeros((0, 64)))
    assert np.all(z == 0) and np.all(np.isneginf(zl))


def test_incremental_decode_equals_full_causal_recompute():
    """The KV-cache experiment ([MD] "KV Cache"): each decode step with a cache of the earlier
    rows gives the same output as the matching row of full causal attention recomputed over
    the whole sequence."""
    rng = np.random.default_rng(13)
    H, D, T = 2, 16, 9
    w = _tiny_weights(rng, H, D)
    for a in ("w_dkv", "w_kr", "w_q"):
        setattr(w, a, getattr(w, a) / math.sqrt(D))
    w.w_uk /= math.sqrt(512)
    w.w_uv /= math.sqrt(512)
    hs = rng.standard_normal((T, D))
    rows = []
    dec = []
    for t in range(T):
        step = O.decode_step(hs[t], w, np.array(rows).reshape(t, 576), pos=t, n_heads=H,
                             with_out=False)
        rows.append(step["row"])
        dec.append(step["o_heads"])
    rows = np.array(rows)
    for h in range(H):
        q = []
        for t in range(T):
            qn, qr = O.query_heads(hs[t], w.w_q, H, 128, 64, pos=t)
            q.append(np.concatenate([qn[h], qr[h]]))
        k_h, v_h = O.head_keys_values(rows[:, :512], rows[:, 512:], w.w_uk, w.w_uv, h, 128, 128)
        full = O.causal_attention(np.array(q), k_h, v_h, 1 / math.sqrt(192))
        for t in range(T):
            np.testing.assert_allclose(full[t], dec[t][h], rtol=1e-11, atol=1e-13)


def test_brute_force_tiny_dimensions():
    """Scalar loops with math.exp on tiny widths (d_c=6, d_R=4, d_nope=4, d_v=3)."""
    rng = np.random.default_rng(14)
    H, n, d_c, d_r, d_n, d_v = 2, 5, 6, 4, 4, 3
    c = rng.standard_normal((n, d_c))
    kr = rng.standard_normal((n, d_r))
    w_uk = rng.standard_normal((H * d_n, d_c))
    w_uv = rng.standard_normal((H * d_v, d_c))
    qn = rng.standard_normal((H, d_n))
    qr = rng.standard_normal((H, d_r))
    scale = 0.37
    r = O.decode_attention(qn, qr, c, kr, w_uk, w_uv, scale=scale)
    for h in range(H):
        scores = []
        for j in range(n):
            s = 0.0
            for i in range(d_n):
                k_ji = sum(w_uk[h * d_n + i][m] * c[j][m] for m in range(d_c))
                s += qn[h][i] * k_ji
            for i in range(d_r):
                s += qr[h][i] * kr[j][i]
            scores.append(s * scale)
        mx = max(scores)
        e = [math.exp(s - mx) for s in scores]
        tot = sum(e)
        for vv in range(d_v):
            o = 0.0
            for j in range(n):
                v_j = sum(w_uv[h * d_v + vv][m] * c[j][m] for m in range(d_c))
                o += e[j] / tot * v_j
            assert r["o_heads"][h][vv] == pytest.approx(o, rel=1e-12, abs=1e-14)
        assert r["lse"][h] == pytest.approx(mx + math.log(tot), rel=1e-13)


def test_causal_mask_hides_future_positions():
    rng = np.random.default_rng(15)
    T = 6
    q, k, v = (rng.standard_normal((T, 8)) for _ in range(3))
    out = O.causal_attention(q, k, v, 0.5)
    v2 = v.copy()
    v2[4:] = 1e6  # rows 4, 5 are in the future of rows 0..3
    k2 = k.copy()
    k2[4:] = -7.0
    out2 = O.causal_attention(q, k2, v2, 0.5)
    np.testing.assert_array_equal(out[:4], out2[:4])
    np.testing.assert_allclose(out[0], v[0], rtol=1e-14)  # row 0 sees only itself


# ---------------------------------------------------------------------------------------------
# Paged layout
# ---------------------------------------------------------------------------------------------

def test_gather_rows_follows_page_table_and_ignores_unused_slots():
    rng = np.random.default_rng(16)
    n = 150  # 2 full pages + 22 rows
    rows = rng.standard_normal((n, 576))
    table = np.array([5, 0, 3])
    pool = np.full((6, 64, 576), 1e30)
    for j in range(n):
        pool[table[j // 64], j % 64] = rows[j]
    assert np.array_equal(O.gather_rows(pool, table, n), rows)
    pool[table[2], 22:] = -5.0  # change every slot past the length
    assert np.array_equal(O.gather_rows(pool, table, n), rows)
    assert O.gather_rows(pool, table, 0).shape == (0, 576)


def test_decode_step_appends_at_position_and_attends_to_itself():
    rng = np.random.default_rng(17)
    H, D = 2, 16
    w = _tiny_weights(rng, H, D)
    h = rng.standard_normal(D)
    step = O.decode_step(h, w, np.zeros((0, 576)), pos=0, n_heads=H)
    # with an empty history the new token sees only itself: o_h = W_UV_h c_new
    c_new = w.w_dkv @ h
    for hh in range(H):
        np.testing.assert_allclose(step["o_heads"][hh], w.w_uv[hh * 128:(hh + 1) * 128] @ c_new,
                                   rtol=1e-12)
    # position 0: the rotary part is unrotated
    np.testing.assert_allclose(step["row"][512:], w.w_kr @ h, rtol=1e-14)
    np.testing.assert_allclose(step["out"], w.w_o @ step["o_heads"].reshape(-1), rtol=1e-13)


# ---------------------------------------------------------------------------------------------
# FP8 (E4M3) weight storage: values the format definition fixes, invariants, brute force
# ---------------------------------------------------------------------------------------------
E4M3_KNOWN = {  # code: value, from the E4M3 definition (bias 7, 3 mantissa bits, max 448)
    0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x38: 1.0,
    0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x77: 240.0, 0x78: 256.0, 0x7E: 448.0,
    0x81: -(2.0 ** -9), 0xB8: -1.0, 0xFE: -448.0,
}


def test_e4m3_decode_known_codes():
    for code, value in E4M3_KNOWN.items():
        assert O.e4m3_decode([code])[0] == value, hex(code)
    assert np.signbit(O.e4m3_decode([0x80])[0]) and O.e4m3_decode([0x80])[0] == 0.0
    assert np.isnan(O.e4m3_decode([0x7F, 0xFF])).all()


def test_e4m3_decode_is_monotone_and_symmetric():
    pos = O.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(pos) > 0)                       # 0 .. 448, strictly increasing
    neg = O.e4m3_decode(np.arange(0x7F) | 0x80)
    assert np.array_equal(neg, -pos)
    # spacing doubles with each exponent step: 8 values per binade above the subnormals
    assert np.allclose(np.diff(pos[8:16]), 2.0 ** -9) and np.allclose(np.diff(pos[16:24]), 2.0 ** -8)


def test_e4m3_quantize_round_trip_ties_and_saturation():
    codes = np.arange(256)
    finite = codes[(codes & 0x7F) != 0x7F]
    assert np.array_equal(O.e4m3_quantize(O.e4m3_decode(finite)), finite.astype(np.uint8))
    # ties go to the code with an even last mantissa bit
    assert O.e4m3_quantize([1.0625])[0] == 0x38 and O.e4m3_quantize([1.1875])[0] == 0x3A
    assert O.e4m3_quantize([-1.0625])[0] == 0xB8
    assert O.e4m3_quantize([2.0 ** -10])[0] == 0x00   # halfway to the smallest subnormal
    assert O.e4m3_quantize([500.0, -1e9])[0] == 0x7E and O.e4m3_quantize([-1e9])[0] == 0xFE


def test_e4m3_quantize_is_nearest_by_brute_force():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 3, 2000), rng.uniform(-450, 450, 2000),
                        rng.uniform(-0.02, 0.02, 2000)])
    grid = O.e4m3_decode(np.arange(256))
    grid = grid[~np.isnan(grid)]
    got = O.e4m3_decode(O.e4m3_quantize(x))
    best = np.abs(x[:, None] - grid[None, :]).min(axis=1)
    assert np.allclose(np.abs(x - np.clip(got, -448, 448)), best, rtol=0, atol=0)


def test_quantize_rows_maps_each_row_max_to_448():
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (5, 300)).astype(np.float32)
    w[3] = 0.0
    codes, s = O.quantize_rows_e4m3(w)
    deq = O.dequantize_rows_e4m3(codes, s)
    for r in (0, 1, 2, 4):
        j = np.argmax(np.abs(w[r]))
        assert abs(O.e4m3_decode([codes[r, j]])[0]) == 448.0
        # every element within half a spacing of its binade (3 mantissa bits: 2^-4 relative)
        assert np.all(np.abs(deq[r] - w[r]) <= 2.0 ** -4 * np.abs(w[r]) + 2.0 ** -10 * s[r])
    assert s[3] == 1.0 and np.all(codes[3] == 0)
