"""End-to-end parity of one decode step (mla_cache_append -> mla_absorb_q -> mla_decode_attn
-> mla_out_proj) against the oracle's reconstructed (non-absorbed) attention in fp64, plus the
bit-exact paging properties of mla_cache_append."""
import numpy as np
import pytest
import torch

import mla_inputs as I
from oracle import mla_oracle as O
from tests.gpu_common import Workload, assert_close, dev, to_np

pytestmark = pytest.mark.gpu


def _check_step(wl: Workload, got, seqs, heads=None, check_out=True):
    for b in seqs:
        ref = wl.oracle(b, heads=heads, with_out=check_out and heads is None)
        hsel = list(range(wl.H)) if heads is None else list(heads)
        assert_close(to_np(got["o_heads"][b][hsel]), ref["o_heads"], wl.dtype, f"o_heads b={b}")
        if check_out and heads is None:
            assert_close(to_np(got["out"][b]), ref["out"], wl.dtype, f"out b={b}")


def test_tiny_fp32():
    """batch 1, 16 heads, d_model 1024, context 256, fp32, seed 0."""
    wl = Workload(0, 1, 16, 1024, [255], dtype=torch.float32, shuffle=False)
    got = wl.run_gpu()
    assert got["status"] == 0
    _check_step(wl, got, [0])
    ref = wl.oracle(0)
    np.testing.assert_allclose(to_np(got["o_lat"][0]), ref["o_lat"], rtol=1e-5, atol=1e-6)


def test_single_layer_v3_shapes():
    """batch 1, 128 heads, d_model 7168, context 4096 contiguous, bf16."""
    wl = Workload(1, 1, 128, 7168, [4095], shuffle=False)
    got = wl.run_gpu()
    assert got["status"] == 0
    _check_step(wl, got, [0])


@pytest.mark.parametrize("hist", [[0], [63, 64, 1], [100, 7, 200, 64]])
def test_small_batches_paged(hist):
    wl = Workload(20 + len(hist), len(hist), 128, 1024, hist)
    got = wl.run_gpu()
    assert got["status"] == 0
    _check_step(wl, got, range(len(hist)))


@pytest.mark.parametrize("H", [16, 64])
def test_fewer_heads(H):
    wl = Workload(30, 3, H, 512, [90, 1, 300])
    got = wl.run_gpu()
    assert got["status"] == 0
    _check_step(wl, got, range(3))


def test_batched_paged_v3_shapes_sampled():
    """batch 64, lengths uniform in [1024, 8192], d_model 7168: two sequences checked on every
    output, eight more on a sample of heads."""
    lens = I.uniform_lengths(2, 64, 1024, 8192)
    wl = Workload(2, 64, 128, 7168, [n - 1 for n in lens])
    got = wl.run_gpu()
    assert got["status"] == 0
    _check_step(wl, got, [0, 37])
    rng = np.random.default_rng(5)
    for b in rng.choice(64, 8, replace=False):
        _check_step(wl, got, [int(b)], heads=sorted(rng.choice(128, 8, replace=False).tolist()))


def test_append_rows_match_oracle_and_touch_one_slot():
    wl = Workload(40, 4, 128, 7168, [0, 63, 64, 1000])
    before = wl.cache.pool.clone()
    got = wl.run_gpu(want_out=False)
    pool = got["pool"]
    changed = (pool.view(pool.shape[0], 64, -1) != before.view(pool.shape[0], 64, -1)).any(-1)
    for b, pos in enumerate(wl.history):
        page = int(wl.cache.page_table[b, pos // 64])
        row = pool[page, pos % 64]
        c, k = O.latent_row(wl.h[b], wl.w.w_dkv, wl.w.w_kr, pos)
        exp = np.concatenate([c, k])
        exp_bf16 = torch.from_numpy(exp.astype(np.float32)).to(torch.bfloat16)
        # rounding of an fp32-accumulated value may land one bf16 step away from the rounding
        # of the exact value; everything else is identical
        diff = (row.view(torch.int16).int() - exp_bf16.view(torch.int16).int()).abs()
        assert int(diff.max()) <= 1 and float((diff == 0).float().mean()) > 0.95
        changed[page, pos % 64] = False
    assert not changed.any(), "append wrote outside the addressed slots"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_append_scatter_is_bit_exact(dtype):
    import mla_latent_kv_37_b200 as M
    B = 5
    cache = I.paged_cache(50, [200] * B, [10, 64, 130, 0, 199], dtype=dtype)
    rows = I.hidden(51, B, 576, 3.0, dtype)
    pos = torch.tensor([10, 64, 130, 0, 199], dtype=torch.int32)
    d = M.dims(B, 128, 1024, dtype)
    pool = dev(cache.pool)
    M.mla_cache_append(d, dev(rows), None, None, dev(pos), dev(cache.page_table), pool)
    assert M.mla_get_status() == 0
    exp = cache.pool.clone()
    for b in range(B):
        exp[int(cache.page_table[b, pos[b] // 64]), int(pos[b]) % 64] = rows[b]
    assert torch.equal(pool.cpu(), exp)


def test_append_bad_position_is_reported():
    import mla_latent_kv_37_b200 as M
    cache = I.paged_cache(52, [64], [3])
    d = M.dims(1, 128, 1024)
    pool = dev(cache.pool)
    M.mla_cache_append(d, dev(I.hidden(53, 1, 576)), None, None,
                       dev(torch.tensor([64], dtype=torch.int32)), dev(cache.page_table), pool)
    assert M.mla_get_status() & M.STATUS_BAD_POSITION
    assert torch.equal(pool.cpu(), cache.pool)


def test_absorbed_query_matches_oracle_projection():
    wl = Workload(60, 3, 128, 7168, [5, 6, 7])
    got = wl.run_gpu(want_out=False)
    for b in range(3):
        qn, qr = O.query_heads(wl.h[b], wl.w.w_q, 128, 128, 64, wl.history[b])
        w_uk = O.f64(wl.w.w_uk)
        q_lat = np.stack([w_uk[h * 128:(h + 1) * 128].T @ qn[h] for h in range(128)])
        assert_close(to_np(got["q_cat"][b, :, :512]), q_lat, torch.bfloat16, "q_lat")
        assert_close(to_np(got["q_cat"][b, :, 512:]), qr, torch.bfloat16, "q_rope")


@pytest.mark.parametrize("dtype,B,H,D", [(torch.bfloat16, 32, 128, 7168),
                                         (torch.bfloat16, 5, 16, 1024),
                                         (torch.bfloat16, 1, 64, 512),
                                         (torch.float32, 3, 16, 1024)])
def test_append_absorb_matches_the_two_calls(dtype, B, H, D):
    """mla_append_absorb (one shared projection launch) gives what mla_cache_append followed
    by mla_absorb_q give: the same cache rows and absorbed queries within the tolerance (the
    fp32 sums are split differently), every other pool byte untouched."""
    import mla_latent_kv_37_b200 as M
    hist = [(37 * i + 5) % 300 for i in range(B)]
    wl = Workload(40 + B, B, H, D, hist, dtype=dtype)
    d = M.dims(B, H, D, dtype)
    w = wl.w
    args = dict(h=dev(wl.h), pos=dev(wl.pos), table=dev(wl.cache.page_table))
    outs = []
    for fused in (False, True):
        pool = dev(wl.cache.pool)
        q = torch.empty(B, H, 576, dtype=dtype, device="cuda")
        ws = M.workspace(d)
        if fused:
            M.mla_append_absorb(d, args["h"], dev(w.w_dkv), dev(w.w_kr), dev(w.w_q), dev(w.w_uk),
                                args["pos"], args["table"], pool, q, ws)
        else:
            M.mla_cache_append(d, args["h"], dev(w.w_dkv), dev(w.w_kr), args["pos"],
                               args["table"], pool, ws)
            M.mla_absorb_q(d, args["h"], dev(w.w_q), dev(w.w_uk), args["pos"], q, ws)
        torch.cuda.synchronize()
        assert M.mla_get_status() == 0
        outs.append((pool.cpu(), q.cpu()))
    (p0, q0), (p1, q1) = outs
    assert_close(to_np(q1), to_np(q0), dtype, "q_cat")
    changed = (p0 != wl.cache.pool).any(dim=-1) | (p1 != wl.cache.pool).any(dim=-1)
    rows0, rows1 = p0[changed], p1[changed]
    assert changed.sum().item() == B  # one slot per sequence
    assert_close(to_np(rows1), to_np(rows0), dtype, "appended rows")
    assert torch.equal(p1[~changed], wl.cache.pool[~changed])


@pytest.mark.parametrize("B", [128, 100])
def test_max_and_ragged_batch(B):
    """The largest batch the bf16 path takes (128: the hi/lo products run the tensor core at
    N = 256) and a batch that is not a multiple of 16 (100 -> N padded to 112 / 224), against
    the oracle on sampled sequences; 16 heads and d_model 1024 keep the oracle quick."""
    hist = [(53 * i + 11) % 257 for i in range(B)]
    wl = Workload(70 + B, B, 16, 1024, hist)
    got = wl.run_gpu()
    assert got["status"] == 0
    _check_step(wl, got, [0, B // 2, B - 1])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_append_rope_at_position_131071(dtype):
    """The appended row at the largest position of the long-context workload (angles up to
    ~1.3e5 rad): the rotary part is checked against the oracle's fp64 RoPE on both arithmetic
    paths (fp32 at 1e-5, bf16 within the row's rounding).  Only the addressed page exists: the
    page table maps page index 2047 to pool page 0."""
    import mla_latent_kv_37_b200 as M
    B, D, pos = 1, 1024, 131071
    w = I.weights(50, 16, D, dtype, with_w_o=False)
    h = I.hidden(51, B, D, 1.0, dtype)
    table = torch.full((B, 2048), -1, dtype=torch.int32)
    table[0, pos // 64] = 0
    pool = torch.zeros(1, 64, 576, dtype=dtype)
    d = M.dims(B, 16, D, dtype)
    ws = M.workspace(d)
    pool_d = dev(pool)
    M.mla_cache_append(d, dev(h), dev(w.w_dkv), dev(w.w_kr), dev(torch.tensor([pos], dtype=torch.int32)),
                       dev(table), pool_d, ws)
    assert M.mla_get_status() == 0
    got = to_np(pool_d.cpu()[0, pos % 64])
    c_kv, k_r = O.latent_row(h[0], w.w_dkv, w.w_kr, pos)
    exp = np.concatenate([c_kv, k_r])
    if dtype == torch.float32:
        np.testing.assert_allclose(got, exp, rtol=1e-5, atol=1e-5 * np.abs(exp).max())
    else:
        # bf16 storage: within one rounding (2^-8 relative) of the exact value
        assert np.all(np.abs(got - exp) <= 2.0 ** -8 * np.abs(exp) + 1e-5)
