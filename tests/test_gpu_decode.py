"""Parity of mla_decode_attn (tcgen05 split-KV kernel + combine) against the oracle's latent
space form, on seeded inputs: page-boundary lengths, ragged batches, empty sequences, several
head counts and split counts, masked-slot invariance, long contexts, bad inputs."""
import numpy as np
import pytest
import torch

import mla_inputs as I
from tests.gpu_common import assert_close, dev, errors, latent_reference

pytestmark = pytest.mark.gpu


def _run(q_cat, cache, lens, H, num_splits=0, dtype=torch.bfloat16):
    import mla_latent_kv_37_b200 as M
    B = q_cat.shape[0]
    d = M.dims(B, H, 1024, dtype)
    ws = M.workspace(d, num_splits)
    o_lat = torch.full((B, H, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    M.mla_decode_attn(d, dev(q_cat), dev(cache.pool), dev(cache.page_table),
                      dev(torch.tensor(lens, dtype=torch.int32)), o_lat, ws, lse=lse,
                      num_splits=num_splits)
    st = M.mla_get_status()
    return o_lat.cpu(), lse.cpu(), st


def _case(seed, lens, H, scale=1.0, dtype=torch.bfloat16, sentinel=I.SENTINEL):
    q = I.query_cat(seed, len(lens), H, scale, dtype)
    cache = I.paged_cache(seed + 1, lens, lens, scale, dtype, sentinel=sentinel)
    return q, cache


def _check(q, cache, lens, o_lat, lse, dtype=torch.bfloat16):
    ref_o, ref_l = latent_reference(q, cache, lens)
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o_lat[b] == 0)
            assert torch.all(torch.isneginf(lse[b]))
            continue
        assert_close(o_lat[b].double().numpy(), ref_o[b], dtype, f"o_lat b={b} n={n}")
        np.testing.assert_allclose(lse[b].double().numpy(), ref_l[b], rtol=2e-4, atol=2e-4)


@pytest.mark.parametrize("lens", [[1], [63], [64], [65], [127], [128], [129], [1000],
                                  [5, 64, 200, 3], [0, 70, 0], [4097]])
def test_lengths(lens):
    q, cache = _case(100 + sum(lens), lens, 128)
    o, l, st = _run(q, cache, lens, 128)
    assert st == 0
    _check(q, cache, lens, o, l)


@pytest.mark.parametrize("H", [16, 64, 96, 128])
def test_head_counts(H):
    lens = [300, 65]
    q, cache = _case(7, lens, H)
    o, l, st = _run(q, cache, lens, H)
    assert st == 0
    _check(q, cache, lens, o, l)


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 64, 0])
def test_split_counts_agree(splits):
    lens = [900, 333, 64, 1]
    q, cache = _case(8, lens, 128)
    o, l, st = _run(q, cache, lens, 128, num_splits=splits)
    assert st == 0
    _check(q, cache, lens, o, l)
    o1, l1, _ = _run(q, cache, lens, 128, num_splits=1)
    rel, _ = errors(o.numpy(), o1.numpy())
    assert rel < 5e-3


def test_masked_slots_have_no_influence():
    lens = [70, 129, 1]
    q, c1 = _case(9, lens, 128, sentinel=1e30)
    _, c2 = _case(9, lens, 128, sentinel=-3.0e4)
    o1, l1, _ = _run(q, c1, lens, 128, num_splits=3)
    o2, l2, _ = _run(q, c2, lens, 128, num_splits=3)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_deterministic_at_fixed_split():
    lens = [2000, 513]
    q, cache = _case(10, lens, 128)
    a = _run(q, cache, lens, 128, num_splits=5)
    b = _run(q, cache, lens, 128, num_splits=5)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_batched_paged_uniform_lengths():
    """Batched paged workload: batch 64, lengths uniform in [1024, 8192], random page table."""
    lens = I.uniform_lengths(2, 64, 1024, 8192)
    q, cache = _case(2, lens, 128)
    o, l, st = _run(q, cache, lens, 128)
    assert st == 0
    _check(q, cache, lens, o, l)


@pytest.mark.parametrize("scale", [1.0, 4.0])
def test_long_context(scale):
    """Long-context split-KV: batch 4 x 131072 tokens; inputs x{1,4} make logits ~N(0,16^2)."""
    lens = [131072] * 4
    q, cache = _case(3, lens, 128, scale=scale)
    o, l, st = _run(q, cache, lens, 128)
    assert st == 0
    _check(q, cache, lens, o, l)


def test_headline_shape():
    """The attention of one layer of the full decode step: batch 32 x 32768 tokens, 128 heads,
    the automatic split (every sequence spread over several parts), every sequence checked."""
    lens = [32768] * 32
    q, cache = _case(5, lens, 128)
    o, l, st = _run(q, cache, lens, 128)
    assert st == 0
    _check(q, cache, lens, o, l)


def test_max_batch_long_context_sampled():
    """The largest shape of the attention sweep: batch 128 (the bf16 path's maximum) x 32768
    tokens, 128 heads, the automatic split; inputs made on the device; four sequences (the
    first, the last and two inside) checked on every head against the oracle."""
    import mla_latent_kv_37_b200 as M
    from oracle import mla_oracle as O
    B, N, H = 128, 32768, 128
    lens = [N] * B
    q = I.query_cat(17, B, H, device="cuda")
    cache = I.paged_cache(18, lens, lens, device="cuda")
    d = M.dims(B, H)
    ws = M.workspace(d)
    o = torch.full((B, H, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    M.mla_decode_attn(d, q, cache.pool, cache.page_table, cache.seq_lens, o, ws, lse=lse)
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    for b in (0, 41, 97, 127):
        rows = O.f64(cache.pool[cache.page_table[b].long()].reshape(-1, 576)[:N].cpu())
        qb = O.f64(q[b].cpu())
        o_ref, l_ref = O.latent_attention(qb[:, :512], qb[:, 512:], rows[:, :512],
                                          rows[:, 512:])
        assert_close(o[b].double().cpu().numpy(), o_ref, torch.bfloat16, f"o_lat b={b}")
        np.testing.assert_allclose(lse[b].double().cpu().numpy(), l_ref, rtol=2e-4, atol=2e-4)


def test_fp32_path():
    lens = [256, 100, 1]
    q, cache = _case(11, lens, 16, dtype=torch.float32)
    o, l, st = _run(q, cache, lens, 16, dtype=torch.float32)
    assert st == 0
    _check(q, cache, lens, o, l, dtype=torch.float32)


def test_bad_page_id_sets_status_not_fault():
    import mla_latent_kv_37_b200 as M
    lens = [200, 100]
    q, cache = _case(12, lens, 128)
    cache.page_table[0, 1] = cache.num_pages + 5
    _, _, st = _run(q, cache, lens, 128)
    assert st & M.STATUS_BAD_PAGE


def test_bad_length_sets_status():
    import mla_latent_kv_37_b200 as M
    lens = [100, 50]
    q, cache = _case(13, lens, 128)
    _, _, st = _run(q, cache, [100, 10_000], 128)
    assert st & M.STATUS_BAD_LENGTH


# ---------------------------------------------------------------------------------------------
# Query carried as bf16 hi + lo (q_lo): the scores use ~16 significant bits of the query.
# ---------------------------------------------------------------------------------------------
def _split_query(seed, B, H, scale):
    """An fp32 absorbed query and its bf16 hi/lo split; the oracle gets hi + lo exactly."""
    q = I.query_cat(seed, B, H, scale, torch.float32)
    hi = q.to(torch.bfloat16)
    lo = (q - hi.float()).to(torch.bfloat16)
    exact = hi.double() + lo.double()
    return hi, lo, exact


def _run_lo(hi, lo, cache, lens, H, num_splits=0):
    import mla_latent_kv_37_b200 as M
    B = hi.shape[0]
    d = M.dims(B, H, 1024)
    ws = M.workspace(d, num_splits)
    o_lat = torch.full((B, H, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    M.mla_decode_attn(d, dev(hi), dev(cache.pool), dev(cache.page_table),
                      dev(torch.tensor(lens, dtype=torch.int32)), o_lat, ws, lse=lse,
                      q_lo=dev(lo), num_splits=num_splits)
    st = M.mla_get_status()
    return o_lat.cpu(), lse.cpu(), st


@pytest.mark.parametrize("H,lens,splits", [(128, [5, 64, 200, 3], 0), (96, [300, 65], 0),
                                           (16, [129, 1], 2), (64, [0, 700, 63], 3),
                                           (128, [900, 333, 64, 1], 7)])
def test_query_remainder(H, lens, splits):
    hi, lo, exact = _split_query(40 + H, len(lens), H, 4.0)
    cache = I.paged_cache(41 + H, lens, lens, 4.0)
    o, l, st = _run_lo(hi, lo, cache, lens, H, splits)
    assert st == 0
    _check(exact, cache, lens, o, l)


def test_query_remainder_long_context_scaled():
    """Long context (4 x 131072) at inputs x4 (logit spread ~16): with the remainder the
    attention output is within tolerance of the oracle fed the ~16-bit query."""
    lens = [131072] * 4
    hi, lo, exact = _split_query(3, 4, 128, 4.0)
    cache = I.paged_cache(4, lens, lens, 4.0)
    o, l, st = _run_lo(hi, lo, cache, lens, 128)
    assert st == 0
    _check(exact, cache, lens, o, l)


def test_query_remainder_zero_matches_plain_call():
    """A zero remainder gives the plain call's result to within the split's rounding."""
    lens = [777, 64]
    q, cache = _case(14, lens, 128)
    o1, l1, _ = _run(q, cache, lens, 128, num_splits=4)
    o2, l2, st = _run_lo(q, torch.zeros_like(q), cache, lens, 128, num_splits=4)
    assert st == 0
    rel, _ = errors(o2.numpy(), o1.numpy())
    assert rel < 1e-3
    np.testing.assert_allclose(l2.numpy(), l1.numpy(), rtol=1e-4, atol=1e-4)


def test_timeout_path_reports_and_recovers(monkeypatch):
    """A wait that can only run out (MLA_TEST_STALL: one warp of every CTA waits on a barrier
    nothing arrives on, with a 20 ms limit): the call reports MLA_STATUS_TIMEOUT instead of
    hanging, the other roles unwind, and the next ordinary call, in the same context, is
    correct."""
    import mla_latent_kv_37_b200 as M
    lens = [4096, 1000, 64]
    q, cache = _case(15, lens, 128)
    monkeypatch.setenv("MLA_TEST_STALL", "1")
    monkeypatch.setenv("MLA_WAIT_NS", "20000000")
    _, _, st = _run(q, cache, lens, 128)
    assert st & M.STATUS_TIMEOUT
    monkeypatch.delenv("MLA_TEST_STALL")
    monkeypatch.delenv("MLA_WAIT_NS")
    o, l, st = _run(q, cache, lens, 128)
    assert st == 0
    _check(q, cache, lens, o, l)


@pytest.mark.parametrize("splits", [1, 5, 0, 200, 1000])
def test_plan_many_short_and_empty_sequences(splits):
    """The planner's cost model (each sequence start weighs as a few pages) on a hard mix: 128
    sequences of 0 to 700 tokens (a quarter empty, many under one page), split into 1 to 1000
    parts, so that parts begin inside sequences' start-up, some parts stay empty and most
    sequences are cut several times; every sequence against the oracle."""
    import random
    rnd = random.Random(splits + 17)
    lens = [0 if rnd.random() < 0.25 else rnd.choice([1, 2, 63, 64, 65, rnd.randint(1, 700)])
            for _ in range(128)]
    q, cache = _case(300 + splits, lens, 128)
    o, l, st = _run(q, cache, lens, 128, num_splits=splits)
    assert st == 0
    _check(q, cache, lens, o, l)


def test_plan_many_parts_fp32():
    """The fp32 path's planner with more parts than pages in some sequences."""
    lens = [1, 0, 130, 64, 65, 300, 2, 0]
    q, cache = _case(23, lens, 16, dtype=torch.float32)
    o, l, st = _run(q, cache, lens, 16, num_splits=37, dtype=torch.float32)
    assert st == 0
    _check(q, cache, lens, o, l, dtype=torch.float32)
