"""mla_decode_attn_static_scratch: decode attention whose split-KV scratch is the library's own
fixed device array, for callers that cannot allocate.  It must give what mla_decode_attn gives
on the same inputs, call after call, although every call reuses (and leaves behind) the same
scratch contents."""
from __future__ import annotations

import pytest
import torch

import mla_inputs as I
from tests.gpu_common import assert_close, dev, to_np

pytestmark = pytest.mark.gpu


def _case(seed, history, n_heads, dtype):
    q = I.query_cat(seed, len(history), n_heads, dtype=dtype)
    cache = I.paged_cache(seed + 1, history, history, dtype=dtype)
    lens = torch.tensor(history, dtype=torch.int32)
    return dev(q), dev(cache.pool), dev(cache.page_table), dev(lens)


def _both(seed, history, n_heads, dtype, num_splits):
    import mla_latent_kv_37_b200 as M
    B = len(history)
    d = M.dims(B, n_heads, dtype=dtype)
    q, pool, table, lens = _case(seed, history, n_heads, dtype)
    ws = M.workspace(d, num_splits)
    o_ref = torch.empty(B, n_heads, 512, dtype=torch.float32, device="cuda")
    l_ref = torch.empty(B, n_heads, dtype=torch.float32, device="cuda")
    M.mla_decode_attn(d, q, pool, table, lens, o_ref, ws, lse=l_ref, num_splits=num_splits)
    # Fill the outputs with garbage so that a slot the static path fails to write shows up.
    o_new = torch.full_like(o_ref, float("nan"))
    l_new = torch.full_like(l_ref, float("nan"))
    M.mla_decode_attn_static_scratch(d, q, pool, table, lens, o_new, lse=l_new,
                                     num_splits=num_splits)
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    return o_ref, l_ref, o_new, l_new


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_workspace_path_two_calls(dtype):
    # Two calls in a row with different shapes and split counts: the second one finds the
    # first one's plan and partials in the shared scratch and must not be affected by them.
    calls = [
        (11, [200, 1, 4097, 64, 0, 1000], 128, 7),
        (23, [65, 3000], 128, 0),
    ]
    for seed, history, n_heads, splits in calls:
        o_ref, l_ref, o_new, l_new = _both(seed, history, n_heads, dtype, splits)
        # An empty sequence has lse = -inf on both paths; no NaN fill may survive.
        assert not torch.isnan(o_new).any() and not torch.isnan(l_new).any()
        assert_close(to_np(o_new), to_np(o_ref), dtype, f"o_lat {history}")
        fin = torch.isfinite(l_ref)
        assert torch.equal(fin, torch.isfinite(l_new))
        assert torch.equal(l_new[~fin], l_ref[~fin])
        assert_close(to_np(l_new[fin]), to_np(l_ref[fin]), dtype, f"lse {history}")


def test_static_scratch_rejects_oversize():
    import mla_latent_kv_37_b200 as M
    B, H = 128, 128  # (B + parts) * H * ~2 KiB of partials is beyond the fixed array
    d = M.dims(B, H)
    q, pool, table, lens = _case(5, [1] * B, H, torch.bfloat16)
    o = torch.empty(B, H, 512, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_attn_static_scratch(d, q, pool, table, lens, o, num_splits=200)
    assert e.value.code == -4  # MLA_ERR_WORKSPACE
    # The rejected call launched nothing; a following call that fits still works.
    o_ref, l_ref, o_new, l_new = _both(31, [300, 129], H, torch.bfloat16, 3)
    assert_close(to_np(o_new), to_np(o_ref), torch.bfloat16, "after rejection")


def test_static_scratch_matches_oracle():
    # The static-scratch call on its own, against the oracle's latent-space attention (not
    # only against the workspace path, which runs the same kernels).
    import mla_latent_kv_37_b200 as M
    from tests.gpu_common import latent_reference
    history = [700, 64, 129, 1]
    B, H = len(history), 128
    q = I.query_cat(41, B, H)
    cache = I.paged_cache(42, history, history)
    d = M.dims(B, H)
    o = torch.full((B, H, 512), float("nan"), dtype=torch.float32, device="cuda")
    M.mla_decode_attn_static_scratch(d, dev(q), dev(cache.pool), dev(cache.page_table),
                                     dev(torch.tensor(history, dtype=torch.int32)), o,
                                     num_splits=5)
    assert M.mla_get_status() == 0
    ref, _ = latent_reference(q, cache, history)
    for b in range(B):
        assert_close(to_np(o[b]), ref[b], torch.bfloat16, f"o_lat b={b}")


def test_static_scratch_near_capacity():
    # 128 sequences x 128 heads split into 127 parts: the plan and partials fill the fixed
    # array to within a fraction of a percent of MLA_STATIC_SCRATCH_BYTES, so its far end is
    # written and read; the result must match the workspace path and leave no NaN behind.
    history = [256] * 128
    o_ref, l_ref, o_new, l_new = _both(61, history, 128, torch.bfloat16, 127)
    assert not torch.isnan(o_new).any() and not torch.isnan(l_new).any()
    assert_close(to_np(o_new), to_np(o_ref), torch.bfloat16, "near capacity")
    assert_close(to_np(l_new), to_np(l_ref), torch.bfloat16, "near capacity lse")
