"""Split-KV across GPUs, device side, with the ranks emulated in one process: every rank's
mla_decode_attn over its own pages (a page table holding only its share of each sequence),
the parts stacked as the all-gather would deliver them, mla_merge_partials; the merged result
is compared with the oracle over all the rows and with the one-GPU call."""
import numpy as np
import pytest
import torch

import mla_inputs as I
from mla_latent_kv_37_b200.splitkv import local_view
from tests.gpu_common import _check_all, dev, errors, latent_reference

pytestmark = pytest.mark.gpu


def _rank_inputs(cache, lens, world, rank):
    B = len(lens)
    views = [local_view(cache.page_table[b], lens[b], world, rank) for b in range(B)]
    width = max(1, max(len(v[0]) for v in views))
    table = torch.full((B, width), -1, dtype=torch.int32)
    for b, (pages, _) in enumerate(views):
        table[b, :len(pages)] = pages
    return table, torch.tensor([n for _, n in views], dtype=torch.int32)


@pytest.mark.parametrize("world", [2, 3])
def test_split_kv_over_emulated_ranks(world):
    import mla_latent_kv_37_b200 as M
    lens = [5000, 300, 64, 1]
    B, H = len(lens), 128
    q = I.query_cat(80, B, H, 4.0, torch.float32)
    hi = q.to(torch.bfloat16)
    lo = (q - hi.float()).to(torch.bfloat16)
    cache = I.paged_cache(81, lens, lens, 4.0)
    d = M.dims(B, H, 1024)
    pool = dev(cache.pool)
    ws = M.workspace(d)
    o_parts = torch.empty(world, B, H, 512, dtype=torch.float32, device="cuda")
    l_parts = torch.empty(world, B, H, dtype=torch.float32, device="cuda")
    for r in range(world):
        table, n = _rank_inputs(cache, lens, world, r)
        M.mla_decode_attn(d, dev(hi), pool, dev(table), dev(n), o_parts[r], ws, lse=l_parts[r],
                          q_lo=dev(lo))
    o = torch.full((B, H, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    M.mla_merge_partials(d, o_parts, l_parts, o, lse)
    assert M.mla_get_status() == 0
    exact = hi.double() + lo.double()
    _check_all(exact, cache, lens, o.cpu(), lse.cpu())
    # the same as one GPU attending over every page
    o1 = torch.empty_like(o)
    M.mla_decode_attn(d, dev(hi), pool, dev(cache.page_table), dev(torch.tensor(lens, dtype=torch.int32)),
                      o1, ws, q_lo=dev(lo))
    rel, _ = errors(o.cpu().numpy(), o1.cpu().numpy())
    assert rel < 1e-3


def test_merge_of_empty_parts():
    import mla_latent_kv_37_b200 as M
    B, H = 2, 16
    d = M.dims(B, H, 1024)
    o_parts = torch.randn(3, B, H, 512, device="cuda")
    l_parts = torch.full((3, B, H), float("-inf"), device="cuda")
    l_parts[1, 0] = 0.5  # sequence 0 has rows in part 1 only; sequence 1 in none
    o = torch.full((B, H, 512), float("nan"), device="cuda")
    lse = torch.full((B, H), float("nan"), device="cuda")
    M.mla_merge_partials(d, o_parts, l_parts, o, lse)
    torch.cuda.synchronize()
    assert torch.equal(o[0], o_parts[1, 0]) and torch.all(lse[0] == 0.5)
    assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1]))
