"""Split-KV across ranks, host side: the page partition, and two gloo ranks that each attend
over their share of a sequence (the oracle stands in for the GPU kernel here) and gather the
parts with the library's plumbing; the merged result equals the oracle over all the rows."""
import math
import os
import socket

import numpy as np
import pytest
import torch

from mla_latent_kv_37_b200.splitkv import gather_partials, local_view, partition_tokens


@pytest.mark.parametrize("n,world", [(0, 2), (1, 2), (63, 3), (64, 2), (65, 2), (1000, 3),
                                     (131072, 8), (200, 8)])
def test_partition_covers_whole_pages(n, world):
    parts = partition_tokens(n, world)
    assert len(parts) == world
    assert parts[0][0] == 0 and parts[-1][1] == n
    for (b0, e0), (b1, e1) in zip(parts, parts[1:]):
        assert e0 == b1  # contiguous, disjoint
    for b, e in parts:
        assert b <= e and b % 64 == 0
        assert e % 64 == 0 or e == n  # only the last non-empty part ends mid-page
    sizes = [math.ceil(e / 64) - b // 64 for b, e in parts]
    assert max(sizes) - min(sizes) <= 1  # the page count is divided evenly


def test_local_view_pages():
    row = torch.arange(100, 120, dtype=torch.int32)  # a sequence's 20 page ids
    pages, n = local_view(row, 1250, 3, 1)  # 20 pages: ranks get 6, 7, 7
    assert n == 7 * 64 and pages.tolist() == list(range(106, 113))
    pages, n = local_view(row, 1250, 3, 2)
    assert n == 1250 - 13 * 64 and pages.tolist() == list(range(113, 120))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, n, out_path):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import mla_inputs as I
        from oracle import mla_oracle as O
        H = 16
        q = I.query_cat(70, 1, H, 4.0, torch.float32)[0]
        rows = O.f64(torch.randn(n, 576, generator=I.generator(71), dtype=torch.float32) * 2.0)
        b, e = partition_tokens(n, world)[rank]
        o, lse = O.latent_attention(O.f64(q)[:, :512], O.f64(q)[:, 512:], rows[b:e, :512],
                                    rows[b:e, 512:])
        o_all, l_all = gather_partials(torch.from_numpy(o), torch.from_numpy(lse))
        if rank == 0:
            # log-sum-exp merge of the gathered parts (reference arithmetic, test side)
            L = l_all.numpy()
            m = L.max(axis=0)
            w = np.exp(L - m)
            merged = (w[:, :, None] * o_all.numpy()).sum(axis=0) / w.sum(axis=0)[:, None]
            ref, ref_l = O.latent_attention(O.f64(q)[:, :512], O.f64(q)[:, 512:], rows[:, :512],
                                            rows[:, 512:])
            err = float(np.abs(merged - ref).max() / np.abs(ref).max())
            lerr = float(np.abs(m + np.log(w.sum(axis=0)) - ref_l).max())
            with open(out_path, "w") as f:
                f.write(f"{err} {lerr} {o_all.shape[0]}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n", [1000, 130])
def test_two_gloo_ranks_merge_to_full_attention(tmp_path, n):
    import torch.multiprocessing as mp
    out = tmp_path / "res.txt"
    mp.start_processes(_rank_main, args=(2, _free_port(), n, str(out)), nprocs=2, join=True,
                       start_method="spawn")
    err, lerr, parts = out.read_text().split()
    assert int(parts) == 2
    assert float(err) < 1e-12 and float(lerr) < 1e-10
