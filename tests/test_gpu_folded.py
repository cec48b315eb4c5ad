"""The folded execution mode -- W_UK multiplied into W_Q and W_UV into W_O once, ahead of time --
against the oracle's non-absorbed fp64 step: the same cache rows as the absorbed path, the
query and the layer output within the bf16 tolerance, and the folded weights themselves."""
import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from tests.gpu_common import Workload, assert_close, dev, to_np

pytestmark = pytest.mark.gpu


def _folded_step(wl: Workload, num_splits=0):
    import mla_latent_kv_37_b200 as M
    B, H, D = wl.B, wl.H, wl.D
    d = M.dims(B, H, D)
    sq, so = M.fold_shapes(d)
    w = wl.w
    w_qf = torch.empty(sq, dtype=torch.bfloat16, device="cuda")
    w_of = torch.empty(so, dtype=torch.bfloat16, device="cuda")
    M.mla_fold_weights(d, w_q=dev(w.w_q), w_uk=dev(w.w_uk), w_uv=dev(w.w_uv), w_o=dev(w.w_o),
                       w_qf=w_qf, w_of=w_of)
    ws = M.workspace(d, num_splits)
    pool = dev(wl.cache.pool)
    table = dev(wl.cache.page_table)
    q_cat = torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
    o_lat = torch.empty(B, H, 512, dtype=torch.float32, device="cuda")
    out = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")
    M.mla_append_absorb_folded(d, dev(wl.h), dev(w.w_dkv), dev(w.w_kr), w_qf, dev(wl.pos), table,
                               pool, q_cat, ws)
    M.mla_decode_attn(d, q_cat, pool, table, dev(wl.lens), o_lat, ws, num_splits=num_splits)
    M.mla_out_proj_folded(d, o_lat, w_of, out, ws)
    torch.cuda.synchronize()
    return dict(pool=pool.cpu(), q_cat=q_cat.cpu(), out=out.cpu(), w_qf=w_qf.cpu(),
                w_of=w_of.cpu(), status=M.mla_get_status())


@pytest.mark.parametrize("B,H,D,hist", [(3, 16, 1024, [100, 1, 300]),
                                        (2, 128, 7168, [64, 500])])
def test_folded_step_matches_oracle(B, H, D, hist):
    wl = Workload(70 + B, B, H, D, hist)
    got = _folded_step(wl)
    assert got["status"] == 0
    # the cache append: the appended rows match the oracle's; every other pool byte is the
    # input's (the same product as the absorbed path, but its fp32 sums may be split over
    # other CTAs, so its rows are compared within the tolerance, not bit for bit)
    pool_in = wl.cache.pool.clone()
    w_uk = O.f64(wl.w.w_uk)
    for b in range(B):
        page = int(wl.cache.page_table[b, wl.history[b] // 64])
        slot = wl.history[b] % 64
        c_kv, k_r = O.latent_row(wl.h[b], wl.w.w_dkv, wl.w.w_kr, wl.history[b])
        row = to_np(got["pool"][page, slot])
        assert_close(row[:512], c_kv, torch.bfloat16, f"appended c_KV b={b}")
        assert_close(row[512:], k_r, torch.bfloat16, f"appended k_R b={b}")
        pool_in[page, slot] = got["pool"][page, slot]
    assert torch.equal(got["pool"], pool_in)
    for b in range(B):
        qn, qr = O.query_heads(wl.h[b], wl.w.w_q, H, 128, 64, wl.history[b])
        q_lat = np.stack([w_uk[h * 128:(h + 1) * 128].T @ qn[h] for h in range(H)])
        assert_close(to_np(got["q_cat"][b, :, :512]), q_lat, torch.bfloat16, f"q_lat b={b}")
        assert_close(to_np(got["q_cat"][b, :, 512:]), qr, torch.bfloat16, f"q_rope b={b}")
        ref = wl.oracle(b)
        assert_close(to_np(got["out"][b]), ref["out"], torch.bfloat16, f"out b={b}")


def test_folded_weights():
    """The folded matrices: RoPE rows copied bit for bit; sampled latent rows and output columns
    against the fp64 products of the bf16 weights, within one bf16 rounding."""
    H, D = 16, 1024
    wl = Workload(91, 1, H, D, [3])
    got = _folded_step(wl)
    w = wl.w
    wq = w.w_q.view(H, 192, D)
    assert torch.equal(got["w_qf"][:, 512:], wq[:, 128:])
    uk, q64 = O.f64(w.w_uk), O.f64(w.w_q)
    uv, o64 = O.f64(w.w_uv), O.f64(w.w_o)
    rng = np.random.default_rng(5)
    for h in rng.choice(H, 4, replace=False):
        ms = rng.choice(512, 8, replace=False)
        exp = uk[h * 128:(h + 1) * 128, ms].T @ q64[h * 192:h * 192 + 128]
        gotq = to_np(got["w_qf"][h, ms])
        assert np.abs(gotq - exp).max() <= 2.0 ** -8 * np.abs(exp).max()
        exp_o = o64[:, h * 128:(h + 1) * 128] @ uv[h * 128:(h + 1) * 128][:, ms]
        goto = to_np(got["w_of"][:, h * 512 + ms])
        assert np.abs(goto - exp_o).max() <= 2.0 ** -8 * np.abs(exp_o).max()
