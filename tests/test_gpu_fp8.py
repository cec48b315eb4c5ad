"""E4M3 (FP8) weights: the GPU quantization against the oracle's (codes and scales bit for
bit), and the output projection with W_O stored as E4M3 (tcgen05 kind::f8f6f4, o_heads as three
scaled E4M3 planes) against the oracle's fp64 step computed with the weights the codes stand
for."""
import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
import mla_inputs as I
from tests.gpu_common import Workload, assert_close, dev, to_np

pytestmark = pytest.mark.gpu


def untile(codes, rows, cols):
    """Codes in 128 x 128 tiles (row tile, then column tile; row-major inside) -> [rows][cols]."""
    rt = codes.numel() // (128 * cols)
    t = codes.reshape(rt, cols // 128, 128, 128).permute(0, 2, 1, 3).reshape(rt * 128, cols)
    return t[:rows].numpy()


def tiled_rows(rows):
    return (rows + 127) // 128 * 128


@pytest.mark.parametrize("rows,cols,std", [(300, 1024, 0.02), (7, 16384, 1.0), (129, 128, 3e-3)])
def test_quantize_matches_oracle_bit_for_bit(rows, cols, std):
    import mla_latent_kv_37_b200 as M
    g = torch.Generator().manual_seed(rows + cols)
    w = (torch.randn(rows, cols, generator=g) * std).to(torch.bfloat16)
    w[1, :] = 0.0                      # a zero row: scale 1, all codes 0
    w[0, 5] = 1e-30                    # far below the smallest step of its row: a zero code
    codes = torch.empty(tiled_rows(rows), cols, dtype=torch.uint8, device="cuda")
    scale = torch.empty(rows, dtype=torch.float32, device="cuda")
    M.mla_quantize_weights_fp8(dev(w), codes, scale)
    torch.cuda.synchronize()
    exp_codes, exp_scale = O.quantize_rows_e4m3(w.float().numpy())
    assert np.array_equal(scale.cpu().numpy(), exp_scale)
    assert np.array_equal(untile(codes.cpu(), rows, cols), exp_codes)


@pytest.mark.parametrize("B,H,D", [(3, 16, 1024), (32, 128, 7168), (33, 16, 1024),
                                   (64, 32, 512), (128, 16, 1024)])
def test_out_proj_fp8_matches_oracle(B, H, D):
    import mla_latent_kv_37_b200 as M
    hist = [(41 * i + 3) % 200 for i in range(B)]
    wl = Workload(80 + B, B, H, D, hist)
    d = M.dims(B, H, D)
    codes = torch.empty(D, H * 128, dtype=torch.uint8, device="cuda")
    scale = torch.empty(D, dtype=torch.float32, device="cuda")
    M.mla_quantize_weights_fp8(dev(wl.w.w_o), codes, scale)
    ws = M.workspace(d)
    q_cat = torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
    pool, table = dev(wl.cache.pool), dev(wl.cache.page_table)
    o_lat = torch.empty(B, H, 512, dtype=torch.float32, device="cuda")
    w = wl.w
    M.mla_append_absorb(d, dev(wl.h), dev(w.w_dkv), dev(w.w_kr), dev(w.w_q), dev(w.w_uk),
                        dev(wl.pos), table, pool, q_cat, ws)
    M.mla_decode_attn(d, q_cat, pool, table, dev(wl.lens), o_lat, ws)
    out = torch.full((B, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    o_heads = torch.empty(B, H, 128, dtype=torch.bfloat16, device="cuda")
    M.mla_out_proj_fp8(d, o_lat, dev(w.w_uv), codes, scale, out, ws, o_heads=o_heads)
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    w_o_deq = O.dequantize_rows_e4m3(untile(codes.cpu(), D, H * 128), scale.cpu().numpy())
    for b in sorted({0, B // 2, B - 1}):
        ref = wl.oracle(b)  # o_heads from the bf16 W_UV; out recomputed with the E4M3 W_O
        assert_close(to_np(o_heads[b].cpu()), ref["o_heads"], torch.bfloat16, f"o_heads b={b}")
        exp = O.output_projection(ref["o_heads"], w_o_deq)
        assert_close(to_np(out[b].cpu()), exp, torch.bfloat16, f"out b={b}")


def test_out_proj_fp8_rejects_large_batch():
    """Batch 129: above the bf16 path's 128 (two E4M3 planes of round16(129) = 144 columns would
    exceed the MMA's 256)."""
    import mla_latent_kv_37_b200 as M
    d = M.dims(129, 16, 1024)
    with pytest.raises(M.MlaError) as e:
        M.mla_out_proj_fp8(d, torch.empty(129, 16, 512, device="cuda"),
                           torch.empty(16 * 128, 512, dtype=torch.bfloat16, device="cuda"),
                           torch.empty(1024, 16 * 128, dtype=torch.uint8, device="cuda"),
                           torch.empty(1024, device="cuda"),
                           torch.empty(129, 1024, dtype=torch.bfloat16, device="cuda"),
                           M.workspace(d))
    assert e.value.code == -2


def _quantize(M, w):
    """E4M3 codes and scales of a bf16 matrix on the GPU, and the weights they stand for."""
    rows, cols = w.shape
    codes = torch.empty(tiled_rows(rows), cols, dtype=torch.uint8, device="cuda")
    scale = torch.empty(rows, dtype=torch.float32, device="cuda")
    M.mla_quantize_weights_fp8(dev(w), codes, scale)
    torch.cuda.synchronize()
    deq = O.dequantize_rows_e4m3(untile(codes.cpu(), rows, cols), scale.cpu().numpy())
    return (codes, scale), deq


@pytest.mark.parametrize("B,H,D,scale", [(32, 128, 7168, 1.0), (5, 16, 1024, 4.0),
                                         (33, 32, 512, 1.0), (128, 16, 1024, 1.0)])
def test_append_absorb_fp8_matches_oracle(B, H, D, scale):
    """Cache append + absorbed query with W_DKV, W_KR and W_Q stored as E4M3: the appended cache
    rows and q_cat against the oracle's fp64 projections with the weights the codes stand for
    (the hidden states enter exactly as two E4M3 planes); every other pool byte untouched."""
    import mla_latent_kv_37_b200 as M
    hist = [(53 * i + 7) % 300 for i in range(B)]
    wl = Workload(90 + B, B, H, D, hist, scale=scale)
    w = wl.w
    dkv, dkv_deq = _quantize(M, w.w_dkv)
    kr, kr_deq = _quantize(M, w.w_kr)
    wq, wq_deq = _quantize(M, w.w_q)
    d = M.dims(B, H, D)
    pool = dev(wl.cache.pool)
    before = wl.cache.pool.clone()
    q_cat = torch.full((B, H, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    q_lo = torch.full((B, H, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.mla_append_absorb_fp8(d, dev(wl.h), dkv, kr, wq, dev(w.w_uk), dev(wl.pos),
                            dev(wl.cache.page_table), pool, q_cat, M.workspace(d), q_lo=q_lo)
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    pool, q_cat, q_lo = pool.cpu(), q_cat.cpu(), q_lo.cpu()
    changed = (pool.view(pool.shape[0], 64, -1) != before.view(pool.shape[0], 64, -1)).any(-1)
    w_uk = O.f64(w.w_uk)
    for b, pos in enumerate(wl.history):
        page = int(wl.cache.page_table[b, pos // 64])
        c, k = O.latent_row(wl.h[b], dkv_deq, kr_deq, pos)
        assert_close(to_np(pool[page, pos % 64]), np.concatenate([c, k]), torch.bfloat16,
                     f"cache row b={b}")
        changed[page, pos % 64] = False
        if b in (0, B // 2, B - 1):
            qn, qr = O.query_heads(wl.h[b], wq_deq, H, 128, 64, pos)
            q_lat = np.stack([w_uk[i * 128:(i + 1) * 128].T @ qn[i] for i in range(H)])
            assert_close(to_np(q_cat[b, :, :512]), q_lat, torch.bfloat16, f"q_lat b={b}")
            assert_close(to_np(q_cat[b, :, 512:]), qr, torch.bfloat16, f"q_rope b={b}")
            # with the rounding remainder the query carries ~16 significant bits
            exact = to_np(q_cat[b]) + to_np(q_lo[b])
            rel = np.linalg.norm(exact[:, :512] - q_lat) / np.linalg.norm(q_lat)
            assert rel < 1e-4, f"q_lat + q_lo b={b}: {rel:.2e}"
    assert not changed.any(), "append wrote outside the addressed slots"


def test_append_absorb_fp8_rejects_large_batch():
    import mla_latent_kv_37_b200 as M
    B, H, D = 129, 16, 1024
    d = M.dims(B, H, D)

    def pair(rows):
        return (torch.empty(*M.fp8_codes_shape(rows, D), dtype=torch.uint8, device="cuda"),
                torch.empty(rows, device="cuda"))
    cache = I.paged_cache(3, [8] * B, [0] * B)
    with pytest.raises(M.MlaError) as e:
        M.mla_append_absorb_fp8(d, torch.empty(B, D, dtype=torch.bfloat16, device="cuda"),
                                pair(512), pair(64), pair(H * 192),
                                torch.empty(H * 128, 512, dtype=torch.bfloat16, device="cuda"),
                                torch.zeros(B, dtype=torch.int32, device="cuda"),
                                dev(cache.page_table), dev(cache.pool),
                                torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda"),
                                M.workspace(d))
    assert e.value.code == -2


def test_e4m3_step_matches_the_oracle():
    """A two-layer decode step (graph replay) with every layer's W_DKV, W_KR, W_Q and W_O stored as
    E4M3 (step.quantize_layer): each layer's o_heads and out against the oracle's non-absorbed
    fp64 step run with the weights the codes stand for."""
    import mla_latent_kv_37_b200 as M
    from mla_latent_kv_37_b200.step import DecodeStep, Layer, quantize_layer
    B, H, D = 4, 128, 1024
    hist = [100, 0, 700, 64]
    wls = [Workload(70 + 10 * l, B, H, D, hist) for l in range(2)]
    layers = [quantize_layer(Layer(dev(wl.w.w_dkv), dev(wl.w.w_kr), dev(wl.w.w_q),
                                   dev(wl.w.w_uk), dev(wl.w.w_uv), dev(wl.w.w_o),
                                   dev(wl.cache.pool), dev(wl.cache.page_table)))
              for wl in wls]
    step = DecodeStep(layers, B, H, D, graph=True)
    h = torch.stack([dev(wl.h) for wl in wls])
    for _ in range(2):
        step.run(h, dev(wls[0].pos), dev(wls[0].lens))
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    for l, (wl, ly) in enumerate(zip(wls, layers)):
        w = I.Weights(*[O.dequantize_rows_e4m3(
            M.fp8_codes_rows(ly.e4m3[n][0], *getattr(ly, n).shape).cpu().numpy(),
            ly.e4m3[n][1].cpu().numpy()) if n in ly.e4m3 else getattr(wl.w, n)
            for n in ("w_dkv", "w_kr", "w_q", "w_uk", "w_uv", "w_o")])
        for b in range(B):
            rows = O.gather_rows(wl.cache.pool, wl.cache.page_table[b].numpy(), hist[b])
            ref = O.decode_step(wl.h[b], w, rows, hist[b], H,
                                round_row=lambda r: torch.from_numpy(
                                    np.asarray(r, dtype=np.float32)).to(torch.bfloat16))
            assert_close(to_np(step.o_heads[l, b]), ref["o_heads"], torch.bfloat16,
                         f"o_heads l={l} b={b}")
            assert_close(to_np(step.out[l, b]), ref["out"], torch.bfloat16, f"out l={l} b={b}")
    # the native executor (host buffers in and out) gives the device step's bytes
    out_host = torch.full((2, B, D), float("nan"), dtype=torch.bfloat16).pin_memory()
    step.run_native(h.cpu().pin_memory(), wls[0].pos.pin_memory(), wls[0].lens.pin_memory(),
                    out_host)
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    assert torch.equal(out_host, step.out.cpu())
