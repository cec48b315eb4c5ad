"""The multi-layer decode step runner (DecodeStep) on the GPU.  It only orders the C-ABI calls,
so every way of launching a step must give the same bytes, and every layer must match the oracle:

- eager launches, graph replay of the whole step, and the host path (per-layer input and output
  copies overlapped with the kernels; one graph per layer) agree bit for bit;
- programmatic dependent launch switched off (MLA_NO_PDL=1, read once per process, so in a child
  process) gives the same bytes as the default launches;
- each layer's o_heads and out match the oracle's non-absorbed fp64 decode step.

A step appends the new token's row and then attends to it.  Running a step again writes the same
row into the same slot, so repeated runs see identical caches."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

from tests.gpu_common import Workload, assert_close, dev, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L, B, H, D = 3, 4, 128, 1024
HIST = [100, 0, 700, 64]


def _workloads():
    return [Workload(60 + 10 * l, B, H, D, HIST) for l in range(L)]


def _step(wls, graph):
    from mla_latent_kv_37_b200.step import DecodeStep, Layer
    layers = [Layer(w_dkv=dev(wl.w.w_dkv), w_kr=dev(wl.w.w_kr), w_q=dev(wl.w.w_q),
                    w_uk=dev(wl.w.w_uk), w_uv=dev(wl.w.w_uv), w_o=dev(wl.w.w_o),
                    pool=dev(wl.cache.pool), page_table=dev(wl.cache.page_table))
              for wl in wls]
    step = DecodeStep(layers, B, H, D, graph=graph)
    h = torch.stack([dev(wl.h) for wl in wls])
    pos = dev(wls[0].pos)
    lens = dev(wls[0].lens)
    return step, h, pos, lens


def eager_outputs():
    """out and o_heads of one eager step (also run by the child process below)."""
    import mla_latent_kv_37_b200 as M
    step, h, pos, lens = _step(_workloads(), graph=False)
    step.run(h, pos, lens)
    torch.cuda.synchronize()
    assert M.mla_get_status() == 0
    return step.out.cpu(), step.o_heads.cpu()


def test_launch_modes_agree_bit_for_bit():
    import mla_latent_kv_37_b200 as M
    out_e, oh_e = eager_outputs()

    step, h, pos, lens = _step(_workloads(), graph=True)
    for _ in range(2):  # capture (after one eager step), then a replay
        step.run(h, pos, lens)
    torch.cuda.synchronize()
    assert torch.equal(step.out.cpu(), out_e) and torch.equal(step.o_heads.cpu(), oh_e)

    for graph in (False, True):
        step, h, pos, lens = _step(_workloads(), graph=graph)
        step.run(h, pos, lens)  # library set-up outside any capture
        torch.cuda.synchronize()
        step.out.zero_()
        h_host, pos_host, lens_host = h.cpu().pin_memory(), pos.cpu().pin_memory(), lens.cpu().pin_memory()
        out_host = torch.full(step.out.shape, float("nan"), dtype=step.out.dtype).pin_memory()
        h_dev, pos_dev, lens_dev = torch.zeros_like(h), torch.zeros_like(pos), torch.zeros_like(lens)
        for _ in range(2):
            step.run_host(h_host, pos_host, lens_host, out_host, h_dev, pos_dev, lens_dev)
        torch.cuda.synchronize()
        assert torch.equal(out_host, out_e), f"host path, graph={graph}"
        assert torch.equal(step.o_heads.cpu(), oh_e), f"host path, graph={graph}"
    assert M.mla_get_status() == 0


def test_without_programmatic_launch_same_bytes(tmp_path):
    out_e, oh_e = eager_outputs()
    path = tmp_path / "no_pdl.pt"
    code = ("import sys, torch; sys.path.insert(0, %r); import tests.test_gpu_step as T; "
            "torch.save(T.eager_outputs(), %r)" % (ROOT, str(path)))
    env = dict(os.environ, MLA_NO_PDL="1")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    out_n, oh_n = torch.load(path)
    assert torch.equal(out_n, out_e) and torch.equal(oh_n, oh_e)


def test_every_layer_matches_the_oracle():
    wls = _workloads()
    step, h, pos, lens = _step(wls, graph=True)
    for _ in range(2):
        step.run(h, pos, lens)
    torch.cuda.synchronize()
    for l, wl in enumerate(wls):
        for b in (range(B) if l == 0 else [2]):
            ref = wl.oracle(b)
            assert_close(to_np(step.o_heads[l, b]), ref["o_heads"], wl.dtype, f"o_heads l={l} b={b}")
            assert_close(to_np(step.out[l, b]), ref["out"], wl.dtype, f"out l={l} b={b}")


def test_native_step_executor_matches_device_step():
    """mla_decode_step_host (the C++ executor: host buffers in, copies and launches in the
    library, `out` back in host memory) gives the device-resident step's bytes, from page-locked
    and from pageable host memory, and twice in a row on the same buffers."""
    import mla_latent_kv_37_b200 as M
    out_e, _ = eager_outputs()
    wls = _workloads()
    step, h, pos, lens = _step(wls, graph=False)
    for pinned in (True, False):
        h_host = h.cpu()
        pos_host, lens_host = pos.cpu(), lens.cpu()
        out_host = torch.full((L, B, D), float("nan"), dtype=torch.bfloat16)
        if pinned:
            h_host, pos_host, lens_host = (t.pin_memory() for t in (h_host, pos_host, lens_host))
            out_host = out_host.pin_memory()
        for _ in range(2):
            step.run_native(h_host, pos_host, lens_host, out_host)
            torch.cuda.synchronize()
            assert M.mla_get_status() == 0
            assert torch.equal(out_host, out_e)


def test_native_step_rejects_bad_host_arguments():
    import mla_latent_kv_37_b200 as M
    wls = _workloads()
    step, h, pos, lens = _step(wls, graph=False)
    with pytest.raises(ValueError):
        step.run_native(h, pos.cpu(), lens.cpu(), torch.empty(L, B, D, dtype=torch.bfloat16))
    d = M.dims(B, H, D)
    arr = M.layer_structs(d, step.layers)
    ws = M.step_workspace(d, L)
    small = ws[: ws.numel() // 2]
    with pytest.raises(M.MlaError) as e:
        M.mla_decode_step_host(d, arr, h.cpu(), pos.cpu(), lens.cpu(),
                               torch.empty(L, B, D, dtype=torch.bfloat16), small)
    assert e.value.code == -4


def test_native_step_executor_fp32_and_fixed_split():
    """The native executor on the fp32 path (16 heads) and with a fixed split count: the same
    bytes as the device-resident step."""
    import mla_latent_kv_37_b200 as M
    from mla_latent_kv_37_b200.step import DecodeStep, Layer
    for dtype, splits in ((torch.float32, 0), (torch.bfloat16, 3)):
        Lf, Bf, Hf, Df = 2, 3, 16, 1024
        wls = [Workload(90 + l, Bf, Hf, Df, [70, 1, 130], dtype=dtype) for l in range(Lf)]
        layers = [Layer(w_dkv=dev(wl.w.w_dkv), w_kr=dev(wl.w.w_kr), w_q=dev(wl.w.w_q),
                        w_uk=dev(wl.w.w_uk), w_uv=dev(wl.w.w_uv), w_o=dev(wl.w.w_o),
                        pool=dev(wl.cache.pool), page_table=dev(wl.cache.page_table))
                  for wl in wls]
        step = DecodeStep(layers, Bf, Hf, Df, dtype=dtype, num_splits=splits)
        h = torch.stack([dev(wl.h) for wl in wls])
        pos, lens = dev(wls[0].pos), dev(wls[0].lens)
        step.run(h, pos, lens)
        torch.cuda.synchronize()
        ref = step.out.cpu()
        out_host = torch.full((Lf, Bf, Df), float("nan"), dtype=dtype).pin_memory()
        step.run_native(h.cpu().pin_memory(), pos.cpu().pin_memory(), lens.cpu().pin_memory(),
                        out_host)
        torch.cuda.synchronize()
        assert M.mla_get_status() == 0
        assert torch.equal(out_host, ref), (dtype, splits)
