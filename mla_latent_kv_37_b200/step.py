"""One MLA decode step over a stack of layers, driven through the C ABI.

A step, per layer l (each layer has its own weights, paged cache and hidden state h[l]):
    mla_append_absorb (= mla_cache_append + mla_absorb_q) -> mla_decode_attn -> mla_out_proj
Everything stays on the device; `run_host` adds the host<->device copies of the step's inputs
and results (pinned buffers) for end-to-end measurement.  Marshalling only: no arithmetic.
"""
from __future__ import annotations

import dataclasses

import torch

from . import (dims as make_dims, mla_append_absorb, mla_decode_attn, mla_launch_count,
               mla_out_proj, workspace)


@dataclasses.dataclass
class Layer:
    w_dkv: torch.Tensor
    w_kr: torch.Tensor
    w_q: torch.Tensor
    w_uk: torch.Tensor
    w_uv: torch.Tensor
    w_o: torch.Tensor | None
    pool: torch.Tensor        # [num_pages, 64, 576]
    page_table: torch.Tensor  # [B, max_pages] int32


class DecodeStep:
    def __init__(self, layers: list[Layer], batch: int, n_heads: int, d_model: int,
                 dtype=torch.bfloat16, num_splits: int = 0, device="cuda", graph: bool = False):
        self.layers = layers
        self.B, self.H, self.D, self.dtype = batch, n_heads, d_model, dtype
        self.dims = make_dims(batch, n_heads, d_model, dtype)
        self.num_splits = num_splits
        L = len(layers)
        self.ws = workspace(self.dims, num_splits, device)
        self.q_cat = torch.empty(batch, n_heads, 576, dtype=dtype, device=device)
        self.o_lat = torch.empty(batch, n_heads, 512, dtype=torch.float32, device=device)
        self.lse = torch.empty(batch, n_heads, dtype=torch.float32, device=device)
        self.o_heads = torch.empty(L, batch, n_heads, 128, dtype=dtype, device=device)
        self.out = torch.empty(L, batch, d_model, dtype=dtype, device=device)
        # graph mode: the step's launches are captured once per set of input buffers (a CUDA
        # graph) and replayed; every launch keeps the arguments it was captured with
        self.graph = graph
        self._graphs: dict = {}
        self.launches_per_step = 0

    def run(self, h, positions, seq_lens, stream=None):
        """h [L, B, D] on the device; positions [B] (append slot), seq_lens [B] = positions+1."""
        if not self.graph:
            self._run(h, positions, seq_lens, stream)
            return
        key = (h.data_ptr(), positions.data_ptr(), seq_lens.data_ptr())
        g = self._graphs.get(key)
        if g is None:
            g = self.capture(h, positions, seq_lens)
        if stream is None:
            g.replay()
        else:
            with torch.cuda.stream(stream):
                g.replay()

    def capture(self, h, positions, seq_lens, before_capture=None):
        """(Re)capture the step for these input buffers.  One eager step first, so that every
        one-time set-up of the library (device context, kernel attributes) happens outside the
        capture; `before_capture` runs between the two."""
        self._run(h, positions, seq_lens)
        torch.cuda.synchronize()
        if before_capture is not None:
            before_capture()
        g = torch.cuda.CUDAGraph()
        n0 = mla_launch_count()
        with torch.cuda.graph(g):
            self._run(h, positions, seq_lens)
        self.launches_per_step = mla_launch_count() - n0
        self._graphs[(h.data_ptr(), positions.data_ptr(), seq_lens.data_ptr())] = g
        return g

    def _run(self, h, positions, seq_lens, stream=None):
        d = self.dims
        for l, ly in enumerate(self.layers):
            mla_append_absorb(d, h[l], ly.w_dkv, ly.w_kr, ly.w_q, ly.w_uk, positions,
                              ly.page_table, ly.pool, self.q_cat, self.ws, stream=stream)
            mla_decode_attn(d, self.q_cat, ly.pool, ly.page_table, seq_lens, self.o_lat, self.ws,
                            lse=self.lse, num_splits=self.num_splits, stream=stream)
            mla_out_proj(d, self.o_lat, ly.w_uv, self.ws, w_o=ly.w_o, o_heads=self.o_heads[l],
                         out=self.out[l] if ly.w_o is not None else None, stream=stream)

    def run_host(self, h_host, pos_host, lens_host, out_host, h_dev, pos_dev, lens_dev,
                 stream=None):
        """End-to-end: copy the step's inputs from pinned host memory, run, copy `out` back."""
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            h_dev.copy_(h_host, non_blocking=True)
            pos_dev.copy_(pos_host, non_blocking=True)
            lens_dev.copy_(lens_host, non_blocking=True)
            self.run(h_dev, pos_dev, lens_dev, stream=s)
            out_host.copy_(self.out, non_blocking=True)
