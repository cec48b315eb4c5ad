"""One MLA decode step over a stack of layers, driven through the C ABI.

A step, per layer l (each layer has its own weights, paged cache and hidden state h[l]):
    mla_append_absorb (= mla_cache_append + mla_absorb_q) -> mla_decode_attn -> mla_out_proj
or, for a layer with E4M3 weights (`Layer.e4m3`, see `quantize_layer`),
    mla_append_absorb_fp8 -> mla_decode_attn -> mla_out_proj_fp8
Everything stays on the device; `run_host` adds the host<->device copies of the step's inputs
and results (pinned buffers), overlapped layer by layer with the kernels, for end-to-end use.
Marshalling only: no arithmetic.
"""
from __future__ import annotations

import dataclasses

import torch

from . import (dims as make_dims, fp8_codes_shape, mla_append_absorb, mla_append_absorb_fp8,
               mla_decode_attn, mla_launch_count, mla_out_proj, mla_out_proj_fp8,
               mla_quantize_weights_fp8, workspace)


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
    # E4M3 copies {"w_dkv", "w_kr", "w_q", "w_o"} -> (codes, scale); None: bf16 weights
    e4m3: dict | None = None


def quantize_layer(layer: Layer) -> Layer:
    """The layer with E4M3 copies of W_DKV, W_KR, W_Q and W_O (mla_quantize_weights_fp8, on the
    weights' device and the current stream); W_UK and W_UV stay bf16."""
    q = {}
    for name in ("w_dkv", "w_kr", "w_q", "w_o"):
        w = getattr(layer, name)
        codes = torch.empty(fp8_codes_shape(*w.shape), dtype=torch.uint8, device=w.device)
        scale = torch.empty(w.shape[0], dtype=torch.float32, device=w.device)
        mla_quantize_weights_fp8(w, codes, scale)
        q[name] = (codes, scale)
    return dataclasses.replace(layer, e4m3=q)


class DecodeStep:
    def __init__(self, layers: list[Layer], batch: int, n_heads: int, d_model: int,
                 dtype=torch.bfloat16, num_splits: int = 0, device="cuda", graph: bool = False,
                 query_remainder: bool = False):
        """`query_remainder` carries the absorbed query's bf16 rounding remainder (q_lo) from
        the projection into the attention, for inputs with large logits."""
        self.layers = layers
        self.B, self.H, self.D, self.dtype = batch, n_heads, d_model, dtype
        self.dims = make_dims(batch, n_heads, d_model, dtype)
        self.num_splits = num_splits
        L = len(layers)
        self.ws = workspace(self.dims, num_splits, device)
        self.q_cat = torch.empty(batch, n_heads, 576, dtype=dtype, device=device)
        self.q_lo = (torch.empty(batch, n_heads, 576, dtype=torch.bfloat16, device=device)
                     if query_remainder else None)
        self.o_lat = torch.empty(batch, n_heads, 512, dtype=torch.float32, device=device)
        self.lse = torch.empty(batch, n_heads, dtype=torch.float32, device=device)
        self.o_heads = torch.empty(L, batch, n_heads, 128, dtype=dtype, device=device)
        self.out = torch.empty(L, batch, d_model, dtype=dtype, device=device)
        # graph mode: the step's launches are captured once per set of input buffers (a CUDA
        # graph) and replayed; every launch keeps the arguments it was captured with
        self.graph = graph
        self._graphs: dict = {}
        self.launches_per_step = 0
        # end-to-end path: one copy stream per direction, one event per layer and direction
        self._copy_in = self._copy_out = None
        self._ev_in: list = []
        self._ev_out: list = []

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

    def _layer(self, l, h_l, positions, seq_lens, stream=None):
        d, ly, q = self.dims, self.layers[l], self.layers[l].e4m3
        if q is not None:
            mla_append_absorb_fp8(d, h_l, q["w_dkv"], q["w_kr"], q["w_q"], ly.w_uk, positions,
                                  ly.page_table, ly.pool, self.q_cat, self.ws, q_lo=self.q_lo,
                                  stream=stream)
        else:
            mla_append_absorb(d, h_l, ly.w_dkv, ly.w_kr, ly.w_q, ly.w_uk, positions,
                              ly.page_table, ly.pool, self.q_cat, self.ws, q_lo=self.q_lo,
                              stream=stream)
        mla_decode_attn(d, self.q_cat, ly.pool, ly.page_table, seq_lens, self.o_lat, self.ws,
                        lse=self.lse, q_lo=self.q_lo, num_splits=self.num_splits, stream=stream)
        if q is not None:
            mla_out_proj_fp8(d, self.o_lat, ly.w_uv, q["w_o"][0], q["w_o"][1], self.out[l],
                             self.ws, o_heads=self.o_heads[l], stream=stream)
        else:
            mla_out_proj(d, self.o_lat, ly.w_uv, self.ws, w_o=ly.w_o, o_heads=self.o_heads[l],
                         out=self.out[l] if ly.w_o is not None else None, stream=stream)

    def _run(self, h, positions, seq_lens, stream=None):
        for l in range(len(self.layers)):
            self._layer(l, h[l], positions, seq_lens, stream)

    def _host_step(self, h_host, pos_host, lens_host, out_host, h_dev, pos_dev, lens_dev):
        """Enqueue one host-path step on the current stream, eagerly or under graph capture.
        Every layer's hidden state goes up on one copy stream ahead of that layer, every
        layer's output comes back on another as soon as the layer has written it, and the
        step ends when the last output is on the host."""
        s = torch.cuda.current_stream()
        L = len(self.layers)
        cin, cout = self._copy_in, self._copy_out
        # the device buffers are free once everything already queued on `s` has run
        cin.wait_stream(s)
        cout.wait_stream(s)
        with torch.cuda.stream(cin):
            pos_dev.copy_(pos_host, non_blocking=True)
            lens_dev.copy_(lens_host, non_blocking=True)
            for l in range(L):
                h_dev[l].copy_(h_host[l], non_blocking=True)
                self._ev_in[l].record(cin)
        for l in range(L):
            s.wait_event(self._ev_in[l])
            self._layer(l, h_dev[l], pos_dev, lens_dev)
            self._ev_out[l].record(s)
            cout.wait_event(self._ev_out[l])
            with torch.cuda.stream(cout):
                out_host[l].copy_(self.out[l], non_blocking=True)
        s.wait_stream(cout)

    def run_native(self, h_host, pos_host, lens_host, out_host, stream=None):
        """End-to-end through the library's native step executor (mla_decode_step_host): the
        host buffers go in and `out` comes back with every copy and launch made in C++."""
        from . import layer_structs, mla_decode_step_host, step_workspace
        if getattr(self, "_native", None) is None:
            self._native = (layer_structs(self.dims, self.layers),
                            step_workspace(self.dims, len(self.layers), self.num_splits,
                                           self.ws.device))
        arr, ws = self._native
        mla_decode_step_host(self.dims, arr, h_host, pos_host, lens_host, out_host, ws,
                             self.num_splits, stream)

    def run_host(self, h_host, pos_host, lens_host, out_host, h_dev, pos_dev, lens_dev,
                 stream=None):
        """End-to-end: the step's inputs come from pinned host memory and `out` goes back to
        pinned host memory, the copies overlapped with the kernels (only the first layer's
        input and the last layer's output are exposed).  In graph mode the whole host-path
        step, copies and both copy streams included, is one graph per set of buffers, captured
        after one eager run of it."""
        s = torch.cuda.current_stream() if stream is None else stream
        if self._copy_in is None:
            L = len(self.layers)
            self._copy_in, self._copy_out = torch.cuda.Stream(), torch.cuda.Stream()
            self._ev_in = [torch.cuda.Event() for _ in range(L)]
            self._ev_out = [torch.cuda.Event() for _ in range(L)]
        bufs = (h_host, pos_host, lens_host, out_host, h_dev, pos_dev, lens_dev)
        if not self.graph:
            with torch.cuda.stream(s):
                self._host_step(*bufs)
            return
        key = ("host",) + tuple(t.data_ptr() for t in bufs)
        g = self._graphs.get(key)
        if g is None:
            with torch.cuda.stream(s):
                self._host_step(*bufs)  # one-time library set-up happens outside the capture
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._host_step(*bufs)
            self._graphs[key] = g
        with torch.cuda.stream(s):
            g.replay()
