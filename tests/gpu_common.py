"""Shared helpers for the GPU parity tests: tolerances, input staging, oracle comparisons."""
from __future__ import annotations

import math

import numpy as np
import torch

import mla_inputs as I
from oracle import mla_oracle as O

# Tolerances stated for this path: bf16 inputs with fp32 accumulation -> relative L2 <= 5e-3 and
# max |err| <= 2e-2 * max |oracle|; fp32 path -> 1e-5 relative.
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 2e-2
FP32_REL = 1e-5


def errors(got, exp):
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    den = np.linalg.norm(exp)
    rel = np.linalg.norm(got - exp) / (den if den > 0 else 1.0)
    mx = np.abs(got - exp).max() / max(np.abs(exp).max(), 1e-300)
    return rel, mx


def assert_close(got, exp, dtype, what=""):
    rel, mx = errors(got, exp)
    if dtype == torch.bfloat16:
        assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, f"{what}: rel-L2 {rel:.3e} max {mx:.3e}"
    else:
        assert rel <= FP32_REL and mx <= FP32_REL, f"{what}: rel-L2 {rel:.3e} max {mx:.3e}"
    return rel, mx


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def round_to(dtype):
    def f(row):
        return torch.from_numpy(np.asarray(row, dtype=np.float32)).to(dtype)
    return f


def dev(t):
    return t.to("cuda")


def latent_reference(q_cat, cache: I.PagedCache, seq_lens, scale=None):
    """Diagnostic o_lat / lse per sequence from the oracle's latent-space form."""
    q = O.f64(q_cat)
    outs, lses = [], []
    for b in range(q.shape[0]):
        n = int(seq_lens[b])
        rows = O.gather_rows(cache.pool, cache.page_table[b].numpy(), n)
        o, l = O.latent_attention(q[b, :, :512], q[b, :, 512:], rows[:, :512], rows[:, 512:],
                                  scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


class Workload:
    """One decode step of one layer: weights, hidden states, a paged cache with history."""

    def __init__(self, seed, batch, n_heads, d_model, history, dtype=torch.bfloat16,
                 scale=1.0, shuffle=True, with_w_o=True):
        self.B, self.H, self.D, self.dtype = batch, n_heads, d_model, dtype
        self.history = list(history)
        self.w = I.weights(seed, n_heads, d_model, dtype, with_w_o=with_w_o)
        self.h = I.hidden(seed + 1, batch, d_model, scale, dtype)
        self.cache = I.paged_cache(seed + 2, [n + 1 for n in history], history, scale, dtype,
                                   shuffle=shuffle)
        self.pos = torch.tensor(history, dtype=torch.int32)
        self.lens = self.pos + 1

    def run_gpu(self, num_splits=0, want_out=True, fused=False, query_remainder=False):
        """One decode step through the C ABI: cache append and absorbed query (two calls, or
        the fused mla_append_absorb), attention, output projection.  `query_remainder` also
        carries the query's bf16 rounding remainder from the projection to the attention."""
        import mla_latent_kv_37_b200 as M
        B, H, D = self.B, self.H, self.D
        d = M.dims(B, H, D, self.dtype)
        ws = M.workspace(d, num_splits)
        pool = dev(self.cache.pool)
        table = dev(self.cache.page_table)
        q_cat = torch.empty(B, H, 576, dtype=self.dtype, device="cuda")
        q_lo = (torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
                if query_remainder else None)
        o_lat = torch.empty(B, H, 512, dtype=torch.float32, device="cuda")
        lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
        o_heads = torch.empty(B, H, 128, dtype=self.dtype, device="cuda")
        out = torch.empty(B, D, dtype=self.dtype, device="cuda") if want_out else None
        w = self.w
        if fused:
            M.mla_append_absorb(d, dev(self.h), dev(w.w_dkv), dev(w.w_kr), dev(w.w_q),
                                dev(w.w_uk), dev(self.pos), table, pool, q_cat, ws, q_lo=q_lo)
        else:
            M.mla_cache_append(d, dev(self.h), dev(w.w_dkv), dev(w.w_kr), dev(self.pos), table,
                               pool, ws)
            M.mla_absorb_q(d, dev(self.h), dev(w.w_q), dev(w.w_uk), dev(self.pos), q_cat, ws,
                           q_lo=q_lo)
        M.mla_decode_attn(d, q_cat, pool, table, dev(self.lens), o_lat, ws, lse=lse,
                          q_lo=q_lo, num_splits=num_splits)
        M.mla_out_proj(d, o_lat, dev(w.w_uv), ws, w_o=dev(w.w_o) if want_out else None,
                       o_heads=o_heads, out=out)
        status = M.mla_get_status()
        return dict(pool=pool.cpu(), q_cat=q_cat.cpu(), o_lat=o_lat.cpu(), lse=lse.cpu(),
                    o_heads=o_heads.cpu(), out=None if out is None else out.cpu(), status=status)

    def oracle(self, b, heads=None, with_out=True):
        hist = O.gather_rows(self.cache.pool, self.cache.page_table[b].numpy(), self.history[b])
        return O.decode_step(self.h[b], self.w, hist, self.history[b], self.H,
                             round_row=round_to(self.dtype), heads=heads, with_out=with_out)


def _check_all(q_exact, cache, lens, o_lat, lse, dtype=torch.bfloat16):
    """o_lat / lse of every sequence against the oracle's latent-space attention."""
    ref_o, ref_l = latent_reference(q_exact, cache, lens)
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o_lat[b] == 0)
            assert torch.all(torch.isneginf(lse[b]))
            continue
        assert_close(o_lat[b].double().numpy(), ref_o[b], dtype, f"o_lat b={b} n={n}")
        np.testing.assert_allclose(lse[b].double().numpy(), ref_l[b], rtol=2e-4, atol=2e-4)
