"""Seeded synthetic inputs for MLA decode, shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and lays them out; it holds none of the method's arithmetic
(no projection, no RoPE, no softmax).  Every tensor is produced by a ``torch.Generator`` with a
fixed seed, so the bytes are machine-independent on CPU.  Large workloads (tens of GB) are drawn
on the device with a seeded CUDA generator instead; those bytes are reproducible on the same GPU
type and are copied back to the host whenever the oracle needs them.

Distributions follow the workloads the MLA pages discuss (DeepSeek-V2/V3 shapes: latent width
512, decoupled RoPE key 64, 128 heads, 61 layers):
  * hidden state h_t ~ N(0, 1) * s
  * weights ~ N(0, 1/fan_in), fan_in = input width of the projection as written in the
    non-absorbed form (W_DKV, W_KR, W_Q: d_model; W_UK, W_UV: d_c; W_O: n_heads * d_v)
  * prefilled cache rows (history) ~ N(0, 1) * s, already in post-RoPE form
  * pages of 64 tokens placed by a seeded random permutation of the pool
  * unused slots of a sequence's last page hold a finite sentinel
"""
from __future__ import annotations

import dataclasses
import math

import torch

D_C = 512      # latent width of c_KV
D_R = 64       # decoupled RoPE key width k_R
D_NOPE = 128   # per-head non-rotary query/key width
D_V = 128      # per-head value width
ROW = D_C + D_R  # 576 numbers cached per token per layer
PAGE = 64      # tokens per cache page

SENTINEL = 1.0e30  # finite filler for cache slots past a sequence's length


def generator(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, std, g, dtype, device):
    x = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


@dataclasses.dataclass
class Weights:
    w_dkv: torch.Tensor  # [d_c, D]
    w_kr: torch.Tensor   # [d_R, D]
    w_q: torch.Tensor    # [H*(d_nope+d_R), D], per head: d_nope rows then d_R rows
    w_uk: torch.Tensor   # [H*d_nope, d_c]
    w_uv: torch.Tensor   # [H*d_v, d_c]
    w_o: torch.Tensor    # [D, H*d_v]


def weights(seed: int, n_heads: int, d_model: int, dtype=torch.bfloat16, device: str = "cpu",
            with_w_o: bool = True) -> Weights:
    g = generator(seed, device)
    H, D = n_heads, d_model
    w_dkv = _randn((D_C, D), 1.0 / math.sqrt(D), g, dtype, device)
    w_kr = _randn((D_R, D), 1.0 / math.sqrt(D), g, dtype, device)
    w_q = _randn((H * (D_NOPE + D_R), D), 1.0 / math.sqrt(D), g, dtype, device)
    w_uk = _randn((H * D_NOPE, D_C), 1.0 / math.sqrt(D_C), g, dtype, device)
    w_uv = _randn((H * D_V, D_C), 1.0 / math.sqrt(D_C), g, dtype, device)
    if with_w_o:
        w_o = _randn((D, H * D_V), 1.0 / math.sqrt(H * D_V), g, dtype, device)
    else:
        w_o = torch.empty(0, dtype=dtype, device=device)
    return Weights(w_dkv, w_kr, w_q, w_uk, w_uv, w_o)


def hidden(seed: int, batch: int, d_model: int, scale: float = 1.0, dtype=torch.bfloat16,
           device: str = "cpu") -> torch.Tensor:
    g = generator(seed, device)
    return _randn((batch, d_model), scale, g, dtype, device)


def query_cat(seed: int, batch: int, n_heads: int, scale: float = 1.0, dtype=torch.bfloat16,
              device: str = "cpu") -> torch.Tensor:
    """A random absorbed query [B, H, 576] for attention-only tests (latent part std 0.5,
    RoPE part std 1, the statistics the N(0, 1/fan_in) weights give at s = 1)."""
    g = generator(seed, device)
    q = torch.randn(batch, n_heads, ROW, generator=g, dtype=torch.float32, device=device)
    q[..., :D_C].mul_(0.5 * scale)
    q[..., D_C:].mul_(scale)
    return q.to(dtype)


@dataclasses.dataclass
class PagedCache:
    pool: torch.Tensor        # [num_pages, PAGE, ROW]
    page_table: torch.Tensor  # [B, max_pages] int32, unused entries = -1
    seq_lens: torch.Tensor    # [B] int32, rows already present (history)
    num_pages: int


def pages_needed(n_tokens: int) -> int:
    return (n_tokens + PAGE - 1) // PAGE


def paged_cache(seed: int, capacity: list[int], history: list[int], scale: float = 1.0,
                dtype=torch.bfloat16, device: str = "cpu", shuffle: bool = True,
                sentinel: float = SENTINEL, extra_pages: int = 0) -> PagedCache:
    """Pool of pages for B sequences.

    capacity[b] tokens of room are reserved for sequence b (so a decode step may append at
    position history[b] when capacity[b] > history[b]); rows [0, history[b]) hold N(0,1)*s
    history and every other slot of the reserved pages holds ``sentinel``.  ``shuffle`` places
    pages by a seeded permutation of the pool, otherwise sequence b owns a contiguous run.
    """
    assert len(capacity) == len(history)
    B = len(capacity)
    g = generator(seed, device)
    n_pages = [pages_needed(c) for c in capacity]
    total = sum(n_pages) + extra_pages
    max_pages = max(max(n_pages), 1)
    pool = torch.full((total, PAGE, ROW), sentinel, dtype=dtype, device=device)
    if shuffle:
        perm = torch.randperm(total, generator=g, device=device)
    else:
        perm = torch.arange(total, device=device)
    table = torch.full((B, max_pages), -1, dtype=torch.int32, device=device)
    cursor = 0
    for b in range(B):
        ids = perm[cursor:cursor + n_pages[b]]
        cursor += n_pages[b]
        table[b, :n_pages[b]] = ids.to(torch.int32)
        n = history[b]
        if n == 0:
            continue
        rows = _randn((n, ROW), scale, g, dtype, device)
        full, rem = divmod(n, PAGE)
        if full:
            pool[ids[:full].long()] = rows[: full * PAGE].view(full, PAGE, ROW)
        if rem:
            pool[ids[full].long(), :rem] = rows[full * PAGE:]
    seq_lens = torch.tensor(history, dtype=torch.int32, device=device)
    return PagedCache(pool, table, seq_lens, total)


def uniform_lengths(seed: int, batch: int, lo: int, hi: int) -> list[int]:
    """Context lengths drawn uniformly from the integers [lo, hi] (inclusive)."""
    g = generator(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=g)]
