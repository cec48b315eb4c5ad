"""Benchmark: MLA decode step throughput on B200, with roofline, end-to-end and CPU baselines.

Default workload: the full 61-layer DeepSeek-V3-shaped MLA decode step -- batch 32, context
32768 per sequence, 128 heads, d_c 512, d_R 64, d_model 7168, bf16 -- where each layer runs
cache append -> absorbed query -> split-KV attention -> W_UV and W_O projections.  Inputs are
seeded synthetic tensors generated on the device (73.7 GB of latent cache + 38.4 GB of weights,
far larger than the 126 MB L2, so no L2 flush is needed between steps).

    python bench.py [--gpus N --steps K --warmup W] [--config NAME] [--impl reference]

One process per GPU (torchrun for N > 1); every GPU runs its own independent replica of the
workload (the path has no exchange step), timing is the max over ranks, value = all tokens /
that time.  `--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "MLA decode tokens/s and latent-cache GB/s / TFLOP/s vs B200 roofline"
ROW_BYTES = 1152           # 576 bf16 numbers per cached token per layer
FLOP_PER_TOKEN_HEAD = 2 * 576 + 2 * 512  # QK^T and PV per cached token per head

CONFIGS = {
    # name: batch, context, layers, heads, d_model, dtype, scale, length mode
    "full_61": dict(batch=32, context=32768, layers=61, heads=128, d_model=7168,
                    workload="full 61-layer MLA decode step (append + absorb + decode attention"
                             " + W_UV/W_O out-proj per layer)"),
    "v3_single": dict(batch=1, context=4096, layers=1, heads=128, d_model=7168,
                      workload="single-layer DeepSeek-V3-shaped MLA decode, context 4096"),
    "paged_b64": dict(batch=64, context=None, layers=1, heads=128, d_model=7168,
                      workload="batched paged MLA decode, batch 64, context U[1024,8192]"),
    "long_128k": dict(batch=4, context=131072, layers=1, heads=128, d_model=7168,
                      workload="long-context split-KV MLA decode, batch 4 x 131072"),
    "long_128k_x4": dict(batch=4, context=131072, layers=1, heads=128, d_model=7168, scale=4.0,
                         remainder=True,
                         workload="long-context split-KV MLA decode, batch 4 x 131072, inputs x4"
                                  " (query carried as bf16 hi + lo)"),
}
# the single-layer configurations reported beside the headline: (name, sequences, heads) sampled
# for the parity check against the oracle
EXTRA_CONFIGS = (("v3_single", 1, 8), ("paged_b64", 2, 4), ("long_128k", 1, 4),
                 ("long_128k_x4", 1, 4))


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------------------------
# distributed plumbing (replicas only: used for the barrier and the max over ranks)
# ---------------------------------------------------------------------------------------------
def dist_setup():
    """One process per GPU under torchrun: NCCL when CUDA is present, gloo otherwise (the
    replicas exchange nothing but a barrier and the max over ranks of the step time)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return rank, ws, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock and throttle-reason samples, every `interval_ms`, each stamped with the
    host time it arrived.  stop(t0, t1) summarises the samples that arrived inside the timed
    window [t0, t1] (host seconds); if none did (a window shorter than the interval), the
    sample nearest to the window's middle is used."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 200):
        self.gpu = gpu_index
        self.interval_ms = interval_ms
        self.lines = []  # (host time, csv line)
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval_ms), "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    @staticmethod
    def parse(line):
        """(sm MHz, max sm MHz, active reasons) of one csv line, or None."""
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            return None
        try:
            sm, mx = float(parts[1]), float(parts[2])
        except ValueError:
            return None
        active = {n for n, v in zip(ClockSampler.REASONS, parts[5:9])
                  if v.lower().startswith("active")}
        return sm, mx, active

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return self.summarise(self.lines, t0, t1)

    @staticmethod
    def summarise(lines, t0, t1, slack=0.0):
        samples = [(t, r) for t, r in ((t, ClockSampler.parse(ln)) for t, ln in lines) if r]
        if t0 is not None and t1 is not None and samples:
            inside = [(t, r) for t, r in samples if t0 - slack <= t <= t1 + slack]
            if not inside:
                mid = 0.5 * (t0 + t1)
                inside = [min(samples, key=lambda s: abs(s[0] - mid))]
            samples = inside
        sm = sorted(r[0] for _, r in samples)
        reasons = set()
        for _, r in samples:
            reasons |= r[2]
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": samples[-1][1][1] if samples else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------------------------
def context_lengths(cfg, seed):
    import mla_inputs as I
    if cfg["context"] is None:
        return I.uniform_lengths(seed, cfg["batch"], 1024, 8192)
    return [cfg["context"]] * cfg["batch"]


def make_workload(cfg, device, seed=4):
    """Per-layer weights, paged cache (history = context - 1 rows) and hidden states, drawn on
    the device with seeded generators; hidden states and history are scaled by cfg["scale"]."""
    import mla_inputs as I
    from mla_latent_kv_37_b200.step import Layer
    B, H, D, L = cfg["batch"], cfg["heads"], cfg["d_model"], cfg["layers"]
    lens = context_lengths(cfg, seed)
    hist = [n - 1 for n in lens]
    layers = []
    for l in range(L):
        w = I.weights(seed * 1000 + l, H, D, torch.bfloat16, device)
        c = I.paged_cache(seed * 1000 + 500 + l, lens, hist, cfg.get("scale", 1.0),
                          torch.bfloat16, device)
        layers.append(Layer(w.w_dkv, w.w_kr, w.w_q, w.w_uk, w.w_uv, w.w_o, c.pool, c.page_table))
        if l == 0 or (l + 1) % 10 == 0:
            log(f"[bench] generated layer {l + 1}/{L}")
    h = torch.stack([I.hidden(seed * 1000 + 900 + l, B, D, cfg.get("scale", 1.0),
                              torch.bfloat16, device) for l in range(L)])
    pos = torch.tensor(hist, dtype=torch.int32, device=device)
    return layers, h, pos, pos + 1, lens


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# ---------------------------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample_inputs(layer, h_layer, b, hist_len):
    """Host copies of what the oracle needs for sequence b of one layer."""
    import numpy as np
    from oracle import mla_oracle as O

    class W:
        pass
    w = W()
    for n in ("w_dkv", "w_kr", "w_q", "w_uk", "w_uv", "w_o"):
        t = getattr(layer, n)
        setattr(w, n, t.cpu() if t is not None else np.zeros(0))
    hist = O.gather_rows(layer.pool, layer.page_table[b].cpu().numpy(), hist_len)
    return w, h_layer[b].cpu(), hist


def time_oracle(w, h, hist, pos, H, budget_s=12.0, min_heads=2):
    """Seconds for one (sequence, layer) of the oracle: projections + per-head attention,
    with the per-head cost measured on as many heads as fit the budget."""
    from oracle import mla_oracle as O
    t0 = time.perf_counter()
    O.decode_step(h, w, hist, pos, H, heads=[], with_out=False)
    t_proj = time.perf_counter() - t0
    c_kv = O.f64(hist)[:, :512]
    k_r = O.f64(hist)[:, 512:]
    qn, qr = O.query_heads(h, w.w_q, H, 128, 64, pos)
    n_heads, t_heads = 0, 0.0
    while n_heads < H and (n_heads < min_heads or t_heads < budget_s):
        t1 = time.perf_counter()
        O.decode_attention(qn, qr, c_kv, k_r, w.w_uk, w.w_uv, heads=[n_heads])
        t_heads += time.perf_counter() - t1
        n_heads += 1
    per_head = t_heads / n_heads
    import numpy as np
    t_out = 0.0
    if O.f64(w.w_o).size:
        t2 = time.perf_counter()
        O.output_projection(np.zeros((H, 128)), w.w_o)
        t_out = time.perf_counter() - t2
    return t_proj + H * per_head + t_out, n_heads, t_proj + t_heads + t_out


def cpu_baseline_from(seconds_per_seq_layer, cfg, heads_timed, wall):
    B, L = cfg["batch"], cfg["layers"]
    step_s = seconds_per_seq_layer * B * L
    return {"value": B / step_s, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"1 sequence x 1 layer of the workload: fp64 projections + {heads_timed} of "
                      f"{cfg['heads']} heads of reconstructed attention over the full context, "
                      f"timed {wall:.1f} s and scaled to {B} sequences x {L} layers x "
                      f"{cfg['heads']} heads"}


# ---------------------------------------------------------------------------------------------
# parity sample on the timed workload
# ---------------------------------------------------------------------------------------------
def parity_sample(layers, h, hist, step, cfg, n_layers=2, n_seqs=2, n_heads=8, seed=0):
    import numpy as np
    from oracle import mla_oracle as O
    rng = np.random.default_rng(seed)
    L, B, H = cfg["layers"], cfg["batch"], cfg["heads"]
    worst = {"o_heads_rel_l2": 0.0, "o_heads_max_abs": 0.0}
    checked = 0
    for l in sorted(set([0, L - 1][:n_layers])):
        for b in rng.choice(B, min(n_seqs, B), replace=False):
            b = int(b)
            w, hb, rows = oracle_sample_inputs(layers[l], h[l], b, hist[b])
            heads = sorted(rng.choice(H, min(n_heads, H), replace=False).tolist())
            to_bf16 = lambda r: torch.from_numpy(np.asarray(r, dtype=np.float32)).to(torch.bfloat16)
            ref = O.decode_step(hb, w, rows, hist[b], H, round_row=to_bf16, heads=heads,
                                with_out=False)
            got = step.o_heads[l, b][heads].float().cpu().numpy().astype(np.float64)
            exp = ref["o_heads"]
            rel = float(np.linalg.norm(got - exp) / np.linalg.norm(exp))
            mx = float(np.abs(got - exp).max() / np.abs(exp).max())
            worst["o_heads_rel_l2"] = max(worst["o_heads_rel_l2"], rel)
            worst["o_heads_max_abs"] = max(worst["o_heads_max_abs"], mx)
            checked += 1
    worst["samples"] = f"{checked} (layer, sequence) pairs x {n_heads} heads"
    worst["pass"] = worst["o_heads_rel_l2"] <= 5e-3 and worst["o_heads_max_abs"] <= 2e-2
    return worst


# ---------------------------------------------------------------------------------------------
# traffic figure from a committed ncu summary, valid only for the exact kernel source
# ---------------------------------------------------------------------------------------------
def kernel_source_hash():
    """Hash of the split kernel's code: its two source files without // comments and blank
    lines, so that editing a comment does not invalidate the recorded counters."""
    hsh = hashlib.sha256()
    for f in ("attn_sm100.cuh", "ptx_sm100.cuh"):
        with open(os.path.join(ROOT, "mla_latent_kv_37_b200", "csrc", f)) as fh:
            lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in fh.read().splitlines()]
        hsh.update("\n".join(ln for ln in lines if ln.strip()).encode())
    return hsh.hexdigest()[:16]


def committed_traffic(config_name):
    path = os.path.join(ROOT, "profiles", "decode_split_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_hash") != kernel_source_hash():
        return None
    return rec.get("bytes_per_launch", {}).get(config_name)


# ---------------------------------------------------------------------------------------------
# single-layer attention sweep: mla_decode_attn alone over batch x context
# ---------------------------------------------------------------------------------------------
SWEEP_BATCH = (32, 64, 128)
SWEEP_CONTEXT = (8192, 16384, 32768)


def load_peaks():
    """MEASURED_PEAKS.json (written on the GPU machine) or {} when it is absent."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return {}


def attention_roofline(tokens, B, H, seconds, peaks, sustained):
    """Roofline numbers of one mla_decode_attn call over `tokens` cached tokens: algorithmic
    bytes (cache rows + query + o_lat) and flops, against the HBM and bf16 tensor peaks (the
    sustained GEMM rate for a kernel timed inside a long step, the burst rate for one timed
    alone); bound = the slower of the two."""
    hbm = peaks.get("hbm_gbs", 6650.0)
    tc_burst = peaks.get("bf16_tflops", 1590.0)
    tc = peaks.get("bf16_tflops_sustained", 1400.0) if sustained else tc_burst
    nbytes = tokens * ROW_BYTES + B * H * 576 * 2 + B * H * 512 * 4
    flops = tokens * H * FLOP_PER_TOKEN_HEAD
    t_hbm, t_tc = nbytes / (hbm * 1e9), flops / (tc * 1e12)
    gbs, tfs = nbytes / seconds / 1e9, flops / seconds / 1e12
    return {"bound": "hbm" if t_hbm >= t_tc else "tensor", "us": seconds * 1e6,
            "roofline_us": max(t_hbm, t_tc) * 1e6, "frac": max(t_hbm, t_tc) / seconds,
            "gbs": gbs, "hbm_frac": gbs / hbm, "tflops": tfs,
            "tensor_frac_burst": tfs / tc_burst,
            "tensor_frac_sustained": tfs / peaks.get("bf16_tflops_sustained", 1400.0),
            "bytes": nbytes, "flops": flops}


def sweep_shape(B, N, warmup, iters, peaks, dev, flush, H=128):
    """mla_decode_attn (plan + split + combine) alone on one layer: B sequences of N tokens in
    full pages at random places, the L2 flushed (a 256 MB write) before every timed call, CUDA
    events around each call; median / p10 / p90 and the roofline fraction at the median against
    the burst peaks (the call is timed alone)."""
    import mla_inputs as I
    import mla_latent_kv_37_b200 as M
    q = I.query_cat(7, B, H, device=dev)
    cache = I.paged_cache(8, [N] * B, [N] * B, device=dev)
    lens = torch.full((B,), N, dtype=torch.int32, device=dev)
    d = M.dims(B, H, 7168)
    ws = M.workspace(d, 0, dev)
    o = torch.empty(B, H, 512, dtype=torch.float32, device=dev)
    lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    for _ in range(warmup):
        M.mla_decode_attn(d, q, cache.pool, cache.page_table, lens, o, ws, lse=lse)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for i, (e0, e1) in enumerate(ev):
        flush.fill_(i & 0xFF)
        e0.record()
        M.mla_decode_attn(d, q, cache.pool, cache.page_table, lens, o, ws, lse=lse)
        e1.record()
    torch.cuda.synchronize()
    st = M.mla_get_status()
    if st:
        raise RuntimeError(f"device status {st:#x} in the sweep (B={B}, N={N})")
    us = sorted(e0.elapsed_time(e1) * 1e3 for e0, e1 in ev)
    pick = lambda f: us[min(len(us) - 1, int(f * (len(us) - 1) + 0.5))]
    r = attention_roofline(B * N, B, H, pick(0.5) * 1e-6, peaks, sustained=False)
    del q, cache, lens, ws, o, lse
    torch.cuda.empty_cache()
    return {"batch": B, "context": N, "heads": H, "us_median": pick(0.5), "us_p10": pick(0.1),
            "us_p90": pick(0.9), "frac": r["frac"], "bound": r["bound"], "gbs": r["gbs"],
            "tflops": r["tflops"], "hbm_frac": r["hbm_frac"],
            "tensor_frac_burst": r["tensor_frac_burst"]}


def run_sweep(args):
    """`--sweep`: every batch x context of SWEEP_BATCH x SWEEP_CONTEXT, one JSON line each."""
    from mla_latent_kv_37_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    src = "of measured" if peaks else "of fallback"
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for B in SWEEP_BATCH:
        for N in SWEEP_CONTEXT:
            line = sweep_shape(B, N, args.sweep_warmup, args.sweep_iters, peaks, dev, flush)
            line.update({"metric": "mla_decode_attn, one layer (plan + split + combine)",
                         "peaks": {"hbm_gbs": peaks.get("hbm_gbs", 6650.0),
                                   "bf16_tflops": peaks.get("bf16_tflops", 1590.0),
                                   "source": src + " (burst)"},
                         "warmup": args.sweep_warmup, "timed": args.sweep_iters,
                         "l2": "flushed by a 256 MB write before every timed call"})
            print(json.dumps(line), flush=True)


# the attention sweep carried in the default JSON line (batch >= 32, context >= 8K)
COMPACT_SWEEP = ((32, 8192), (32, 32768), (64, 8192), (64, 32768), (128, 8192), (128, 32768))


def compact_sweep(dev, peaks, warmup=5, iters=20):
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    shapes = [sweep_shape(B, N, warmup, iters, peaks, dev, flush) for B, N in COMPACT_SWEEP]
    del flush
    torch.cuda.empty_cache()
    fr = [x["frac"] for x in shapes]
    return {"what": "mla_decode_attn alone (plan + split + combine), one layer, 128 heads, "
                    f"{warmup} warm-up + {iters} timed calls per shape, L2 flushed before each, "
                    "median; roofline against the burst peaks",
            "shapes": [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in x.items()}
                       for x in shapes],
            "min_frac": min(fr), "max_frac": max(fr), "target_frac": 0.7,
            "meets_target": min(fr) >= 0.7}


def run_extra_configs(dev, peaks, steps=10):
    """The single-layer configurations beside the headline: each one decode step (append +
    absorbed query + attention + W_UV/W_O) timed over `steps` eager steps, its split-KV kernel
    timed by CUDA events on its stream, and a parity sample against the oracle."""
    import mla_latent_kv_37_b200 as M
    from mla_latent_kv_37_b200.step import DecodeStep
    out = {}
    for name, n_seqs, n_heads in EXTRA_CONFIGS:
        cfg = dict(CONFIGS[name])
        B, H, D = cfg["batch"], cfg["heads"], cfg["d_model"]
        layers, h, pos, lens_dev, lens = make_workload(cfg, dev, seed=7)
        step = DecodeStep(layers, B, H, D, device=dev, graph=False,
                          query_remainder=cfg.get("remainder", False))
        for _ in range(3):
            step.run(h, pos, lens_dev)
        torch.cuda.synchronize()
        ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        M.mla_set_profile_events(ev_b, ev_e)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            step.run(h, pos, lens_dev)
        e1.record()
        torch.cuda.synchronize()
        used = M.mla_profile_events_used()
        M.mla_set_profile_events([], [])
        st = M.mla_get_status()
        if st:
            raise RuntimeError(f"device status {st:#x} in config {name}")
        ms = e0.elapsed_time(e1) / steps
        split_s = sorted(b.elapsed_time(e) for b, e in zip(ev_b[:used], ev_e[:used]))
        split_s = split_s[len(split_s) // 2] / 1e3
        r = attention_roofline(sum(lens), B, H, split_s, peaks, sustained=False)
        par = parity_sample(layers, h, [n - 1 for n in lens], step, cfg, n_layers=1,
                            n_seqs=n_seqs, n_heads=n_heads, seed=1)
        out[name] = {"workload": cfg["workload"], "batch": B, "tokens_read": sum(lens),
                     "ms_per_step": ms, "tokens_per_s": B / (ms / 1e3),
                     "attention": {k: r[k] for k in ("us", "roofline_us", "frac", "bound",
                                                     "gbs", "tflops")},
                     "query_remainder": bool(cfg.get("remainder", False)), "parity": par}
        del layers, h, pos, lens_dev, step
        torch.cuda.empty_cache()
    return out


def graph_us_per_call(call, n_layers, reps=10):
    """Median device time of one call, from replays of a CUDA graph holding call(0) ..
    call(n_layers - 1) back to back (each layer its own weights, together larger than L2): no
    host launch cost in the timed region, and every call streams its weights from HBM."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for l in range(n_layers):  # eager once: the library's one-time set-up stays outside
            call(l)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for l in range(n_layers):
            call(l)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3 / n_layers)
    del g
    return sorted(ts)[len(ts) // 2]


def _nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


def _weight_rate(us, wbytes, peaks):
    gbs = wbytes / (us * 1e-6) / 1e9
    return {"us_per_layer": us, "weight_bytes_per_layer": wbytes, "gbs": gbs,
            "hbm_frac": gbs / peaks.get("hbm_gbs", 6650.0)}


def run_execution_modes(dev, peaks, n_layers=3, B=32, H=128, D=7168):
    """The projections of one layer (cache append + query, then the output product) in the
    absorbed form the step uses and in the folded form (W_UK multiplied into W_Q and W_UV into
    W_O ahead of time): time per layer and weight bytes streamed.  Attention is the same in
    both and is not timed here."""
    import mla_latent_kv_37_b200 as M
    import mla_inputs as I
    d = M.dims(B, H, D)
    ws_ = [I.weights(11 + l, H, D, device=dev) for l in range(n_layers)]
    h = I.hidden(12, B, D, device=dev)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    table = torch.arange(B, dtype=torch.int32, device=dev).view(B, 1)
    pool = torch.zeros(B, 64, 576, dtype=torch.bfloat16, device=dev)
    sq, so = M.fold_shapes(d)
    folded_w = []
    for w in ws_:
        w_qf = torch.empty(sq, dtype=torch.bfloat16, device=dev)
        w_of = torch.empty(so, dtype=torch.bfloat16, device=dev)
        M.mla_fold_weights(d, w_q=w.w_q, w_uk=w.w_uk, w_uv=w.w_uv, w_o=w.w_o, w_qf=w_qf,
                           w_of=w_of)
        folded_w.append((w_qf, w_of))
    ws = M.workspace(d, 0, dev)
    q_cat = torch.empty(B, H, 576, dtype=torch.bfloat16, device=dev)
    o_lat = torch.randn(B, H, 512, dtype=torch.float32, device=dev)
    o_heads = torch.empty(B, H, 128, dtype=torch.bfloat16, device=dev)
    out = torch.empty(B, D, dtype=torch.bfloat16, device=dev)

    def absorbed(l):
        w = ws_[l]
        M.mla_append_absorb(d, h, w.w_dkv, w.w_kr, w.w_q, w.w_uk, pos, table, pool, q_cat, ws)
        M.mla_out_proj(d, o_lat, w.w_uv, ws, w_o=w.w_o, o_heads=o_heads, out=out)

    def folded(l):
        w, (w_qf, w_of) = ws_[l], folded_w[l]
        M.mla_append_absorb_folded(d, h, w.w_dkv, w.w_kr, w_qf, pos, table, pool, q_cat, ws)
        M.mla_out_proj_folded(d, o_lat, w_of, out, ws)

    w0, (qf0, of0) = ws_[0], folded_w[0]
    res = {"absorbed": _weight_rate(graph_us_per_call(absorbed, n_layers),
                                    _nbytes(w0.w_dkv, w0.w_kr, w0.w_q, w0.w_uk, w0.w_uv, w0.w_o),
                                    peaks),
           "folded": _weight_rate(graph_us_per_call(folded, n_layers),
                                  _nbytes(w0.w_dkv, w0.w_kr, qf0, of0), peaks)}
    st = M.mla_get_status()
    if st:
        raise RuntimeError(f"device status {st:#x} in the execution-mode measurement")
    res["what"] = ("projections of one layer (cache append + query, output product) at "
                   f"B={B}, H={H}, D={D}: CUDA-graph replay of {n_layers} layers with their own "
                   "weights, median of 10; attention is identical in both")
    res["folded_over_absorbed_time"] = res["folded"]["us_per_layer"] / res["absorbed"]["us_per_layer"]
    del ws_, folded_w, ws
    torch.cuda.empty_cache()
    return res


def run_fp8_weights(dev, peaks, n_layers=4, B=32, H=128, D=7168):
    """The two projection calls of one layer with bf16 weights and with W_DKV, W_KR, W_Q and W_O
    stored as E4M3 codes + row scales (one byte per weight streamed from HBM): time per call
    and the weight bytes it streams."""
    import mla_latent_kv_37_b200 as M
    import mla_inputs as I
    from mla_latent_kv_37_b200.step import Layer, quantize_layer
    d = M.dims(B, H, D)
    h = I.hidden(14, B, D, device=dev)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    table = torch.arange(B, dtype=torch.int32, device=dev).view(B, 1)
    pool = torch.zeros(B, 64, 576, dtype=torch.bfloat16, device=dev)
    lys = []
    for l in range(n_layers):
        w = I.weights(13 + l, H, D, device=dev)
        lys.append(quantize_layer(Layer(w.w_dkv, w.w_kr, w.w_q, w.w_uk, w.w_uv, w.w_o, pool,
                                        table)))
    ws = M.workspace(d, 0, dev)
    q_cat = torch.empty(B, H, 576, dtype=torch.bfloat16, device=dev)
    o_lat = torch.randn(B, H, 512, dtype=torch.float32, device=dev)
    out = torch.empty(B, D, dtype=torch.bfloat16, device=dev)
    calls = {
        "append_absorb": (
            lambda l: M.mla_append_absorb(d, h, lys[l].w_dkv, lys[l].w_kr, lys[l].w_q,
                                          lys[l].w_uk, pos, table, pool, q_cat, ws),
            lambda l: M.mla_append_absorb_fp8(d, h, lys[l].e4m3["w_dkv"], lys[l].e4m3["w_kr"],
                                              lys[l].e4m3["w_q"], lys[l].w_uk, pos, table, pool,
                                              q_cat, ws),
            ("w_dkv", "w_kr", "w_q"), ("w_uk",)),
        "out_proj": (
            lambda l: M.mla_out_proj(d, o_lat, lys[l].w_uv, ws, w_o=lys[l].w_o, out=out),
            lambda l: M.mla_out_proj_fp8(d, o_lat, lys[l].w_uv, lys[l].e4m3["w_o"][0],
                                         lys[l].e4m3["w_o"][1], out, ws),
            ("w_o",), ("w_uv",)),
    }
    res = {}
    ly0 = lys[0]
    for name, (f_bf16, f_e4m3, quant, kept) in calls.items():
        kept_b = _nbytes(*[getattr(ly0, k) for k in kept])
        res[name] = {
            "bf16": _weight_rate(graph_us_per_call(f_bf16, n_layers),
                                 kept_b + _nbytes(*[getattr(ly0, k) for k in quant]), peaks),
            "e4m3": _weight_rate(graph_us_per_call(f_e4m3, n_layers),
                                 kept_b + sum(_nbytes(*ly0.e4m3[k]) for k in quant), peaks)}
        res[name]["e4m3_over_bf16_time"] = (res[name]["e4m3"]["us_per_layer"] /
                                            res[name]["bf16"]["us_per_layer"])
    st = M.mla_get_status()
    if st:
        raise RuntimeError(f"device status {st:#x} in the E4M3 measurement")
    res["what"] = (f"the projection calls of one layer at B={B}, H={H}, D={D}: CUDA-graph replay "
                   f"of {n_layers} layers with their own weights, median of 10 (W_UK and W_UV "
                   "stay bf16 in both)")
    del lys, ws
    torch.cuda.empty_cache()
    return res


def run_fp8_step(layers, h, pos, lens_dev, lens, cfg, dev, steps):
    """The headline step with W_DKV, W_KR, W_Q and W_O of every layer stored as E4M3 (the rest
    unchanged): tokens/s from CUDA-graph replays, and a parity sample against the oracle run
    with the weights the codes stand for."""
    import numpy as np
    import mla_latent_kv_37_b200 as M
    from oracle import mla_oracle as O
    from mla_latent_kv_37_b200.step import DecodeStep, quantize_layer
    B, H, D = cfg["batch"], cfg["heads"], cfg["d_model"]
    q_layers = [quantize_layer(ly) for ly in layers]
    step = DecodeStep(q_layers, B, H, D, device=dev, graph=True)
    for _ in range(3):
        step.run(h, pos, lens_dev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step.run(h, pos, lens_dev)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    # end to end through the native executor, host buffers in and out (as the headline's e2e)
    h_host = h.cpu().pin_memory()
    pos_host, lens_host = pos.cpu().pin_memory(), lens_dev.cpu().pin_memory()
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    for _ in range(2):
        step.run_native(h_host, pos_host, lens_host, out_host)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(steps):
        step.run_native(h_host, pos_host, lens_host, out_host)
    f1.record()
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1) / steps
    st = M.mla_get_status()
    if st:
        raise RuntimeError(f"device status {st:#x} in the E4M3 step")
    # parity: layer 0, sequence 0, 8 heads, oracle with the dequantized weights
    ly, b = q_layers[0], 0
    hist = lens[b] - 1
    w, hb, rows = oracle_sample_inputs(ly, h[0], b, hist)
    for name in ("w_dkv", "w_kr", "w_q", "w_o"):
        codes, scale = ly.e4m3[name]
        n_rows, n_cols = getattr(ly, name).shape
        setattr(w, name, O.dequantize_rows_e4m3(
            M.fp8_codes_rows(codes, n_rows, n_cols).cpu().numpy(), scale.cpu().numpy()))
    heads = list(range(0, H, max(1, H // 8)))[:8]
    to_bf16 = lambda r: torch.from_numpy(np.asarray(r, dtype=np.float32)).to(torch.bfloat16)
    ref = O.decode_step(hb, w, rows, hist, H, round_row=to_bf16, heads=heads, with_out=False)
    got = step.o_heads[0, b][heads].float().cpu().numpy().astype(np.float64)
    exp = ref["o_heads"]
    rel = float(np.linalg.norm(got - exp) / np.linalg.norm(exp))
    mx = float(np.abs(got - exp).max() / np.abs(exp).max())
    res = {"value": B / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "launch": "CUDA graph of the step",
           "e2e": {"value": B / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": h_host.numel() * h_host.element_size() + 2 * B * 4,
                   "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
                   "path": "mla_decode_step_host with E4M3 layers"},
           "what": "the headline step with W_DKV, W_KR, W_Q, W_O in E4M3 (W_UK, W_UV bf16; "
                   "cache bf16)",
           "parity": {"o_heads_rel_l2": rel, "o_heads_max_abs": mx,
                      "samples": "layer 0, sequence 0, 8 heads; oracle with the dequantized "
                                 "weights",
                      "pass": rel <= 5e-3 and mx <= 2e-2}}
    del step, q_layers
    torch.cuda.empty_cache()
    return res


def config_block(cfg, lens, world):
    """The workload description both arms print (identical for the same configuration)."""
    B, L = cfg["batch"], cfg["layers"]
    tokens = sum(lens)
    return {"workload": cfg["workload"], "batch": B,
            "context": lens[0] if cfg["context"] else "U[1024,8192]", "layers": L,
            "heads": cfg["heads"], "d_model": cfg["d_model"], "d_c": 512, "d_rope": 64,
            "page_size": 64, "global_batch": B * world, "parallelism": f"replicas x{world}",
            "l2": "no flush: inputs per step exceed L2 "
                  f"({(tokens * ROW_BYTES * L + 0.629e9 * L) / 1e9:.0f} GB vs 0.126 GB)"}


# ---------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The oracle arm: times the fp64 CPU oracle on bounded samples of the same workload."""
    if rank != 0:
        return
    import numpy as np
    import mla_inputs as I
    cfg = CONFIGS[args.config]
    B, H, D = cfg["batch"], cfg["heads"], cfg["d_model"]
    lens = context_lengths(cfg, 4)
    n = lens[0]
    w = I.weights(4000, H, D, torch.bfloat16)
    h = I.hidden(4900, 1, D)[0]
    g = I.generator(4500)
    hist = torch.randn(n - 1, 576, generator=g).to(torch.bfloat16)
    per_step = []
    heads_timed = 0
    for i in range(args.warmup + args.steps):
        budget = args.ref_seconds or max(2.0, min(20.0, 150.0 / max(1, args.warmup + args.steps)))
        t, heads_timed, wall = time_oracle(w, h, hist, n - 1, H, budget_s=budget)
        if i >= args.warmup:
            per_step.append(t)
    sec = float(np.mean(per_step))
    cb = cpu_baseline_from(sec, cfg, heads_timed, wall)
    step_s = sec * B * cfg["layers"]
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, lens, world),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="full_61", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (profiling runs on a slice of the workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-check", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other single-layer configurations and the attention sweep")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel eagerly instead of replaying a captured step")
    ap.add_argument("--ref-seconds", type=float, default=0.0,
                    help="reference arm: CPU seconds per timed sample (0 = fit a few minutes)")
    ap.add_argument("--sweep", action="store_true",
                    help="time mla_decode_attn alone on one layer over batch {32,64,128} x "
                         "context {8K,16K,32K} (one JSON line per shape) instead of the step")
    ap.add_argument("--sweep-warmup", type=int, default=10)
    ap.add_argument("--sweep-iters", type=int, default=50)
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        # the CPU oracle arm: rank 0 alone runs it; under torchrun the other ranks exit at once
        run_reference(args, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup()
    args.warmup = max(args.warmup, 3)
    from mla_latent_kv_37_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    import mla_latent_kv_37_b200 as M
    from mla_latent_kv_37_b200.step import DecodeStep
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = dict(CONFIGS[args.config])
    if args.layers:
        cfg["layers"] = args.layers
        cfg["workload"] += f" [sliced to {args.layers} layers]"
    B, H, D, L = cfg["batch"], cfg["heads"], cfg["d_model"], cfg["layers"]
    t_gen = time.time()
    layers, h, pos, lens_dev, lens = make_workload(cfg, dev, seed=4 + rank)
    torch.cuda.synchronize()
    log(f"[bench] rank {rank}: workload ready in {time.time() - t_gen:.1f} s, "
        f"{torch.cuda.memory_allocated() / 1e9:.1f} GB on device")
    graph = not args.no_graph
    step = DecodeStep(layers, B, H, D, num_splits=args.num_splits, device=dev, graph=graph)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step.run(h, pos, lens_dev)
    torch.cuda.synchronize()
    st = M.mla_get_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after warm-up")

    # ---------------- timed region (device-resident inputs) ----------------
    # CUDA events around every split-kernel launch, on the stream it runs on.  In graph mode
    # the events are captured into the step's graph and re-recorded by every replay: after
    # the timed steps they hold the last step's L launches.
    n_prof = L if graph else args.steps * L
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(n_prof)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(n_prof)]
    if graph:
        step.capture(h, pos, lens_dev,
                     before_capture=lambda: M.mla_set_profile_events(ev_b, ev_e))
        used = M.mla_profile_events_used()
        M.mla_set_profile_events([], [])
        for _ in range(2):
            step.run(h, pos, lens_dev)
        torch.cuda.synchronize()
    else:
        M.mla_set_profile_events(ev_b, ev_e)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = M.mla_launch_count()
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step.run(h, pos, lens_dev)
    e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    launches = (step.launches_per_step * args.steps if graph
                else M.mla_launch_count() - launches0)
    barrier(world)
    clocks = sampler.stop(t_wall0, t_wall1)
    if not graph:
        used = M.mla_profile_events_used()
        M.mla_set_profile_events([], [])
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    split_ms = [b.elapsed_time(e) for b, e in zip(ev_b[:used], ev_e[:used])]
    st = M.mla_get_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after timed steps")
    tokens_per_step = B * world
    value = tokens_per_step / (ms / 1e3)

    # ---------------- roofline of the dominant kernel (split-KV decode) ----------------
    peaks = load_peaks()
    peak_src = "of measured" if peaks else "of fallback"
    tokens_read = sum(lens)
    avg_split_s = (sum(split_ms) / len(split_ms)) / 1e3 if split_ms else float("nan")
    # the kernel runs inside a long step: the sustained tensor rate is its ceiling
    r = attention_roofline(tokens_read, B, H, avg_split_s, peaks, sustained=True)
    traffic = committed_traffic(args.config)
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    tc_peak = peaks.get("bf16_tflops_sustained", 1400.0)
    roofline = {"bound": r["bound"],
                "achieved": r["gbs"] if r["bound"] == "hbm" else r["tflops"],
                "peak": hbm_peak if r["bound"] == "hbm" else tc_peak,
                "unit": "GB/s" if r["bound"] == "hbm" else "TFLOP/s",
                "frac": r["frac"],
                "traffic": traffic,
                "kernel": "mla::attn::split_kernel",
                "peak_source": peak_src + (" (HBM copy)" if r["bound"] == "hbm" else
                                           " (sustained bf16 GEMM)"),
                "us_per_launch": r["us"],
                "hbm_gbs": r["gbs"], "hbm_frac": r["hbm_frac"],
                "tflops": r["tflops"],
                "tensor_frac": r["tensor_frac_sustained"],
                "tensor_frac_label": f"achieved TFLOP/s / sustained bf16 GEMM rate, {peak_src}",
                "tensor_frac_burst": r["tensor_frac_burst"],
                "tensor_frac_burst_label": f"achieved TFLOP/s / burst bf16 dense GEMM rate (the "
                                           f"dense peak a kernel timed alone reaches), {peak_src}",
                "bytes_per_launch": r["bytes"], "flops_per_launch": r["flops"],
                "roofline_us": r["roofline_us"],
                "frac_of_roofline_time": r["frac"]}

    # ---------------- end-to-end through the API with host buffers ----------------
    # The headline: the library's native step executor (mla_decode_step_host, one C-ABI call
    # per step: page-locked host inputs in, every copy and launch made in C++, `out` back in
    # host memory).  Beside it, the same step through the Python runner's host path replayed
    # as one CUDA graph.
    e2e = None
    if not args.no_e2e:
        h_host = h.cpu().pin_memory()
        pos_host = pos.cpu().pin_memory()
        lens_host = lens_dev.cpu().pin_memory()
        out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
        bi = h_host.numel() * h_host.element_size() + 2 * B * 4
        bo = out_host.numel() * out_host.element_size()

        def timed(run):
            for _ in range(2):
                run()
            torch.cuda.synchronize()
            barrier(world)
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(args.steps):
                run()
            f1.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(f0.elapsed_time(f1) / args.steps, world)

        native_ms = timed(lambda: step.run_native(h_host, pos_host, lens_host, out_host))
        h_dev = torch.empty_like(h)
        p_dev, l_dev = torch.empty_like(pos), torch.empty_like(lens_dev)
        graph_ms = timed(lambda: step.run_host(h_host, pos_host, lens_host, out_host, h_dev,
                                               p_dev, l_dev))
        st = M.mla_get_status()
        if st:
            raise RuntimeError(f"device status {st:#x} in the end-to-end steps")
        e2e = {"value": tokens_per_step / (native_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": native_ms,
               "path": "mla_decode_step_host (C ABI, page-locked host buffers, eager launches)",
               "python_graph_host_path": {"value": tokens_per_step / (graph_ms / 1e3),
                                          "ms_per_step": graph_ms}}

    # ---------------- CPU oracle baseline and parity sample (rank 0) ----------------
    cpu = None
    parity = None
    if rank == 0 and not args.no_check:
        parity = parity_sample(layers, h, [n - 1 for n in lens], step, cfg)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        w, hb, rows = oracle_sample_inputs(layers[0], h[0], 0, lens[0] - 1)
        sec, heads_timed, wall = time_oracle(w, hb, rows, lens[0] - 1, H)
        cpu = cpu_baseline_from(sec, cfg, heads_timed, wall)

    # ---------------- the other configurations and the attention sweep (one GPU) ----------
    configs = sweep = modes = fp8w = fp8s = None
    if rank == 0 and world == 1 and not args.no_extras:
        if B <= 128:
            del step
            torch.cuda.empty_cache()
            fp8s = run_fp8_step(layers, h, pos, lens_dev, lens, cfg, dev, max(3, args.steps // 2))
        else:
            del step
        del layers, h
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        configs = run_extra_configs(dev, peaks)
        sweep = compact_sweep(dev, peaks)
        modes = run_execution_modes(dev, peaks)
        fp8w = run_fp8_weights(dev, peaks)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded: N(0,1) hidden states and cache history, "
                    "N(0,1/fan_in) weights, random page placement)",
            "config": config_block(cfg, lens, world),
            "launch": "CUDA graph of the step" if graph else "eager",
            "num_splits": args.num_splits or "auto",
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clocks, "parity": parity,
            "attention_us_per_layer": roofline["us_per_launch"],
            "configs": configs, "attention_sweep": sweep, "execution_modes": modes,
            "fp8_weights": fp8w, "fp8_weights_step": fp8s,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
