"""Benchmark of the Gemma-4-style attention hot path on B200.

One step = one pass of the whole hot path on synthetic data shaped like the pages' models:
  * the 5:1 interleaved block prefill at T = 65536 (five local layers: 32 q / 16 kv heads,
    head_dim 256, window 1024, RoPE base 1e4, separate values; one global layer: 32 q / 4 kv
    heads, head_dim 512, p-RoPE 0.25 at base 1e6, keys reused as values, full causal),
  * one global-layer decode step for 16 sequences against a 32768-token K(=V) cache.
`value` is the prefill throughput of the step (algorithmic FLOPs of the six layers over
their device time); the decode half of the metric (cache GB/s) rides along in `decode`.
Inputs are larger than L2 (126 MB), so no flush is needed between steps.

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank runs an independent replica (weak scaling, no collective
on the data path); timing is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attn TFLOP/s & decode KV GB/s on 1 B200, as % of BF16/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for name in ("prefill.cu", "sm100.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "attention_g4attn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_hash):
    """DRAM bytes per launch of the global prefill kernel from the committed ncu summary,
    valid only while the kernel sources still hash to the recorded value."""
    p = os.path.join(ROOT, "profiles", "prefill_global_T65536_traffic.md")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_hash") != kernel_hash:
        return None
    try:
        return float(vals["dram_bytes_per_full_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._thr = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(
                    ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                     "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
                parts = [x.strip() for x in out.stdout.strip().split(",")]
                if len(parts) >= 7:
                    self.samples.append(parts)
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thr.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4)
                          if s[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


# --------------------------------------------------------------------------- workload

def make_step(device, seed_base=0):
    """Device-resident inputs and outputs of one step, plus a callable that runs it."""
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads

    blk = workloads.BLOCK_5TO1_64K
    dec = workloads.GLOBAL_DECODE_32K
    layers = []
    for ly, seed in zip(blk.layers, blk.seeds):
        inp = synth.layer_inputs(blk.B, blk.T, ly.n_q_heads, ly.n_kv_heads, ly.head_dim,
                                 ly.separate_v, seed=seed + seed_base, device=device)
        cfg = b.LayerCfg.from_layer(ly)
        ws = torch.empty(b.g4attn_prefill_workspace_size(blk.B, blk.T, cfg), dtype=torch.uint8,
                         device=device)
        out = torch.empty_like(inp.q)
        layers.append((inp, cfg, ws, out))
    dly = dec.layer
    dinp = synth.decode_inputs(dec.B, dec.L, dly.n_q_heads, dly.n_kv_heads, dly.head_dim, False,
                               seed=100 + seed_base, device=device)
    dcfg = b.LayerCfg.from_layer(dly)
    dws = torch.empty(b.g4attn_decode_workspace_size(dec.B, dec.L, dcfg), dtype=torch.uint8,
                      device=device)
    dout = torch.empty_like(dinp.q)
    return dict(blk=blk, dec=dec, layers=layers, dinp=dinp, dcfg=dcfg, dws=dws, dout=dout)


def run_step(S, stream, ev=None):
    """Launch the step on `stream`; ev = list of 4 events (prefill start/end, decode
    start/end) recorded on the same stream when timing."""
    from attention_g4attn_b200 import binding as b
    if ev:
        ev[0].record(stream)
    for inp, cfg, ws, out in S["layers"]:
        b.g4attn_prefill(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, cfg, out=out,
                         workspace=ws, stream=stream)
    if ev:
        ev[1].record(stream)
        ev[2].record(stream)
    d = S["dinp"]
    b.g4attn_decode(d.q, d.k, None, S["dcfg"], out=S["dout"], workspace=S["dws"], stream=stream)
    if ev:
        ev[3].record(stream)


LAUNCHES_PER_STEP = 6 * 2 + 2   # per layer: key pre-pass + flash kernel; decode + combine


def time_global_32k(device, stream, reps=3):
    """Global-layer prefill at T=32768 alone (the workload of the prefill target)."""
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads
    wl = workloads.GLOBAL_PREFILL_32K
    ly = wl.layers[0]
    inp = synth.layer_inputs(wl.B, wl.T, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                             seed=7, device=device)
    cfg = b.LayerCfg.from_layer(ly)
    ws = torch.empty(b.g4attn_prefill_workspace_size(wl.B, wl.T, cfg), dtype=torch.uint8,
                     device=device)
    out = torch.empty_like(inp.q)
    for _ in range(2):
        b.g4attn_prefill(inp.q, inp.k, None, inp.gamma_q, inp.gamma_k, cfg, out=out,
                         workspace=ws, stream=stream)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        b.g4attn_prefill(inp.q, inp.k, None, inp.gamma_q, inp.gamma_k, cfg, out=out,
                         workspace=ws, stream=stream)
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    t = statistics.median(ts)
    return {"workload": wl.name, "ms": t * 1e3, "tflops": wl.flops() / t / 1e12}


def time_decode_128k(device, stream, reps=5):
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads
    wl = workloads.GLOBAL_DECODE_128K
    ly = wl.layer
    d = synth.decode_inputs(wl.B, wl.L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                            seed=8, device=device)
    cfg = b.LayerCfg.from_layer(ly)
    ws = torch.empty(b.g4attn_decode_workspace_size(wl.B, wl.L, cfg), dtype=torch.uint8,
                     device=device)
    out = torch.empty_like(d.q)
    for _ in range(3):
        b.g4attn_decode(d.q, d.k, None, cfg, out=out, workspace=ws, stream=stream)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        b.g4attn_decode(d.q, d.k, None, cfg, out=out, workspace=ws, stream=stream)
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    t = statistics.median(ts)
    return {"workload": wl.name, "ms": t * 1e3, "gbs": wl.cache_bytes() / t / 1e9}


def time_local_ring_decode(device, stream, reps=10, rotated=False):
    """Decode step of the block's local layer (32 q / 16 kv heads, d 256, window 1024,
    separate values) for 16 sequences at position 65535, against ring caches of 1024 rows:
    the keys and values of the window, each read once.  rotated: the ring holds the keys
    turned to their positions (g4attn_decode_rotated), so none is turned on the fly."""
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads
    ly = workloads.LOCAL_W1024
    B, L, C = 16, 65536, 1024
    d = synth.decode_inputs(B, C, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, True, seed=9,
                            device=device)   # the ring's rows are random: any ring content works
    cfg = b.LayerCfg.from_layer(ly)
    ws = torch.empty(b.g4attn_decode_ring_workspace_size(B, L, C, cfg), dtype=torch.uint8,
                     device=device)
    out = torch.empty_like(d.q)
    def call():
        if rotated:
            b.g4attn_decode_rotated(d.q, d.k, d.v, L, cfg, ring=True, out=out, workspace=ws,
                                    stream=stream)
        else:
            b.g4attn_decode_ring(d.q, d.k, d.v, L, cfg, out=out, workspace=ws, stream=stream)

    for _ in range(3):
        call()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    t = statistics.median(ts)
    nbytes = 2.0 * B * ly.n_kv_heads * ly.window * ly.head_dim * 2
    name = "local_decode_ring%s_B16_pos65535_C1024_h32x16_d256_w1024" % ("_turned_keys" if rotated else "")
    return {"workload": name, "ms": t * 1e3, "gbs": nbytes / t / 1e9}


def time_decode_graph(device, reps=20):
    """The global decode step (B=16, L=32768) captured once in a CUDA graph and replayed back
    to back: the per-step time without host launch overhead (serving loops replay a captured
    decode step)."""
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads
    ly = workloads.GLOBAL_8TO1
    B, L = 16, 32768
    d = synth.decode_inputs(B, L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=7,
                            device=device)
    cfg = b.LayerCfg.from_layer(ly)
    ws = torch.empty(b.g4attn_decode_workspace_size(B, L, cfg), dtype=torch.uint8, device=device)
    out = torch.empty_like(d.q)
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        for _ in range(3):
            b.g4attn_decode(d.q, d.k, None, cfg, out=out, workspace=ws)
    torch.cuda.current_stream(device).wait_stream(side)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        b.g4attn_decode(d.q, d.k, None, cfg, out=out, workspace=ws)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    e1.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    assert b.g4attn_device_status() == 0
    del g
    return {"workload": "global_decode_B16_L32768_h32x4_d512_cuda_graph_replay", "ms": t * 1e3,
            "gbs": B * ly.n_kv_heads * L * ly.head_dim * 2 / t / 1e9}


def time_chunked_prefill(device, stream, chunk=4096, reps=3):
    """The global layer's T = 32768 prefill (32 q / 4 kv heads, d 512, causal) fed as
    chunks of `chunk` tokens, each against the linear cache the earlier chunks wrote
    (g4attn_prefill_chunk): the time of the whole sequence of calls, and of the last chunk
    (the 4096 queries at positions 28672 .. 32767 against all 32768 keys)."""
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads
    ly = workloads.GLOBAL_8TO1
    T = 32768
    inp = synth.layer_inputs(1, T, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=21,
                             device=device)
    cfg = b.LayerCfg.from_layer(ly)
    gq, gk = inp.gamma_q.to(device), inp.gamma_k.to(device)
    kc = torch.empty((1, T, ly.n_kv_heads, ly.head_dim), dtype=torch.bfloat16, device=device)
    out = torch.empty_like(inp.q)
    ws = torch.empty(b.g4attn_prefill_chunk_workspace_size(1, T - chunk, chunk, cfg),
                     dtype=torch.uint8, device=device)
    cuts = list(range(0, T + 1, chunk))
    pieces = [(P, inp.q[:, P:P + chunk], inp.k[:, P:P + chunk], out[:, P:P + chunk])
              for P in cuts[:-1]]

    def one(P, q, k, o):
        b.g4attn_prefill_chunk(q, k, None, gq, gk, kc, None, P, cfg, out=o, workspace=ws,
                               stream=stream)

    def timed(calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for c in calls:
            one(*c)
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3

    for _ in range(2):
        timed(pieces)
    t_all = statistics.median([timed(pieces) for _ in range(reps)])
    t_last = statistics.median([timed(pieces[-1:]) for _ in range(reps)])
    assert b.g4attn_device_status(stream) == 0
    flops_all = 4.0 * ly.head_dim * ly.n_q_heads * workloads.visible_pairs(T, 0)
    P = T - chunk
    flops_last = 4.0 * ly.head_dim * ly.n_q_heads * (chunk * P + chunk * (chunk + 1) / 2)
    return {"workload": "global_prefill_T32768_in_chunks_of_%d_h32x4_d512" % chunk,
            "ms_all_chunks": t_all * 1e3, "tflops_all_chunks": flops_all / t_all / 1e12,
            "ms_last_chunk": t_last * 1e3, "tflops_last_chunk": flops_last / t_last / 1e12}


# --------------------------------------------------------------------------- CPU oracle

def oracle_sample(max_seconds=20.0, seed=0):
    """Time the fp64 oracle on a bounded sample of the step: query rows of the global layer
    of the block (all 32 heads) against their full causal prefix of T=65536 keys.  Only the
    sampled query rows are drawn (the rest of q stays untouched zero pages); keys are drawn
    in full.  Returns (TFLOP/s, info, seconds)."""
    import numpy as np
    import torch
    import oracle
    from attention_g4attn_b200 import workloads

    blk = workloads.BLOCK_5TO1_64K
    ly = blk.layers[5]
    gen = torch.Generator().manual_seed(1234 + seed)
    k = torch.randn((blk.B, blk.T, ly.n_kv_heads, ly.head_dim), generator=gen).bfloat16()
    kb = oracle.bf16_bits(k)
    gq = (1.0 + 0.1 * torch.randn(ly.head_dim, generator=gen)).numpy()
    gk = (1.0 + 0.1 * torch.randn(ly.head_dim, generator=gen)).numpy()
    qb = np.zeros((blk.B, blk.T, ly.n_q_heads, ly.head_dim), np.uint16)
    cfg = oracle.OracleCfg(ly.n_q_heads, ly.n_kv_heads, ly.head_dim, ly.rope_p, ly.rope_base,
                           ly.window, ly.scale, ly.kv_is_k, ly.qk_norm, ly.qk_norm_eps)
    rng = np.random.default_rng(seed)
    nrows = 1
    flops = 0.0
    done_rows = 0
    t_total = 0.0
    while t_total < max_seconds and nrows <= 64:
        rows = np.sort(rng.integers(blk.T // 2, blk.T, size=nrows)).astype(np.int32)
        for r in rows:
            qr = torch.randn((blk.B, ly.n_q_heads, ly.head_dim), generator=gen).bfloat16()
            qb[:, r] = oracle.bf16_bits(qr)
        t0 = time.perf_counter()
        oracle.prefill_rows(qb, kb, None, gq, gk, cfg, rows)
        t_total += time.perf_counter() - t0
        flops += float(sum(4.0 * ly.head_dim * ly.n_q_heads * (int(r) + 1) for r in rows))
        done_rows += nrows
        nrows *= 2
    cores = os.cpu_count() or 1
    info = {"kind": "oracle", "cores": cores,
            "sample": "%d query rows x 32 heads of the block's global layer (T=65536, causal "
                      "prefix of each row, key normalisation included)" % done_rows}
    return flops / t_total / 1e12, info, t_total


# --------------------------------------------------------------------------- main

CASES = {
    # small cases for profiler captures: inputs larger than L2, a few GB on the device
    "global_prefill_T8192": ("prefill", dict(B=1, T=8192, layer="GLOBAL_8TO1")),
    "global_prefill_T65536": ("prefill", dict(B=1, T=65536, layer="GLOBAL_8TO1")),
    "local_prefill_T16384": ("prefill", dict(B=1, T=16384, layer="LOCAL_W1024")),
    "global_decode_L8192": ("decode", dict(B=16, L=8192, layer="GLOBAL_8TO1")),
    "global_decode_L32768": ("decode", dict(B=16, L=32768, layer="GLOBAL_8TO1")),
    # the local layer's decode at position 65535 over rings of 1024 rows (1.07 GB of window)
    "local_decode_ring_B64": ("ring", dict(B=64, L=65536, C=1024, layer="LOCAL_W1024")),
    "local_decode_ring_turned_B64": ("ring_turned", dict(B=64, L=65536, C=1024,
                                                         layer="LOCAL_W1024")),
}


def run_case(name, steps, warmup):
    """One named workload alone, `steps` timed calls (used under profilers)."""
    import torch
    from attention_g4attn_b200 import binding as b, synth, workloads
    kind, p = CASES[name]
    ly = getattr(workloads, p["layer"])
    dev = torch.device("cuda:0")
    stream = torch.cuda.Stream(dev)
    cfg = b.LayerCfg.from_layer(ly)
    if kind == "prefill":
        inp = synth.layer_inputs(p["B"], p["T"], ly.n_q_heads, ly.n_kv_heads, ly.head_dim,
                                 ly.separate_v, seed=3, device=dev)
        ws = torch.empty(b.g4attn_prefill_workspace_size(p["B"], p["T"], cfg), dtype=torch.uint8,
                         device=dev)
        out = torch.empty_like(inp.q)

        def call():
            b.g4attn_prefill(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, cfg, out=out,
                             workspace=ws, stream=stream)
        work = 4.0 * ly.head_dim * ly.n_q_heads * p["B"] * workloads.visible_pairs(p["T"], ly.window)
        unit = "TFLOP/s"
    elif kind in ("ring", "ring_turned"):
        # the ring's rows are random draws: any ring content is a valid cache
        d = synth.decode_inputs(p["B"], p["C"], ly.n_q_heads, ly.n_kv_heads, ly.head_dim, True,
                                seed=3, device=dev)
        ws = torch.empty(b.g4attn_decode_ring_workspace_size(p["B"], p["L"], p["C"], cfg),
                         dtype=torch.uint8, device=dev)
        out = torch.empty_like(d.q)

        def call():
            if kind == "ring":
                b.g4attn_decode_ring(d.q, d.k, d.v, p["L"], cfg, out=out, workspace=ws,
                                     stream=stream)
            else:
                b.g4attn_decode_rotated(d.q, d.k, d.v, p["L"], cfg, ring=True, out=out,
                                        workspace=ws, stream=stream)
        work = float(2 * p["B"] * ly.n_kv_heads * ly.window * ly.head_dim * 2) * 1e3   # -> GB/s
        unit = "GB/s"
    else:
        d = synth.decode_inputs(p["B"], p["L"], ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                                seed=3, device=dev)
        ws = torch.empty(b.g4attn_decode_workspace_size(p["B"], p["L"], cfg), dtype=torch.uint8,
                         device=dev)
        out = torch.empty_like(d.q)

        def call():
            b.g4attn_decode(d.q, d.k, None, cfg, out=out, workspace=ws, stream=stream)
        work = float(p["B"] * ly.n_kv_heads * p["L"] * ly.head_dim * 2) * 1e3   # -> GB/s
        unit = "GB/s"
    for _ in range(warmup):
        call()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    e1.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / steps
    assert b.g4attn_device_status(stream) == 0
    print(json.dumps({"case": name, "ms": t * 1e3, "value": work / t / 1e12, "unit": unit}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=sorted(CASES), default=None,
                    help="time one small workload alone (profiler captures)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="g4attn", choices=["g4attn", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.case:
        run_case(args.case, max(args.steps, 1), max(args.warmup, 0))
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        v, info, secs = oracle_sample(max_seconds=20.0)
        steps = max(args.steps, 1)
        info["value"] = v
        line = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": steps, "warmup": args.warmup, "ms_per_step": secs * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": {"workload": "block_5local_1global_T65536+global_decode_B16_L32768",
                           "sample": info["sample"]},
                "impl": "reference", "cpu_baseline": info,
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    from attention_g4attn_b200 import replicas
    dist, rank, world, local_rank = replicas.init_from_env("nccl")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    from attention_g4attn_b200 import binding as b  # noqa: F401  (fails loudly without the .so)

    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        S = make_step(device, seed_base=rank)
    stream.synchronize()

    for _ in range(max(args.warmup, 0)):
        run_step(S, stream)
    stream.synchronize()
    assert b.g4attn_device_status(stream) == 0

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for k in range(args.steps):
            run_step(S, stream, ev[k])
        t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    status = b.g4attn_device_status(stream)
    total_s = t_start.elapsed_time(t_end) / 1e3
    pre_s = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    dec_s = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    total_s, pre_s, dec_s = replicas.max_over_ranks([total_s, pre_s, dec_s], dist, device)

    blk, dec = S["blk"], S["dec"]
    flops_step = blk.flops()
    value = replicas.job_rate(flops_step * args.steps, pre_s, world, 1e12)
    dec_gbs = replicas.job_rate(dec.cache_bytes() * args.steps, dec_s, world, 1e9)
    peaks, peak_src = load_peaks()
    tf_peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    # dominant kernel: the global layer of the block (about 93% of the step's FLOPs)
    g_inp, g_cfg, g_ws, g_out = S["layers"][5]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gt = []
    for _ in range(3):
        e0.record(stream)
        b.g4attn_prefill(g_inp.q, g_inp.k, None, g_inp.gamma_q, g_inp.gamma_k, g_cfg, out=g_out,
                         workspace=g_ws, stream=stream)
        e1.record(stream)
        e1.synchronize()
        gt.append(e0.elapsed_time(e1) / 1e3)
    g_s = statistics.median(gt)
    from attention_g4attn_b200 import workloads
    g_flops = 4.0 * 512 * 32 * blk.B * workloads.visible_pairs(blk.T, 0)
    khash = kernel_source_hash()
    roofline = {"bound": "tensor", "achieved": g_flops / g_s / 1e12, "peak": tf_peak,
                "unit": "TFLOP/s", "frac": g_flops / g_s / 1e12 / tf_peak,
                "traffic": recorded_traffic(khash),
                "kernel": "prefill_kernel<512> (+ key pre-pass) on the block's global layer",
                "peak_source": "%s bf16_tflops_sustained" % peak_src}

    extra = {}
    if rank == 0:
        extra["global_prefill_T32768"] = time_global_32k(device, stream)
        extra["global_prefill_T32768"]["frac_of_sustained"] = \
            extra["global_prefill_T32768"]["tflops"] / tf_peak
        extra["global_prefill_T32768"]["frac_of_burst"] = \
            extra["global_prefill_T32768"]["tflops"] / float(peaks.get("bf16_tflops", 1590.0))
        extra["global_decode_L131072"] = time_decode_128k(device, stream)
        extra["global_decode_L131072"]["frac_of_hbm"] = \
            extra["global_decode_L131072"]["gbs"] / hbm_peak
        extra["local_decode_ring"] = time_local_ring_decode(device, stream)
        extra["local_decode_ring"]["frac_of_hbm"] = extra["local_decode_ring"]["gbs"] / hbm_peak
        extra["local_decode_ring_turned_keys"] = time_local_ring_decode(device, stream, rotated=True)
        extra["local_decode_ring_turned_keys"]["frac_of_hbm"] = \
            extra["local_decode_ring_turned_keys"]["gbs"] / hbm_peak
        extra["global_decode_L32768_graph"] = time_decode_graph(device)
        extra["global_decode_L32768_graph"]["frac_of_hbm"] = \
            extra["global_decode_L32768_graph"]["gbs"] / hbm_peak
        extra["chunked_prefill"] = time_chunked_prefill(device, stream)
        extra["chunked_prefill"]["frac_of_sustained"] = \
            extra["chunked_prefill"]["tflops_all_chunks"] / tf_peak

    # end to end through the public API with host buffers (pinned), copies inside the region
    e2e = None
    if not args.no_e2e:
        try:
            e2e = run_e2e(S, stream, device, steps=min(args.steps, 2))
        except RuntimeError as exc:   # pinned host memory refused
            e2e = {"error": str(exc)[:200]}
    if e2e is not None and "error" not in e2e:
        e2e["seconds"] = replicas.max_over_ranks([e2e["seconds"]], dist, device)[0]
        e2e = {"value": replicas.job_rate(flops_step * e2e["steps"], e2e["seconds"], world, 1e12),
               "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["h2d"],
               "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, info, _ = oracle_sample(max_seconds=15.0)
        info["value"] = v
        info["unit"] = "TFLOP/s"
        cpu = info

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_s * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "block_5local_1global_T65536+global_decode_B16_L32768",
                   "prefill": "5 x (32q/16kv, d256, window 1024, RoPE 1e4, separate v) + "
                              "1 x (32q/4kv, d512, p-RoPE 0.25 @ 1e6, K=V, causal), B=1, T=65536",
                   "decode": "B=16, 32q/4kv, d512, K=V cache L=32768",
                   "l2": "inputs larger than L2, no flush", "parallelism": "replicas"},
        "decode": {"value": dec_gbs, "unit": "GB/s", "frac": dec_gbs / world / hbm_peak,
                   "peak": hbm_peak, "peak_source": "%s hbm_gbs" % peak_src},
        "roofline": roofline,
        "clocks": clk.summary(),
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "device_status": status,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    line.update(extra)
    print(json.dumps(line))


def run_e2e(S, stream, device, steps):
    """The same step through the public API with inputs in pinned host memory: every step
    copies its inputs host->device, runs, and copies the outputs device->host."""
    import torch
    from attention_g4attn_b200 import binding as b

    def pin(t):
        return None if t is None else t.to("cpu").pin_memory()

    host = []
    h2d = d2h = 0
    for inp, cfg, ws, out in S["layers"]:
        hq, hk, hv = pin(inp.q), pin(inp.k), pin(inp.v)
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        host.append((hq, hk, hv, ho))
        h2d += sum(t.numel() * t.element_size() for t in (hq, hk, hv) if t is not None)
        d2h += ho.numel() * ho.element_size()
    d = S["dinp"]
    hdq, hdk = pin(d.q), pin(d.k)
    hdo = torch.empty(S["dout"].shape, dtype=S["dout"].dtype).pin_memory()
    h2d += hdq.numel() * 2 + hdk.numel() * 2
    d2h += hdo.numel() * 2
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            for (inp, cfg, ws, out), (hq, hk, hv, ho) in zip(S["layers"], host):
                inp.q.copy_(hq, non_blocking=True)
                inp.k.copy_(hk, non_blocking=True)
                if hv is not None:
                    inp.v.copy_(hv, non_blocking=True)
                b.g4attn_prefill(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, cfg, out=out,
                                 workspace=ws, stream=stream)
                ho.copy_(out, non_blocking=True)
            d.q.copy_(hdq, non_blocking=True)
            d.k.copy_(hdk, non_blocking=True)
            b.g4attn_decode(d.q, d.k, None, S["dcfg"], out=S["dout"], workspace=S["dws"],
                            stream=stream)
            hdo.copy_(S["dout"], non_blocking=True)
    e1.record(stream)
    e1.synchronize()
    secs = e0.elapsed_time(e1) / 1e3
    return {"seconds": secs, "steps": steps, "h2d": h2d, "d2h": d2h,
            "wall": time.perf_counter() - t0}


if __name__ == "__main__":
    main()
