"""Benchmark of the Gemma-4-style attention hot path on B200.

One step = one pass of the whole hot path on synthetic data shaped like the pages' models:
  * the 5:1 interleaved block prefill at T = 65536 (five local layers: 32 q / 16 kv heads,
    head_dim 256, window 1024, RoPE base 1e4, separate values; one global layer: 32 q / 4 kv
    heads, head_dim 512, p-RoPE 0.25 at base 1e6, keys reused as values, full causal),
  * one global-layer decode step for 16 sequences against a 32768-token K(=V) cache.
`value` is the prefill throughput of the step (algorithmic FLOPs of the six layers over
their device time); the decode half of the metric (cache GB/s) rides along in `decode`.
Inputs are larger than L2 (126 MB), so no flush is needed between steps.

--impl reference times the fp64 CPU oracle on the host cores, each step a bounded sample of
the same workload.  Multi-GPU: `--gpus N` runs N ranks (under torchrun, or re-launched as N
processes of torch.distributed.run when started plainly); every rank runs an independent
replica (weak scaling, no collective on the data path) and the timing is the max over ranks.
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


def _code_lines(text):
    """The lines of a C++ source without its // comments and blank lines (a // inside a
    string literal, i.e. after an odd number of quotes on the line, is kept)."""
    out = []
    for line in text.splitlines():
        cut = len(line)
        start = 0
        while True:
            i = line.find("//", start)
            if i < 0:
                break
            if line.count('"', 0, i) % 2 == 0:
                cut = i
                break
            start = i + 2
        code = line[:cut].rstrip()
        if code.strip():
            out.append(code)
    return out


def kernel_source_hash():
    """Hash of the global prefill kernel's code (its sources less comments and blank lines),
    so that a recorded DRAM-traffic figure stays attached to the code it was measured on."""
    h = hashlib.sha256()
    for name in ("prefill.cu", "sm100.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "attention_g4attn_b200", "csrc", name), encoding="utf-8") as f:
            h.update("\n".join(_code_lines(f.read())).encode())
    return h.hexdigest()[:16]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "prefill_global_T65536_traffic.json")


def recorded_traffic(kernel_hash):
    """DRAM bytes per launch of the global prefill kernel from the committed ncu record
    (profiles/prefill_global_T65536_traffic.json), valid only while the kernel sources still
    hash to the value recorded there."""
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_hash") != kernel_hash:
        return None
    try:
        return float(rec["dram_bytes_per_full_launch"])
    except (KeyError, TypeError, ValueError):
        return None


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled every 50 ms for the whole
    run in a background thread (NVML, read-only; `nvidia-smi` queries when NVML is missing).
    `window()` marks a stretch of wall-clock time; `summary(w)` covers the samples inside it."""
    # NVML clock-event reason bits (nvml.h: clocks event reasons)
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.samples = []          # (time, sm_mhz, max_mhz, watts, reasons)
        self._stop = threading.Event()
        self._thr = None
        self._nvml = None
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._handle = self._find_handle(pynvml, cuda_index)
        except Exception:
            self._nvml = None

    @staticmethod
    def _find_handle(pynvml, cuda_index):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(cuda_index)

    def _sample_nvml(self):
        n, h = self._nvml, self._handle
        sm = n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM)
        w = n.nvmlDeviceGetPowerUsage(h) / 1000.0
        get = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = int(get(h))
        return (float(sm), float(mx), w, sorted(k for k, b in self.REASONS.items() if bits & b))

    def _sample_smi(self):
        out = subprocess.run(["nvidia-smi", "-i", str(self.cuda_index),
                              "--query-gpu=" + self.SMI_FIELDS, "--format=csv,noheader,nounits"],
                             capture_output=True, text=True, timeout=5)
        p = [x.strip() for x in out.stdout.strip().split(",")]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        return (float(p[0]), float(p[1]), float(p[2]) if p[2].replace(".", "").isdigit() else None,
                sorted(names[i] for i in range(4) if p[3 + i].lower() == "active"))

    def _run(self):
        while not self._stop.is_set():
            try:
                s = self._sample_nvml() if self._nvml else self._sample_smi()
                self.samples.append((time.time(),) + s)
            except Exception:
                pass
            self._stop.wait(0.05 if self._nvml else 0.2)

    def start(self):
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def stop(self):
        self._stop.set()
        if self._thr:
            self._thr.join(timeout=10)

    class _Window:
        def __init__(self):
            self.t0 = self.t1 = None

        def __enter__(self):
            self.t0 = time.time()
            return self

        def __exit__(self, *exc):
            self.t1 = time.time()

    def window(self):
        return self._Window()

    def summary(self, w=None):
        s = [x for x in self.samples if w is None or (w.t0 <= x[0] <= (w.t1 or time.time()))]
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(x[1] for x in s),
                "sm_min_mhz": min(x[1] for x in s),
                "sm_max_mhz": max(x[2] for x in s),
                "reasons": sorted({r for x in s for r in x[4]}),
                "samples": len(s),
                "source": "nvml" if self._nvml else "nvidia-smi"}


def timed_calls(call, stream, min_seconds=0.5, min_reps=5, max_reps=5000):
    """Back-to-back calls on `stream`, each bracketed by CUDA events, until `min_seconds` of
    device time: the median per-call seconds and the number of calls."""
    import torch
    evs = []
    total = 0.0
    while len(evs) < max_reps and (len(evs) < min_reps or total < min_seconds):
        batch = []
        for _ in range(min_reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            batch.append((e0, e1))
        batch[-1][1].synchronize()
        for e0, e1 in batch:
            total += e0.elapsed_time(e1) / 1e3
        evs.extend(batch)
    ts = [e0.elapsed_time(e1) / 1e3 for e0, e1 in evs]
    return statistics.median(ts), len(ts)


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


def time_global_32k(device, stream):
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

    def call():
        b.g4attn_prefill(inp.q, inp.k, None, inp.gamma_q, inp.gamma_k, cfg, out=out,
                         workspace=ws, stream=stream)
    for _ in range(2):
        call()
    t, n = timed_calls(call, stream, min_seconds=1.0, min_reps=3)
    return {"workload": wl.name, "ms": t * 1e3, "calls": n, "tflops": wl.flops() / t / 1e12}


def time_decode(device, stream, wl, seed):
    """Global-layer decode step (K=V bf16 cache), back-to-back calls."""
    import torch
    from attention_g4attn_b200 import binding as b, synth
    ly = wl.layer
    d = synth.decode_inputs(wl.B, wl.L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                            seed=seed, device=device)
    cfg = b.LayerCfg.from_layer(ly)
    ws = torch.empty(b.g4attn_decode_workspace_size(wl.B, wl.L, cfg), dtype=torch.uint8,
                     device=device)
    out = torch.empty_like(d.q)

    def call():
        b.g4attn_decode(d.q, d.k, None, cfg, out=out, workspace=ws, stream=stream)
    for _ in range(3):
        call()
    t, n = timed_calls(call, stream, min_seconds=0.5)
    return {"workload": wl.name, "ms": t * 1e3, "calls": n, "gbs": wl.cache_bytes() / t / 1e9}


def time_decode_int8(device, stream, wl, seed):
    """The global decode step against an int8 cache (codes + one fp32 scale per row, the
    layout g4attn_quantize_int8 writes): GB/s of the int8 bytes read (codes and scales)."""
    import torch
    from attention_g4attn_b200 import binding as b, synth
    ly = wl.layer
    kc, ks = synth.int8_cache(wl.B, wl.L, ly.n_kv_heads, ly.head_dim, seed=seed, device=device)
    q = synth.decode_inputs(wl.B, 1, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                            seed=seed, device=device).q
    cfg = b.LayerCfg.from_layer(ly)
    ws = torch.empty(b.g4attn_decode_int8_workspace_size(wl.B, wl.L, 0, cfg), dtype=torch.uint8,
                     device=device)
    out = torch.empty_like(q)

    def call():
        b.g4attn_decode_int8(q, kc, ks, None, None, wl.L, cfg, out=out, workspace=ws,
                             stream=stream)
    for _ in range(3):
        call()
    t, n = timed_calls(call, stream, min_seconds=0.5)
    nbytes = float(kc.numel() + 4 * ks.numel())
    return {"workload": wl.name.replace("global_decode", "global_decode_int8"), "ms": t * 1e3,
            "calls": n, "gbs": nbytes / t / 1e9, "bytes": nbytes,
            "bf16_equivalent_gbs": wl.cache_bytes() / t / 1e9}


def time_local_ring_decode(device, stream, rotated=False):
    """Decode step of the block's local layer (32 q / 16 kv heads, d 256, window 1024,
    separate values) for 16 sequences at position 65535, against ring caches of 1024 rows:
    the keys and values of the window, each read once.  rotated: the ring holds the keys
    turned to their positions (g4attn_decode_rotated, the local layers' serving layout), so
    none is turned on the fly."""
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
    t, n = timed_calls(call, stream, min_seconds=0.3)
    nbytes = 2.0 * B * ly.n_kv_heads * ly.window * ly.head_dim * 2
    name = "local_decode_ring%s_B16_pos65535_C1024_h32x16_d256_w1024" % ("_turned_keys" if rotated else "")
    return {"workload": name, "ms": t * 1e3, "calls": n, "gbs": nbytes / t / 1e9}


def time_decode_graph(device, reps=1000):
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
            "calls": reps, "gbs": B * ly.n_kv_heads * L * ly.head_dim * 2 / t / 1e9}


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

class OracleSample:
    """The fp64 CPU oracle on a bounded sample of the step: `rows` query rows (all 32 heads)
    of the block's global layer (T=65536, causal), each against its full prefix, key
    normalisation included.  The keys are drawn once; every call draws its own rows
    (positions uniform in [T/2, T)) and their queries from `seed`."""

    def __init__(self, rows=8):
        import numpy as np
        import torch
        import oracle
        from attention_g4attn_b200 import workloads
        self.np, self.torch, self.oracle = np, torch, oracle
        self.blk = workloads.BLOCK_5TO1_64K
        self.ly = ly = self.blk.layers[5]
        self.rows = rows
        gen = torch.Generator().manual_seed(1234)
        k = torch.randn((self.blk.B, self.blk.T, ly.n_kv_heads, ly.head_dim), generator=gen).bfloat16()
        self.kb = oracle.bf16_bits(k)
        self.gq = (1.0 + 0.1 * torch.randn(ly.head_dim, generator=gen)).numpy()
        self.gk = (1.0 + 0.1 * torch.randn(ly.head_dim, generator=gen)).numpy()
        self.qb = np.zeros((self.blk.B, self.blk.T, ly.n_q_heads, ly.head_dim), np.uint16)
        self.cfg = oracle.OracleCfg(ly.n_q_heads, ly.n_kv_heads, ly.head_dim, ly.rope_p,
                                    ly.rope_base, ly.window, ly.scale, ly.kv_is_k, ly.qk_norm,
                                    ly.qk_norm_eps)

    def step(self, seed):
        """One sample: returns (FLOPs, seconds)."""
        np, torch, ly, T = self.np, self.torch, self.ly, self.blk.T
        rng = np.random.default_rng(seed)
        rows = np.sort(rng.choice(np.arange(T // 2, T), size=self.rows, replace=False)).astype(np.int32)
        gen = torch.Generator().manual_seed(10_000 + seed)
        for r in rows:
            qr = torch.randn((self.blk.B, ly.n_q_heads, ly.head_dim), generator=gen).bfloat16()
            self.qb[:, r] = self.oracle.bf16_bits(qr)
        t0 = time.perf_counter()
        self.oracle.prefill_rows(self.qb, self.kb, None, self.gq, self.gk, self.cfg, rows)
        secs = time.perf_counter() - t0
        flops = float(sum(4.0 * ly.head_dim * ly.n_q_heads * (int(r) + 1) for r in rows))
        return flops, secs

    def describe(self, steps, seconds):
        return ("%d steps x %d query rows x %d heads of the block's global layer (T=65536, "
                "positions uniform in [T/2, T), causal prefix of each row, key normalisation "
                "included), %.1f s of oracle time"
                % (steps, self.rows, self.ly.n_q_heads, seconds))


def reference_arm(args, rank):
    """--impl reference: the fp64 oracle (the only reference implementation of the pages'
    method) on the host cores.  Each step is one bounded sample of the workload (OracleSample);
    `warmup` untimed steps, then `steps` timed ones.  Under torchrun only rank 0 runs."""
    if rank != 0:
        return
    steps, warmup = max(args.steps, 1), max(args.warmup, 0)
    sampler = OracleSample(rows=8)
    for w in range(warmup):
        sampler.step(seed=w)
    flops = secs = 0.0
    for k in range(steps):
        f, s = sampler.step(seed=1000 + k)
        flops += f
        secs += s
    v = flops / secs / 1e12
    cores = os.cpu_count() or 1
    info = {"kind": "oracle", "cores": cores, "value": v, "unit": "TFLOP/s",
            "sample": sampler.describe(steps, secs)}
    line = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": secs * 1e3 / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": "block_5local_1global_T65536+global_decode_B16_L32768",
                       "step": "one sample of %d query rows x %d heads of the global layer"
                               % (sampler.rows, sampler.ly.n_q_heads),
                       "sample": info["sample"], "rows_per_step": sampler.rows,
                       "heads": sampler.ly.n_q_heads, "oracle_seconds": secs},
            "impl": "reference", "cpu_baseline": info,
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def cpu_baseline(max_seconds=15.0):
    """The oracle timed on a bounded sample (rank 0, one GPU): OracleSample steps until about
    `max_seconds` of oracle time."""
    sampler = OracleSample(rows=8)
    flops = secs = 0.0
    n = 0
    while secs < max_seconds and n < 64:
        f, s = sampler.step(seed=2000 + n)
        flops += f
        secs += s
        n += 1
    return {"kind": "oracle", "cores": os.cpu_count() or 1, "value": flops / secs / 1e12,
            "unit": "TFLOP/s", "sample": sampler.describe(n, secs)}


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
    "global_decode_int8_L32768": ("decode_int8", dict(B=16, L=32768, layer="GLOBAL_8TO1")),
    "global_decode_int8_L8192": ("decode_int8", dict(B=16, L=8192, layer="GLOBAL_8TO1")),
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
    elif kind == "decode_int8":
        kc, ks = synth.int8_cache(p["B"], p["L"], ly.n_kv_heads, ly.head_dim, seed=3, device=dev)
        q = synth.decode_inputs(p["B"], 1, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                                seed=3, device=dev).q
        ws = torch.empty(b.g4attn_decode_int8_workspace_size(p["B"], p["L"], 0, cfg),
                         dtype=torch.uint8, device=dev)
        out = torch.empty_like(q)

        def call():
            b.g4attn_decode_int8(q, kc, ks, None, None, p["L"], cfg, out=out, workspace=ws,
                                 stream=stream)
        work = float(kc.numel() + 4 * ks.numel()) * 1e3   # -> GB/s
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
    ap.add_argument("--no-extras", action="store_true")
    args = ap.parse_args()
    if args.case:
        run_case(args.case, max(args.steps, 1), max(args.warmup, 0))
        return

    if args.impl == "reference":
        reference_arm(args, int(os.environ.get("RANK", "0")))
        return

    from attention_g4attn_b200 import replicas
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: run this same command as --gpus ranks under torch.distributed.run
        sys.exit(replicas.launch_ranks(args.gpus, [os.path.abspath(__file__)] + sys.argv[1:]))
    world_env = int(os.environ.get("WORLD_SIZE", "1"))
    if world_env != args.gpus:
        print("bench.py: --gpus %d but WORLD_SIZE=%d" % (args.gpus, world_env), file=sys.stderr)
        sys.exit(2)

    import torch
    dist, rank, world, local_rank = replicas.init_from_env("nccl")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    from attention_g4attn_b200 import binding as b  # noqa: F401  (fails loudly without the .so)
    clk = ClockSampler(local_rank).start()

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
    with clk.window() as w_main:
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
    tf_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    # dominant kernel: the global layer of the block (about 93% of the step's FLOPs), timed
    # by CUDA events on its launching stream
    g_inp, g_cfg, g_ws, g_out = S["layers"][5]

    def g_call():
        b.g4attn_prefill(g_inp.q, g_inp.k, None, g_inp.gamma_q, g_inp.gamma_k, g_cfg, out=g_out,
                         workspace=g_ws, stream=stream)
    with clk.window() as w_roof:
        g_s, g_n = timed_calls(g_call, stream, min_seconds=0.4, min_reps=3)
    from attention_g4attn_b200 import workloads
    g_flops = 4.0 * 512 * 32 * blk.B * workloads.visible_pairs(blk.T, 0)
    khash = kernel_source_hash()
    roofline = {"bound": "tensor", "achieved": g_flops / g_s / 1e12, "peak": tf_peak,
                "unit": "TFLOP/s", "frac": g_flops / g_s / 1e12 / tf_peak,
                "traffic": recorded_traffic(khash),
                "algorithmic_flops_per_launch": g_flops, "launch_ms": g_s * 1e3,
                "launches_timed": g_n,
                "kernel": "prefill_kernel<512> (+ key pre-pass) on the block's global layer",
                "peak_source": "%s bf16_tflops_sustained" % peak_src,
                "clocks": clk.summary(w_roof)}

    extra = {}
    # single-GPU extras: under N ranks the others would wait at the next reduction while rank 0
    # ran them
    if rank == 0 and world == 1 and not args.no_extras:
        def run_extra(name, fn, frac_key, num_key, peak):
            with clk.window() as w:
                r = fn()
            r[frac_key] = r[num_key] / peak
            r["clocks"] = clk.summary(w)
            extra[name] = r
        run_extra("global_prefill_T32768", lambda: time_global_32k(device, stream),
                  "frac_of_sustained", "tflops", tf_peak)
        extra["global_prefill_T32768"]["frac_of_burst"] = \
            extra["global_prefill_T32768"]["tflops"] / tf_burst
        run_extra("global_decode_L32768_alone",
                  lambda: time_decode(device, stream, workloads.GLOBAL_DECODE_32K, 8),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("global_decode_L131072",
                  lambda: time_decode(device, stream, workloads.GLOBAL_DECODE_128K, 8),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("global_decode_L32768_graph", lambda: time_decode_graph(device),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("global_decode_int8_L32768",
                  lambda: time_decode_int8(device, stream, workloads.GLOBAL_DECODE_32K, 18),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("global_decode_int8_L131072",
                  lambda: time_decode_int8(device, stream, workloads.GLOBAL_DECODE_128K, 18),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("local_decode_ring", lambda: time_local_ring_decode(device, stream),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("local_decode_ring_turned_keys",
                  lambda: time_local_ring_decode(device, stream, rotated=True),
                  "frac_of_hbm", "gbs", hbm_peak)
        run_extra("chunked_prefill", lambda: time_chunked_prefill(device, stream),
                  "frac_of_sustained", "tflops_all_chunks", tf_peak)

    # end to end through the public API with host buffers (pinned), copies inside the region
    e2e = None
    if not args.no_e2e:
        try:
            with clk.window() as w_e2e:
                e2e = run_e2e(S, stream, device, steps=max(args.steps, 1),
                              warmup=min(max(args.warmup, 0), 1))
        except RuntimeError as exc:   # pinned host memory refused
            e2e = {"error": str(exc)[:200]}
    if e2e is not None:
        # every rank takes the same reduction, a rank whose leg failed included (as +inf)
        ok = "error" not in e2e
        secs = replicas.max_over_ranks([e2e["seconds"] if ok else math.inf], dist, device)[0]
        if ok and not math.isfinite(secs):
            e2e = {"error": "the end-to-end leg failed on another rank"}
    if e2e is not None and "error" not in e2e:
        e2e["seconds"] = secs
        e2e = {"value": replicas.job_rate(flops_step * e2e["steps"], e2e["seconds"], world, 1e12),
               "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["h2d"],
               "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"],
               "warmup": e2e["warmup"],
               "ms_per_step": e2e["seconds"] * 1e3 / e2e["steps"],
               "overlap": "host-to-device copies on one stream, kernels on a second, "
                          "device-to-host copies on a third, ordered per layer by events",
               "clocks": clk.summary(w_e2e)}
    clk.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(max_seconds=15.0)

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
                   "l2": "inputs larger than L2, no flush",
                   "parallelism": "replicas" if world == 1 else "replicas x%d" % world},
        "decode": {"value": dec_gbs, "unit": "GB/s", "frac": dec_gbs / world / hbm_peak,
                   "peak": hbm_peak, "peak_source": "%s hbm_gbs" % peak_src,
                   "ms_per_step": dec_s * 1e3 / args.steps},
        "roofline": roofline,
        "clocks": clk.summary(w_main),
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "device_status": status,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    line.update(extra)
    print(json.dumps(line))


def run_e2e(S, stream, device, steps, warmup):
    """The same step through the public API with inputs in pinned host memory: every step
    copies each layer's inputs host->device, runs the layer, and copies its output
    device->host.  Copies in and out run on streams of their own, so layer i+1's inputs and
    layer i-1's output cross PCIe while layer i computes; events order each layer's buffers
    (its inputs are overwritten only after its previous compute, its output only after the
    previous copy out).  Like the device-timed steps: `warmup` untimed steps, then `steps`
    timed ones between synchronizes (the first timed step's copies have nothing to overlap
    with; later steps' copies overlap the step before)."""
    import torch
    from attention_g4attn_b200 import binding as b

    def pin(t):
        return None if t is None else t.to("cpu").pin_memory()

    units = []   # (host inputs, device inputs, host out, device out, launch)
    h2d = d2h = 0
    for inp, cfg, ws, out in S["layers"]:
        hin = [pin(t) for t in (inp.q, inp.k, inp.v)]
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def launch(inp=inp, cfg=cfg, ws=ws, out=out):
            b.g4attn_prefill(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, cfg, out=out,
                             workspace=ws, stream=stream)
        units.append((hin, [inp.q, inp.k, inp.v], ho, out, launch))
        h2d += sum(t.numel() * t.element_size() for t in hin if t is not None)
        d2h += ho.numel() * ho.element_size()
    d = S["dinp"]
    hin = [pin(d.q), pin(d.k)]
    hdo = torch.empty(S["dout"].shape, dtype=S["dout"].dtype).pin_memory()

    def dlaunch():
        b.g4attn_decode(d.q, d.k, None, S["dcfg"], out=S["dout"], workspace=S["dws"],
                        stream=stream)
    units.append((hin, [d.q, d.k], hdo, S["dout"], dlaunch))
    h2d += sum(t.numel() * t.element_size() for t in hin)
    d2h += hdo.numel() * hdo.element_size()

    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    n = len(units)
    in_ready = [torch.cuda.Event() for _ in range(n)]
    computed = [torch.cuda.Event() for _ in range(n)]
    drained = [torch.cuda.Event() for _ in range(n)]

    def run(nsteps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for s in range(nsteps):
            for i, (hin, din, ho, dout, launch) in enumerate(units):
                if s > 0:
                    s_in.wait_event(computed[i])      # the previous step's layer i read its inputs
                with torch.cuda.stream(s_in):
                    for h, dv in zip(hin, din):
                        if h is not None:
                            dv.copy_(h, non_blocking=True)
                in_ready[i].record(s_in)
                stream.wait_event(in_ready[i])
                if s > 0:
                    stream.wait_event(drained[i])     # the previous output of layer i is on the host
                launch()
                computed[i].record(stream)
                s_out.wait_event(computed[i])
                with torch.cuda.stream(s_out):
                    ho.copy_(dout, non_blocking=True)
                drained[i].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / 1e3

    if warmup > 0:
        run(warmup)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    secs = run(steps)
    return {"seconds": secs, "steps": steps, "warmup": warmup, "h2d": h2d, "d2h": d2h,
            "wall": time.perf_counter() - t0}


if __name__ == "__main__":
    main()
