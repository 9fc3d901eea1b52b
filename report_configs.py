"""Per-config report: GPU time and roofline fraction, oracle time, and parity for the five
named workloads (needs a CUDA device: `python report_configs.py`; prints a markdown table).

GPU: CUDA events on the launching stream, 3 warm-up calls, median of 10 timed calls (3 for the
T=65536 layers), inputs resident in device memory.  Oracle: the fp64 CPU oracle on all host
cores, in full for the tiny prefill, the local prefill and both decode lengths, on a row
sample (boundary rows plus 64 seeded random rows) for the T=32768 prefill and for the
global and first local layer of the 5:1 block.  Parity: max-abs and
relative L2 of out (and lse) against the oracle on the same rows.
"""
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))   # the parity helpers the GPU tests use

import oracle  # noqa: E402
from attention_g4attn_b200 import binding as b, synth, workloads  # noqa: E402
from gpu_common import ocfg, sample_rows  # noqa: E402
from parity import errors, to_np  # noqa: E402

DEV = torch.device("cuda:0")
PEAKS = {"bf16_tflops": 1601.1, "hbm_gbs": 6553.9}


def load_peaks():
    p = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            PEAKS.update(json.load(f))


def time_gpu(call, n):
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    return statistics.median(ts)


def prefill_case(layer, B, T, seed, rows, n_time):
    inp = synth.layer_inputs(B, T, layer.n_q_heads, layer.n_kv_heads, layer.head_dim,
                             layer.separate_v, seed=seed)
    cfg = b.LayerCfg.from_layer(layer)
    q, k, gq, gk = (x.to(DEV) for x in (inp.q, inp.k, inp.gamma_q, inp.gamma_k))
    v = inp.v.to(DEV) if inp.v is not None else None
    ws = torch.empty(b.g4attn_prefill_workspace_size(B, T, cfg), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    lse = torch.empty((B, layer.n_q_heads, T), dtype=torch.float32, device=DEV)
    sec = time_gpu(lambda: b.g4attn_prefill(q, k, v, gq, gk, cfg, out=out, lse=lse, workspace=ws), n_time)
    assert b.g4attn_device_status() == 0
    rows = np.arange(T, dtype=np.int32) if rows is None else rows
    t0 = time.perf_counter()
    ro, rl = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, ocfg(layer), rows)
    osec = time.perf_counter() - t0
    go, gl = to_np(out.cpu())[:, rows], to_np(lse.cpu())[:, :, rows]
    flops = 4.0 * layer.head_dim * layer.n_q_heads * B * workloads.visible_pairs(T, layer.window)
    return sec, flops, osec, len(rows), T, errors(go, ro), errors(gl, rl)


def decode_case(wl, n_time):
    ly = wl.layer
    d = synth.decode_inputs(wl.B, wl.L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=wl.seed)
    cfg = b.LayerCfg.from_layer(ly)
    q, kc = d.q.to(DEV), d.k.to(DEV)
    ws = torch.empty(b.g4attn_decode_workspace_size(wl.B, wl.L, cfg), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, ly.n_q_heads), dtype=torch.float32, device=DEV)
    sec = time_gpu(lambda: b.g4attn_decode(q, kc, None, cfg, out=out, lse=lse, workspace=ws), n_time)
    assert b.g4attn_device_status() == 0
    t0 = time.perf_counter()
    ro, rl = oracle.decode(d.q[:, 0], d.k, None, ocfg(ly))
    osec = time.perf_counter() - t0
    go, gl = to_np(out.cpu())[:, 0], to_np(lse.cpu())
    return sec, wl.cache_bytes(), osec, errors(go, ro), errors(gl, rl)


def fmt_err(e):
    return "%.1e / %.1e" % e


def main():
    load_peaks()
    tf_peak, hbm = float(PEAKS["bf16_tflops"]), float(PEAKS["hbm_gbs"])
    cores = os.cpu_count() or 1
    lines = ["| Config | GPU time | GPU TFLOP/s or GB/s | %% of roofline (measured peak) | Oracle time "
             "(%d cores) | Parity out: max-abs / rel-L2 | Parity lse |" % cores,
             "|---|---|---|---|---|---|---|"]

    def pre_row(name, res, full):
        sec, flops, osec, nrows, T, eo, el = res
        tf = flops / sec / 1e12
        otime = ("%.2f s" % osec) if full else ("%.2f s for %d of %d rows (extrapolated %.0f s)"
                                               % (osec, nrows, T, osec * T / nrows))
        lines.append("| %s | %.3f ms | %.1f TFLOP/s | %.1f%% of %.0f | %s | %s | %s |"
                     % (name, sec * 1e3, tf, 100 * tf / tf_peak, tf_peak, otime, fmt_err(eo), fmt_err(el)))

    pre_row("1 global prefill tiny (T=128)",
            prefill_case(workloads.GLOBAL_TINY, 1, 128, 0, None, 10), True)
    pre_row("2 local prefill (B2, T4096, W512)",
            prefill_case(workloads.LOCAL_W512, 2, 4096, 0, None, 10), True)
    pre_row("3 global prefill (T=32768)",
            prefill_case(workloads.GLOBAL_8TO1, 1, 32768, 0, sample_rows(32768, 0, 64, 3), 10), False)
    for wl in (workloads.GLOBAL_DECODE_32K, workloads.GLOBAL_DECODE_128K):
        sec, nbytes, osec, eo, el = decode_case(wl, 10)
        gbs = nbytes / sec / 1e9
        lines.append("| 4 global decode (B16, L=%d) | %.3f ms | %.0f GB/s | %.1f%% of %.0f | %.2f s | %s | %s |"
                     % (wl.L, sec * 1e3, gbs, 100 * gbs / hbm, hbm, osec, fmt_err(eo), fmt_err(el)))
    blk = workloads.BLOCK_5TO1_64K
    tot_s, tot_f = 0.0, 0.0
    for i, ly in enumerate(blk.layers):
        checked = i in (0, 5)
        rows = sample_rows(blk.T, ly.window, 64, 5 + i) if checked else np.array([0], np.int32)
        res = prefill_case(ly, blk.B, blk.T, blk.seeds[i], rows, 3)
        tot_s += res[0]
        tot_f += res[1]
        if checked:
            pre_row("5 block layer %d (%s)" % (i, "global" if ly.head_dim == 512 else "local"), res, False)
    tf = tot_f / tot_s / 1e12
    lines.append("| 5 block, six layers | %.1f ms | %.1f TFLOP/s | %.1f%% of %.0f | — | — | — |"
                 % (tot_s * 1e3, tf, 100 * tf / tf_peak, tf_peak))
    print("\n".join(lines))


if __name__ == "__main__":
    main()
