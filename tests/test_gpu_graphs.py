"""The entry points inside CUDA graphs: a decode step and a prefill captured once (argument
checks, plans and tensor maps are fixed at capture), then replayed with new inputs written into
the same buffers, each replay checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import binding, ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _capture(call):
    """Warm up on a side stream (first launches load the kernels), then capture one call."""
    s = torch.cuda.Stream(DEV)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        call()
    return g


def test_decode_replays_from_a_cuda_graph():
    b = binding()
    ly = workloads.GLOBAL_8TO1
    cfg = b.LayerCfg.from_layer(ly)
    B, L = 4, 3000
    decs = [synth.decode_inputs(B, L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=s)
            for s in (31, 32)]
    q, k = decs[0].q.to(DEV), decs[0].k.to(DEV)
    out = torch.empty_like(q)
    lse = torch.empty((B, ly.n_q_heads), dtype=torch.float32, device=DEV)
    ws = torch.empty(b.g4attn_decode_workspace_size(B, L, cfg), dtype=torch.uint8, device=DEV)
    g = _capture(lambda: b.g4attn_decode(q, k, None, cfg, out=out, lse=lse, workspace=ws))
    for i, dec in enumerate(decs):
        q.copy_(dec.q.to(DEV))
        k.copy_(dec.k.to(DEV))
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert b.g4attn_device_status() == 0
        ro, rl = oracle.decode(dec.q[:, 0], dec.k, None, ocfg(ly))
        assert_parity(to_np(out.cpu())[:, 0], ro, "graph decode replay %d out" % i)
        assert_parity(to_np(lse.cpu()), rl, "graph decode replay %d lse" % i)


def test_local_prefill_replays_from_a_cuda_graph():
    b = binding()
    ly = workloads.LOCAL_W512
    cfg = b.LayerCfg.from_layer(ly)
    B, T = 1, 700
    inps = [synth.layer_inputs(B, T, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, True, seed=s)
            for s in (33, 34)]
    q, k, v = (x.to(DEV) for x in (inps[0].q, inps[0].k, inps[0].v))
    gq, gk = inps[0].gamma_q.to(DEV), inps[0].gamma_k.to(DEV)
    out = torch.empty_like(q)
    lse = torch.empty((B, ly.n_q_heads, T), dtype=torch.float32, device=DEV)
    ws = torch.empty(b.g4attn_prefill_workspace_size(B, T, cfg), dtype=torch.uint8, device=DEV)
    g = _capture(lambda: b.g4attn_prefill(q, k, v, gq, gk, cfg, out=out, lse=lse, workspace=ws))
    for i, inp in enumerate(inps):
        for dst, src in ((q, inp.q), (k, inp.k), (v, inp.v), (gq, inp.gamma_q), (gk, inp.gamma_k)):
            dst.copy_(src.to(DEV))
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert b.g4attn_device_status() == 0
        rows = np.arange(T, dtype=np.int32)
        ro, rl = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, ocfg(ly), rows)
        assert_parity(to_np(out.cpu()), ro, "graph prefill replay %d out" % i)
        assert_parity(to_np(lse.cpu()), rl, "graph prefill replay %d lse" % i)
