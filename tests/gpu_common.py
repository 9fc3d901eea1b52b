"""Shared plumbing of the GPU parity tests: run the CUDA path through the C ABI and the
fp64 oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
from oracle import OracleCfg
from parity import assert_parity, to_np


def binding():
    from attention_g4attn_b200 import binding as b
    return b


def ocfg(layer, **kw):
    d = dict(n_q_heads=layer.n_q_heads, n_kv_heads=layer.n_kv_heads, head_dim=layer.head_dim,
             rope_p=layer.rope_p, rope_base=layer.rope_base, window=layer.window,
             scale=layer.scale, kv_is_k=layer.kv_is_k, qk_norm=layer.qk_norm,
             qk_norm_eps=layer.qk_norm_eps)
    d.update(kw)
    return OracleCfg(**d)


def gpu_prefill(inp, layer, **kw):
    b = binding()
    cfg = b.LayerCfg.from_layer(layer, **kw)
    dev = torch.device("cuda:0")
    v = inp.v.to(dev) if inp.v is not None else None
    out, lse = b.g4attn_prefill(inp.q.to(dev), inp.k.to(dev), v, inp.gamma_q.to(dev),
                                inp.gamma_k.to(dev), cfg, want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    return out.cpu(), lse.cpu()


def check_prefill(inp, layer, rows=None, what="prefill", **kw):
    out, lse = gpu_prefill(inp, layer, **kw)
    T = inp.q.shape[1]
    rows = np.arange(T, dtype=np.int32) if rows is None else np.asarray(rows, np.int32)
    ro, rl = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k,
                                 ocfg(layer, **kw), rows)
    go = to_np(out)[:, rows]
    gl = to_np(lse)[:, :, rows]
    r1 = assert_parity(go, ro, what + " out")
    r2 = assert_parity(gl, rl, what + " lse")
    return r1, r2, out, lse


def sample_rows(T, window=0, n_random=16, seed=0):
    rows = {0, 1, min(127, T - 1), min(128, T - 1), T // 2, max(T - 2, 0), T - 1}
    if window > 0:
        for r in (window - 1, window, window + 1):
            if r < T:
                rows.add(r)
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, T, size=n_random).tolist())
    return np.array(sorted(rows), np.int32)
