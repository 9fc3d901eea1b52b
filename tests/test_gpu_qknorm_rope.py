"""GPU parity of the standalone QKNorm + p-RoPE prologue (g4attn_qknorm_rope)."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import binding, ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layer,B,T,pos0", [
    (workloads.GLOBAL_8TO1, 2, 37, 0),
    (workloads.GLOBAL_8TO1, 1, 5, 131000),          # positions of a 128K context
    (workloads.LOCAL_W512, 2, 19, 3),
    (workloads.LOCAL_W1024, 1, 9, 65530),
])
def test_qknorm_rope_parity(layer, B, T, pos0):
    b = binding()
    inp = synth.layer_inputs(B, T, layer.n_q_heads, layer.n_kv_heads, layer.head_dim, False,
                             seed=100 + T)
    dev = torch.device("cuda:0")
    cfg = b.LayerCfg.from_layer(layer)
    qo, ko, kr = b.g4attn_qknorm_rope(inp.q.to(dev), inp.k.to(dev), inp.gamma_q.to(dev),
                                      inp.gamma_k.to(dev), cfg, pos0=pos0)
    torch.cuda.synchronize()
    rq, rk, rr = oracle.qknorm_rope(inp.q, inp.k, inp.gamma_q, inp.gamma_k, ocfg(layer), pos0)
    assert_parity(to_np(qo), rq, "q_out")
    assert_parity(to_np(ko), rk, "kcache_out")
    assert_parity(to_np(kr), rr, "krot_out")


def test_qknorm_rope_without_norm_is_pure_rope():
    b = binding()
    layer = workloads.GLOBAL_8TO1
    inp = synth.layer_inputs(1, 7, 32, 4, 512, False, seed=7)
    dev = torch.device("cuda:0")
    cfg = b.LayerCfg.from_layer(layer, qk_norm=0)
    qo, ko, kr = b.g4attn_qknorm_rope(inp.q.to(dev), inp.k.to(dev), None, None, cfg, pos0=11)
    torch.cuda.synchronize()
    rq, rk, rr = oracle.qknorm_rope(inp.q, inp.k, None, None, ocfg(layer, qk_norm=0), 11)
    assert_parity(to_np(qo), rq, "q_out")
    np.testing.assert_array_equal(to_np(ko), to_np(inp.k))   # no norm, no rotation: a copy
    assert_parity(to_np(kr), rr, "krot_out")


def test_qknorm_rope_k_only_and_empty():
    b = binding()
    layer = workloads.GLOBAL_8TO1
    inp = synth.layer_inputs(1, 3, 32, 4, 512, False, seed=8)
    dev = torch.device("cuda:0")
    cfg = b.LayerCfg.from_layer(layer)
    _, ko, kr = b.g4attn_qknorm_rope(None, inp.k.to(dev), None, inp.gamma_k.to(dev), cfg)
    torch.cuda.synchronize()
    _, rk, rr = oracle.qknorm_rope(None, inp.k, None, inp.gamma_k, ocfg(layer))
    assert_parity(to_np(ko), rk, "kcache_out")
    assert_parity(to_np(kr), rr, "krot_out")
    e = torch.empty(1, 0, 32, 512, dtype=torch.bfloat16, device=dev)
    b.g4attn_qknorm_rope(e, None, inp.gamma_q.to(dev), None, cfg)   # T = 0: no-op
