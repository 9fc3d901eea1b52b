"""Failure detection inside the attention kernels themselves: with the device wait limit set
to one poll, the first wait of a prefill or decode that is not satisfied at once gives up.
The kernel then records G4ATTN_ERR_TIMEOUT, raises its abort flags, drains what it started
(the key / value copies of both CTAs of a pair, its MMAs) and returns.  The test checks the
status each launch leaves and that normal launches afterwards still match the oracle, so the
context stayed usable.  Nothing here faults or hangs a GPU: every wait is bounded."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import binding, check_prefill, ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _prefill(layer, T, seed):
    b = binding()
    inp = synth.layer_inputs(1, T, layer.n_q_heads, layer.n_kv_heads, layer.head_dim,
                             layer.separate_v, seed=seed)
    cfg = b.LayerCfg.from_layer(layer)
    v = None if inp.v is None else inp.v.to(DEV)
    b.g4attn_prefill(inp.q.to(DEV), inp.k.to(DEV), v, inp.gamma_q.to(DEV), inp.gamma_k.to(DEV), cfg)


def _decode(seed):
    b = binding()
    ly = workloads.GLOBAL_8TO1
    dec = synth.decode_inputs(4, 3000, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=seed)
    b.g4attn_decode(dec.q.to(DEV), dec.k.to(DEV), None, b.LayerCfg.from_layer(ly))
    return dec


@pytest.mark.parametrize("what", ["global_prefill", "local_prefill", "decode"])
def test_kernels_give_up_on_a_one_poll_wait_limit_and_the_context_recovers(what):
    b = binding()
    assert b.g4attn_device_status() == 0
    old = b.g4attn_set_wait_limit(1)
    try:
        if what == "global_prefill":
            _prefill(workloads.GLOBAL_8TO1, 2048, 500)
        elif what == "local_prefill":
            _prefill(workloads.LOCAL_W1024, 4096, 501)
        else:
            _decode(502)
        torch.cuda.synchronize()
        status = b.g4attn_device_status()
    finally:
        b.g4attn_set_wait_limit(old)
    assert status == b.G4ATTN_ERR_TIMEOUT
    assert b.g4attn_device_status() == 0
    # the same kinds of launch run normally afterwards and match the oracle
    ly = workloads.GLOBAL_8TO1
    inp = synth.layer_inputs(1, 300, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=503)
    check_prefill(inp, ly, what="prefill after a timeout")
    loc = workloads.LOCAL_W1024
    inp = synth.layer_inputs(1, 1500, loc.n_q_heads, loc.n_kv_heads, loc.head_dim, True, seed=504)
    check_prefill(inp, loc, what="local prefill after a timeout")
    dec = synth.decode_inputs(2, 777, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=505)
    out, lse = b.g4attn_decode(dec.q.to(DEV), dec.k.to(DEV), None, b.LayerCfg.from_layer(ly),
                               want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    ro, rl = oracle.decode(dec.q[:, 0], dec.k, None, ocfg(ly))
    assert_parity(to_np(out.cpu())[:, 0], ro, "decode after a timeout out")
    assert_parity(to_np(lse.cpu()), rl, "decode after a timeout lse")
