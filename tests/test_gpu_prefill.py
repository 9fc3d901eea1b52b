"""GPU parity of the fused flash-attention prefill (g4attn_prefill) against the oracle."""
import numpy as np
import pytest
import torch

from attention_g4attn_b200 import synth, workloads
from gpu_common import check_prefill, gpu_prefill, sample_rows
from parity import to_np

pytestmark = pytest.mark.gpu

GLOBAL = workloads.GLOBAL_8TO1
TINY = workloads.GLOBAL_TINY
LOCAL = workloads.LOCAL_W512


def _inp(B, T, ly, seed):
    return synth.layer_inputs(B, T, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, ly.separate_v,
                              seed=seed)


def test_global_prefill_tiny_workload():
    wl = workloads.GLOBAL_PREFILL_TINY
    check_prefill(_inp(wl.B, wl.T, TINY, wl.seeds[0]), TINY, what=wl.name)


@pytest.mark.parametrize("T", [1, 5, 16, 17, 129, 300])
def test_global_prefill_ragged(T):
    check_prefill(_inp(1, T, TINY, 40 + T), TINY, what="global T=%d" % T)


def test_global_prefill_two_kv_heads_two_batches():
    ly = workloads.with_layer(GLOBAL, n_q_heads=16, n_kv_heads=2)
    check_prefill(_inp(2, 200, ly, 3), ly, what="global 16/2 B=2")


def test_global_prefill_rotated_values():
    check_prefill(_inp(1, 150, TINY, 4), TINY, kv_is_k=2, what="global kv_is_k=2")


def test_global_prefill_separate_values():
    ly = workloads.with_layer(TINY, kv_is_k=0)
    check_prefill(_inp(1, 140, ly, 5), ly, what="global separate v")


def test_global_prefill_full_rope_cos_sin_from_table():
    # full RoPE at head_dim 512: the (cos, sin) rows are too wide for the TMA staging, so the
    # prologue reads them from the workspace table; T = 37 leaves a ragged last row tile
    ly = workloads.with_layer(TINY, rope_p=1.0)
    check_prefill(_inp(1, 37, ly, 8), ly, what="global full RoPE T=37")


def test_local_prefill_one_query_head_per_kv_head():
    # G = 1: 128 tokens per row tile, whose (cos, sin) rows also come from the table
    ly = workloads.with_layer(LOCAL, n_q_heads=8, n_kv_heads=8, window=100)
    check_prefill(_inp(1, 201, ly, 9), ly, what="local G=1 T=201 W=100")


def test_prefill_without_qknorm():
    check_prefill(_inp(1, 150, TINY, 10), TINY, what="global no QKNorm", qk_norm=0)
    ly = workloads.with_layer(LOCAL, window=64)
    check_prefill(_inp(1, 150, ly, 11), ly, what="local no QKNorm", qk_norm=0)


@pytest.mark.parametrize("T,W", [(700, 512), (333, 100), (130, 1)])
def test_local_prefill_window(T, W):
    ly = workloads.with_layer(LOCAL, window=W)
    check_prefill(_inp(2, T, ly, 6 + W), ly, what="local T=%d W=%d" % (T, W))


def test_window_at_least_T_equals_causal():
    ly = workloads.with_layer(LOCAL, window=0)
    inp = _inp(1, 300, ly, 7)
    a, la = gpu_prefill(inp, ly)
    b, lb = gpu_prefill(inp, workloads.with_layer(ly, window=300))
    c, lc = gpu_prefill(inp, workloads.with_layer(ly, window=5000))
    assert torch.equal(a, b) and torch.equal(a, c)
    assert torch.equal(la, lb) and torch.equal(la, lc)


def test_local_prefill_workload_sampled():
    wl = workloads.LOCAL_PREFILL
    ly = wl.layers[0]
    inp = _inp(wl.B, wl.T, ly, wl.seeds[0])
    check_prefill(inp, ly, rows=sample_rows(wl.T, ly.window), what=wl.name)


def test_global_prefill_32k_sampled():
    wl = workloads.GLOBAL_PREFILL_32K
    ly = wl.layers[0]
    inp = _inp(wl.B, wl.T, ly, wl.seeds[0])
    check_prefill(inp, ly, rows=sample_rows(wl.T, 0, n_random=8), what=wl.name)


@pytest.mark.parametrize("layer_idx", [0, 1, 2, 3, 4, 5])
def test_block_5to1_layers_sampled(layer_idx):
    wl = workloads.BLOCK_5TO1_64K
    ly = wl.layers[layer_idx]
    inp = _inp(wl.B, wl.T, ly, wl.seeds[layer_idx])
    check_prefill(inp, ly, rows=sample_rows(wl.T, ly.window, n_random=6),
                  what="%s layer %d" % (wl.name, layer_idx))
