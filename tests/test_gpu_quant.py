"""GPU parity of the int8 KV cache writer (g4attn_quantize_int8) against the oracle: codes and
scales are integer decisions taken in IEEE fp32 on both sides, so they must match exactly."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth
from gpu_common import binding

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _check(x):
    b = binding()
    codes, scales = b.g4attn_quantize_int8(x.to(DEV))
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_int8(x)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("d", [128, 256, 512])
def test_quantize_int8_random_caches(d):
    # N(0,1) caches, rows scaled over six decades (small scales reach fp32 subnormal quotients)
    dec = synth.decode_inputs(3, 257, 4, 2, d, False, seed=d)
    gen = torch.Generator().manual_seed(d)
    mag = torch.pow(10.0, torch.empty((3, 257, 2, 1)).uniform_(-3, 3, generator=gen))
    _check((dec.k.float() * mag).to(torch.bfloat16))


def test_quantize_int8_special_rows():
    # zero rows, exact multiples of a power-of-two scale with half-way quotients, tiny values
    d = 256
    x = torch.zeros((6, d), dtype=torch.float32)
    x[1, :4] = torch.tensor([127.0, 0.5, 1.5, 2.5])
    x[2, :4] = torch.tensor([-127.0, -0.5, -1.5, 126.5])
    x[3] = torch.linspace(-3, 3, d)
    x[4, 7] = 1e-30
    x[5, :] = 1e-38
    _check(x.to(torch.bfloat16))


def test_quantize_int8_non_finite_rows():
    # rows holding +inf, -inf or NaN get scale NaN and codes 0 on both sides
    d = 128
    x = torch.randn((5, d), generator=torch.Generator().manual_seed(5))
    x[0, 3] = float("inf")
    x[2, 100] = float("-inf")
    x[4, 0] = float("nan")
    _check(x.to(torch.bfloat16))


def test_quantize_int8_full_size_global_cache():
    # the global decode workload's cache (B=16, L=32768, 4 kv heads, d 512), rows sampled
    b = binding()
    dec = synth.decode_inputs(16, 32768, 32, 4, 512, False, seed=3, device="cuda")
    codes, scales = b.g4attn_quantize_int8(dec.k)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    idx = [(0, 0), (15, 32767)] + [tuple(rng.integers([0, 0], [16, 32768])) for _ in range(64)]
    for bb, ll in idx:
        rc, rs = oracle.quantize_int8(dec.k[bb, ll].cpu())
        np.testing.assert_array_equal(codes[bb, ll].cpu().numpy(), rc)
        np.testing.assert_array_equal(scales[bb, ll].cpu().numpy().view(np.uint32), rs.view(np.uint32))
