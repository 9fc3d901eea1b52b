"""GPU parity of the int8 KV-cache decode (g4attn_decode_int8) against the fp64 oracle's
decode_int8 on the same codes and scales.  The caches are the oracle's own quantisation of a
seeded N(0,1) bf16 cache (small sizes) or seeded random codes and scales (full sizes); the
expected values come from the oracle alone."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import binding, ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
GLOBAL = workloads.GLOBAL_8TO1


def _q8(x):
    """The oracle's int8 cache of a bf16 cache, as torch tensors."""
    c, s = oracle.quantize_int8(x)
    return torch.from_numpy(c), torch.from_numpy(s)


def _ring8(codes, scales, L, C):
    """Ring of C rows (position p in row p % C) holding the last C positions of a linear int8
    cache.  Rows never written hold code 127 and scale NaN: they must never reach a result."""
    B = codes.shape[0]
    rc = torch.full((B, C) + tuple(codes.shape[2:]), 127, dtype=torch.int8)
    rs = torch.full((B, C) + tuple(scales.shape[2:]), float("nan"), dtype=torch.float32)
    for p in range(max(0, L - C), L):
        rc[:, p % C] = codes[:, p]
        rs[:, p % C] = scales[:, p]
    return rc, rs


def run_int8(q, kc, ks, vc, vs, L, layer, ring=False, **kw):
    b = binding()
    cfg = b.LayerCfg.from_layer(layer, **kw)
    dv = lambda t: None if t is None else t.to(DEV)   # noqa: E731
    out, lse = b.g4attn_decode_int8(q.to(DEV), dv(kc), dv(ks), dv(vc), dv(vs), L, cfg, ring=ring,
                                    want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    return to_np(out.cpu())[:, 0], to_np(lse.cpu())


def compare(go, gl, ro, rl, what, items=None, layer=None):
    if items is not None:
        G = layer.n_q_heads // layer.n_kv_heads
        sel = [(it // layer.n_kv_heads, (it % layer.n_kv_heads) * G + h)
               for it in items for h in range(G)]
        bi, hi = [s[0] for s in sel], [s[1] for s in sel]
        go, ro, gl, rl = go[bi, hi], ro[bi, hi], gl[bi, hi], rl[bi, hi]
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl)), what
    assert_parity(go, ro, what + " out")
    assert_parity(gl, rl, what + " lse")


def check_linear(dec, layer, what, **kw):
    kc, ks = _q8(dec.k)
    vc, vs = _q8(dec.v) if dec.v is not None else (None, None)
    L = dec.k.shape[1]
    go, gl = run_int8(dec.q, kc, ks, vc, vs, L, layer, **kw)
    ro, rl = oracle.decode_int8(dec.q[:, 0], kc.numpy(), ks.numpy(),
                                None if vc is None else vc.numpy(),
                                None if vs is None else vs.numpy(), ocfg(layer, **kw))
    compare(go, gl, ro, rl, what)


@pytest.mark.parametrize("L", [1, 129, 3001])
def test_decode_int8_global_layer(L):
    # 32 q / 4 kv heads, head_dim 512, p-RoPE 0.25 at 1e6, keys as values (one int8 cache)
    dec = synth.decode_inputs(3, L, 32, 4, 512, False, seed=300 + L)
    check_linear(dec, GLOBAL, "int8 decode global L=%d" % L)


def test_decode_int8_rotated_values_variant():
    dec = synth.decode_inputs(2, 777, 32, 4, 512, False, seed=311)
    check_linear(dec, GLOBAL, "int8 decode kv_is_k=2", kv_is_k=2)


def test_decode_int8_separate_values_with_window():
    dec = synth.decode_inputs(2, 1500, 32, 4, 512, True, seed=312)
    check_linear(dec, GLOBAL, "int8 decode separate v, window 300", kv_is_k=0, window=300)


@pytest.mark.parametrize("Hq,Hkv,L,window", [
    (32, 16, 2000, 1024),   # the block's local layer: two turned slots (2 q heads per kv head)
    (32, 4, 1300, 512),     # 8 q heads per kv head: the absolute-angle path
])
def test_decode_int8_local_shapes(Hq, Hkv, L, window):
    ly = workloads.with_layer(workloads.LOCAL_W1024, n_q_heads=Hq, n_kv_heads=Hkv, window=window)
    dec = synth.decode_inputs(2, L, Hq, Hkv, 256, True, seed=320 + Hkv)
    check_linear(dec, ly, "int8 decode d256 G=%d W=%d" % (Hq // Hkv, window))


@pytest.mark.parametrize("L,C", [(1, 1024), (700, 1024), (1024, 1024), (5000, 1024)])
def test_decode_int8_ring_local_layer(L, C):
    # the block's local layer (32 q / 16 kv heads, d 256, window 1024, separate values) on
    # ring caches; never-written rows are poisoned
    ly = workloads.LOCAL_W1024
    dec = synth.decode_inputs(2, L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, True, seed=330 + L)
    kc, ks = _q8(dec.k)
    vc, vs = _q8(dec.v)
    rkc, rks = _ring8(kc, ks, L, C)
    rvc, rvs = _ring8(vc, vs, L, C)
    go, gl = run_int8(dec.q, rkc, rks, rvc, rvs, L, ly, ring=True)
    ro, rl = oracle.decode_int8(dec.q[:, 0], kc.numpy(), ks.numpy(), vc.numpy(), vs.numpy(),
                                ocfg(ly))
    compare(go, gl, ro, rl, "int8 ring decode L=%d C=%d" % (L, C))


def test_decode_int8_empty_cache():
    b = binding()
    q = torch.randn(2, 1, 32, 512, device=DEV).bfloat16()
    kc = torch.empty(2, 0, 4, 512, dtype=torch.int8, device=DEV)
    ks = torch.empty(2, 0, 4, dtype=torch.float32, device=DEV)
    out, lse = b.g4attn_decode_int8(q, kc, ks, None, None, 0, b.LayerCfg.from_layer(GLOBAL),
                                    want_lse=True)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert torch.all(torch.isinf(lse)) and torch.all(lse < 0)


def test_decode_int8_matches_bf16_decode_of_the_dequantised_cache():
    # scales that are powers of two make scale * code exact in bf16: the int8 decode and the
    # bf16 decode of the dequantised cache compute the same attention
    b = binding()
    gen = torch.Generator().manual_seed(340)
    B, L = 2, 2222
    kc = torch.randint(-127, 128, (B, L, 4, 512), generator=gen, dtype=torch.int8)
    ks = torch.pow(2.0, torch.randint(-7, -5, (B, L, 4), generator=gen).float())   # |x| < 2
    q = torch.randn((B, 1, 32, 512), generator=gen).bfloat16()
    kb = (kc.float() * ks[..., None]).bfloat16()
    assert torch.equal(kb.float(), kc.float() * ks[..., None])
    cfg = b.LayerCfg.from_layer(GLOBAL)
    o8, l8 = run_int8(q, kc, ks, None, None, L, GLOBAL)
    o16, l16 = b.g4attn_decode(q.to(DEV), kb.to(DEV), None, cfg, want_lse=True)
    torch.cuda.synchronize()
    assert_parity(o8, to_np(o16.cpu())[:, 0], "int8 vs bf16 decode out")
    assert_parity(l8, to_np(l16.cpu()), "int8 vs bf16 decode lse")


@pytest.mark.parametrize("L", [32768, 131072])
def test_decode_int8_full_size_sampled(L):
    # the global decode workload (B=16, 32 q / 4 kv heads, d 512) at full length, codes and
    # scales drawn on the device; the oracle runs the sampled (batch, kv head) items
    ly = GLOBAL
    B = 16
    kc, ks = synth.int8_cache(B, L, ly.n_kv_heads, ly.head_dim, seed=L, device="cuda")
    q = synth.decode_inputs(B, 1, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=350).q
    go, gl = run_int8(q, kc, ks, None, None, L, ly)
    items = [0, 17, B * ly.n_kv_heads - 1]   # (b, g) = (0, 0), (4, 1), (15, 3)
    # only the sampled sequences go to the host: batch entry i of the small cache holds item i
    n = len(items)
    kch = torch.zeros((n, L, ly.n_kv_heads, ly.head_dim), dtype=torch.int8)
    ksh = torch.zeros((n, L, ly.n_kv_heads), dtype=torch.float32)
    for i, it in enumerate(items):
        bb, g = divmod(it, ly.n_kv_heads)
        kch[i, :, g] = kc[bb, :, g].cpu()
        ksh[i, :, g] = ks[bb, :, g].cpu()
    qs = torch.stack([q[it // ly.n_kv_heads, 0] for it in items])
    sub = np.array([i * ly.n_kv_heads + it % ly.n_kv_heads for i, it in enumerate(items)], np.int32)
    ro, rl = oracle.decode_int8(qs, kch.numpy(), ksh.numpy(), None, None, ocfg(ly), items=sub)
    G = ly.n_q_heads // ly.n_kv_heads
    for i, it in enumerate(items):
        bb, g = divmod(it, ly.n_kv_heads)
        hs = slice(g * G, g * G + G)
        assert_parity(go[bb, hs], ro[i, hs], "int8 decode B16 L=%d item %d out" % (L, it))
        assert_parity(gl[bb, hs], rl[i, hs], "int8 decode B16 L=%d item %d lse" % (L, it))
