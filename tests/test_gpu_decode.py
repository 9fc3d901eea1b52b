"""GPU parity of split-KV decode (g4attn_decode) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import binding, ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu

GLOBAL = workloads.GLOBAL_8TO1


def run_decode(dec, layer, **kw):
    b = binding()
    dev = torch.device("cuda:0")
    cfg = b.LayerCfg.from_layer(layer, **kw)
    v = dec.v.to(dev) if dec.v is not None else None
    out, lse = b.g4attn_decode(dec.q.to(dev), dec.k.to(dev), v, cfg, want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    return out.cpu(), lse.cpu()


def check(dec, layer, items=None, what="decode", **kw):
    out, lse = run_decode(dec, layer, **kw)
    ro, rl = oracle.decode(dec.q[:, 0], dec.k, dec.v, ocfg(layer, **kw), items=items)
    go, gl = to_np(out)[:, 0], to_np(lse)
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
    if items is not None:
        G = layer.n_q_heads // layer.n_kv_heads
        sel = [(it // layer.n_kv_heads, (it % layer.n_kv_heads) * G + h)
               for it in items for h in range(G)]
        bi = [s[0] for s in sel]
        hi = [s[1] for s in sel]
        go, ro, gl, rl = go[bi, hi], ro[bi, hi], gl[bi, hi], rl[bi, hi]
    assert_parity(go, ro, what + " out")
    assert_parity(gl, rl, what + " lse")


@pytest.mark.parametrize("L", [1, 100, 128, 129, 1000, 3001])
def test_decode_global_small(L):
    dec = synth.decode_inputs(2, L, 32, 4, 512, False, seed=L)
    check(dec, GLOBAL, what="decode L=%d" % L)


def test_decode_rotated_values_variant():
    dec = synth.decode_inputs(2, 777, 32, 4, 512, False, seed=5)
    check(dec, GLOBAL, kv_is_k=2, what="decode kv_is_k=2")


def test_decode_separate_values_and_window():
    dec = synth.decode_inputs(2, 1500, 32, 4, 512, True, seed=6)
    check(dec, GLOBAL, kv_is_k=0, what="decode separate v")
    check(dec, GLOBAL, kv_is_k=0, window=300, what="decode separate v, window 300")


def test_decode_local_layer_shape():
    loc = workloads.LOCAL_W1024
    dec = synth.decode_inputs(2, 2000, loc.n_q_heads, loc.n_kv_heads, loc.head_dim, True, seed=9)
    check(dec, loc, what="decode local")


@pytest.mark.parametrize("p,L,window,Hq,Hkv", [
    (1.0, 9000, 0, 16, 8),      # full RoPE, two turned slots, 70 pair-tiles per sequence
    (0.75, 3001, 1024, 16, 8),  # R = 96: slot 1 turned in part
    (0.5, 2500, 700, 16, 8),    # R = 64: one turned slot
    (1.0, 1800, 1024, 32, 2),   # 16 query heads per kv head: the absolute-angle path
    (1.0, 1500, 1024, 32, 4),   # 8 query heads per kv head: the absolute-angle path too
    (1.0, 1400, 512, 16, 4),    # 4 query heads per kv head: two turned slots
])
def test_decode_head_dim_256_rotation_variants(p, L, window, Hq, Hkv):
    # the relative rotation turns up to two slots at head_dim 256 (separate values); each
    # variant against the oracle
    ly = workloads.with_layer(workloads.LOCAL_W1024, rope_p=p, window=window, n_q_heads=Hq,
                              n_kv_heads=Hkv)
    dec = synth.decode_inputs(2, L, Hq, Hkv, 256, True, seed=int(100 * p) + L)
    check(dec, ly, what="decode d256 p=%.2f L=%d W=%d G=%d" % (p, L, window, Hq // Hkv))


def test_decode_empty_cache():
    b = binding()
    dev = torch.device("cuda:0")
    q = torch.randn(2, 1, 32, 512, device=dev).bfloat16()
    k = torch.empty(2, 0, 4, 512, dtype=torch.bfloat16, device=dev)
    out, lse = b.g4attn_decode(q, k, None, b.LayerCfg.from_layer(GLOBAL), want_lse=True)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert torch.all(torch.isinf(lse)) and torch.all(lse < 0)


@pytest.mark.parametrize("wl", [workloads.GLOBAL_DECODE_32K, workloads.GLOBAL_DECODE_128K])
def test_decode_full_size_sampled(wl):
    ly = wl.layer
    dec = synth.decode_inputs(wl.B, wl.L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                              seed=wl.seed)
    items = [0, 17, wl.B * ly.n_kv_heads - 1]      # (b, g) = (0,0), (4,1), (15,3)
    check(dec, ly, items=items, what=wl.name)


def test_decode_matches_last_prefill_row():
    """Decode at position T-1 against the normalised cache equals prefill row T-1."""
    b = binding()
    dev = torch.device("cuda:0")
    T = 517
    inp = synth.layer_inputs(1, T, 32, 4, 512, False, seed=21)
    cfg = b.LayerCfg.from_layer(GLOBAL)
    q, k, gq, gk = (x.to(dev) for x in (inp.q, inp.k, inp.gamma_q, inp.gamma_k))
    pre, pre_lse = b.g4attn_prefill(q, k, None, gq, gk, cfg, want_lse=True)
    _, kc, _ = b.g4attn_qknorm_rope(None, k, None, gk, cfg, pos0=0, want_krot=False)
    # the query of the last token sits at position T-1
    qn, _, _ = b.g4attn_qknorm_rope(q[:, T - 1:T].contiguous(), None, gq, None, cfg, pos0=T - 1)
    dout, dlse = b.g4attn_decode(qn, kc, None, cfg, want_lse=True)
    torch.cuda.synchronize()
    assert_parity(to_np(dout)[:, 0], to_np(pre)[:, T - 1], "decode vs prefill row")
    assert_parity(to_np(dlse), to_np(pre_lse)[:, :, T - 1], "decode vs prefill lse")


def test_bounded_wait_gives_up_and_reports_timeout():
    # a device wait that nothing satisfies gives up after its poll bound and records
    # G4ATTN_ERR_TIMEOUT; the status read clears it and the context stays usable
    b = binding()
    assert b.g4attn_device_status() == 0
    assert b.g4attn_wait_selftest(4096) == 0
    assert b.g4attn_device_status() == b.G4ATTN_ERR_TIMEOUT
    assert b.g4attn_device_status() == 0
    # the 2-second wall-clock bound applies with the default (unbounded) poll limit too
    assert b.g4attn_wait_selftest(0) == 0
    assert b.g4attn_device_status() == b.G4ATTN_ERR_TIMEOUT
    test_decode_global_small(300)   # kernels still run and match the oracle afterwards


# ------------------------------------------------------------ ring-buffer (local) decode
LOCAL = workloads.LOCAL_W512


def _ring(lin, L, C):
    """Ring of C rows (position p in row p % C) holding the last C positions of a linear
    [B, L, H, d] bf16 cache; rows never written hold NaN, which must never reach a result."""
    ring = torch.full((lin.shape[0], C) + tuple(lin.shape[2:]), float("nan"), dtype=torch.bfloat16)
    for p in range(max(0, L - C), L):
        ring[:, p % C] = lin[:, p]
    return ring


def check_ring(dec, layer, L, C, what, **kw):
    b = binding()
    dev = torch.device("cuda:0")
    cfg = b.LayerCfg.from_layer(layer, **kw)
    kr = _ring(dec.k, L, C)
    vr = None if dec.v is None else _ring(dec.v, L, C)
    out, lse = b.g4attn_decode_ring(dec.q.to(dev), kr.to(dev), None if vr is None else vr.to(dev),
                                    L, cfg, want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    ro, rl = oracle.decode_ring(dec.q[:, 0], kr, vr, L, ocfg(layer, **kw))
    go, gl = to_np(out.cpu())[:, 0], to_np(lse.cpu())
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
    assert_parity(go, ro, what + " out")
    assert_parity(gl, rl, what + " lse")


@pytest.mark.parametrize("L,C", [(1, 512), (100, 512), (512, 512), (513, 512), (700, 576),
                                 (3001, 512), (5000, 1024)])
def test_decode_ring_local_layer(L, C):
    # local layer: 16 q / 8 kv heads, d 256, full RoPE base 1e4, window 512, separate values
    dec = synth.decode_inputs(2, L, LOCAL.n_q_heads, LOCAL.n_kv_heads, LOCAL.head_dim, True,
                              seed=60 + L)
    check_ring(dec, LOCAL, L, C, "ring decode L=%d C=%d" % (L, C))


def test_decode_ring_keys_as_values_with_window():
    # a head_dim-512 keys-as-values layer with a window (the turned-slot path) on a ring
    dec = synth.decode_inputs(2, 1000, 32, 4, 512, False, seed=61)
    check_ring(dec, GLOBAL, 1000, 384, "ring decode K=V W=300", window=300)


def test_decode_ring_rejects_bad_rings():
    b = binding()
    dev = torch.device("cuda:0")
    dec = synth.decode_inputs(1, 10, 16, 8, 256, True, seed=62)
    q = dec.q.to(dev)
    kr = torch.zeros(1, 100, 8, 256, dtype=torch.bfloat16, device=dev)   # C not a multiple of 64
    with pytest.raises(b.G4AttnError):
        b.g4attn_decode_ring(q, kr, kr.clone(), 10, b.LayerCfg.from_layer(LOCAL))
    kr = torch.zeros(1, 256, 8, 256, dtype=torch.bfloat16, device=dev)   # window 512 > C
    with pytest.raises(b.G4AttnError):
        b.g4attn_decode_ring(q, kr, kr.clone(), 10, b.LayerCfg.from_layer(LOCAL))


# ------------------------------------------------------------------- split cache (37.5%)
def _split_cache(k_pre, R, base):
    """Rotated keys (each turned to its position, rounded to bf16) and the side copy of the
    pre-RoPE rotated dims [0, R) and [d/2, d/2 + R) of a pre-RoPE bf16 cache."""
    import bruteforce as bf
    kf = bf.bf16_to_f64(oracle.bf16_bits(k_pre))
    L, d = kf.shape[1], kf.shape[-1]
    krot = torch.from_numpy(bf.rope_complex(kf, np.arange(L), R, base)).to(torch.bfloat16)
    vside = torch.cat([k_pre[..., :R], k_pre[..., d // 2:d // 2 + R]], dim=-1).contiguous()
    return krot, vside


@pytest.mark.parametrize("L", [1, 129, 1000, 4097])
def test_decode_split_cache_matches_keys_as_values(L):
    b = binding()
    dev = torch.device("cuda:0")
    dec = synth.decode_inputs(2, L, 32, 4, 512, False, seed=70 + L)
    krot, vside = _split_cache(dec.k, 64, GLOBAL.rope_base)
    cfg = b.LayerCfg.from_layer(GLOBAL)
    out, lse = b.g4attn_decode_split_cache(dec.q.to(dev), krot.to(dev), vside.to(dev), cfg,
                                           want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    ro, rl = oracle.decode(dec.q[:, 0], dec.k, None, ocfg(GLOBAL))
    assert_parity(to_np(out.cpu())[:, 0], ro, "split cache L=%d out" % L)
    assert_parity(to_np(lse.cpu()), rl, "split cache L=%d lse" % L)


def test_decode_split_cache_needs_keys_as_values_and_r64():
    b = binding()
    dev = torch.device("cuda:0")
    dec = synth.decode_inputs(1, 10, 16, 8, 256, False, seed=71)
    z = torch.zeros(1, 10, 8, 128, dtype=torch.bfloat16, device=dev)
    with pytest.raises(b.G4AttnError):   # local layer: R = 128
        b.g4attn_decode_split_cache(dec.q.to(dev), dec.k.to(dev), z,
                                    b.LayerCfg.from_layer(workloads.LOCAL_W512, kv_is_k=1))


# ------------------------------------------- cache of turned keys (separate-value layers)
def _turned(k_pre, R, base):
    """Each cached key turned to its position (complex-number RoPE in fp64, rounded to bf16)."""
    import bruteforce as bf
    kf = bf.bf16_to_f64(oracle.bf16_bits(k_pre))
    return torch.from_numpy(bf.rope_complex(kf, np.arange(kf.shape[1]), R, base)).to(torch.bfloat16)


@pytest.mark.parametrize("L,C", [(1, 0), (700, 0), (3000, 0), (300, 512), (1500, 1024),
                                 (5000, 512)])
def test_decode_rotated_cache(L, C):
    # against the definition (scores on the stored keys as they are: the oracle without
    # rotation) and against the decode of the unrotated cache (within the bf16 rounding of the
    # stored keys)
    b = binding()
    dev = torch.device("cuda:0")
    dec = synth.decode_inputs(2, L, LOCAL.n_q_heads, LOCAL.n_kv_heads, LOCAL.head_dim, True,
                              seed=90 + L + C)
    R = oracle.rope_pairs(LOCAL.head_dim, LOCAL.rope_p)
    krot = _turned(dec.k, R, LOCAL.rope_base)
    kc, vc = (krot, dec.v) if C == 0 else (_ring(krot, L, C), _ring(dec.v, L, C))
    cfg = b.LayerCfg.from_layer(LOCAL)
    out, lse = b.g4attn_decode_rotated(dec.q.to(dev), kc.to(dev), vc.to(dev), L, cfg,
                                       ring=C > 0, want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    go, gl = to_np(out.cpu())[:, 0], to_np(lse.cpu())
    what = "turned-key decode L=%d C=%d" % (L, C)
    ro, rl = oracle.decode(dec.q[:, 0], krot, dec.v, ocfg(LOCAL, rope_p=0.0))
    assert_parity(go, ro, what + " out")
    assert_parity(gl, rl, what + " lse")
    ro2, rl2 = oracle.decode(dec.q[:, 0], dec.k, dec.v, ocfg(LOCAL))
    assert_parity(go, ro2, what + " out vs unrotated cache")
    assert_parity(gl, rl2, what + " lse vs unrotated cache")


def test_decode_rotated_refuses_keys_as_values():
    b = binding()
    dev = torch.device("cuda:0")
    dec = synth.decode_inputs(1, 10, 32, 4, 512, False, seed=91)
    with pytest.raises(b.G4AttnError):
        b.g4attn_decode_rotated(dec.q.to(dev), dec.k.to(dev), None, 10, b.LayerCfg.from_layer(GLOBAL))
