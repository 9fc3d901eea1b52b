"""GPU parity of the chunked prefill (g4attn_prefill_chunk) against the oracle: one chunk
against a linear or ring cache, the keys and values it appends, and a prompt fed in
chunks against the full-sequence prefill."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import binding, ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
GLOBAL = workloads.GLOBAL_TINY                      # 8 query heads on 1 kv head, d = 512
LOCAL = workloads.LOCAL_W512                        # 16 / 8 heads, d = 256, W = 512
POISON = 0x7F80                                     # bf16 +inf: rows that must not be read


def _bits(t):
    return oracle.bf16_bits(t)


def _from_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _cache(lin_bits, P, rows, ring):
    """The cache the kernel reads: positions 0 .. P-1 of lin_bits (linear: row p; ring:
    row p % rows, last `rows` positions), every other row poisoned."""
    shape = (lin_bits.shape[0], rows) + lin_bits.shape[2:]
    c = np.full(shape, POISON, np.uint16)
    for p in range(max(0, P - rows) if ring else 0, P):
        c[:, p % rows if ring else p] = lin_bits[:, p]
    return c


def _turned(k_pre, R, base):
    """Keys turned to their positions (complex-number RoPE in fp64, rounded to bf16)."""
    import bruteforce as bf
    kf = bf.bf16_to_f64(_bits(k_pre))
    return torch.from_numpy(bf.rope_complex(kf, np.arange(kf.shape[1]), R, base)).to(torch.bfloat16)


def _run_chunk(ch, ly, P, rows, ring, rotated=False):
    b = binding()
    cfg = b.LayerCfg.from_layer(ly)
    kpre = ch.kcache
    if rotated:
        kpre = _turned(kpre, oracle.rope_pairs(ly.head_dim, ly.rope_p), ly.rope_base)
    kc = _from_bits(_cache(_bits(kpre), P, rows, ring)).to(DEV)
    vc = None
    if ch.vcache is not None:
        vc = _from_bits(_cache(_bits(ch.vcache), P, rows, ring)).to(DEV)
    v = None if ch.v is None else ch.v.to(DEV)
    out, lse = b.g4attn_prefill_chunk(ch.q.to(DEV), ch.k.to(DEV), v, ch.gamma_q.to(DEV),
                                      ch.gamma_k.to(DEV), kc, vc, P, cfg, ring=ring,
                                      rotated=rotated, want_lse=True)
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    return out.cpu(), lse.cpu(), kc.cpu(), None if vc is None else vc.cpu()


def _check_appended(ch, ly, P, Tn, rows, ring, kc, vc, before_k, before_v, rotated=False):
    """Rows of positions P .. P+Tn-1 hold RMS(k) * gamma_k (turned to its position when
    rotated) rounded to bf16, and v as given; every other row is as it was."""
    _, kh, kr = oracle.qknorm_rope(None, ch.k, None, ch.gamma_k, ocfg(ly), pos0=P)
    if rotated:
        kh = kr
    got_k, got_v = _bits(kc), None if vc is None else _bits(vc)
    written = set()
    for t in range(max(0, Tn - rows) if ring else 0, Tn):
        r = (P + t) % rows if ring else P + t
        written.add(r)
        g = to_np(_from_bits(got_k[:, r]))
        # one bf16 rounding, plus the fp32 turn's error on components that cancel
        np.testing.assert_allclose(g, kh[:, t], rtol=2.0 ** -8, atol=1e-5 if rotated else 1e-30)
        if vc is not None:
            np.testing.assert_array_equal(got_v[:, r], _bits(ch.v)[:, t])
    keep = [r for r in range(rows) if r not in written]
    np.testing.assert_array_equal(got_k[:, keep], before_k[:, keep])
    if vc is not None:
        np.testing.assert_array_equal(got_v[:, keep], before_v[:, keep])


def _chunk_case(ly, B, P, Tn, rows, ring, seed, rotated=False):
    ch = synth.chunk_inputs(B, P, Tn, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, ly.separate_v,
                            seed=seed)
    out, lse, kc, vc = _run_chunk(ch, ly, P, rows, ring, rotated)
    ro, rl = oracle.prefill_chunk(ch.q, ch.k, ch.v, ch.kcache, ch.vcache, ch.gamma_q,
                                  ch.gamma_k, P, ocfg(ly))
    what = "chunk P=%d Tn=%d rows=%d ring=%d" % (P, Tn, rows, ring)
    assert_parity(to_np(out), ro, what + " out")
    assert_parity(to_np(lse), rl, what + " lse")
    kpre = ch.kcache
    if rotated:
        kpre = _turned(kpre, oracle.rope_pairs(ly.head_dim, ly.rope_p), ly.rope_base)
    before_k = _cache(_bits(kpre), P, rows, ring)
    before_v = None if ch.vcache is None else _cache(_bits(ch.vcache), P, rows, ring)
    _check_appended(ch, ly, P, Tn, rows, ring, kc, vc, before_k, before_v, rotated)


@pytest.mark.parametrize("P,Tn", [(0, 200), (128, 128), (300, 77), (1000, 256), (4097, 130),
                                  (50, 1)])
def test_global_chunk_linear_cache(P, Tn):
    _chunk_case(GLOBAL, 1, P, Tn, P + Tn + 64, False, 100 + P)


def test_global_chunk_full_rope_cos_sin_from_table():
    # full RoPE at head_dim 512: the prologue reads the (cos, sin) rows of the chunk's
    # positions from the workspace table, at the chunk's offset into it
    _chunk_case(workloads.with_layer(GLOBAL, rope_p=1.0), 1, 333, 37, 400, False, 8)


def test_global_chunk_two_kv_heads_two_batches():
    ly = workloads.with_layer(workloads.GLOBAL_8TO1, n_q_heads=16, n_kv_heads=2)
    _chunk_case(ly, 2, 700, 300, 1000, False, 7)


@pytest.mark.parametrize("P,Tn", [(700, 300), (100, 600), (2000, 129), (511, 1)])
def test_local_chunk_linear_cache(P, Tn):
    _chunk_case(LOCAL, 2, P, Tn, P + Tn, False, 200 + P)


@pytest.mark.parametrize("P,Tn,C", [(1500, 300, 512), (1500, 300, 1024), (300, 200, 512),
                                    (600, 1100, 512), (4000, 64, 640)])
def test_local_chunk_ring_cache(P, Tn, C):
    _chunk_case(LOCAL, 1, P, Tn, C, True, 300 + P + C)


@pytest.mark.parametrize("P,Tn,C", [(700, 300, 0), (1500, 300, 512), (600, 1100, 512)])
def test_local_chunk_turned_key_cache(P, Tn, C):
    # the cache holds keys turned to their positions: read as stored, appended turned; the
    # oracle works on the unrotated cache (within the bf16 rounding of the turned keys)
    _chunk_case(LOCAL, 1, P, Tn, C if C else P + Tn, C > 0, 400 + P, rotated=True)


def test_local_chunk_keys_as_values_window():
    ly = workloads.with_layer(LOCAL, kv_is_k=1, window=100)
    _chunk_case(ly, 1, 450, 200, 700, False, 9)


@pytest.mark.parametrize("ly,cuts,ring_rows,rotated", [
    (GLOBAL, (0, 700, 1300, 2000), 0, False),
    (workloads.with_layer(LOCAL, window=256), (0, 300, 301, 900, 1500), 0, False),
    (workloads.with_layer(LOCAL, window=256), (0, 300, 301, 900, 1500), 320, False),
    (workloads.with_layer(LOCAL, window=256), (0, 300, 301, 900, 1500), 320, True),
    # the 5:1 block's local layer (32 q / 16 kv heads, d 256, window 1024) in its serving
    # layout: a ring of 1024 rows holding turned keys, then a decode step
    (workloads.LOCAL_W1024, (0, 1500, 2600, 3000), 1024, True)])
def test_prompt_in_chunks_matches_the_full_prefill(ly, cuts, ring_rows, rotated):
    # a prompt fed in chunks, each against the cache the previous chunks wrote, gives the
    # full-sequence prefill (the cache rounds the normalised keys to bf16: within the bar)
    b = binding()
    T = cuts[-1]
    inp = synth.layer_inputs(1, T, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, ly.separate_v,
                             seed=11 + T)
    cfg = b.LayerCfg.from_layer(ly)
    rows = ring_rows or T
    kc = torch.zeros((1, rows, ly.n_kv_heads, ly.head_dim), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc) if ly.separate_v else None
    outs, lses = [], []
    for P, E in zip(cuts[:-1], cuts[1:]):
        sl = slice(P, E)
        v = None if inp.v is None else inp.v[:, sl].contiguous().to(DEV)
        o, l = b.g4attn_prefill_chunk(inp.q[:, sl].contiguous().to(DEV),
                                      inp.k[:, sl].contiguous().to(DEV), v,
                                      inp.gamma_q.to(DEV), inp.gamma_k.to(DEV), kc, vc, P, cfg,
                                      ring=bool(ring_rows), rotated=rotated, want_lse=True)
        outs.append(o.cpu())
        lses.append(l.cpu())
    torch.cuda.synchronize()
    assert b.g4attn_device_status() == 0
    out, lse = torch.cat(outs, dim=1), torch.cat(lses, dim=2)
    ro, rl = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, ocfg(ly))
    assert_parity(to_np(out), ro, "chunked prompt out")
    assert_parity(to_np(lse), rl, "chunked prompt lse")
    if ring_rows and rotated:
        # the next token's decode against the cache the chunks left (turned keys, ring)
        gen = torch.Generator().manual_seed(5)
        qn = torch.randn((1, 1, ly.n_q_heads, ly.head_dim), generator=gen).to(torch.bfloat16)
        o, l = b.g4attn_decode_rotated(qn.to(DEV), kc, vc, T, cfg, ring=True, want_lse=True)
        torch.cuda.synchronize()
        assert b.g4attn_device_status() == 0
        # the oracle's cache: the normalised keys of the whole prompt (exact, unrotated)
        _, kh, _ = oracle.qknorm_rope(None, inp.k, None, inp.gamma_k, ocfg(ly))
        kh_bits = oracle.bf16_bits(torch.from_numpy(kh).to(torch.bfloat16))
        ro, rl = oracle.decode(qn[:, 0], kh_bits, inp.v, ocfg(ly))
        assert_parity(to_np(o.cpu())[:, 0], ro, "decode after chunks out")
        assert_parity(to_np(l.cpu()), rl, "decode after chunks lse")
