"""Host-only checks of the C ABI: the library loads without a GPU, exports every entry
point declared in include/g4attn.h, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "g4attn.h")


@pytest.fixture(scope="module")
def lib():
    from attention_g4attn_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


@pytest.fixture(scope="module")
def b():
    from attention_g4attn_b200 import build
    build.build()
    from attention_g4attn_b200 import binding
    return binding


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"G4ATTN_API\s+[\w\s\*]+?\b(g4attn_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ("g4attn_qknorm_rope", "g4attn_prefill", "g4attn_decode",
              "g4attn_prefill_workspace_size", "g4attn_decode_workspace_size",
              "g4attn_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(b):
    assert b.g4attn_status_string(0) == "ok"
    for code in range(-7, 0):
        s = b.g4attn_status_string(code)
        assert s and s != "unknown status"
    assert b.g4attn_status_string(-99) == "unknown status"
    assert "sm_100a" in b.g4attn_version()


def test_wait_limit_roundtrip(b):
    old = b.g4attn_set_wait_limit(1234)
    assert b.g4attn_set_wait_limit(0) == 1234       # < 1 restores the default
    assert b.g4attn_set_wait_limit(old) == old


def _align(x):
    return (x + 255) // 256 * 256


def test_prefill_workspace_formula(b):
    # normalised keys + rotated keys (bf16) + the (cos, sin) table of every position
    g = b.LayerCfg(32, 4, 512, 0.25, 1e6, 0, None, 1)
    B, T = 1, 32768
    rows = B * T * 4 * 512 * 2
    assert b.g4attn_prefill_workspace_size(B, T, g) == 2 * _align(rows) + _align(T * 64 * 8)
    # local layer: every chunk rotated and separate values -> no pre-RoPE copy
    loc = b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0)
    rows = 2 * 4096 * 8 * 256 * 2
    assert b.g4attn_prefill_workspace_size(2, 4096, loc) == _align(rows) + _align(4096 * 128 * 8)


def _decode_segments(B, Hkv, L, window, pairs=74, ring=0):
    """Stream-K split of a decode step, by brute force: the sequences' 128-key tiles form one
    flat range cut evenly over the CTA pairs; returns the most pairs any sequence meets.
    With a ring cache the tiles start at the 64-aligned position at or below the window."""
    key_lo = L - window if (window > 0 and L > window) else 0
    base = key_lo // 64 * 64 if ring else key_lo
    nt = -(-(L - base) // 128)
    W = B * Hkv * nt
    P = min(pairs, W)
    if W == 0:
        return 0
    starts = [p * W // P for p in range(P + 1)]
    most = 0
    for bg in range(B * Hkv):
        lo, hi = bg * nt, (bg + 1) * nt
        most = max(most, sum(1 for p in range(P) if starts[p] < hi and starts[p + 1] > lo))
    return most


@pytest.mark.parametrize("B,L,layer", [(16, 32768, "g"), (16, 131072, "g"), (2, 1000, "g"),
                                       (3, 5000, "l"), (1, 1, "g"), (37, 300, "g"), (5, 129, "l"),
                                       (1, 0, "g")])
def test_decode_workspace_follows_the_stream_k_split(b, B, L, layer):
    # two fp32 partials (d outputs + max, sum) per segment and (b, h), 256-byte aligned parts
    cfg = (b.LayerCfg(32, 4, 512, 0.25, 1e6, 0, None, 1) if layer == "g"
           else b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0))
    Hq, Hkv, d, window = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.window
    S = _decode_segments(B, Hkv, L, window)
    n = 2 * max(S, 1) * B * Hq
    assert b.g4attn_decode_workspace_size(B, L, cfg) == _align(n * d * 4) + _align(n * 2 * 4)


@pytest.mark.parametrize("B,L,C", [(2, 3001, 512), (16, 1024, 1024), (1, 1, 512), (3, 700, 576),
                                   (16, 70000, 1024)])
def test_decode_ring_workspace_follows_the_aligned_split(b, B, L, C):
    loc = b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0)
    S = _decode_segments(B, 8, L, 512, ring=C)
    n = 2 * max(S, 1) * B * 16
    assert b.g4attn_decode_ring_workspace_size(B, L, C, loc) == _align(n * 256 * 4) + _align(n * 2 * 4)


def test_decode_ring_rejects_bad_rings_without_gpu(b):
    loc = b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0)
    assert b.g4attn_decode_ring_workspace_size(1, 10, 100, loc) == 0   # C not a multiple of 64
    assert b.g4attn_decode_ring_workspace_size(1, 10, 256, loc) == 0   # window 512 > C
    assert b.g4attn_decode_ring_workspace_size(1, 10, 0, loc) == 0
    nowin = b.LayerCfg(16, 8, 256, 1.0, 1e4, 0, None, 0)
    assert b.g4attn_decode_ring_workspace_size(1, 10, 512, nowin) == 0  # no window: no ring


def test_invalid_configs_are_rejected(b):
    bad = [
        b.LayerCfg(6, 4, 512, 0.25, 1e6),        # Hq % Hkv != 0
        b.LayerCfg(8, 1, 384, 0.25, 1e6),        # head_dim not handled by the kernels
        b.LayerCfg(8, 1, 512, 1.5, 1e6),         # p outside [0, 1]
        b.LayerCfg(8, 1, 512, 0.25, -1.0),       # base <= 0
        b.LayerCfg(8, 1, 512, 0.25, 1e6, -3),    # negative window
        b.LayerCfg(8, 1, 512, 0.25, 1e6, 0, None, 3),   # kv_is_k out of range
        b.LayerCfg(256, 1, 512, 0.25, 1e6),      # G = 256 does not divide 128
        b.LayerCfg(8, 1, 512, 0.25, 1e6, 0, -0.1),   # non-positive softmax scale
    ]
    for cfg in bad:
        assert b.g4attn_prefill_workspace_size(1, 16, cfg) == 0
        assert b.g4attn_decode_workspace_size(1, 16, cfg) == 0


def _call_prefill(lib, b, cfg, q=0x1000, k=0x2000, v=None, gq=0x3000, gk=0x4000, out=0x5000,
                  ws=0x100000, ws_bytes=1 << 40, B=1, T=16):
    c = cfg.c()
    P = ctypes.c_void_p
    f = lib.g4attn_prefill
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, P, ctypes.c_size_t, ctypes.c_int, ctypes.c_int,
                  ctypes.POINTER(type(c)), P]
    return f(q, k, v, gq, gk, out, None, ws, ws_bytes, B, T, ctypes.byref(c), None)


def test_prefill_argument_checks_without_gpu(lib, b):
    g = b.LayerCfg(8, 1, 512, 0.25, 1e6)
    assert _call_prefill(lib, b, b.LayerCfg(6, 4, 512, 0.25, 1e6)) == b.G4ATTN_ERR_INVALID_ARG
    assert _call_prefill(lib, b, g, v=0x6000) == b.G4ATTN_ERR_INVALID_ARG     # K=V takes no v
    assert _call_prefill(lib, b, b.LayerCfg(8, 1, 512, 1.0, 1e4, 0, None, 0)) == \
        b.G4ATTN_ERR_INVALID_ARG                                              # v missing
    assert _call_prefill(lib, b, g, q=0x1001) == b.G4ATTN_ERR_MISALIGNED
    assert _call_prefill(lib, b, g, ws_bytes=16) == b.G4ATTN_ERR_WORKSPACE
    assert _call_prefill(lib, b, g, ws=None) == b.G4ATTN_ERR_WORKSPACE
    assert _call_prefill(lib, b, g, ws=0x100010) == b.G4ATTN_ERR_MISALIGNED  # 256 B rule
    assert _call_prefill(lib, b, g, gq=None) == b.G4ATTN_ERR_INVALID_ARG      # QKNorm gains
    assert _call_prefill(lib, b, g, B=-1) == b.G4ATTN_ERR_INVALID_ARG
    assert _call_prefill(lib, b, g, T=0) == b.G4ATTN_OK                       # empty: no-op


def test_decode_argument_checks_without_gpu(lib, b):
    P = ctypes.c_void_p
    f = lib.g4attn_decode
    f.restype = ctypes.c_int
    g = b.LayerCfg(32, 4, 512, 0.25, 1e6).c()
    f.argtypes = [P, P, P, ctypes.c_int, P, P, P, ctypes.c_size_t, ctypes.c_int,
                  ctypes.POINTER(type(g)), P]
    assert f(0x1000, 0x2000, 0x3000, 16, 0x4000, None, 0x10000, 1 << 30, 1, ctypes.byref(g),
             None) == b.G4ATTN_ERR_INVALID_ARG   # K=V layer given a value cache
    assert f(0x1000, 0x2000, None, -1, 0x4000, None, 0x10000, 1 << 30, 1, ctypes.byref(g),
             None) == b.G4ATTN_ERR_INVALID_ARG
    g32 = b.LayerCfg(64, 2, 512, 0.25, 1e6).c()     # 32 query heads per KV head
    assert f(0x1000, 0x2000, None, 16, 0x4000, None, 0x10000, 1 << 30, 1, ctypes.byref(g32),
             None) == b.G4ATTN_ERR_UNSUPPORTED
    assert f(0x1000, 0x2001, None, 16, 0x4000, None, 0x10000, 1 << 30, 1, ctypes.byref(g),
             None) == b.G4ATTN_ERR_MISALIGNED


def test_binding_refuses_host_tensors(b):
    import torch
    q = torch.zeros(1, 4, 8, 512, dtype=torch.bfloat16)
    k = torch.zeros(1, 4, 1, 512, dtype=torch.bfloat16)
    g = torch.ones(512)
    with pytest.raises(b.G4AttnError):
        b.g4attn_prefill(q, k, None, g, g, b.LayerCfg(8, 1, 512, 0.25, 1e6), out=q.clone(),
                         workspace=torch.zeros(16, dtype=torch.uint8))


def test_prefill_chunk_workspace_covers_the_visible_positions(b):
    # causal layer: every earlier position is visible, so the key rows are those of a
    # prefill of P + Tn tokens
    g = b.LayerCfg(32, 4, 512, 0.25, 1e6, 0, None, 1)
    assert b.g4attn_prefill_chunk_workspace_size(1, 30000, 2768, g) == \
        b.g4attn_prefill_workspace_size(1, 32768, g)
    # window 512: positions P-511 .. P+Tn-1, plus a copy of their values
    loc = b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0)
    Tk = 511 + 100
    rows = 2 * Tk * 8 * 256 * 2
    assert b.g4attn_prefill_chunk_workspace_size(2, 3000, 100, loc) == \
        2 * _align(rows) + _align(Tk * 128 * 8)
    Tk = 300 + 100   # P < W: all P earlier positions
    rows = 2 * Tk * 8 * 256 * 2
    assert b.g4attn_prefill_chunk_workspace_size(2, 300, 100, loc) == \
        2 * _align(rows) + _align(Tk * 128 * 8)
    assert b.g4attn_prefill_chunk_workspace_size(1, -1, 10, g) == 0


def _call_chunk(lib, b, cfg, v=None, kc=0x7000, vc=None, rows=1 << 20, ring=0, ws=0x100000,
                ws_bytes=1 << 40, B=1, P=100, Tn=16):
    c = cfg.c()
    Pt, I = ctypes.c_void_p, ctypes.c_int
    f = lib.g4attn_prefill_chunk
    f.restype = I
    f.argtypes = [Pt, Pt, Pt, Pt, Pt, Pt, Pt, I, I, Pt, Pt, Pt, ctypes.c_size_t, I, I, I,
                  ctypes.POINTER(type(c)), Pt]
    return f(0x1000, 0x2000, v, 0x3000, 0x4000, kc, vc, rows, ring, 0x5000, None, ws, ws_bytes,
             B, P, Tn, ctypes.byref(c), None)


def test_prefill_chunk_argument_checks_without_gpu(lib, b):
    g = b.LayerCfg(8, 1, 512, 0.25, 1e6)
    loc = b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0)
    E = b.G4ATTN_ERR_INVALID_ARG
    assert _call_chunk(lib, b, g, rows=115) == E                     # linear cache < P + Tn
    assert _call_chunk(lib, b, g, rows=512, ring=1) == E             # ring without a window
    assert _call_chunk(lib, b, loc, v=0x6000, vc=0x8000, rows=256, ring=1) == E   # W > ring
    assert _call_chunk(lib, b, g, ring=2) == E                       # turned keys: K=V layer
    assert _call_chunk(lib, b, g, ring=4) == E                       # unknown flag
    assert _call_chunk(lib, b, loc, v=0x6000, vc=0x8000, ring=8) == E
    assert _call_chunk(lib, b, g, P=-1) == E
    assert _call_chunk(lib, b, g, vc=0x8000) == E                    # K=V layer: no values
    assert _call_chunk(lib, b, loc, v=0x6000) == E                   # values but no value cache
    assert _call_chunk(lib, b, g, kc=None) == E
    assert _call_chunk(lib, b, g, kc=0x7008) == b.G4ATTN_ERR_MISALIGNED
    assert _call_chunk(lib, b, g, ws_bytes=16) == b.G4ATTN_ERR_WORKSPACE
    assert _call_chunk(lib, b, g, Tn=0) == b.G4ATTN_OK               # empty chunk: no-op


def test_decode_rotated_workspace_and_checks_without_gpu(lib, b):
    loc = b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0)
    assert b.g4attn_decode_rotated_workspace_size(4, 5000, 0, loc) == \
        b.g4attn_decode_workspace_size(4, 5000, loc)
    assert b.g4attn_decode_rotated_workspace_size(4, 5000, 1024, loc) == \
        b.g4attn_decode_ring_workspace_size(4, 5000, 1024, loc)
    assert b.g4attn_decode_rotated_workspace_size(4, 5000, 100, loc) == 0   # C % 64 != 0
    assert b.g4attn_decode_rotated_workspace_size(4, 5000, -64, loc) == 0
    Pt, I = ctypes.c_void_p, ctypes.c_int
    f = lib.g4attn_decode_rotated
    f.restype = I
    g = b.LayerCfg(32, 4, 512, 0.25, 1e6).c()
    lc = loc.c()
    f.argtypes = [Pt, Pt, Pt, I, I, Pt, Pt, Pt, ctypes.c_size_t, I, ctypes.POINTER(type(g)), Pt]
    # keys-as-values layer: its cache holds unrotated keys
    assert f(0x1000, 0x2000, None, 16, 0, 0x4000, None, 0x10000, 1 << 30, 1, ctypes.byref(g),
             None) == b.G4ATTN_ERR_UNSUPPORTED
    assert f(0x1000, 0x2000, 0x3000, 16, 100, 0x4000, None, 0x10000, 1 << 30, 1,
             ctypes.byref(lc), None) == b.G4ATTN_ERR_INVALID_ARG              # bad ring
    assert f(0x1000, 0x2000, None, 16, 0, 0x4000, None, 0x10000, 1 << 30, 1, ctypes.byref(lc),
             None) == b.G4ATTN_ERR_INVALID_ARG                                # values missing


def test_quantize_int8_argument_checks_without_gpu(lib, b):
    Pt = ctypes.c_void_p
    f = lib.g4attn_quantize_int8
    f.restype = ctypes.c_int
    f.argtypes = [Pt, Pt, Pt, ctypes.c_longlong, ctypes.c_int, Pt]
    assert f(0x1000, 0x2000, 0x3000, 10, 384, None) == b.G4ATTN_ERR_INVALID_ARG   # d
    assert f(0x1000, 0x2000, 0x3000, -1, 512, None) == b.G4ATTN_ERR_INVALID_ARG
    assert f(None, 0x2000, 0x3000, 10, 512, None) == b.G4ATTN_ERR_INVALID_ARG
    assert f(0x1008, 0x2000, 0x3000, 10, 512, None) == b.G4ATTN_ERR_MISALIGNED
    assert f(0x1000, 0x2000, 0x3002, 10, 512, None) == b.G4ATTN_ERR_MISALIGNED
    assert f(None, None, None, 0, 512, None) == b.G4ATTN_OK                       # empty


def test_decode_int8_argument_checks_without_gpu(lib, b):
    loc = b.LayerCfg(32, 16, 256, 1.0, 1e4, 1024, None, 0)
    glb = b.LayerCfg(32, 4, 512, 0.25, 1e6)
    # same split-KV partials as the bf16 decode of the same geometry
    assert b.g4attn_decode_int8_workspace_size(16, 32768, 0, glb) == \
        b.g4attn_decode_workspace_size(16, 32768, glb)
    assert b.g4attn_decode_int8_workspace_size(16, 65536, 1024, loc) == \
        b.g4attn_decode_ring_workspace_size(16, 65536, 1024, loc)
    assert b.g4attn_decode_int8_workspace_size(16, 65536, 1000, loc) == 0   # C % 64 != 0
    Pt, I = ctypes.c_void_p, ctypes.c_int
    f = lib.g4attn_decode_int8
    f.restype = I
    g, lc = glb.c(), loc.c()
    f.argtypes = [Pt, Pt, Pt, Pt, Pt, I, I, Pt, Pt, Pt, ctypes.c_size_t, I,
                  ctypes.POINTER(type(g)), Pt]
    ws = (0x100000, 1 << 30)
    # keys as values: no value codes; separate values: both codes and scales
    assert f(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 16, 0, 0x6000, None, *ws, 1,
             ctypes.byref(g), None) == b.G4ATTN_ERR_INVALID_ARG
    assert f(0x1000, 0x2000, 0x3000, 0x4000, None, 16, 1024, 0x6000, None, *ws, 1,
             ctypes.byref(lc), None) == b.G4ATTN_ERR_INVALID_ARG
    assert f(0x1000, 0x2000, None, None, None, 16, 0, 0x6000, None, *ws, 1,
             ctypes.byref(g), None) == b.G4ATTN_ERR_INVALID_ARG               # key scales missing
    assert f(0x1000, 0x2008, 0x3000, None, None, 16, 0, 0x6000, None, *ws, 1,
             ctypes.byref(g), None) == b.G4ATTN_ERR_MISALIGNED                # codes
    assert f(0x1000, 0x2000, 0x3002, None, None, 16, 0, 0x6000, None, *ws, 1,
             ctypes.byref(g), None) == b.G4ATTN_ERR_MISALIGNED                # scales
    assert f(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 16, 100, 0x6000, None, *ws, 1,
             ctypes.byref(lc), None) == b.G4ATTN_ERR_INVALID_ARG              # bad ring
    g16 = b.LayerCfg(32, 2, 512, 0.25, 1e6).c()                               # 16 q heads per kv head
    assert f(0x1000, 0x2000, 0x3000, None, None, 16, 0, 0x6000, None, *ws, 1,
             ctypes.byref(g16), None) == b.G4ATTN_ERR_UNSUPPORTED


def test_header_compiles_as_plain_c(tmp_path):
    # the boundary is a C ABI: the public header must stand alone in a C99 translation unit
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "g4attn.h"\n'
                   "int probe(void) { g4attn_layer_cfg c; (void)c; "
                   "return G4ATTN_CACHE_RING | G4ATTN_CACHE_ROTATED; }\n")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                        "-c", str(src), "-o", str(tmp_path / "use_header.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.parametrize("seed", range(4))
def test_prefill_chunk_frame_over_random_chunks(b, seed):
    # the frame holds the positions any chunk query can see: from max(0, P - W + 1) (0 when
    # causal) to P + Tn - 1; its workspace is the fp16 key copies, the (cos, sin) table and,
    # with separate values, a bf16 value copy of those rows
    rng = np.random.default_rng(seed)
    layers = [b.LayerCfg(32, 4, 512, 0.25, 1e6, 0, None, 1),       # global: pre-RoPE + rotated
              b.LayerCfg(16, 8, 256, 1.0, 1e4, 512, None, 0),      # local: rotated + values
              b.LayerCfg(16, 8, 256, 0.5, 1e4, 100, None, 1)]      # both copies, K=V
    for _ in range(25):
        c = layers[rng.integers(len(layers))]
        B, P, Tn = int(rng.integers(1, 4)), int(rng.integers(0, 5000)), int(rng.integers(1, 3000))
        W, d, Hkv, kvk = c.window, c.head_dim, c.n_kv_heads, c.kv_is_k
        kb = max(0, P - W + 1) if W > 0 else 0
        Tk = P + Tn - kb
        R = int(c.rope_p * d / 2)
        rows = _align(B * Tk * Hkv * d * 2)
        need_kn = kvk == 1 or R < d // 2
        want = (2 if need_kn else 1) * rows + _align(Tk * max(R, 1) * 8) + (rows if kvk == 0 else 0)
        assert b.g4attn_prefill_chunk_workspace_size(B, P, Tn, c) == want, (B, P, Tn, W)
