"""Python binding of the g4attn C ABI (include/g4attn.h).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
libg4attn.so.  torch provides device memory and the current stream.  Importing this
module raises G4AttnError when the shared library is missing; there is no fallback.
"""
import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libg4attn.so")

G4ATTN_OK = 0
G4ATTN_ERR_INVALID_ARG = -1
G4ATTN_ERR_UNSUPPORTED = -2
G4ATTN_ERR_MISALIGNED = -3
G4ATTN_ERR_WORKSPACE = -4
G4ATTN_ERR_CUDA = -5
G4ATTN_ERR_TIMEOUT = -6
G4ATTN_ERR_TOO_LARGE = -7


class G4AttnError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        msg = "%s (status %d)" % (_status_str(code), code)
        super().__init__(what + ": " + msg if what else msg)


class _CCfg(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("rope_p", ctypes.c_float),
        ("rope_base", ctypes.c_double),
        ("window", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("kv_is_k", ctypes.c_int),
        ("qk_norm", ctypes.c_int),
        ("qk_norm_eps", ctypes.c_float),
    ]


@dataclass
class LayerCfg:
    """Mirror of g4attn_layer_cfg."""
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_p: float
    rope_base: float
    window: int = 0
    scale: Optional[float] = None
    kv_is_k: int = 1
    qk_norm: int = 1
    qk_norm_eps: float = 1e-6

    def c(self) -> _CCfg:
        scale = self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)
        return _CCfg(self.n_q_heads, self.n_kv_heads, self.head_dim, self.rope_p,
                     self.rope_base, self.window, scale, self.kv_is_k, self.qk_norm,
                     self.qk_norm_eps)

    @classmethod
    def from_layer(cls, ly, **kw):
        d = dict(n_q_heads=ly.n_q_heads, n_kv_heads=ly.n_kv_heads, head_dim=ly.head_dim,
                 rope_p=ly.rope_p, rope_base=ly.rope_base, window=ly.window,
                 scale=ly.scale, kv_is_k=ly.kv_is_k, qk_norm=ly.qk_norm,
                 qk_norm_eps=ly.qk_norm_eps)
        d.update(kw)
        return cls(**d)


def _load():
    if not os.path.exists(LIB_PATH):
        raise G4AttnError(G4ATTN_ERR_UNSUPPORTED,
                          "libg4attn.so is missing at %s; build it with "
                          "`python -m attention_g4attn_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    CFG = ctypes.POINTER(_CCfg)
    sig = {
        "g4attn_qknorm_rope": (I, [P, P, P, P, P, P, P, I, I, LL, CFG, P]),
        "g4attn_prefill_workspace_size": (SZ, [I, I, CFG]),
        "g4attn_prefill": (I, [P, P, P, P, P, P, P, P, SZ, I, I, CFG, P]),
        "g4attn_prefill_chunk_workspace_size": (SZ, [I, I, I, CFG]),
        "g4attn_prefill_chunk": (I, [P, P, P, P, P, P, P, I, I, P, P, P, SZ, I, I, I, CFG, P]),
        "g4attn_decode_workspace_size": (SZ, [I, I, CFG]),
        "g4attn_decode": (I, [P, P, P, I, P, P, P, SZ, I, CFG, P]),
        "g4attn_decode_noalloc": (I, [P, P, P, I, P, P, I, CFG, P]),
        "g4attn_decode_ring_workspace_size": (SZ, [I, I, I, CFG]),
        "g4attn_decode_ring": (I, [P, P, P, I, I, P, P, P, SZ, I, CFG, P]),
        "g4attn_decode_split_cache": (I, [P, P, P, I, P, P, P, SZ, I, CFG, P]),
        "g4attn_decode_rotated_workspace_size": (SZ, [I, I, I, CFG]),
        "g4attn_decode_rotated": (I, [P, P, P, I, I, P, P, P, SZ, I, CFG, P]),
        "g4attn_quantize_int8": (I, [P, P, P, LL, I, P]),
        "g4attn_decode_int8_workspace_size": (SZ, [I, I, I, CFG]),
        "g4attn_decode_int8": (I, [P, P, P, P, P, I, I, P, P, P, SZ, I, CFG, P]),
        "g4attn_status_string": (ctypes.c_char_p, [I]),
        "g4attn_device_status": (I, [P]),
        "g4attn_set_wait_limit": (LL, [LL]),
        "g4attn_wait_selftest": (I, [LL, P]),
        "g4attn_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library_path() -> str:
    return LIB_PATH


def _status_str(code: int) -> str:
    try:
        return _lib.g4attn_status_string(code).decode()
    except NameError:
        return "status"


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise G4AttnError(G4ATTN_ERR_INVALID_ARG, "tensors must live in device memory")
    if not t.is_contiguous():
        raise G4AttnError(G4ATTN_ERR_INVALID_ARG, "tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc, what):
    if rc != G4ATTN_OK:
        raise G4AttnError(rc, what)


def _bf16(t, what):
    if t is not None and t.dtype != torch.bfloat16:
        raise G4AttnError(G4ATTN_ERR_INVALID_ARG, what + " must be bfloat16")


def g4attn_status_string(code: int) -> str:
    return _status_str(code)


def g4attn_version() -> str:
    return _lib.g4attn_version().decode()


def g4attn_set_wait_limit(polls: int) -> int:
    return _lib.g4attn_set_wait_limit(int(polls))


def g4attn_device_status(stream=None) -> int:
    return _lib.g4attn_device_status(_stream(stream))


def g4attn_wait_selftest(polls: int = 0, stream=None) -> int:
    """Launch the bounded-wait self-test (a wait that nothing satisfies); read the outcome
    with g4attn_device_status."""
    return _lib.g4attn_wait_selftest(int(polls), _stream(stream))


def g4attn_prefill_workspace_size(B: int, T: int, cfg: LayerCfg) -> int:
    c = cfg.c()
    return _lib.g4attn_prefill_workspace_size(B, T, ctypes.byref(c))


def g4attn_decode_workspace_size(B: int, L: int, cfg: LayerCfg) -> int:
    c = cfg.c()
    return _lib.g4attn_decode_workspace_size(B, L, ctypes.byref(c))


def g4attn_qknorm_rope(q_in, k_in, gamma_q, gamma_k, cfg: LayerCfg, pos0: int = 0,
                       q_out=None, kcache_out=None, krot_out=None, want_krot=True,
                       stream=None):
    """QKNorm + RoPE of a block of tokens.  Returns (q_out, kcache_out, krot_out)."""
    for t, n in ((q_in, "q_in"), (k_in, "k_in")):
        _bf16(t, n)
    if q_in is not None and q_out is None:
        q_out = torch.empty_like(q_in)
    if k_in is not None:
        if kcache_out is None:
            kcache_out = torch.empty_like(k_in)
        if krot_out is None and want_krot:
            krot_out = torch.empty_like(k_in)
    ref = q_in if q_in is not None else k_in
    B, T = ref.shape[0], ref.shape[1]
    c = cfg.c()
    rc = _lib.g4attn_qknorm_rope(_ptr(q_in), _ptr(k_in), _ptr(q_out), _ptr(kcache_out),
                                 _ptr(krot_out), _ptr(gamma_q), _ptr(gamma_k), B, T, pos0,
                                 ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_qknorm_rope")
    return q_out, kcache_out, krot_out


def g4attn_prefill(q, k, v, gamma_q, gamma_k, cfg: LayerCfg, out=None, lse=None,
                   want_lse=False, workspace=None, stream=None):
    """Prefill attention.  q [B,T,Hq,d], k/v [B,T,Hkv,d] bf16 raw.  Returns (out, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n)
    B, T = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads, T), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_prefill_workspace_size(B, T, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma_q), _ptr(gamma_k),
                             _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), B, T,
                             ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_prefill")
    return out, lse


def g4attn_prefill_chunk_workspace_size(B: int, P: int, Tn: int, cfg: LayerCfg) -> int:
    c = cfg.c()
    return _lib.g4attn_prefill_chunk_workspace_size(B, P, Tn, ctypes.byref(c))


G4ATTN_CACHE_RING = 1
G4ATTN_CACHE_ROTATED = 2


def g4attn_prefill_chunk(q, k, v, gamma_q, gamma_k, kcache, vcache, P: int, cfg: LayerCfg,
                         ring=False, rotated=False, out=None, lse=None, want_lse=False,
                         workspace=None, stream=None):
    """Prefill of a chunk: q [B,Tn,Hq,d], k/v [B,Tn,Hkv,d] raw, at positions P..P+Tn-1,
    against kcache/vcache [B, rows, Hkv, d] (normalised keys, turned to their positions
    with rotated=True; position p in row p, or in row p % rows with ring=True), which
    receive the chunk's keys and values.  Returns (out, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (kcache, "kcache"), (vcache, "vcache")):
        _bf16(t, n)
    B, Tn = q.shape[0], q.shape[1]
    rows = kcache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads, Tn), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_prefill_chunk_workspace_size(B, int(P), Tn, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma_q), _ptr(gamma_k),
                                   _ptr(kcache), _ptr(vcache), rows,
                                   (G4ATTN_CACHE_RING if ring else 0) |
                                   (G4ATTN_CACHE_ROTATED if rotated else 0), _ptr(out),
                                   _ptr(lse), _ptr(workspace), workspace.numel(), B, int(P), Tn,
                                   ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_prefill_chunk")
    return out, lse


def g4attn_decode(q, kcache, vcache, cfg: LayerCfg, out=None, lse=None, want_lse=False,
                  workspace=None, stream=None):
    """Decode one token.  q [B,1,Hq,d] normalised + rotated, kcache [B,L,Hkv,d]."""
    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache")):
        _bf16(t, n)
    B, L = kcache.shape[0], kcache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_decode_workspace_size(B, L, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), L, _ptr(out), _ptr(lse),
                            _ptr(workspace), workspace.numel(), B, ctypes.byref(c),
                            _stream(stream))
    _check(rc, "g4attn_decode")
    return out, lse


def g4attn_decode_ring_workspace_size(B: int, L: int, C: int, cfg: LayerCfg) -> int:
    c = cfg.c()
    return _lib.g4attn_decode_ring_workspace_size(B, L, C, ctypes.byref(c))


def g4attn_decode_ring(q, kring, vring, L: int, cfg: LayerCfg, out=None, lse=None,
                       want_lse=False, workspace=None, stream=None):
    """Decode one token at position L-1 against ring caches kring/vring [B, C, Hkv, d]
    (position p in row p % C; window = cfg.window <= C)."""
    for t, n in ((q, "q"), (kring, "kring"), (vring, "vring")):
        _bf16(t, n)
    B, C = kring.shape[0], kring.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_decode_ring_workspace_size(B, L, C, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_decode_ring(_ptr(q), _ptr(kring), _ptr(vring), int(L), C, _ptr(out),
                                 _ptr(lse), _ptr(workspace), workspace.numel(), B,
                                 ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_decode_ring")
    return out, lse


def g4attn_decode_rotated_workspace_size(B: int, L: int, C: int, cfg: LayerCfg) -> int:
    c = cfg.c()
    return _lib.g4attn_decode_rotated_workspace_size(B, L, C, ctypes.byref(c))


def g4attn_decode_rotated(q, krot, vcache, L: int, cfg: LayerCfg, ring=False, out=None,
                          lse=None, want_lse=False, workspace=None, stream=None):
    """Decode one token at position L-1 against keys stored turned to their positions and
    separate values: krot/vcache [B, L, Hkv, d], or ring caches [B, C, Hkv, d] (row p % C)
    with ring=True."""
    for t, n in ((q, "q"), (krot, "krot"), (vcache, "vcache")):
        _bf16(t, n)
    B = krot.shape[0]
    C = krot.shape[1] if ring else 0
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_decode_rotated_workspace_size(B, int(L), C, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_decode_rotated(_ptr(q), _ptr(krot), _ptr(vcache), int(L), C, _ptr(out),
                                    _ptr(lse), _ptr(workspace), workspace.numel(), B,
                                    ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_decode_rotated")
    return out, lse


def g4attn_quantize_int8(x, codes=None, scales=None, stream=None):
    """int8 cache of a bf16 cache x [..., d] (d 128, 256 or 512), one fp32 scale per row of d:
    returns (codes int8 [..., d], scales fp32 [...])."""
    _bf16(x, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    rc = _lib.g4attn_quantize_int8(_ptr(x), _ptr(codes), _ptr(scales), rows, d, _stream(stream))
    _check(rc, "g4attn_quantize_int8")
    return codes, scales


def g4attn_decode_int8_workspace_size(B: int, L: int, C: int, cfg: LayerCfg) -> int:
    c = cfg.c()
    return _lib.g4attn_decode_int8_workspace_size(B, L, C, ctypes.byref(c))


def g4attn_decode_int8(q, kcodes, kscales, vcodes, vscales, L: int, cfg: LayerCfg, ring=False,
                       out=None, lse=None, want_lse=False, workspace=None, stream=None):
    """Decode one token at position L-1 against an int8 cache: codes [B, L, Hkv, d] int8 and
    scales [B, L, Hkv] fp32 (g4attn_quantize_int8's layout), keys not rotated; values likewise
    when kv_is_k == 0, else vcodes / vscales None.  ring=True: ring caches of C rows (row
    p % C)."""
    _bf16(q, "q")
    for t, n in ((kcodes, "kcodes"), (vcodes, "vcodes")):
        if t is not None and t.dtype != torch.int8:
            raise G4AttnError(G4ATTN_ERR_INVALID_ARG, n + " must be int8")
    for t, n in ((kscales, "kscales"), (vscales, "vscales")):
        if t is not None and t.dtype != torch.float32:
            raise G4AttnError(G4ATTN_ERR_INVALID_ARG, n + " must be float32")
    B = kcodes.shape[0]
    C = kcodes.shape[1] if ring else 0
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_decode_int8_workspace_size(B, int(L), C, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_decode_int8(_ptr(q), _ptr(kcodes), _ptr(kscales), _ptr(vcodes),
                                 _ptr(vscales), int(L), C, _ptr(out), _ptr(lse), _ptr(workspace),
                                 workspace.numel(), B, ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_decode_int8")
    return out, lse


def g4attn_decode_split_cache(q, krot, vside, cfg: LayerCfg, out=None, lse=None, want_lse=False,
                              workspace=None, stream=None):
    """Decode one token against the split cache: krot [B,L,Hkv,d] rotated keys and vside
    [B,L,Hkv,128] pre-RoPE values of the rotated dims."""
    for t, n in ((q, "q"), (krot, "krot"), (vside, "vside")):
        _bf16(t, n)
    B, L = krot.shape[0], krot.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads), dtype=torch.float32, device=q.device)
    c = cfg.c()
    ws_bytes = _lib.g4attn_decode_workspace_size(B, L, ctypes.byref(c))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    rc = _lib.g4attn_decode_split_cache(_ptr(q), _ptr(krot), _ptr(vside), L, _ptr(out),
                                        _ptr(lse), _ptr(workspace), workspace.numel(), B,
                                        ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_decode_split_cache")
    return out, lse


def g4attn_decode_noalloc(q, kcache, vcache, cfg: LayerCfg, out=None, lse=None, want_lse=False,
                          stream=None):
    """Decode one token without a workspace: for callers that cannot allocate device memory
    (a plugin whose host framework owns all device memory and hands it only input and
    output buffers, a service that reserves the whole device up front).  The split
    partials go to a fixed 8 MiB scratch inside the library; problems that do not fit are
    refused with G4ATTN_ERR_TOO_LARGE.  Calls share that scratch, so calls that overlap on
    the GPU race; keep them on one stream.  `out` and `lse` are allocated here only when
    not given."""
    for t, n in ((q, "q"), (kcache, "kcache"), (vcache, "vcache")):
        _bf16(t, n)
    B, L = kcache.shape[0], kcache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.n_q_heads), dtype=torch.float32, device=q.device)
    c = cfg.c()
    rc = _lib.g4attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), L, _ptr(out), _ptr(lse),
                                    B, ctypes.byref(c), _stream(stream))
    _check(rc, "g4attn_decode_noalloc")
    return out, lse
