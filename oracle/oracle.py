"""ctypes front end of the fp64 CPU oracle (test infrastructure only).

Inputs arrive as bf16 bit patterns (numpy uint16) or as torch bf16 CPU tensors; the C side
widens them exactly to double.  Outputs are float64 numpy arrays.
"""
import ctypes
import math
from dataclasses import dataclass, replace

import numpy as np

from . import build as _build

_lib = None


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("rope_p", ctypes.c_double),
        ("rope_base", ctypes.c_double),
        ("window", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("kv_is_k", ctypes.c_int),
        ("qk_norm", ctypes.c_int),
        ("qk_norm_eps", ctypes.c_double),
    ]


@dataclass
class OracleCfg:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_p: float
    rope_base: float
    window: int = 0
    scale: float = None
    kv_is_k: int = 1
    qk_norm: int = 1
    qk_norm_eps: float = 1e-6

    def c(self) -> _Cfg:
        scale = self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)
        return _Cfg(self.n_q_heads, self.n_kv_heads, self.head_dim, float(self.rope_p),
                    float(self.rope_base), int(self.window), float(scale), int(self.kv_is_k),
                    int(self.qk_norm), float(self.qk_norm_eps))


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.g4o_rope_pairs.argtypes = [ctypes.c_int, ctypes.c_double]
        lib.g4o_rope_pairs.restype = ctypes.c_int
        lib.g4o_rmsnorm.argtypes = [P, P, ctypes.c_int, ctypes.c_double, P]
        lib.g4o_rmsnorm.restype = None
        lib.g4o_rope.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                 ctypes.c_int64, P]
        lib.g4o_rope.restype = None
        lib.g4o_qknorm_rope.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                        ctypes.POINTER(_Cfg), P, P, P]
        lib.g4o_qknorm_rope.restype = ctypes.c_int
        lib.g4o_prefill_rows.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(_Cfg), P, ctypes.c_int, ctypes.c_int,
                                         P, P]
        lib.g4o_prefill_rows.restype = ctypes.c_int
        lib.g4o_decode.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_Cfg),
                                   P, ctypes.c_int, ctypes.c_int, P, P]
        lib.g4o_decode.restype = ctypes.c_int
        lib.g4o_decode_int8.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(_Cfg), P, ctypes.c_int, ctypes.c_int, P, P]
        lib.g4o_decode_int8.restype = ctypes.c_int
        _lib = lib
    return _lib


def bf16_bits(x) -> np.ndarray:
    """Return the bf16 bit patterns of a torch bf16 tensor (CPU) or pass uint16 through."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


def _f32(x):
    if x is None:
        return None
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def rope_pairs(head_dim: int, p: float) -> int:
    return _load().g4o_rope_pairs(head_dim, p)


def rmsnorm(x: np.ndarray, gamma=None, eps: float = 1e-6) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float64)
    y = np.empty_like(x)
    _load().g4o_rmsnorm(_ptr(x), _ptr(g), x.shape[-1], eps, _ptr(y))
    return y


def rope(x: np.ndarray, R: int, base: float, pos: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().g4o_rope(_ptr(x), x.shape[-1], R, base, pos, _ptr(y))
    return y


def qknorm_rope(q, k, gamma_q, gamma_k, cfg: OracleCfg, pos0: int = 0, want_krot=True):
    """Returns (q_out, k_out, krot_out) as float64 arrays shaped like the inputs."""
    qb = None if q is None else bf16_bits(q)
    kb = None if k is None else bf16_bits(k)
    ref = qb if qb is not None else kb
    B, T = ref.shape[0], ref.shape[1]
    qo = None if qb is None else np.empty(qb.shape, np.float64)
    ko = None if kb is None else np.empty(kb.shape, np.float64)
    kr = None if (kb is None or not want_krot) else np.empty(kb.shape, np.float64)
    c = cfg.c()
    rc = _load().g4o_qknorm_rope(_ptr(qb), _ptr(kb), _ptr(_f32(gamma_q)), _ptr(_f32(gamma_k)),
                                 B, T, pos0, ctypes.byref(c), _ptr(qo), _ptr(ko), _ptr(kr))
    if rc != 0:
        raise ValueError("oracle qknorm_rope rejected its arguments (%d)" % rc)
    return qo, ko, kr


def prefill_rows(q, k, v, gamma_q, gamma_k, cfg: OracleCfg, rows=None, nthreads: int = 0):
    """Attention output for query positions `rows` (all by default).

    Returns (out [B, nrows, Hq, d], lse [B, Hq, nrows]) in float64."""
    qb, kb = bf16_bits(q), bf16_bits(k)
    vb = None if v is None else bf16_bits(v)
    B, T = qb.shape[0], qb.shape[1]
    if rows is None:
        rows = np.arange(T, dtype=np.int32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    out = np.zeros((B, len(rows), cfg.n_q_heads, cfg.head_dim), np.float64)
    lse = np.zeros((B, cfg.n_q_heads, len(rows)), np.float64)
    c = cfg.c()
    rc = _load().g4o_prefill_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(_f32(gamma_q)),
                                  _ptr(_f32(gamma_k)), B, T, ctypes.byref(c), _ptr(rows),
                                  len(rows), nthreads, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments (%d)" % rc)
    return out, lse


def decode(q, kcache, vcache, cfg: OracleCfg, items=None, nthreads: int = 0):
    """One query per (b, h) at position L-1.  Returns (out [B, Hq, d], lse [B, Hq]).

    `items` optionally restricts the work to b * Hkv + g entries (others stay NaN)."""
    qb, kb = bf16_bits(q), bf16_bits(kcache)
    vb = None if vcache is None else bf16_bits(vcache)
    B, L = kb.shape[0], kb.shape[1]
    out = np.full((B, cfg.n_q_heads, cfg.head_dim), np.nan)
    lse = np.full((B, cfg.n_q_heads), np.nan)
    it = None if items is None else np.ascontiguousarray(items, dtype=np.int32)
    c = cfg.c()
    rc = _load().g4o_decode(_ptr(qb), _ptr(kb), _ptr(vb), B, L, ctypes.byref(c), _ptr(it),
                            0 if it is None else len(it), nthreads, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments (%d)" % rc)
    return out, lse


def decode_ring(q, kring, vring, L: int, cfg: OracleCfg, nthreads: int = 0):
    """Decode of a sliding-window layer against ring caches (Gemma 4 report section 2 and the
    explainer's "interleaved layers": a local layer attends to the last W tokens, so its cache
    keeps only the last C >= W positions, position p in row p % C).

    Written out as the definition: the ring is unrolled into a linear cache of L positions
    (row p = ring row p % C for the last C positions; earlier positions, outside the window,
    are zero) and the linear decode above runs on it with the same window."""
    kb = bf16_bits(kring)
    vb = None if vring is None else bf16_bits(vring)
    B, C = kb.shape[0], kb.shape[1]
    if not (cfg.window and 0 < cfg.window <= C):
        raise ValueError("ring decode needs 0 < window <= C")
    shape = (B, L) + kb.shape[2:]
    k_lin = np.zeros(shape, np.uint16)
    v_lin = None if vb is None else np.zeros(shape, np.uint16)
    for p in range(max(0, L - C), L):
        k_lin[:, p] = kb[:, p % C]
        if vb is not None:
            v_lin[:, p] = vb[:, p % C]
    return decode(q, k_lin, v_lin, cfg, nthreads=nthreads)


def _widen(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns to float64, exactly (the bits are the top half of an fp32)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def prefill_chunk(q, k, v, kcache, vcache, gamma_q, gamma_k, P: int, cfg: OracleCfg, rows=None):
    """Prefill of one chunk of a longer prompt (the attention of Gemma 4 report section 2,
    taken a chunk at a time against the cache the earlier chunks left).

    The chunk's Tn tokens sit at positions P .. P+Tn-1.  Keys at positions j < P are the
    cache rows 0 .. P-1 as stored (already normalised, not rotated); the chunk's keys get
    QKNorm here.  Key j is turned to angle j and the query of chunk token t, after QKNorm,
    to angle P + t.  Token t sees the keys j <= P + t, and on a window-W layer only those
    with j > P + t - W.  Softmax of the scaled scores weighs the values: the unrotated key
    (kv_is_k = 1), the rotated key (2), or the separate value (0: vcache rows 0 .. P-1, then
    the chunk's v).

    Written out as that definition; the scores and the weighted sums are float64 numpy
    matrix products over all P + Tn keys of a (batch, head).
    Returns (out [B, nrows, Hq, d], lse [B, Hq, nrows]) for the chunk tokens `rows`."""
    qb, kb, cb = bf16_bits(q), bf16_bits(k), bf16_bits(kcache)
    B, Tn, Hq, d = qb.shape
    Hkv = cfg.n_kv_heads
    G = Hq // Hkv
    if cb.shape[1] < P:
        raise ValueError("the cache holds fewer than P positions")
    rows = np.arange(Tn) if rows is None else np.asarray(rows, dtype=np.int64)
    # the chunk: queries normalised and turned to P + t, keys normalised (and turned)
    qr, kh_new, kr_new = qknorm_rope(qb, kb, gamma_q, gamma_k, cfg, pos0=P)
    if P > 0:
        # the cached keys are used as stored: rotation only
        _, kh_old, kr_old = qknorm_rope(None, cb[:, :P], None, None, replace(cfg, qk_norm=0))
        kh = np.concatenate([kh_old, kh_new], axis=1)
        kr = np.concatenate([kr_old, kr_new], axis=1)
    else:
        kh, kr = kh_new, kr_new
    if cfg.kv_is_k == 1:
        vals = kh
    elif cfg.kv_is_k == 2:
        vals = kr
    else:
        vb = _widen(bf16_bits(v))
        vals = np.concatenate([_widen(bf16_bits(vcache)[:, :P]), vb], axis=1) if P > 0 else vb
    scale = cfg.scale if cfg.scale is not None else 1.0 / math.sqrt(d)
    pos_q = P + rows                                  # positions of the chunk rows asked for
    pos_k = np.arange(P + Tn)
    vis = pos_k[None, :] <= pos_q[:, None]
    if cfg.window and cfg.window > 0:
        vis &= pos_k[None, :] > pos_q[:, None] - cfg.window
    out = np.zeros((B, len(rows), Hq, d))
    lse = np.zeros((B, Hq, len(rows)))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = scale * (qr[b, rows, h] @ kr[b, :, g].T)          # [nrows, P + Tn]
            s = np.where(vis, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            den = e.sum(axis=1, keepdims=True)
            out[b, :, h] = (e / den) @ vals[b, :, g]
            lse[b, h] = m[:, 0] + np.log(den[:, 0])
    return out, lse


def quantize_int8(x):
    """int8 cache of a bf16 cache [..., d]: one scale per row (the last axis), symmetric.

    The pages count the KV cache in int8 (Gemma 4 report, memory table) but give no scheme;
    the reading taken: scale = max_c |x_c| / 127 and code_c = round(x_c / scale) (half to
    even), clamped to [-127, 127]; a row of zeros has scale 0 and codes 0.  These steps take
    integer decisions, so they run in IEEE fp32 (each operation rounded to nearest), the
    precision the device quantiser uses, and the codes and scales are exact to compare.
    A row holding an infinity or a NaN (outside the reading: max|x|/127 is not a scale)
    gets scale NaN and codes 0.
    Returns (codes int8 [..., d], scales float32 [...])."""
    xf = _widen(bf16_bits(x)).astype(np.float32)          # exact: bf16 values fit fp32
    finite = np.all(np.isfinite(xf), axis=-1)
    amax = np.max(np.abs(np.where(np.isfinite(xf), xf, np.float32(0))), axis=-1)
    scales = (amax / np.float32(127.0)).astype(np.float32)
    # a row holding an infinity or a NaN has no finite max|x|: scale NaN, codes 0, so every
    # element it stands for reads as NaN
    scales = np.where(finite, scales, np.float32(np.nan)).astype(np.float32)
    safe = np.where(scales > 0, scales, np.float32(1.0)).astype(np.float32)
    with np.errstate(invalid="ignore"):
        ratio = (xf / safe[..., None]).astype(np.float32)
        codes = np.clip(np.rint(ratio), -127, 127)
    codes = np.where(scales[..., None] > 0, codes, 0).astype(np.int8)
    return codes, scales


def dequantize_int8(codes, scales):
    """scale * code per element, in float64 (exact)."""
    return np.asarray(scales, np.float64)[..., None] * np.asarray(codes, np.float64)


def decode_int8(q, kcodes, kscales, vcodes, vscales, cfg: OracleCfg, items=None, nthreads: int = 0):
    """decode() against an int8 cache: codes [B, L, Hkv, d] int8 and scales [B, L, Hkv] fp32
    (values likewise when kv_is_k = 0); each element is scale * code, exact in double."""
    qb = bf16_bits(q)
    kq = np.ascontiguousarray(kcodes, np.int8)
    ks = np.ascontiguousarray(kscales, np.float32)
    vq = None if vcodes is None else np.ascontiguousarray(vcodes, np.int8)
    vs = None if vscales is None else np.ascontiguousarray(vscales, np.float32)
    B, L = kq.shape[0], kq.shape[1]
    out = np.full((B, cfg.n_q_heads, cfg.head_dim), np.nan)
    lse = np.full((B, cfg.n_q_heads), np.nan)
    it = None if items is None else np.ascontiguousarray(items, dtype=np.int32)
    c = cfg.c()
    rc = _load().g4o_decode_int8(_ptr(qb), _ptr(kq), _ptr(ks), _ptr(vq), _ptr(vs), B, L,
                                 ctypes.byref(c), _ptr(it), 0 if it is None else len(it),
                                 nthreads, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle int8 decode rejected its arguments (%d)" % rc)
    return out, lse
