"""A second, unblocked formulation of the attention layer for tiny inputs (numpy, fp64).

It shares no code with the C oracle and is written differently on purpose: RoPE is a
complex multiplication z * exp(i * pos * theta) on the pairs (x_i, x_{i+d/2}), the mask is
an explicit T x T boolean matrix, the softmax is taken over the full masked score matrix
with numpy's exp, and GQA is done by repeating KV heads up to Hq.  Only used for T <= 64.
"""
import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rms(x, gamma, eps):
    # y = x / sqrt(mean(x^2) + eps) * gamma, over the last axis
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * (1.0 if gamma is None else gamma)


def rope_complex(x, positions, R, base):
    """Rotate pairs (i, i + d/2), i < R, by positions * base^(-2i/d) as complex numbers.
    x: [..., T, H, d]; positions: [T]."""
    d = x.shape[-1]
    half = d // 2
    y = x.copy()
    if R == 0:
        return y
    i = np.arange(R)
    theta = base ** (-2.0 * i / d)                          # [R]
    ang = positions[:, None].astype(np.float64) * theta    # [T, R]
    rot = np.exp(1j * ang)[:, None, :]                     # [T, 1, R] broadcast over heads
    z = x[..., :R] + 1j * x[..., half:half + R]
    z = z * rot
    y[..., :R] = z.real
    y[..., half:half + R] = z.imag
    return y


def attention(q_bits, k_bits, v_bits, gamma_q, gamma_k, Hq, Hkv, d, p, base, window,
              scale, kv_is_k, qk_norm=1, eps=1e-6):
    """Returns out [B, T, Hq, d] and lse [B, Hq, T]."""
    q = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_bits)
    B, T = q.shape[0], q.shape[1]
    R = int(np.floor(p * d / 2))
    gq = None if gamma_q is None else np.asarray(gamma_q, np.float64)
    gk = None if gamma_k is None else np.asarray(gamma_k, np.float64)
    qh = rms(q, gq, eps) if qk_norm else q
    kh = rms(k, gk, eps) if qk_norm else k
    pos = np.arange(T)
    qr = rope_complex(qh, pos, R, base)
    kr = rope_complex(kh, pos, R, base)
    if kv_is_k == 1:
        v = kh
    elif kv_is_k == 2:
        v = kr
    else:
        v = bf16_to_f64(v_bits)
    G = Hq // Hkv
    kr_rep = np.repeat(kr, G, axis=2)     # head h reads kv head h // G
    v_rep = np.repeat(v, G, axis=2)
    ii = pos[:, None]
    jj = pos[None, :]
    mask = jj <= ii
    if window > 0:
        mask &= jj > ii - window
    s = scale * np.einsum("bihc,bjhc->bhij", qr, kr_rep)
    s = np.where(mask[None, None], s, -np.inf)
    smax = s.max(axis=-1, keepdims=True)
    e = np.exp(s - smax)
    den = e.sum(axis=-1, keepdims=True)
    pmat = e / den
    out = np.einsum("bhij,bjhc->bihc", pmat, v_rep)
    lse = (smax + np.log(den))[..., 0]
    return out, lse
