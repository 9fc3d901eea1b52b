"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no arithmetic of the attention method: it only draws random numbers.
Recipe (same for every workload): a torch Generator seeded with `seed` draws, in this
order, q ~ N(0,1) [B,T,Hq,d], k ~ N(0,1) [B,T,Hkv,d], v ~ N(0,1) [B,T,Hkv,d] (only for
layers with a separate value), then gamma_q = 1 + 0.1 N(0,1) [d] and
gamma_k = 1 + 0.1 N(0,1) [d] in fp32.  q, k and v are drawn in fp32 (in pieces of 2^24
elements for tensors larger than that) and rounded to bf16 (round to nearest even).  On the CPU the bytes are reproducible across machines; `device="cuda"` uses the
CUDA generator instead (fast for the largest workloads, different bytes for the same seed).
"""
from dataclasses import dataclass
from typing import Optional

import torch


@dataclass
class LayerInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: Optional[torch.Tensor]
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor


_CHUNK = 1 << 24


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _randn_bf16(shape, gen, device):
    """N(0,1) draws rounded to bf16.  Large tensors are drawn in fixed 2^24-element pieces
    (fp32, then rounded) so host memory stays bounded; the piece size is part of the
    recipe, so the bytes are the same on every run."""
    n = 1
    for x in shape:
        n *= x
    if n <= _CHUNK:
        return _randn(shape, gen, device).to(torch.bfloat16)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for i in range(0, n, _CHUNK):
        m = min(_CHUNK, n - i)
        out[i:i + m] = _randn((m,), gen, device).to(torch.bfloat16)
    return out.view(shape)


def layer_inputs(B, T, n_q_heads, n_kv_heads, head_dim, separate_v, seed, device="cpu"):
    gen = torch.Generator(device=device).manual_seed(int(seed))
    q = _randn_bf16((B, T, n_q_heads, head_dim), gen, device)
    k = _randn_bf16((B, T, n_kv_heads, head_dim), gen, device)
    v = None
    if separate_v:
        v = _randn_bf16((B, T, n_kv_heads, head_dim), gen, device)
    gamma_q = 1.0 + 0.1 * _randn((head_dim,), gen, device)
    gamma_k = 1.0 + 0.1 * _randn((head_dim,), gen, device)
    return LayerInputs(q, k, v, gamma_q.contiguous(), gamma_k.contiguous())


def decode_inputs(B, L, n_q_heads, n_kv_heads, head_dim, separate_v, seed, device="cpu"):
    """A decode step: q [B,1,Hq,d] and a cache [B,L,Hkv,d] of N(0,1) bf16 values that is
    used as if it already held normalised keys (the cache of the decode workload)."""
    gen = torch.Generator(device=device).manual_seed(int(seed))
    q = _randn_bf16((B, 1, n_q_heads, head_dim), gen, device)
    kcache = _randn_bf16((B, L, n_kv_heads, head_dim), gen, device)
    vcache = None
    if separate_v:
        vcache = _randn_bf16((B, L, n_kv_heads, head_dim), gen, device)
    gamma_q = 1.0 + 0.1 * _randn((head_dim,), gen, device)
    gamma_k = 1.0 + 0.1 * _randn((head_dim,), gen, device)
    return LayerInputs(q, kcache, vcache, gamma_q.contiguous(), gamma_k.contiguous())


@dataclass
class ChunkInputs:
    q: torch.Tensor                 # [B, Tn, Hq, d] raw queries of the chunk
    k: torch.Tensor                 # [B, Tn, Hkv, d] raw keys of the chunk
    v: Optional[torch.Tensor]       # [B, Tn, Hkv, d] raw values of the chunk
    kcache: torch.Tensor            # [B, P, Hkv, d] cached (already normalised) keys
    vcache: Optional[torch.Tensor]  # [B, P, Hkv, d] cached values
    gamma_q: torch.Tensor
    gamma_k: torch.Tensor


def chunk_inputs(B, P, Tn, n_q_heads, n_kv_heads, head_dim, separate_v, seed, device="cpu"):
    """One prefill chunk: raw q/k/v of Tn tokens (as layer_inputs) plus the cache of the P
    earlier positions, N(0,1) bf16 values used as if already normalised (as decode_inputs)."""
    gen = torch.Generator(device=device).manual_seed(int(seed))
    q = _randn_bf16((B, Tn, n_q_heads, head_dim), gen, device)
    k = _randn_bf16((B, Tn, n_kv_heads, head_dim), gen, device)
    kcache = _randn_bf16((B, P, n_kv_heads, head_dim), gen, device)
    v = vcache = None
    if separate_v:
        v = _randn_bf16((B, Tn, n_kv_heads, head_dim), gen, device)
        vcache = _randn_bf16((B, P, n_kv_heads, head_dim), gen, device)
    gamma_q = 1.0 + 0.1 * _randn((head_dim,), gen, device)
    gamma_k = 1.0 + 0.1 * _randn((head_dim,), gen, device)
    return ChunkInputs(q, k, v, kcache, vcache, gamma_q.contiguous(), gamma_k.contiguous())


def int8_cache(B, L, n_kv_heads, head_dim, seed, device="cpu"):
    """A random int8 cache in g4attn_quantize_int8's layout, drawn directly (for the sizes
    where quantising a drawn bf16 cache on the host would be slow), with the statistics of a
    quantised N(0,1) cache of head_dim 256-512 (row maximum about 3.3, so scale about 0.026 and
    codes about N(0, 38^2)): codes = clamp(round(38 N(0,1)), -127, 127) int8 [B, L, Hkv, d],
    scales = 0.026 (1 + 0.05 N(0,1)) fp32 [B, L, Hkv]; the elements scale * code are then
    close to N(0,1)."""
    gen = torch.Generator(device=device).manual_seed(int(seed))
    codes = torch.empty((B, L, n_kv_heads, head_dim), dtype=torch.int8, device=device)
    flat = codes.view(-1)
    for i in range(0, flat.numel(), _CHUNK):
        m = min(_CHUNK, flat.numel() - i)
        flat[i:i + m] = torch.round(38.0 * _randn((m,), gen, device)).clamp_(-127, 127).to(torch.int8)
    scales = 0.026 * (1.0 + 0.05 * _randn((B, L, n_kv_heads), gen, device))
    return codes, scales.contiguous()
