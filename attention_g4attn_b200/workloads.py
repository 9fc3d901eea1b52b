"""The five named workloads of the Gemma-4-style attention hot path.

Shapes follow the pages: global layers use p-RoPE p=0.25 at base 1e6, 8 query heads per
KV head, head_dim 512 and keys reused as values (Gemma 4 report section 2; explainer
"GQA", "K=V" and "p-RoPE" sections); local layers use full RoPE at base 1e4, 2 query
heads per KV head, head_dim 256 and a causal sliding window of 512 or 1024 (explainer
"interleaved layers" section; talk notes on GQA 2:1 / 8:1 and head_dim 256 -> 512).
The 5:1 block interleaves five local layers with one global layer (report section 2).
"""
import math
from dataclasses import dataclass, field, replace
from typing import List


@dataclass(frozen=True)
class Layer:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_p: float
    rope_base: float
    window: int
    kv_is_k: int
    qk_norm: int = 1
    qk_norm_eps: float = 1e-6

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def separate_v(self) -> bool:
        return self.kv_is_k == 0


GLOBAL_8TO1 = Layer(32, 4, 512, 0.25, 1e6, 0, 1)
GLOBAL_TINY = Layer(8, 1, 512, 0.25, 1e6, 0, 1)
LOCAL_W512 = Layer(16, 8, 256, 1.0, 1e4, 512, 0)
LOCAL_W1024 = Layer(32, 16, 256, 1.0, 1e4, 1024, 0)


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    T: int
    layers: List[Layer] = field(default_factory=list)
    seeds: List[int] = field(default_factory=list)

    def flops(self) -> float:
        """4 * d * Hq * B * (unmasked query-key pairs) summed over layers."""
        total = 0.0
        for ly in self.layers:
            total += 4.0 * ly.head_dim * ly.n_q_heads * self.B * visible_pairs(self.T, ly.window)
        return total


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    L: int
    layer: Layer
    seed: int = 0

    def cache_bytes(self) -> float:
        """Bytes of cache that one decode step must read once (bf16; K=V: one cache)."""
        n = 1 if self.layer.kv_is_k else 2
        return float(n * self.B * self.layer.n_kv_heads * self.L * self.layer.head_dim * 2)


def visible_pairs(T: int, window: int) -> int:
    """Number of (query, key) pairs a causal (window = 0) or sliding-window layer attends."""
    if window <= 0 or window >= T:
        return T * (T + 1) // 2
    return window * (window + 1) // 2 + (T - window) * window


GLOBAL_PREFILL_TINY = Prefill("global_prefill_T128_h8x1_d512", 1, 128, [GLOBAL_TINY], [0])
LOCAL_PREFILL = Prefill("local_prefill_B2_T4096_h16x8_d256_w512", 2, 4096, [LOCAL_W512], [0])
GLOBAL_PREFILL_32K = Prefill("global_prefill_T32768_h32x4_d512", 1, 32768, [GLOBAL_8TO1], [0])
GLOBAL_DECODE_32K = Decode("global_decode_B16_L32768_h32x4_d512", 16, 32768, GLOBAL_8TO1)
GLOBAL_DECODE_128K = Decode("global_decode_B16_L131072_h32x4_d512", 16, 131072, GLOBAL_8TO1)
BLOCK_5TO1_64K = Prefill("block_5local_1global_T65536", 1, 65536,
                         [LOCAL_W1024] * 5 + [GLOBAL_8TO1], [0, 1, 2, 3, 4, 5])

ALL = {w.name: w for w in (GLOBAL_PREFILL_TINY, LOCAL_PREFILL, GLOBAL_PREFILL_32K,
                           GLOBAL_DECODE_32K, GLOBAL_DECODE_128K, BLOCK_5TO1_64K)}


def with_layer(layer: Layer, **kw) -> Layer:
    return replace(layer, **kw)
