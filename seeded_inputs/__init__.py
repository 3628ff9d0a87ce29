"""Seeded synthetic inputs and workload definitions shared by the oracle and the GPU path.

This module holds no arithmetic of the attention method: it only draws random
numbers (in a fixed order, from a fixed seed) and names the workloads. Both the
fp64 CPU oracle and the CUDA path consume exactly these tensors, so a parity test
compares the two on identical inputs.

Recipe (the same for every workload):
  * ``torch.Generator('cpu').manual_seed(seed)``, then ``torch.randn`` in fp32 in
    the order q, k, v (prefill), or kcache, vcache, then per decode step q, k, v.
  * Values are iid N(0, 1); bf16 workloads round the fp32 draw to bf16.
  * Query rows sampled for the oracle at long lengths come from
    ``numpy.random.default_rng(seed + 1000)`` and always include the rows that sit
    next to the local-window edge, the tile edges and the pretrained-window edge.

The workloads carry Qwen3 attention-layer head shapes (the pages evaluate the
method on Qwen3-1.7B/4B/8B up to 128K tokens); no dataset or model weight is used.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

FREQ_INTERP = "freq_interp"
POS_ALIAS = "pos_alias"


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    L: int
    hq: int
    hkv: int
    head_dim: int
    w0: int
    w_pretrained: int
    theta: float
    mode: str
    seed: int
    dtype: str  # "fp32" or "bf16": the dtype the inputs are drawn in

    @property
    def causal_flops(self) -> float:
        """Counted work of one prefill: 2 GEMMs x 2 FLOP x (L^2/2) pairs x D x Hq."""
        return 4.0 * (self.L * self.L / 2.0) * self.head_dim * self.hq


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    prefix_len: int  # cache filled at positions 0 .. prefix_len-1
    steps: int
    capacity: int
    hq: int
    hkv: int
    head_dim: int
    w0: int
    w_pretrained: int
    theta: float
    mode: str
    seed: int

    def cache_bytes(self, L: int) -> int:
        """Algorithmic HBM bytes of one decode step at length L: K and V, bf16."""
        return 2 * L * self.hkv * self.head_dim * 2


TINY = PrefillWorkload("tiny_L512_hq2_hkv1_d64_fp32", 512, 2, 1, 64, 64, 128, 1e4, FREQ_INTERP, 0, "fp32")
QWEN3_1P7B_32K = PrefillWorkload("qwen3_1.7b_L32768_hq16_hkv8_d128", 32768, 16, 8, 128, 4096, 32768, 1e6,
                                 FREQ_INTERP, 1, "bf16")
QWEN3_4B_64K_FI = PrefillWorkload("qwen3_4b_L65536_hq32_hkv8_d128_fi", 65536, 32, 8, 128, 4096, 32768, 1e6,
                                  FREQ_INTERP, 2, "bf16")
QWEN3_4B_64K_PA = dataclasses.replace(QWEN3_4B_64K_FI, name="qwen3_4b_L65536_hq32_hkv8_d128_pa", mode=POS_ALIAS)


def qwen3_8b_128k(w0: int = 4096, mode: str = FREQ_INTERP) -> PrefillWorkload:
    return PrefillWorkload(f"qwen3_8b_L131072_hq32_hkv8_d128_w{w0}" + ("_pa" if mode == POS_ALIAS else ""),
                           131072, 32, 8, 128, w0, 32768, 1e6, mode, 3, "bf16")


QWEN3_8B_128K_W0 = (1024, 4096, 16384)

DECODE_128K = DecodeWorkload("qwen3_8b_decode_131000_plus200", 131000, 200, 131200, 32, 8, 128, 4096, 32768,
                             1e6, FREQ_INTERP, 4)


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _draw(g: torch.Generator, shape, dtype: str) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "fp32":
        return x
    raise ValueError(f"unknown dtype {dtype!r}")


def prefill_inputs(w: PrefillWorkload, batch: int = 1, L: Optional[int] = None):
    """q [b, L, Hq, D], k and v [b, L, Hkv, D] on the CPU, in the workload's dtype."""
    L = w.L if L is None else L
    g = generator(w.seed)
    q = _draw(g, (batch, L, w.hq, w.head_dim), w.dtype)
    k = _draw(g, (batch, L, w.hkv, w.head_dim), w.dtype)
    v = _draw(g, (batch, L, w.hkv, w.head_dim), w.dtype)
    return q, k, v


def random_qkv(seed: int, batch: int, L: int, hq: int, hkv: int, head_dim: int, dtype: str = "bf16"):
    """Same recipe as :func:`prefill_inputs` for ad-hoc shapes (edge-case tests)."""
    g = generator(seed)
    q = _draw(g, (batch, L, hq, head_dim), dtype)
    k = _draw(g, (batch, L, hkv, head_dim), dtype)
    v = _draw(g, (batch, L, hkv, head_dim), dtype)
    return q, k, v


class DecodeStream:
    """Seeded decode workload: a bf16 cache prefix, then one (q, k, v) draw per step.

    The cache values are iid N(0,1) bf16 and are taken to be keys that already
    carry the original RoPE (a rotation keeps the N(0, I) distribution).
    """

    def __init__(self, w: DecodeWorkload, prefix_len: Optional[int] = None, capacity: Optional[int] = None):
        self.w = w
        self.prefix_len = w.prefix_len if prefix_len is None else prefix_len
        self.capacity = w.capacity if capacity is None else capacity
        self.g = generator(w.seed)

    def cache_prefix(self):
        """kcache, vcache [prefix_len, Hkv, D] bf16 (drawn first, in this order)."""
        shape = (self.prefix_len, self.w.hkv, self.w.head_dim)
        kc = _draw(self.g, shape, "bf16")
        vc = _draw(self.g, shape, "bf16")
        return kc, vc

    def step(self):
        """One decode step's raw inputs: q [Hq, D], k_new and v_new [Hkv, D] (bf16)."""
        q = _draw(self.g, (self.w.hq, self.w.head_dim), "bf16")
        k = _draw(self.g, (self.w.hkv, self.w.head_dim), "bf16")
        v = _draw(self.g, (self.w.hkv, self.w.head_dim), "bf16")
        return q, k, v


def sample_rows(seed: int, L: int, w0: int, w_pretrained: int, n: int = 512) -> np.ndarray:
    """Sorted query rows for oracle checks at long lengths.

    Always contains the rows next to the local-window edge (w0-2 .. w0+1), the first
    and last rows, the 128-row tile edge and the pretrained-window edge; the rest
    are drawn uniformly without replacement from ``default_rng(seed + 1000)``.
    """
    must = {0, 1, w0 - 2, w0 - 1, w0, w0 + 1, L - 2, L - 1, 127, 128, 129, w_pretrained - 1, w_pretrained}
    must = sorted(r for r in must if 0 <= r < L)
    n = min(n, L)
    rest = np.setdiff1d(np.arange(L), np.array(must, dtype=np.int64))
    rng = np.random.default_rng(seed + 1000)
    extra = rng.choice(rest, size=max(0, n - len(must)), replace=False) if len(rest) else np.empty(0, np.int64)
    return np.sort(np.concatenate([np.array(must, dtype=np.int64), extra.astype(np.int64)]))
