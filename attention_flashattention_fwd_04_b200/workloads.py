"""Seeded synthetic inputs for the attention kernels and for the checks on them.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path's tests/bench and the CPU oracle
can take their inputs from it.

Workloads (all values bf16, drawn in fp32 from ``torch.Generator('cpu')`` and
rounded to nearest-even; draw order Q, K, V, then any per-position offset):

* ``tiny``         B=1, H=2, N=128, d=64, non-causal, N(0,1), seed 1
* ``causal_mha``   B=4, H=16, N=2048, d=128, causal, N(0,1), seed 2
* ``causal_gqa``   B=1, Hq=32, Hkv=8, N=8192, d=128, causal, N(0,1) x 0.5, seed 3
* ``paged_decode`` 64 sequences, one query each, Hq=32, Hkv=8, d=128,
  lengths uniform in [512, 8192], 16-token pages, physical pages a seeded
  permutation of exactly the pages needed, seed 4
* ``long_causal``  B=1, H=8, N=32768, d=128, causal, N(0,1) with one offset
  c_j ~ N(0, sigma=2) per key position added to every element of key row j
  (shared by all heads) to make peaked softmax rows, seed 5
* ``long_window``  the ``long_causal`` shapes and draws (seed 7) with a sliding
  window: query i sees keys i-4095 .. i (a 4096-key window, the size used by
  common sliding-window models; the pages name the pattern, not a size)

The page size of 16 tokens is the cache block size of the vLLM example in
"Fast Attention Kernels and Operator Fusion" (wpnews.pro), section "Paged
Attention Kernels".  No public suite is named for these workloads; these
synthetic draws stand in for real activations.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "PrefillConfig",
    "DecodeConfig",
    "PREFILL_CONFIGS",
    "DECODE_CONFIGS",
    "make_prefill_inputs",
    "make_decode_inputs",
    "prefill_flops",
    "visible_pairs",
    "decode_kv_bytes",
]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    seed: int
    value_scale: float = 1.0
    k_offset_sigma: float = 0.0
    window_left: int = -1  # W >= 0: query i sees keys j >= i - W only; -1: no window

    @property
    def scale(self) -> float:
        # 1/sqrt(d), rounded to fp32 once; the kernels and the oracle both get
        # this same fp32 value.
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    num_seqs: int
    Hq: int
    Hkv: int
    d: int
    page_size: int
    min_len: int
    max_len: int
    seed: int
    max_pages: int = field(default=0)

    @property
    def scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))

    @property
    def table_width(self) -> int:
        return self.max_pages or -(-self.max_len // self.page_size)


PREFILL_CONFIGS = {
    "tiny": PrefillConfig("tiny", 1, 2, 2, 128, 64, False, 1),
    "causal_mha": PrefillConfig("causal_mha", 4, 16, 16, 2048, 128, True, 2),
    "causal_gqa": PrefillConfig("causal_gqa", 1, 32, 8, 8192, 128, True, 3, value_scale=0.5),
    "long_causal": PrefillConfig("long_causal", 1, 8, 8, 32768, 128, True, 5, k_offset_sigma=2.0),
    "long_window": PrefillConfig("long_window", 1, 8, 8, 32768, 128, True, 7, k_offset_sigma=2.0,
                                 window_left=4095),
}

DECODE_CONFIGS = {
    "paged_decode": DecodeConfig("paged_decode", 64, 32, 8, 128, 16, 512, 8192, 4),
    # a small decode batch, where per-call host work and launch gaps dominate
    "small_decode": DecodeConfig("small_decode", 4, 32, 8, 128, 16, 256, 1024, 6),
}


def make_prefill_inputs(cfg: PrefillConfig, device: str | torch.device = "cpu"):
    """Q [B,Hq,N,d], K and V [B,Hkv,N,d], bf16, contiguous."""
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed)
    q = torch.randn(cfg.B, cfg.Hq, cfg.N, cfg.d, generator=g, dtype=torch.float32)
    k = torch.randn(cfg.B, cfg.Hkv, cfg.N, cfg.d, generator=g, dtype=torch.float32)
    v = torch.randn(cfg.B, cfg.Hkv, cfg.N, cfg.d, generator=g, dtype=torch.float32)
    if cfg.value_scale != 1.0:
        q.mul_(cfg.value_scale)
        k.mul_(cfg.value_scale)
        v.mul_(cfg.value_scale)
    if cfg.k_offset_sigma:
        off = torch.normal(0.0, cfg.k_offset_sigma, (cfg.N,), generator=g, dtype=torch.float32)
        k.add_(off.view(1, 1, cfg.N, 1))
    out = tuple(t.to(torch.bfloat16).contiguous().to(device) for t in (q, k, v))
    return out


def make_decode_inputs(cfg: DecodeConfig, device: str | torch.device = "cpu",
                       poison_tail: bool = False, seq_lens=None):
    """Paged-KV decode inputs.

    Returns a dict with q [S,Hq,d] bf16, k_pool / v_pool
    [num_pages,page_size,Hkv,d] bf16, block_table [S,max_pages] int32 (unused
    entries -1), seq_lens [S] int32, and the sizes.  Each sequence owns
    ceil(L/page_size) pages; the physical ids are a seeded permutation of
    0..num_pages-1 handed out in sequence order.  ``poison_tail`` fills the
    slots past the end of each sequence's last page with NaN (they must never
    influence a result).  ``seq_lens`` overrides the drawn lengths.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed)
    S, ps = cfg.num_seqs, cfg.page_size
    drawn = torch.randint(cfg.min_len, cfg.max_len + 1, (S,), generator=g, dtype=torch.int64)
    if seq_lens is not None:
        drawn = torch.as_tensor(seq_lens, dtype=torch.int64).clone()
        assert drawn.numel() == S
    pages = (drawn + ps - 1) // ps
    width = max(cfg.table_width, int(pages.max().item()) if S else 0)
    num_pages = int(pages.sum().item())
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((S, width), -1, dtype=torch.int32)
    off = 0
    for s in range(S):
        n = int(pages[s])
        table[s, :n] = perm[off:off + n].to(torch.int32)
        off += n
    q = torch.randn(S, cfg.Hq, cfg.d, generator=g, dtype=torch.float32)
    k_pool = torch.randn(num_pages, ps, cfg.Hkv, cfg.d, generator=g, dtype=torch.float32)
    v_pool = torch.randn(num_pages, ps, cfg.Hkv, cfg.d, generator=g, dtype=torch.float32)
    q, k_pool, v_pool = (t.to(torch.bfloat16) for t in (q, k_pool, v_pool))
    if poison_tail:
        for s in range(S):
            L = int(drawn[s])
            n = int(pages[s])
            if n and L < n * ps:
                last = int(table[s, n - 1])
                k_pool[last, L - (n - 1) * ps:] = float("nan")
                v_pool[last, L - (n - 1) * ps:] = float("nan")
    dev = torch.device(device)
    return {
        "q": q.contiguous().to(dev),
        "k_pool": k_pool.contiguous().to(dev),
        "v_pool": v_pool.contiguous().to(dev),
        "block_table": table.contiguous().to(dev),
        "seq_lens": drawn.to(torch.int32).contiguous().to(dev),
        "page_size": ps,
        "num_pages": num_pages,
        "max_pages": width,
        "scale": cfg.scale,
    }


def visible_pairs(N: int, causal: bool, window_left: int = -1) -> int:
    """Number of (query, key) pairs the mask leaves visible in one head."""
    i = torch.arange(N, dtype=torch.int64)
    last = i if causal else torch.full_like(i, N - 1)
    first = (i - window_left).clamp(min=0) if window_left >= 0 else torch.zeros_like(i)
    return int((last - first + 1).clamp(min=0).sum().item())


def prefill_flops(cfg: PrefillConfig) -> float:
    """Algorithmic FLOPs of QK^T and PV: 4*d per visible (query, key) pair.

    Without a window the usual convention is kept: 4*B*Hq*N^2*d, halved for
    causal.  With a sliding window the visible pairs are counted exactly.
    """
    if cfg.window_left >= 0:
        return 4.0 * cfg.B * cfg.Hq * cfg.d * visible_pairs(cfg.N, cfg.causal, cfg.window_left)
    f = 4.0 * cfg.B * cfg.Hq * cfg.N * cfg.N * cfg.d
    return f / 2.0 if cfg.causal else f


def decode_kv_bytes(seq_lens, Hkv: int, d: int, Hq: int, page_size: int = 16) -> float:
    """Algorithmic HBM bytes of one decode pass.

    K and V of every cached token (2 * Hkv * d * 2 bytes per token), plus the
    bf16 query and output, the fp32 LSE, the used block-table entries and the
    sequence lengths.
    """
    L = torch.as_tensor(seq_lens, dtype=torch.int64)
    S = L.numel()
    kv = float(L.sum().item()) * 2 * Hkv * d * 2
    qo = 2.0 * S * Hq * d * 2
    lse = 4.0 * S * Hq
    table = 4.0 * float(((L + page_size - 1) // page_size).sum().item()) + 4.0 * S
    return kv + qo + lse + table
