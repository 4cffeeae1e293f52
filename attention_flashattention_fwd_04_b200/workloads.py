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
* ``chunked_prefill`` 16 sequences, Hq=32, Hkv=8, d=128, 16-token pages;
  cached context lengths uniform in [0, 6144], new-chunk lengths uniform in
  [256, 2048] (a serving step that appends a prompt chunk to each
  sequence's cache and attends over all of it), seed 8
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
    "make_prefill_inputs_fp8",
    "make_decode_inputs",
    "ChunkedConfig",
    "CHUNKED_CONFIGS",
    "make_chunked_inputs",
    "chunked_flops",
    "chunked_append_bytes",
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
    # causal_gqa cut to 4 query heads (one KV head): a per-head M of 0.5 GB
    # instead of 4.3 GB, small enough for a full ncu capture.
    "causal_gqa_h4": PrefillConfig("causal_gqa_h4", 1, 4, 1, 8192, 128, True, 3, value_scale=0.5),
}

DECODE_CONFIGS = {
    "paged_decode": DecodeConfig("paged_decode", 64, 32, 8, 128, 16, 512, 8192, 4),
    # a small decode batch, where per-call host work and launch gaps dominate
    "small_decode": DecodeConfig("small_decode", 4, 32, 8, 128, 16, 256, 1024, 6),
}


@dataclass(frozen=True)
class ChunkedConfig:
    name: str
    num_seqs: int
    Hq: int
    Hkv: int
    d: int
    page_size: int
    ctx_range: tuple
    q_range: tuple
    seed: int

    @property
    def scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))


CHUNKED_CONFIGS = {
    "chunked_prefill": ChunkedConfig("chunked_prefill", 16, 32, 8, 128, 16, (0, 6144), (256, 2048), 8),
}


def make_chunked_inputs(cfg: ChunkedConfig, device: str | torch.device = "cpu", poison: bool = False,
                        ctx_lens=None, q_lens=None, spare_pages: int = 0):
    """Inputs of one append + chunked-prefill step over a paged cache.

    Sequence s holds ctx_s cached tokens and receives q_s new ones
    (seq_len = ctx + q).  Returns a dict with q [total_q,Hq,d], k_new / v_new
    [total_q,Hkv,d] (packed by sequence, cu_seqlens_q [S+1] int32), pools
    [num_pages,page_size,Hkv,d] holding every sequence's context (pages for
    all seq_len tokens are allocated up front, a seeded permutation of the
    pool), block_table [S,width] int32 (-1 past each sequence's pages),
    seq_lens [S] int32.  The slots of the new tokens and every slot past a
    sequence's end hold NaN when ``poison`` (the append must overwrite the
    former; nothing may read the latter), else random values.
    ``spare_pages`` adds unused pages (filled like the rest) to the pool.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed)
    S, ps = cfg.num_seqs, cfg.page_size
    ctx = torch.randint(cfg.ctx_range[0], cfg.ctx_range[1] + 1, (S,), generator=g, dtype=torch.int64)
    ql = torch.randint(cfg.q_range[0], cfg.q_range[1] + 1, (S,), generator=g, dtype=torch.int64)
    if ctx_lens is not None:
        ctx = torch.as_tensor(ctx_lens, dtype=torch.int64).clone()
    if q_lens is not None:
        ql = torch.as_tensor(q_lens, dtype=torch.int64).clone()
    lens = ctx + ql
    pages = (lens + ps - 1) // ps
    width = max(1, int(pages.max().item()) if S else 1)
    num_pages = int(pages.sum().item()) + spare_pages
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((S, width), -1, dtype=torch.int32)
    off = 0
    for s in range(S):
        n = int(pages[s])
        table[s, :n] = perm[off:off + n].to(torch.int32)
        off += n
    total_q = int(ql.sum().item())
    cu = torch.zeros(S + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(ql, 0).to(torch.int32)
    q = torch.randn(total_q, cfg.Hq, cfg.d, generator=g, dtype=torch.float32)
    k_new = torch.randn(total_q, cfg.Hkv, cfg.d, generator=g, dtype=torch.float32)
    v_new = torch.randn(total_q, cfg.Hkv, cfg.d, generator=g, dtype=torch.float32)
    k_pool = torch.randn(num_pages, ps, cfg.Hkv, cfg.d, generator=g, dtype=torch.float32)
    v_pool = torch.randn(num_pages, ps, cfg.Hkv, cfg.d, generator=g, dtype=torch.float32)
    q, k_new, v_new, k_pool, v_pool = (t.to(torch.bfloat16) for t in (q, k_new, v_new, k_pool, v_pool))
    if poison:
        for s in range(S):
            n = int(pages[s])
            for t in range(int(ctx[s]), n * ps):
                pg = int(table[s, t // ps])
                k_pool[pg, t % ps] = float("nan")
                v_pool[pg, t % ps] = float("nan")
    dev = torch.device(device)
    return {
        "q": q.contiguous().to(dev),
        "k_new": k_new.contiguous().to(dev),
        "v_new": v_new.contiguous().to(dev),
        "k_pool": k_pool.contiguous().to(dev),
        "v_pool": v_pool.contiguous().to(dev),
        "block_table": table.contiguous().to(dev),
        "cu_seqlens_q": cu.contiguous().to(dev),
        "seq_lens": lens.to(torch.int32).contiguous().to(dev),
        "ctx_lens": ctx,
        "q_lens": ql,
        "page_size": ps,
        "num_pages": num_pages,
        "max_pages": width,
        "total_q": total_q,
        "scale": cfg.scale,
    }


def chunked_flops(ctx_lens, q_lens, Hq: int, d: int, causal: bool = True) -> float:
    """4*d per visible (query, key) pair: new query i of a sequence sees
    ctx + i + 1 keys under the causal mask, ctx + q otherwise."""
    total = 0
    for c, q in zip(torch.as_tensor(ctx_lens).tolist(), torch.as_tensor(q_lens).tolist()):
        total += q * c + q * (q + 1) // 2 if causal else q * (c + q)
    return 4.0 * Hq * d * total


def chunked_append_bytes(q_lens, Hkv: int, d: int) -> float:
    """HBM bytes of the append: K and V of every new token read once and
    written once (2 tensors x 2 directions x Hkv x d x 2 bytes), plus the
    block-table entries and lengths it reads."""
    n = float(torch.as_tensor(q_lens).sum().item())
    return n * 2 * 2 * Hkv * d * 2


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


def make_bias_inputs(shape, kind: str = "normal", seed: int = 0, sigma: float = 1.0, neg_inf_frac: float = 0.0,
                     pad_fill: float = 0.0, device: str | torch.device = "cpu"):
    """An additive mask M of ``shape`` = (B', H', R, N) (R = N, or 1 for one
    row per head), bf16, natural-log units, as a view ``[..., :N]`` of a buffer
    whose rows are padded to a multiple of 8 with ``pad_fill``.

    kind "normal": N(0, sigma^2) values; kind "alibi": -slope_h * |i - j| with
    slopes 2^(-8 (h + 1) / H') per head (a linear distance penalty).  A
    fraction ``neg_inf_frac`` of the entries is then set to -inf.  Returns
    (buffer, view)."""
    Bp, Hp, R, N = shape
    padded = -(-N // 8) * 8
    buf = torch.full((Bp, Hp, R, padded), pad_fill, dtype=torch.bfloat16)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    if kind == "normal":
        buf[..., :N] = (torch.randn(Bp, Hp, R, N, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)
    elif kind == "alibi":
        for h in range(Hp):  # one head at a time: no full-size float32 intermediate
            buf[:, h, :, :N] = alibi_rows(Hp, h, 0, R, N)
    else:
        raise ValueError(kind)
    if neg_inf_frac > 0:
        view = buf[..., :N]
        view[torch.rand(view.shape, generator=g) < neg_inf_frac] = float("-inf")
    buf = buf.to(device)
    return buf, buf[..., :N]


def alibi_rows(Hp: int, h: int, r0: int, r1: int, N: int) -> torch.Tensor:
    """Rows r0 .. r1-1 of head h's linear distance penalty (of Hp heads):
    -s_h * |i - j| with s_h = 2^(-8 (h + 1) / Hp), bf16 [r1 - r0, N]."""
    s = 2.0 ** (-8.0 * (h + 1) / Hp)
    i = torch.arange(r0, r1, dtype=torch.float32).view(-1, 1)
    j = torch.arange(N, dtype=torch.float32).view(1, -1)
    return (-s * (i - j).abs()).to(torch.bfloat16)


def longformer_keep(nb: int) -> torch.Tensor:
    """Block mask [nb, nb] (128 x 128 blocks) of a Longformer-style pattern:
    each query block keeps its own key block, the one before it, and key
    block 0 (a global first block)."""
    keep = torch.zeros(nb, nb, dtype=torch.bool)
    for i in range(nb):
        keep[i, max(0, i - 1): i + 1] = True
        keep[i, 0] = True
    return keep


def block_sparse_pairs(keep2d, N: int, causal: bool) -> int:
    """Visible (query, key) pairs of one head under a [nb, nb] block mask of
    128 x 128 blocks (and the causal mask)."""
    import numpy as np
    keep2d = np.asarray(keep2d, dtype=bool)
    nb = keep2d.shape[0]
    total = 0
    for qb in range(nb):
        rows = np.arange(qb * 128, min(N, qb * 128 + 128))
        for kb in np.nonzero(keep2d[qb])[0]:
            c0, c1 = kb * 128, min(N, kb * 128 + 128)
            if causal:
                total += int(np.clip(np.minimum(rows + 1, c1) - c0, 0, None).sum())
            else:
                total += rows.size * (c1 - c0)
    return total


# Prefill workloads with a general mask: (shapes, mask kind).
MASK_WORKLOADS = {
    "longformer_sparse": ("causal_gqa", "longformer"),
    "alibi_bias": ("causal_gqa", "alibi"),
    "alibi_bias_h4": ("causal_gqa_h4", "alibi"),
}


def make_prefill_inputs_fp8(cfg: PrefillConfig, device: str | torch.device = "cpu"):
    """The bf16 draw of ``cfg`` quantised to e4m3 per tensor: descale =
    amax / 448, codes = round-to-nearest-even(x / descale) (PyTorch's
    float8_e4m3fn conversion).  Returns (q8, k8, v8) as uint8 codes and
    (q_descale, k_descale, v_descale) as Python floats (fp32 values)."""
    codes, scales = [], []
    for t in make_prefill_inputs(cfg):
        x = t.float()
        d = float(torch.tensor(max(float(x.abs().max()), 1e-30) / 448.0, dtype=torch.float32))
        codes.append((x / d).to(torch.float8_e4m3fn).view(torch.uint8).contiguous().to(device))
        scales.append(d)
    return tuple(codes), tuple(scales)


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
