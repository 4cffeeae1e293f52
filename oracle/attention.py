"""Plain, slow, fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or helper with the CUDA path.

What it computes, and where the pages define it
-----------------------------------------------
"Fast Attention Kernels and Operator Fusion" (wpnews.pro), section
"FlashAttention-Style Kernels", gives the operation as

    Attention(Q, K, V) = softmax(Q K^T / sqrt(d) + M) V

with M an additive mask; its SDPA example uses ``is_causal=True``, i.e. M is
-inf above the diagonal.  "Kernel Fusion and Custom Kernels" (ai.zenoagi.com),
section 5 "Intra-Attention Fusion", spells the unfused chain out as
S = Q K^T -> P = softmax(S) -> O = P V with S and P full N x N matrices; this
module does exactly that, materialising S and P per head, in float64.  The
anylearn.cc lesson ("Five things", third point) states that the fused method
is exact rather than approximate, so the plain definition is the oracle for
the fused kernel (up to rounding order).

Readings where the pages are silent (each is restated where it is used):

* scale: passed in (1/sqrt(d) in every workload) and multiplied into the
  scores before the mask is added.
* causal alignment: query i sees key j iff j <= i (Nq == Nk, so top-left and
  bottom-right alignment agree and no row is empty).
* LSE: the natural log of sum_j exp(scale * q_i . k_j) over the visible keys.
* GQA: query head h uses key/value head h // (Hq // Hkv) (consecutive query
  heads share one KV head).
* paged KV: pool layout [num_pages, page_size, Hkv, d]; logical token t of a
  sequence lives in physical page block_table[t // page_size], slot
  t % page_size ("Paged Attention Kernels" section and its block-table figure,
  logical blocks 0,1,2,3 -> physical 17,4,29,8).  Decode has one query per
  sequence that sees all seq_len cached keys.
* block-sparse masks (FlashInfer's 2-D block-sparse masks in "Kernel Fusion
  and Custom Kernels", section 4, e.g. the Longformer pattern): a boolean
  [B, Hq, ceil(N/128), ceil(N/128)] block mask; M = -inf for every key of a
  masked 128 x 128 block, on top of the causal mask.  A row that sees no key
  at all outputs zeros with LSE = -inf (the pages leave it open; this is the
  decode's convention for an empty sequence).
* additive M (the attention equation's M in general: any finite values, -inf
  allowed): a [B|1, Hq|1, N, N] array in natural-log units added to the
  scaled scores, S = scale * q k^T + M, on top of the causal mask.
* FP8 inputs ("Kernel Fusion and Custom Kernels", ai.zenoagi.com, section 3
  "FlashAttention: The Milestone of Fusion", under "v3 (2024, H100-Exclusive)":
  Q K^T and P V computed in FP8): Q, K, V arrive as e4m3 codes with one
  descale factor per tensor; the operation is attention over the decoded values times their descales
  (e4m3: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at
  exponent field 0, no infinities, the all-ones code NaN).
* appending to the cache / chunked prefill ("Operator Fusion" section: the
  KV cache is updated as keys and values are produced; "Paged Attention
  Kernels": blocks are allocated as the cache grows): a sequence holding
  seq_len tokens after the step received its last q_len of them in this step,
  packed by sequence ([total_q, H, d], rows cu_seqlens_q[s] ..
  cu_seqlens_q[s+1]-1).  New token i is logical token ctx + i with
  ctx = seq_len - q_len; its K and V are written there, and its query sees
  keys 0 .. ctx + i under the causal mask (every one of the seq_len keys
  without it).

Pins (all in ``tests/test_oracle.py``): rows of P sum to one; constant V rows
are returned unchanged; K == 0 gives the prefix mean of V and LSE = log(count);
causal row 0 returns v_0 with LSE = scale q_0 . k_0; a pure-Python ``math.fsum``
brute force on tiny inputs; PyTorch's fp64 CPU ``scaled_dot_product_attention``
and ``logsumexp`` as a library special case; the pages' block-table example;
paged gather equal to contiguous KV bit for bit; the sliding window against a
closed form, a scalar brute force and SDPA with an explicit mask; the append
against a hand-worked placement on the pages' block table; chunked prefill
against SDPA with an explicit bottom-right mask, a scalar brute force, the
whole-sequence prefill (two chunks give the same rows) and the decode (its
last row).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "gqa_kv_head",
    "block_keep",
    "attention_scores",
    "softmax_with_lse",
    "attention_head",
    "attention_forward",
    "attention_rows",
    "gather_paged_kv",
    "paged_decode",
    "paged_append",
    "paged_prefill",
    "fp8_e4m3_decode",
    "attention_forward_fp8",
]


def _f64(x) -> np.ndarray:
    """Return ``x`` as a float64 ndarray (exact for bf16/fp16/fp32 inputs)."""
    return np.asarray(x, dtype=np.float64)


def gqa_kv_head(h_q: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head ``h_q``: floor(h_q / (Hq / Hkv)).

    The pages do not mention grouped-query attention; this is the reading in
    which consecutive query heads share a KV head.
    """
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h_q // (Hq // Hkv)


def attention_scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
                     row_offset: int = 0, window_left: int | None = None, keep=None, bias=None) -> np.ndarray:
    """S = scale * q k^T + M for one head.

    ``q`` holds query rows ``row_offset .. row_offset + len(q) - 1`` of the head;
    ``k`` holds all keys.  With ``causal`` the additive mask M is -inf where the
    key index exceeds the query index ("FlashAttention-Style Kernels",
    equation with M and the ``is_causal=True`` example).  ``window_left`` = W
    (a sliding window, one more mask M of that equation) also sets M to -inf
    where the key index is below query index - W.
    """
    q = _f64(q)
    k = _f64(k)
    s = float(scale) * (q @ k.T)
    if bias is not None:  # additive M, [len(q), len(k)]
        s = s + _f64(bias)
    rows = np.arange(row_offset, row_offset + q.shape[0])[:, None]
    cols = np.arange(k.shape[0])[None, :]
    if causal:
        s = np.where(cols > rows, -np.inf, s)
    if window_left is not None and window_left >= 0:
        s = np.where(cols < rows - int(window_left), -np.inf, s)
    if keep is not None:  # boolean [len(q), len(k)]: False -> -inf
        s = np.where(np.asarray(keep, dtype=bool), s, -np.inf)
    return s


def softmax_with_lse(s: np.ndarray):
    """Row softmax of ``s`` and its natural-log log-sum-exp.

    LSE_i = m_i + log(sum_j exp(s_ij - m_i)) with m_i the row maximum (the
    shift changes nothing mathematically; it keeps exp finite).  Then
    P = exp(S - LSE).  Returns (P, LSE).
    """
    s = _f64(s)
    m = np.max(s, axis=-1, keepdims=True)
    empty = np.isneginf(m)  # a row with no visible key: P = 0, LSE = -inf
    m = np.where(empty, 0.0, m)
    with np.errstate(divide="ignore"):  # log(0) = -inf is the intended LSE of an empty row
        lse = m + np.log(np.sum(np.exp(s - m), axis=-1, keepdims=True))
    p = np.where(empty, 0.0, np.exp(s - np.where(empty, 0.0, lse)))
    return p, lse[..., 0]


def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                   causal: bool, row_offset: int = 0, window_left: int | None = None, keep=None, bias=None):
    """O and LSE for one head: materialise S, then P, then O = P V."""
    s = attention_scores(q, k, scale, causal, row_offset, window_left, keep, bias)
    p, lse = softmax_with_lse(s)
    o = p @ _f64(v)
    return o, lse


def block_keep(block_mask_bh, rows, n_keys: int, block: int = 128) -> np.ndarray:
    """Element mask of query rows `rows` over keys 0..n_keys-1 from one head's
    [q_blocks, k_blocks] block mask: key j is kept for row i iff block
    (i // block, j // block) is set."""
    bm = np.asarray(block_mask_bh, dtype=bool)
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.arange(int(n_keys))
    return bm[rows[:, None] // block, cols[None, :] // block]


def attention_forward(q, k, v, causal: bool, scale: float, row_chunk: int | None = None,
                      window_left: int | None = None, block_mask=None, bias=None):
    """Full attention forward for [B, Hq, N, d] queries and [B, Hkv, N, d] K/V.

    Returns (O [B, Hq, N, d] float64, LSE [B, Hq, N] float64).  ``row_chunk``
    splits each head into blocks of complete query rows (every row still sees
    its whole key set), which only bounds memory for long sequences.
    ``block_mask``: boolean [B, Hq, ceil(N/128), ceil(N/128)] (see block_keep).
    ``bias``: additive M, [B or 1, Hq or 1, N, N], natural-log units.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    o = np.empty((B, Hq, N, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    step = N if row_chunk is None else int(row_chunk)
    for b in range(B):
        for h in range(Hq):
            hk = gqa_kv_head(h, Hq, Hkv)
            for r0 in range(0, N, step):
                r1 = min(N, r0 + step)
                keep = None if block_mask is None else block_keep(block_mask[b, h], np.arange(r0, r1), N)
                mb = None
                if bias is not None:
                    bb = np.asarray(bias)
                    mb = bb[b if bb.shape[0] > 1 else 0, h if bb.shape[1] > 1 else 0, r0:r1]
                o[b, h, r0:r1], lse[b, h, r0:r1] = attention_head(
                    q[b, h, r0:r1], k[b, hk], v[b, hk], scale, causal, row_offset=r0,
                    window_left=window_left, keep=keep, bias=mb)
    return o, lse


def attention_rows(q, k, v, causal: bool, scale: float, b: int, h: int, rows,
                   window_left: int | None = None, block_mask=None, bias=None):
    """O and LSE of selected query rows of head (b, h), each row exact.

    Used for sampled parity checks at sizes where the full oracle is too slow.
    """
    rows = np.asarray(rows, dtype=np.int64)
    Hq, Hkv = q.shape[1], k.shape[1]
    hk = gqa_kv_head(h, Hq, Hkv)
    kk = _f64(k[b, hk])
    vv = _f64(v[b, hk])
    out_o = np.empty((rows.size, vv.shape[-1]), dtype=np.float64)
    out_l = np.empty(rows.size, dtype=np.float64)
    for i, r in enumerate(rows):
        qr = _f64(q[b, h, r:r + 1])
        keep = None if block_mask is None else block_keep(block_mask[b, h], [int(r)], kk.shape[0])
        mb = None
        if bias is not None:
            bb = np.asarray(bias)
            mb = bb[b if bb.shape[0] > 1 else 0, h if bb.shape[1] > 1 else 0, int(r):int(r) + 1]
        o_r, l_r = attention_head(qr, kk, vv, scale, causal, row_offset=int(r), window_left=window_left,
                                  keep=keep, bias=mb)
        out_o[i] = o_r[0]
        out_l[i] = l_r[0]
    return out_o, out_l


def gather_paged_kv(pool, block_table_row, seq_len: int, page_size: int) -> np.ndarray:
    """Logical KV rows 0..seq_len-1 of one sequence, read through its block table.

    Token t sits in physical page ``block_table_row[t // page_size]`` at slot
    ``t % page_size`` ("Paged Attention Kernels": the kernel translates logical
    positions through the block table).  Returns [seq_len, Hkv, d] in the
    pool's own dtype (no arithmetic, so the gather is exact).
    """
    pool = np.asarray(pool)
    table = np.asarray(block_table_row)
    t = np.arange(int(seq_len))
    pages = table[t // page_size]
    if seq_len > 0 and (pages.min() < 0 or pages.max() >= pool.shape[0]):
        raise IndexError("block table entry outside the pool")
    return pool[pages, t % page_size]


def paged_decode(q, k_pool, v_pool, block_table, seq_lens, page_size: int, scale: float):
    """Single-query decode attention over a paged KV cache.

    q: [S, Hq, d]; pools: [num_pages, page_size, Hkv, d]; block_table:
    [S, max_pages] int; seq_lens: [S].  The one query of sequence s is its
    newest token and sees all ``seq_lens[s]`` cached keys (no mask).
    Returns (O [S, Hq, d] float64, LSE [S, Hq] float64).
    """
    q = _f64(q)
    S, Hq, d = q.shape
    Hkv = np.asarray(k_pool).shape[2]
    o = np.empty((S, Hq, d), dtype=np.float64)
    lse = np.empty((S, Hq), dtype=np.float64)
    for s in range(S):
        L = int(seq_lens[s])
        ks = _f64(gather_paged_kv(k_pool, block_table[s], L, page_size))
        vs = _f64(gather_paged_kv(v_pool, block_table[s], L, page_size))
        for h in range(Hq):
            hk = gqa_kv_head(h, Hq, Hkv)
            o_h, l_h = attention_head(q[s, h][None, :], ks[:, hk], vs[:, hk], scale, causal=False)
            o[s, h] = o_h[0]
            lse[s, h] = l_h[0]
    return o, lse


def _chunk_bounds(cu_seqlens_q, seq_lens, s):
    """(first packed row, q_len, ctx) of sequence s."""
    q0 = int(cu_seqlens_q[s])
    q_len = int(cu_seqlens_q[s + 1]) - q0
    ctx = int(seq_lens[s]) - q_len
    if q_len < 0 or ctx < 0:
        raise ValueError("a sequence has more new tokens than tokens in all")
    return q0, q_len, ctx


def paged_append(k_pool, v_pool, k_new, v_new, block_table, cu_seqlens_q, seq_lens, page_size: int):
    """Write each sequence's new K/V rows into the paged cache.

    k_new/v_new: [total_q, Hkv, d], packed by sequence as the queries are.
    Row i of sequence s becomes logical token ctx + i, stored at physical page
    block_table[s][(ctx + i) // page_size], slot (ctx + i) % page_size.
    Returns new pool arrays (the inputs are not modified); every other slot
    keeps its old contents.  Pure indexing: exact in the pools' own dtype.
    """
    kp = np.array(k_pool, copy=True)
    vp = np.array(v_pool, copy=True)
    kn = np.asarray(k_new)
    vn = np.asarray(v_new)
    table = np.asarray(block_table)
    for s in range(len(seq_lens)):
        q0, q_len, ctx = _chunk_bounds(cu_seqlens_q, seq_lens, s)
        for i in range(q_len):
            t = ctx + i
            page = int(table[s, t // page_size])
            if page < 0 or page >= kp.shape[0]:
                raise IndexError("block table entry outside the pool")
            kp[page, t % page_size] = kn[q0 + i]
            vp[page, t % page_size] = vn[q0 + i]
    return kp, vp


def paged_prefill(q, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens, page_size: int, scale: float,
                  causal: bool = True):
    """Attention of each sequence's new queries over its whole paged cache.

    q: [total_q, Hq, d] packed by sequence; the pools already hold all
    seq_len tokens of every sequence (the new ones included).  Query i of
    sequence s is logical token ctx + i, so under the causal mask it is row
    ctx + i of the sequence's attention (``row_offset`` = ctx).
    Returns (O [total_q, Hq, d] float64, LSE [total_q, Hq] float64).
    """
    q = _f64(q)
    total_q, Hq, d = q.shape
    Hkv = np.asarray(k_pool).shape[2]
    o = np.zeros((total_q, Hq, np.asarray(v_pool).shape[-1]), dtype=np.float64)
    lse = np.zeros((total_q, Hq), dtype=np.float64)
    for s in range(len(seq_lens)):
        q0, q_len, ctx = _chunk_bounds(cu_seqlens_q, seq_lens, s)
        if q_len == 0:
            continue
        L = int(seq_lens[s])
        ks = _f64(gather_paged_kv(k_pool, block_table[s], L, page_size))
        vs = _f64(gather_paged_kv(v_pool, block_table[s], L, page_size))
        for h in range(Hq):
            hk = gqa_kv_head(h, Hq, Hkv)
            o_h, l_h = attention_head(q[q0:q0 + q_len, h], ks[:, hk], vs[:, hk], scale, causal, row_offset=ctx)
            o[q0:q0 + q_len, h] = o_h
            lse[q0:q0 + q_len, h] = l_h
    return o, lse


def fp8_e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 byte code, as float64 (every e4m3 value is exact).

    Field by field: sign s = bit 7, exponent e = bits 6..3, mantissa m = bits
    2..0.  e = 0: (-1)^s * m/8 * 2^-6 (subnormal); 0 < e: (-1)^s * (1 + m/8) *
    2^(e-7); e = 15 and m = 7 is NaN (the format has no infinities, so
    e = 15, m < 7 are ordinary values up to 448).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * val
    return np.where((e == 15) & (m == 7), np.nan, val)


def attention_forward_fp8(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float, causal: bool,
                          scale: float, row_chunk: int | None = None):
    """Attention of e4m3-coded inputs: decode each code, multiply by the
    tensor's descale factor, then the plain definition (attention_forward)."""
    q = fp8_e4m3_decode(q8) * float(q_descale)
    k = fp8_e4m3_decode(k8) * float(k_descale)
    v = fp8_e4m3_decode(v8) * float(v_descale)
    return attention_forward(q, k, v, causal, scale, row_chunk=row_chunk)
