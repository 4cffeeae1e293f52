"""Pins that tie the CPU oracle to facts the pages and the mathematics fix.

Every pin takes an oracle-like module ``o`` (the real ``oracle.attention`` or a
copy with a planted mistake) and raises ``AssertionError`` when the module
disagrees with the fact.  None of them re-types the oracle's own vectorised
formula: they use closed forms, invariants, a scalar brute force written in
the ratio form sum(w v) / sum(w), PyTorch's fp64 SDPA as a library special
case, and the pages' printed block-table example.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(rng, *shape):
    # bf16-representable values, like the kernels' inputs
    x = rng.standard_normal(shape).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)


# -- softmax normalisation ---------------------------------------------------

def pin_rows_sum_to_one(o):
    """Every row of P = softmax(S + M) sums to one (causal and not)."""
    rng = _rng(11)
    q, k = _rand(rng, 37, 16), _rand(rng, 37, 16)
    for causal in (False, True):
        s = o.attention_scores(q, k, 0.25, causal)
        p, _ = o.softmax_with_lse(s)
        assert np.all(np.isfinite(p))
        assert np.max(np.abs(p.sum(axis=-1) - 1.0)) < 1e-12
        if causal:
            assert np.all(p[np.triu_indices(37, 1)] == 0.0)


# -- closed forms ------------------------------------------------------------

def pin_constant_v(o):
    """If every value row equals c, every output row equals c."""
    rng = _rng(12)
    B, Hq, Hkv, N, d = 1, 4, 2, 45, 8
    q = _rand(rng, B, Hq, N, d)
    k = _rand(rng, B, Hkv, N, d)
    c = _rand(rng, B, Hkv, 1, d)
    v = np.broadcast_to(c, (B, Hkv, N, d)).copy()
    for causal in (False, True):
        out, _ = o.attention_forward(q, k, v, causal, 0.3)
        for h in range(Hq):
            want = c[0, h // (Hq // Hkv), 0]
            assert np.max(np.abs(out[0, h] - want)) < 1e-12


def pin_zero_k(o):
    """K == 0 makes every visible score 0: O_i is the mean of the visible value
    rows and LSE_i = log(number of visible keys)."""
    rng = _rng(13)
    B, H, N, d = 1, 2, 33, 8
    q = _rand(rng, B, H, N, d)
    k = np.zeros((B, H, N, d))
    v = _rand(rng, B, H, N, d)
    out, lse = o.attention_forward(q, k, v, True, 0.125)
    for i in range(N):
        assert np.max(np.abs(out[0, :, i] - v[0, :, : i + 1].mean(axis=1))) < 1e-12
        assert np.max(np.abs(lse[0, :, i] - math.log(i + 1))) < 1e-12
    out, lse = o.attention_forward(q, k, v, False, 0.125)
    assert np.max(np.abs(out[0] - v[0].mean(axis=1, keepdims=True))) < 1e-12
    assert np.max(np.abs(lse - math.log(N))) < 1e-12


def pin_causal_row0(o):
    """Causal row 0 sees only key 0: O_0 = v_0 and LSE_0 = scale * q_0 . k_0."""
    rng = _rng(14)
    q, k, v = (_rand(rng, 1, 3, 20, 16) for _ in range(3))
    out, lse = o.attention_forward(q, k, v, True, 0.7)
    assert np.array_equal(out[0, :, 0], v[0, :, 0])
    want = 0.7 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0])
    assert np.max(np.abs(lse[0, :, 0] - want)) < 1e-12


def pin_onehot(o):
    """One key whose score beats all others by ~1000 takes all the weight:
    exp of the others underflows to exactly 0 in fp64, so O equals that value
    row exactly and LSE equals that score."""
    rng = _rng(15)
    N, d = 24, 8
    q = np.zeros((1, 1, N, d))
    q[..., 0] = 1.0
    k = _rand(rng, 1, 1, N, d) * 0.01
    v = _rand(rng, 1, 1, N, d)
    star = 17
    k[0, 0, star, 0] = 1000.0
    out, lse = o.attention_forward(q, k, v, False, 1.0)
    assert np.array_equal(out[0, 0], np.broadcast_to(v[0, 0, star], (N, d)))
    assert np.max(np.abs(lse[0, 0] - k[0, 0, star, 0])) < 1e-9


# -- brute force ---------------------------------------------------------------

def _brute(q, k, v, scale, causal, Hq, Hkv):
    """Scalar loops, no max shift: O_i = sum_j w_ij v_j / sum_j w_ij with
    w_ij = exp(scale q_i . k_j), LSE_i = log(sum_j w_ij), sums by math.fsum."""
    B, _, N, d = q.shape
    out = np.zeros((B, Hq, N, d))
    lse = np.zeros((B, Hq, N))
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            for i in range(N):
                ws = []
                for j in range(N):
                    if causal and j > i:
                        continue
                    dot = math.fsum(float(q[b, h, i, t]) * float(k[b, hk, j, t]) for t in range(d))
                    ws.append((j, math.exp(scale * dot)))
                z = math.fsum(w for _, w in ws)
                lse[b, h, i] = math.log(z)
                for t in range(d):
                    out[b, h, i, t] = math.fsum(w * float(v[b, hk, j, t]) for j, w in ws) / z
    return out, lse


def pin_bruteforce(o):
    """Tiny cases (N <= 8) against the scalar brute force, MHA and GQA."""
    rng = _rng(16)
    for (B, Hq, Hkv, N, d, causal, scale) in [
        (1, 1, 1, 1, 4, True, 0.5),
        (1, 2, 2, 5, 4, False, 0.5),
        (2, 4, 2, 7, 3, True, 0.9),
        (1, 6, 3, 8, 5, False, 0.35),
        (1, 4, 1, 8, 4, True, 1.3),
    ]:
        q = _rand(rng, B, Hq, N, d)
        k = _rand(rng, B, Hkv, N, d)
        v = _rand(rng, B, Hkv, N, d)
        out, lse = o.attention_forward(q, k, v, causal, scale)
        bo, bl = _brute(q, k, v, scale, causal, Hq, Hkv)
        assert np.max(np.abs(out - bo)) < 1e-12, (N, causal)
        assert np.max(np.abs(lse - bl)) < 1e-12, (N, causal)


# -- library special case ------------------------------------------------------

def pin_torch_sdpa(o):
    """PyTorch's CPU fp64 scaled_dot_product_attention (GQA expanded with
    repeat_interleave) and logsumexp of the masked scores."""
    rng = _rng(17)
    for (B, Hq, Hkv, N, d, causal, scale) in [
        (2, 4, 4, 50, 16, True, 0.25),
        (1, 8, 2, 67, 32, True, 1 / math.sqrt(32)),
        (1, 6, 3, 40, 8, False, 0.4),
    ]:
        q = _rand(rng, B, Hq, N, d)
        k = _rand(rng, B, Hkv, N, d)
        v = _rand(rng, B, Hkv, N, d)
        out, lse = o.attention_forward(q, k, v, causal, scale)
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        tk = tk.repeat_interleave(Hq // Hkv, dim=1)
        tv = tv.repeat_interleave(Hq // Hkv, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        s = scale * (tq @ tk.transpose(-1, -2))
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        ref_lse = torch.logsumexp(s, dim=-1)
        assert np.max(np.abs(out - ref.numpy())) < 1e-12
        assert np.max(np.abs(lse - ref_lse.numpy())) < 1e-12


# -- paged layout ------------------------------------------------------------------

def pin_block_table_example(o):
    """The pages' block table: logical blocks 0,1,2,3 live in physical blocks
    17,4,29,8, and a page holds 16 tokens.  Label every pool slot with its
    (page, slot) and check where each logical token is read from."""
    with open(os.path.join(GOLDEN, "block_table_example.json")) as f:
        ex = json.load(f)
    ps = ex["page_size"]
    phys = ex["physical_blocks"]
    pool = np.zeros((32, ps, 1, 2), dtype=np.int64)
    for p in range(32):
        for s in range(ps):
            pool[p, s, 0] = (p, s)
    L = len(ex["logical_blocks"]) * ps
    got = o.gather_paged_kv(pool, np.array(phys), L, ps)
    for t in range(L):
        assert tuple(got[t, 0]) == (phys[t // ps], t % ps)


def pin_paged_equals_contiguous(o):
    """Scatter a contiguous KV sequence into randomly chosen pages (shared
    prefix pages included), read it back through the table: bit-identical.
    Decode over the pages equals attention of the last query over the
    contiguous keys."""
    rng = _rng(18)
    ps, Hkv, Hq, d = 4, 2, 4, 8
    lens = [1, 4, 9, 13]
    num_pages = 16
    pool_k = _rand(rng, num_pages, ps, Hkv, d)
    pool_v = _rand(rng, num_pages, ps, Hkv, d)
    order = rng.permutation(num_pages)
    table = -np.ones((len(lens), 4), dtype=np.int32)
    used = 0
    conts = []
    for s, L in enumerate(lens):
        n = -(-L // ps)
        table[s, :n] = order[used:used + n]
        used += n
    table[3, 0] = table[2, 0]  # sequence 3 shares its first page with sequence 2
    for s, L in enumerate(lens):
        kc = np.stack([pool_k[table[s, t // ps], t % ps] for t in range(L)])
        vc = np.stack([pool_v[table[s, t // ps], t % ps] for t in range(L)])
        assert np.array_equal(o.gather_paged_kv(pool_k, table[s], L, ps), kc)
        assert np.array_equal(o.gather_paged_kv(pool_v, table[s], L, ps), vc)
        conts.append((kc, vc))
    q = _rand(rng, len(lens), Hq, d)
    out, lse = o.paged_decode(q, pool_k, pool_v, table, np.array(lens), ps, 0.3)
    for s, (kc, vc) in enumerate(conts):
        tq = torch.from_numpy(q[s][:, None, :])                       # [Hq,1,d]
        tk = torch.from_numpy(kc.transpose(1, 0, 2)).repeat_interleave(Hq // Hkv, 0)
        tv = torch.from_numpy(vc.transpose(1, 0, 2)).repeat_interleave(Hq // Hkv, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.3)
        ref_lse = torch.logsumexp(0.3 * (tq @ tk.transpose(-1, -2)), dim=-1)
        assert np.max(np.abs(out[s] - ref[:, 0].numpy())) < 1e-12
        assert np.max(np.abs(lse[s] - ref_lse[:, 0].numpy())) < 1e-12


def pin_printed_sizes(o):
    """Numbers the pages print: the N=2048 score matrix holds 4M entries, 16MB
    in fp32, per head; causal SDPA on (2,16,512,64) returns that shape."""
    with open(os.path.join(GOLDEN, "printed_values.json")) as f:
        pv = json.load(f)
    sm = pv["score_matrix"]
    N = sm["N"]
    q = np.ones((N, 1))
    s = o.attention_scores(q, q, 1.0, False)
    assert s.size == sm["elements"]
    assert s.astype(np.float32).nbytes == sm["bytes_fp32"]
    shp = pv["sdpa_example"]["shape"]
    small = [1, 2, 24, shp[3]]  # same head dim; fewer heads/rows keeps it fast
    rng = _rng(19)
    q, k, v = (_rand(rng, *small) for _ in range(3))
    out, lse = o.attention_forward(q, k, v, pv["sdpa_example"]["causal"], 0.125)
    assert list(out.shape) == small and list(lse.shape) == small[:3]


def pin_window_closed_form(o):
    """Sliding window W with K == 0: query i sees keys max(0, i-W) .. i (or
    .. N-1 without the causal mask), all with score 0, so O_i is their mean
    and LSE_i = log(count)."""
    rng = _rng(20)
    N, d = 40, 8
    q = _rand(rng, 1, 2, N, d)
    k = np.zeros((1, 2, N, d))
    v = _rand(rng, 1, 2, N, d)
    for W in (0, 1, 5, 39):
        for causal in (True, False):
            out, lse = o.attention_forward(q, k, v, causal, 0.2, window_left=W)
            for i in range(N):
                lo, hi = max(0, i - W), (i if causal else N - 1)
                assert np.max(np.abs(out[0, :, i] - v[0, :, lo:hi + 1].mean(axis=1))) < 1e-12
                assert np.max(np.abs(lse[0, :, i] - math.log(hi - lo + 1))) < 1e-12


def pin_window_sdpa(o):
    """Sliding window against PyTorch's fp64 SDPA with an explicit boolean
    mask, and against the scalar brute force on tiny inputs."""
    rng = _rng(21)
    B, Hq, Hkv, N, d = 1, 4, 2, 45, 8
    q = _rand(rng, B, Hq, N, d)
    k = _rand(rng, B, Hkv, N, d)
    v = _rand(rng, B, Hkv, N, d)
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    for W, causal in ((7, True), (0, True), (20, False)):
        out, lse = o.attention_forward(q, k, v, causal, 0.3, window_left=W)
        allowed = (j >= i - W) & ((j <= i) if causal else torch.ones_like(j, dtype=torch.bool))
        tq = torch.from_numpy(q)
        tk = torch.from_numpy(k).repeat_interleave(Hq // Hkv, dim=1)
        tv = torch.from_numpy(v).repeat_interleave(Hq // Hkv, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed, scale=0.3)
        ref_lse = torch.logsumexp((0.3 * (tq @ tk.transpose(-1, -2))).masked_fill(~allowed, float("-inf")), -1)
        assert np.max(np.abs(out - ref.numpy())) < 1e-12
        assert np.max(np.abs(lse - ref_lse.numpy())) < 1e-12
    # scalar brute force: keys outside the window simply do not take part
    out, lse = o.attention_forward(q[:, :1, :6], k[:, :1, :6], v[:, :1, :6], True, 0.5, window_left=2)
    for r in range(6):
        ws = [(j, math.exp(0.5 * math.fsum(float(q[0, 0, r, t]) * float(k[0, 0, j, t]) for t in range(d))))
              for j in range(max(0, r - 2), r + 1)]
        z = math.fsum(w for _, w in ws)
        assert abs(lse[0, 0, r] - math.log(z)) < 1e-12
        for t in range(d):
            want = math.fsum(w * float(v[0, 0, j, t]) for j, w in ws) / z
            assert abs(out[0, 0, r, t] - want) < 1e-12


# -- appending to the paged cache and chunked prefill ----------------------------

def pin_append_example(o):
    """The pages' block table with 16-token blocks: a sequence holding 20
    tokens receives 30 more.  Each new row must land at the (page, slot)
    worked out by hand in the golden file; nothing else may change."""
    with open(os.path.join(GOLDEN, "append_example.json")) as f:
        ex = json.load(f)
    ps, phys = ex["page_size"], ex["physical_blocks"]
    ctx, n_new = ex["context_tokens"], ex["new_tokens"]
    num_pages = 32
    # label old slots (page, slot, 0) and new rows (-1, i, 1)
    kp = np.zeros((num_pages, ps, 1, 3), dtype=np.int64)
    for pg in range(num_pages):
        for sl in range(ps):
            kp[pg, sl, 0] = (pg, sl, 0)
    vp = kp.copy()
    kn = np.array([[[-1, i, 1]] for i in range(n_new)], dtype=np.int64)
    vn = kn.copy()
    table = np.array([phys], dtype=np.int32)
    ko, vo = o.paged_append(kp, vp, kn, vn, table, np.array([0, n_new]), np.array([ctx + n_new]), ps)
    for d in ex["destinations"]:
        assert tuple(ko[d["physical_page"], d["slot"], 0]) == (-1, d["new_token"], 1)
        assert tuple(vo[d["physical_page"], d["slot"], 0]) == (-1, d["new_token"], 1)
    changed = {(pg, sl) for pg in range(num_pages) for sl in range(ps) if ko[pg, sl, 0, 2] == 1}
    assert len(changed) == n_new
    for sl in range(16):
        assert tuple(ko[17, sl, 0]) == (17, sl, 0)
    for sl in range(4):
        assert tuple(ko[4, sl, 0]) == (4, sl, 0)
    for sl in range(2, 16):
        assert tuple(ko[8, sl, 0]) == (8, sl, 0)
    assert np.array_equal(kp[:, :, :, 2], np.zeros_like(kp[:, :, :, 2]))  # inputs untouched


def _chunked_setup(seed, lens, q_lens, ps, Hq, Hkv, d, num_pages):
    rng = _rng(seed)
    pool_k = _rand(rng, num_pages, ps, Hkv, d)
    pool_v = _rand(rng, num_pages, ps, Hkv, d)
    order = rng.permutation(num_pages)
    width = max(-(-L // ps) for L in lens)
    table = -np.ones((len(lens), width), dtype=np.int32)
    used = 0
    for s, L in enumerate(lens):
        n = -(-L // ps)
        table[s, :n] = order[used:used + n]
        used += n
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    q = _rand(rng, int(cu[-1]), Hq, d)
    return q, pool_k, pool_v, table, cu


def pin_paged_prefill_sdpa(o):
    """Chunked prefill against PyTorch's fp64 SDPA with an explicit mask in
    which new query i of a sequence with ctx cached tokens sees keys
    0..ctx+i (and, without the causal mask, all keys)."""
    lens, q_lens = [9, 23, 5, 17, 1], [9, 6, 1, 17, 1]
    ps, Hq, Hkv, d = 4, 4, 2, 8
    q, pk, pv, table, cu = _chunked_setup(30, lens, q_lens, ps, Hq, Hkv, d, 24)
    for causal in (True, False):
        out, lse = o.paged_prefill(q, pk, pv, table, cu, np.array(lens), ps, 0.3, causal)
        for s, L in enumerate(lens):
            ql, ctx = q_lens[s], L - q_lens[s]
            kc = np.stack([pk[table[s, t // ps], t % ps] for t in range(L)])
            vc = np.stack([pv[table[s, t // ps], t % ps] for t in range(L)])
            tq = torch.from_numpy(q[cu[s]:cu[s + 1]].transpose(1, 0, 2))            # [Hq, ql, d]
            tk = torch.from_numpy(kc.transpose(1, 0, 2)).repeat_interleave(Hq // Hkv, 0)
            tv = torch.from_numpy(vc.transpose(1, 0, 2)).repeat_interleave(Hq // Hkv, 0)
            i = torch.arange(ql)[:, None]
            j = torch.arange(L)[None, :]
            allowed = (j <= ctx + i) if causal else torch.ones(ql, L, dtype=torch.bool)
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed, scale=0.3)
            ref_lse = torch.logsumexp((0.3 * (tq @ tk.transpose(-1, -2))).masked_fill(~allowed, float("-inf")), -1)
            assert np.max(np.abs(out[cu[s]:cu[s + 1]] - ref.numpy().transpose(1, 0, 2))) < 1e-12
            assert np.max(np.abs(lse[cu[s]:cu[s + 1]] - ref_lse.numpy().T)) < 1e-12


def pin_paged_prefill_brute(o):
    """Scalar brute force, ratio form: the new query i of a sequence with
    ctx = 3 cached tokens averages V over keys 0..3+i with weights
    exp(scale q.k)."""
    lens, q_lens = [7], [4]
    ps, Hq, Hkv, d = 2, 2, 1, 4
    q, pk, pv, table, cu = _chunked_setup(31, lens, q_lens, ps, Hq, Hkv, d, 6)
    out, lse = o.paged_prefill(q, pk, pv, table, cu, np.array(lens), ps, 0.5, True)
    for i in range(4):
        for h in range(Hq):
            keys = range(0, 3 + i + 1)
            w = [math.exp(0.5 * math.fsum(float(q[i, h, c]) * float(pk[table[0, t // ps], t % ps, 0, c])
                                          for c in range(d))) for t in keys]
            z = math.fsum(w)
            for c in range(d):
                want = math.fsum(wt * float(pv[table[0, t // ps], t % ps, 0, c]) for wt, t in zip(w, keys)) / z
                assert abs(out[i, h, c] - want) < 1e-12
            assert abs(lse[i, h] - math.log(z)) < 1e-12


def pin_chunked_equals_whole(o):
    """A sequence prefilled in one chunk, or as a first chunk followed by a
    second one over the cache the first left behind, gives the same rows: a
    row depends only on its own position and keys."""
    L, a, ps, Hq, Hkv, d = 21, 8, 4, 2, 2, 8
    q, pk, pv, table, _ = _chunked_setup(32, [L], [L], ps, Hq, Hkv, d, 8)
    whole_o, whole_l = o.paged_prefill(q, pk, pv, table, np.array([0, L]), np.array([L]), ps, 0.4, True)
    first_o, first_l = o.paged_prefill(q[:a], pk, pv, table, np.array([0, a]), np.array([a]), ps, 0.4, True)
    second_o, second_l = o.paged_prefill(q[a:], pk, pv, table, np.array([0, L - a]), np.array([L]), ps, 0.4,
                                         True)
    assert np.max(np.abs(whole_o[:a] - first_o)) < 1e-12 and np.max(np.abs(whole_l[:a] - first_l)) < 1e-12
    assert np.max(np.abs(whole_o[a:] - second_o)) < 1e-12 and np.max(np.abs(whole_l[a:] - second_l)) < 1e-12
    # the last row is the decode of the same sequence
    dec_o, dec_l = o.paged_decode(q[L - 1:L], pk, pv, table, np.array([L]), ps, 0.4)
    assert np.max(np.abs(whole_o[L - 1] - dec_o[0])) < 1e-12 and np.max(np.abs(whole_l[L - 1] - dec_l[0])) < 1e-12


# -- FP8 (e4m3) inputs ---------------------------------------------------------

def pin_fp8_code_points(o):
    """e4m3 code points worked out by hand from the format's fields."""
    with open(os.path.join(GOLDEN, "fp8_e4m3_codes.json")) as f:
        ex = json.load(f)
    codes = np.array([int(c["code"], 16) for c in ex["codes"]], dtype=np.uint8)
    got = o.fp8_e4m3_decode(codes)
    for c, g in zip(ex["codes"], got):
        if c["value"] == "nan":
            assert np.isnan(g)
        else:
            assert g == c["value"] and math.copysign(1.0, g) == math.copysign(1.0, c["value"]), (c, g)


def pin_fp8_matches_library(o):
    """All 256 codes against PyTorch's float8_e4m3fn conversion (a library
    special case of the same format)."""
    c = np.arange(256, dtype=np.uint8)
    got = o.fp8_e4m3_decode(c)
    ref = torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()
    assert np.all((got == ref) | (np.isnan(got) & np.isnan(ref)))


def pin_fp8_attention(o):
    """FP8 attention: scalar brute force over the decoded codes on a tiny
    case; descales of Q and K act as a factor on the scores, the V descale
    scales O and leaves LSE alone."""
    rng = _rng(33)

    def codes(*shape):  # sign, exponent field 0..8 (|value| < 4), any mantissa
        return (rng.integers(0, 2, shape) * 128 + rng.integers(0, 9, shape) * 8 +
                rng.integers(0, 8, shape)).astype(np.uint8)
    q8, k8, v8 = codes(1, 2, 6, 4), codes(1, 1, 6, 4), codes(1, 1, 6, 4)
    out, lse = o.attention_forward_fp8(q8, k8, v8, 0.5, 0.25, 2.0, True, 0.3)
    dq = torch.from_numpy(q8).view(torch.float8_e4m3fn).double().numpy() * 0.5
    dk = torch.from_numpy(k8).view(torch.float8_e4m3fn).double().numpy() * 0.25
    dv = torch.from_numpy(v8).view(torch.float8_e4m3fn).double().numpy() * 2.0
    for h in range(2):
        for i in range(6):
            w = [math.exp(0.3 * math.fsum(dq[0, h, i, c] * dk[0, 0, j, c] for c in range(4))) for j in range(i + 1)]
            z = math.fsum(w)
            for c in range(4):
                want = math.fsum(wj * dv[0, 0, j, c] for j, wj in enumerate(w)) / z
                assert abs(out[0, h, i, c] - want) <= 1e-12 * max(1.0, abs(want))
            assert abs(lse[0, h, i] - math.log(z)) < 1e-12
    o2, l2 = o.attention_forward_fp8(q8, k8, v8, 1.0, 1.0, 1.0, True, 0.3 * 0.5 * 0.25)
    assert np.max(np.abs(out - 2.0 * o2)) <= 1e-12 * max(1.0, np.max(np.abs(out)))
    assert np.max(np.abs(lse - l2)) < 1e-12


# -- block-sparse masks -----------------------------------------------------------

def _block_case(seed, causal):
    rng = _rng(seed)
    B, Hq, Hkv, N, d = 1, 2, 1, 300, 4   # 3 blocks of 128 (the last one ragged)
    q = _rand(rng, B, Hq, N, d)
    k = _rand(rng, B, Hkv, N, d)
    v = _rand(rng, B, Hkv, N, d)
    bm = rng.random((B, Hq, 3, 3)) < 0.5
    bm[0, 0, 1, :] = False            # query block 1 of head 0 sees nothing
    bm[0, 1] = True
    bm[0, 1, 2, 0] = False            # head 1: the last query block skips the first key block
    return q, k, v, bm


def pin_block_mask_sdpa(o):
    """Block-sparse mask against PyTorch's fp64 SDPA with the mask expanded to
    elements by hand (key j of row i kept iff block (i // 128, j // 128) is
    set), causal or not; rows that see no key give O = 0 and LSE = -inf."""
    for causal in (False, True):
        q, k, v, bm = _block_case(40, causal)
        out, lse = o.attention_forward(q, k, v, causal, 0.5, block_mask=bm)
        N = q.shape[2]
        for h in range(2):
            blk = torch.arange(N) // 128                       # block of each row / key
            allowed = torch.from_numpy(bm[0, h])[blk[:, None], blk[None, :]]
            if causal:
                allowed &= torch.arange(N)[None, :] <= torch.arange(N)[:, None]
            rows = allowed.any(dim=1)
            tq = torch.from_numpy(q[0, h])
            tk = torch.from_numpy(k[0, 0])
            tv = torch.from_numpy(v[0, 0])
            ref = torch.nn.functional.scaled_dot_product_attention(tq[rows][None], tk[None], tv[None],
                                                                    attn_mask=allowed[rows][None], scale=0.5)[0]
            ref_lse = torch.logsumexp((0.5 * (tq @ tk.T)).masked_fill(~allowed, float("-inf")), -1)
            assert np.max(np.abs(out[0, h][rows.numpy()] - ref.numpy())) < 1e-12
            assert np.max(np.abs(lse[0, h][rows.numpy()] - ref_lse[rows].numpy())) < 1e-12
            empty = ~rows.numpy()
            if h == 0:
                assert empty[128:256].all()
            assert np.all(out[0, h][empty] == 0.0) and np.all(np.isneginf(lse[0, h][empty]))


def pin_block_mask_brute(o):
    """Scalar brute force for one row per query block, and an all-ones block
    mask is no mask at all."""
    q, k, v, bm = _block_case(41, True)
    out, lse = o.attention_forward(q, k, v, True, 0.5, block_mask=bm)
    for h in range(2):
        for i in (5, 200, 299):
            keys = [j for j in range(i + 1) if bm[0, h, i // 128, j // 128]]
            if not keys:
                assert np.all(out[0, h, i] == 0.0) and np.isneginf(lse[0, h, i])
                continue
            w = [math.exp(0.5 * math.fsum(q[0, h, i, c] * k[0, 0, j, c] for c in range(4))) for j in keys]
            z = math.fsum(w)
            for c in range(4):
                assert abs(out[0, h, i, c] - math.fsum(wj * v[0, 0, j, c] for wj, j in zip(w, keys)) / z) < 1e-12
            assert abs(lse[0, h, i] - math.log(z)) < 1e-12
    full = np.ones_like(bm)
    o1, l1 = o.attention_forward(q, k, v, True, 0.5, block_mask=full)
    o2, l2 = o.attention_forward(q, k, v, True, 0.5)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# -- additive M ---------------------------------------------------------------------

def pin_bias_sdpa(o):
    """Additive M against PyTorch's fp64 SDPA with a float attn_mask (which is
    added to the scaled scores) and logsumexp of the biased scores, with a
    broadcast over batch and per-head M, causal or not; -inf entries allowed."""
    rng = _rng(50)
    B, Hq, Hkv, N, d = 2, 2, 1, 37, 8
    q = _rand(rng, B, Hq, N, d)
    k = _rand(rng, B, Hkv, N, d)
    v = _rand(rng, B, Hkv, N, d)
    m = rng.standard_normal((1, Hq, N, N)) * 2.0
    m[0, 1, :, :3] = -np.inf                       # head 1: the first three keys masked by M
    m[0, 1, :3, 3:] = 0.0
    for causal in (False, True):
        out, lse = o.attention_forward(q, k, v, causal, 0.3, bias=m)
        for b in range(B):
            for h in range(Hq):
                tm = torch.from_numpy(m[0, h].copy())
                if causal:
                    tm = tm.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
                tq, tk, tv = (torch.from_numpy(x) for x in (q[b, h], k[b, 0], v[b, 0]))
                rows = torch.isfinite(tm).any(dim=1)
                ref = torch.nn.functional.scaled_dot_product_attention(tq[rows][None], tk[None], tv[None],
                                                                        attn_mask=tm[rows][None], scale=0.3)[0]
                ref_lse = torch.logsumexp(0.3 * (tq @ tk.T) + tm, -1)
                assert np.max(np.abs(out[b, h][rows.numpy()] - ref.numpy())) < 1e-12
                assert np.max(np.abs(lse[b, h][rows.numpy()] - ref_lse[rows].numpy())) < 1e-12
                # rows M leaves without a finite score (head 1, rows 0..2 under the causal
                # mask): O = 0, LSE = -inf
                empty = ~rows.numpy()
                if causal and h == 1:
                    assert empty[:3].all()
                assert np.all(out[b, h][empty] == 0.0) and np.all(np.isneginf(lse[b, h][empty]))


def pin_bias_invariants(o):
    """A constant M = c changes nothing but LSE, which moves by c; an M of
    -inf above the diagonal is the causal mask; a scalar brute force."""
    rng = _rng(51)
    q = _rand(rng, 1, 1, 20, 4)
    k = _rand(rng, 1, 1, 20, 4)
    v = _rand(rng, 1, 1, 20, 4)
    o1, l1 = o.attention_forward(q, k, v, False, 0.5)
    o2, l2 = o.attention_forward(q, k, v, False, 0.5, bias=np.full((1, 1, 20, 20), 1.25))
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l2 - l1 - 1.25)) < 1e-12
    upper = np.where(np.triu(np.ones((20, 20)), 1) > 0, -np.inf, 0.0)[None, None]
    o3, l3 = o.attention_forward(q, k, v, False, 0.5, bias=upper)
    o4, l4 = o.attention_forward(q, k, v, True, 0.5)
    assert np.max(np.abs(o3 - o4)) < 1e-12 and np.max(np.abs(l3 - l4)) < 1e-12
    m = rng.standard_normal((1, 1, 20, 20))
    out, lse = o.attention_forward(q, k, v, True, 0.5, bias=m)
    for i in (0, 7, 19):
        w = [math.exp(0.5 * math.fsum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(4)) + m[0, 0, i, j])
             for j in range(i + 1)]
        z = math.fsum(w)
        for c in range(4):
            assert abs(out[0, 0, i, c] - math.fsum(wj * v[0, 0, j, c] for j, wj in enumerate(w)) / z) < 1e-12
        assert abs(lse[0, 0, i] - math.log(z)) < 1e-12


ALL_PINS = [
    pin_rows_sum_to_one,
    pin_constant_v,
    pin_zero_k,
    pin_causal_row0,
    pin_onehot,
    pin_bruteforce,
    pin_torch_sdpa,
    pin_block_table_example,
    pin_paged_equals_contiguous,
    pin_printed_sizes,
    pin_window_closed_form,
    pin_window_sdpa,
    pin_append_example,
    pin_paged_prefill_sdpa,
    pin_paged_prefill_brute,
    pin_chunked_equals_whole,
    pin_fp8_code_points,
    pin_fp8_matches_library,
    pin_fp8_attention,
    pin_block_mask_sdpa,
    pin_block_mask_brute,
    pin_bias_sdpa,
    pin_bias_invariants,
]
