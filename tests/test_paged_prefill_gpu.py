"""Appending to a paged cache and chunked prefill over it: the CUDA path
(through the C ABI) against the fp64 oracle.

The append is pure data movement, so the pools after it must equal the
oracle's bit for bit (compared as raw 16-bit patterns, NaN poison included).
The attention is held to max |O - O_ref| <= 2e-2 and max |LSE - LSE_ref|
<= 1e-3, element by element on small cases and on sampled rows at the full
chunked-prefill workload.
"""

import numpy as np
import pytest
import torch

import oracle
from attention_flashattention_fwd_04_b200 import api
from attention_flashattention_fwd_04_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_TOL = 2e-2
LSE_TOL = 1e-3
ERR_PAGED_TABLE = 1 << 12


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy()


def to_cuda(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) and k not in ("ctx_lens", "q_lens") else v)
            for k, v in inp.items()}


def nan_outputs(g):
    """Outputs pre-filled with NaN: a row the kernel skips cannot pass."""
    o = torch.full_like(g["q"], float("nan"))
    lse = torch.full(g["q"].shape[:2], float("nan"), device=g["q"].device)
    return o, lse


def oracle_append(inp):
    """Pools after the append, as raw bf16 bit patterns (pure indexing)."""
    kp, vp = oracle.paged_append(bits(inp["k_pool"]), bits(inp["v_pool"]), bits(inp["k_new"]), bits(inp["v_new"]),
                                 inp["block_table"].numpy(), inp["cu_seqlens_q"].numpy(), inp["seq_lens"].numpy(),
                                 inp["page_size"])
    return kp, vp


def as_bf16(b):
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16)


def oracle_prefill(inp, kp_bits, vp_bits, causal):
    kp = as_bf16(kp_bits).float().numpy()
    vp = as_bf16(vp_bits).float().numpy()
    return oracle.paged_prefill(f64(inp["q"]), kp, vp, inp["block_table"].numpy(), inp["cu_seqlens_q"].numpy(),
                                inp["seq_lens"].numpy(), inp["page_size"], inp["scale"], causal)


def assert_close(o, lse, ro, rl):
    o = f64(o)
    lse = f64(lse)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    eo = np.abs(o - ro)
    el = np.abs(lse - rl)
    assert eo.max() <= O_TOL, f"O err {eo.max()} at {np.unravel_index(eo.argmax(), eo.shape)}"
    assert el.max() <= LSE_TOL, f"LSE err {el.max()} at {np.unravel_index(el.argmax(), el.shape)}"


CASES = [
    # num_seqs, Hq, Hkv, d, page_size, cached lengths, new-chunk lengths
    (3, 8, 2, 128, 16, [0, 20, 129], [300, 30, 1]),
    (2, 4, 4, 64, 32, [5, 0], [256, 1]),
    (4, 16, 2, 128, 64, [1000, 64, 3, 511], [17, 128, 255, 257]),
    (2, 8, 1, 128, 128, [127, 300], [129, 513]),
    (2, 4, 2, 64, 256, [255, 700], [2, 600]),
    (5, 8, 8, 128, 16, [0, 1, 15, 16, 17], [1, 1, 1, 16, 100]),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S,Hq,Hkv,d,ps,ctx,ql", CASES)
def test_append_then_prefill_matches_the_oracle(S, Hq, Hkv, d, ps, ctx, ql, causal):
    cfg = W.ChunkedConfig("t", S, Hq, Hkv, d, ps, (0, 1), (1, 1), seed=sum(ctx) + sum(ql) + ps)
    inp = W.make_chunked_inputs(cfg, poison=True, ctx_lens=ctx, q_lens=ql, spare_pages=3)
    g = to_cuda(inp)
    o, lse = nan_outputs(g)
    api.paged_prefill_append(g["q"], g["k_new"], g["v_new"], g["k_pool"], g["v_pool"], g["block_table"],
                             g["cu_seqlens_q"], g["seq_lens"], causal=causal, scale=inp["scale"], out=o, lse=lse)
    assert api.device_status() == 0
    kp, vp = oracle_append(inp)
    assert np.array_equal(bits(g["k_pool"]), kp) and np.array_equal(bits(g["v_pool"]), vp)
    ro, rl = oracle_prefill(inp, kp, vp, causal)
    assert_close(o, lse, ro, rl)


@pytest.mark.parametrize("causal", [True, False])
def test_many_sequences_with_empty_chunks(causal):
    """300 sequences (blocks sorted by work on the device, 2 sequences per
    thread in the scan), a third of them with no new tokens."""
    S = 300
    rng = np.random.default_rng(46)
    ctx = rng.integers(0, 400, S).tolist()
    ql = [0 if i % 3 == 0 else int(x) for i, x in enumerate(rng.integers(1, 300, S))]
    cfg = W.ChunkedConfig("t", S, 4, 2, 64, 16, (0, 1), (1, 1), seed=46)
    inp = W.make_chunked_inputs(cfg, poison=True, ctx_lens=ctx, q_lens=ql)
    g = to_cuda(inp)
    o, lse = nan_outputs(g)
    api.paged_prefill_append(g["q"], g["k_new"], g["v_new"], g["k_pool"], g["v_pool"], g["block_table"],
                             g["cu_seqlens_q"], g["seq_lens"], causal=causal, scale=inp["scale"], out=o, lse=lse)
    assert api.device_status() == 0
    kp, vp = oracle_append(inp)
    assert np.array_equal(bits(g["k_pool"]), kp) and np.array_equal(bits(g["v_pool"]), vp)
    ro, rl = oracle_prefill(inp, kp, vp, causal)
    assert_close(o, lse, ro, rl)


def test_one_call_equals_append_then_prefill():
    cfg = W.ChunkedConfig("t", 3, 16, 4, 128, 16, (0, 900), (1, 700), seed=41)
    a = to_cuda(W.make_chunked_inputs(cfg, poison=True))
    b = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in a.items()}
    o1, l1 = api.paged_prefill_append(a["q"], a["k_new"], a["v_new"], a["k_pool"], a["v_pool"], a["block_table"],
                                      a["cu_seqlens_q"], a["seq_lens"], scale=a["scale"])
    api.paged_kv_append(b["k_new"], b["v_new"], b["k_pool"], b["v_pool"], b["block_table"], b["cu_seqlens_q"],
                        b["seq_lens"])
    o2, l2 = api.paged_prefill(b["q"], b["k_pool"], b["v_pool"], b["block_table"], b["cu_seqlens_q"], b["seq_lens"],
                               scale=b["scale"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert np.array_equal(bits(a["k_pool"]), bits(b["k_pool"]))


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("ps", [16, 64, 256])
def test_empty_cache_chunk_is_the_dense_kernel_bit_for_bit(ps, causal):
    """With no cached context the paged prefill computes exactly what
    attn_fwd computes on the same rows laid out contiguously: same tiles,
    same order, so the same bits.  Any mistake in page or row indexing would
    show up here."""
    N, Hq, Hkv, d = 700, 8, 2, 128
    cfg = W.ChunkedConfig("t", 1, Hq, Hkv, d, ps, (0, 0), (N, N), seed=43)
    g = to_cuda(W.make_chunked_inputs(cfg, poison=True, spare_pages=5))
    o, lse = api.paged_prefill_append(g["q"], g["k_new"], g["v_new"], g["k_pool"], g["v_pool"], g["block_table"],
                                      g["cu_seqlens_q"], g["seq_lens"], causal=causal, scale=g["scale"])
    q = g["q"].transpose(0, 1).unsqueeze(0).contiguous()          # [1, Hq, N, d]
    k = g["k_new"].transpose(0, 1).unsqueeze(0).contiguous()      # [1, Hkv, N, d]
    v = g["v_new"].transpose(0, 1).unsqueeze(0).contiguous()
    od, ld = api.attn_fwd(q, k, v, causal, g["scale"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(o, od[0].transpose(0, 1)) and torch.equal(lse, ld[0].transpose(0, 1))


def test_two_chunks_give_the_rows_of_one():
    """Prefill a sequence as one chunk, or as a first chunk and then a second
    over the cache the first one left: the second chunk's rows agree with the
    corresponding rows of the single chunk (to rounding: tiles differ)."""
    L, a, Hq, Hkv, d, ps = 900, 333, 8, 2, 128, 16
    cfg = W.ChunkedConfig("t", 1, Hq, Hkv, d, ps, (0, 0), (L, L), seed=44)
    g = to_cuda(W.make_chunked_inputs(cfg, poison=True))
    whole_o, whole_l = api.paged_prefill_append(g["q"], g["k_new"], g["v_new"], g["k_pool"].clone(),
                                                g["v_pool"].clone(), g["block_table"], g["cu_seqlens_q"],
                                                g["seq_lens"], scale=g["scale"])
    kp, vp = g["k_pool"].clone(), g["v_pool"].clone()
    for lo, hi in ((0, a), (a, L)):
        cu = torch.tensor([0, hi - lo], dtype=torch.int32, device="cuda")
        lens = torch.tensor([hi], dtype=torch.int32, device="cuda")
        o, l = api.paged_prefill_append(g["q"][lo:hi].contiguous(), g["k_new"][lo:hi].contiguous(),
                                        g["v_new"][lo:hi].contiguous(), kp, vp, g["block_table"], cu, lens,
                                        scale=g["scale"])
        assert (o.float() - whole_o[lo:hi].float()).abs().max().item() <= 2e-2
        assert (l - whole_l[lo:hi]).abs().max().item() <= 1e-4
    assert api.device_status() == 0


def test_chunked_prefill_workload_sampled():
    """The bench workload (16 sequences, 19k new tokens over 6k-token
    contexts), run once through the one-call API; appended slots checked bit
    for bit, attention checked on sampled rows against the oracle."""
    cfg = W.CHUNKED_CONFIGS["chunked_prefill"]
    inp = W.make_chunked_inputs(cfg)
    g = to_cuda(inp)
    o, lse = api.paged_prefill_append(g["q"], g["k_new"], g["v_new"], g["k_pool"], g["v_pool"], g["block_table"],
                                      g["cu_seqlens_q"], g["seq_lens"], scale=inp["scale"])
    assert api.device_status() == 0
    kp, vp = g["k_pool"].cpu(), g["v_pool"].cpu()
    o, lse = o.cpu(), lse.cpu()
    ps, table, cu = inp["page_size"], inp["block_table"], inp["cu_seqlens_q"]
    rng = np.random.default_rng(8)
    for s in (0, 7, 15):
        L = int(inp["seq_lens"][s])
        q0, ql = int(cu[s]), int(cu[s + 1] - cu[s])
        ctx = L - ql
        pages = table[s, (torch.arange(ctx, L) // ps)]
        slots = torch.arange(ctx, L) % ps
        assert torch.equal(kp[pages, slots].view(torch.int16), inp["k_new"][q0:q0 + ql].view(torch.int16))
        assert torch.equal(vp[pages, slots].view(torch.int16), inp["v_new"][q0:q0 + ql].view(torch.int16))
        ks = oracle.gather_paged_kv(kp.float().numpy(), table[s].numpy(), L, ps).astype(np.float64)
        vs = oracle.gather_paged_kv(vp.float().numpy(), table[s].numpy(), L, ps).astype(np.float64)
        rows = sorted({0, 1, 127, 128, ql - 1} | set(rng.integers(0, ql, 6).tolist()))
        for h in (0, 13, 31):
            hk = oracle.gqa_kv_head(h, cfg.Hq, cfg.Hkv)
            for r in rows:
                ro, rl = oracle.attention_head(f64(inp["q"][q0 + r, h][None]), ks[:, hk], vs[:, hk], inp["scale"],
                                               True, row_offset=ctx + r)
                assert_close(o[q0 + r, h][None], lse[q0 + r, h][None], ro, rl)


def test_bad_table_entry_and_bad_lengths_are_reported_not_faulted():
    cfg = W.ChunkedConfig("t", 2, 8, 2, 128, 16, (0, 0), (1, 1), seed=45)
    inp = W.make_chunked_inputs(cfg, ctx_lens=[100, 40], q_lens=[50, 10])
    table = inp["block_table"].clone()
    table[0, 7] = inp["num_pages"] + 5          # a page of sequence 0's new chunk
    g = to_cuda(dict(inp, block_table=table))
    before = g["k_pool"].clone()
    api.paged_prefill_append(g["q"], g["k_new"], g["v_new"], g["k_pool"], g["v_pool"], g["block_table"],
                             g["cu_seqlens_q"], g["seq_lens"], scale=inp["scale"])
    assert api.device_status() & ERR_PAGED_TABLE
    # sequence 1 is unaffected and was appended normally
    kp_bits, _ = oracle_append(dict(inp))
    pages = inp["block_table"][1, torch.arange(40, 50) // 16]
    slots = torch.arange(40, 50) % 16
    assert np.array_equal(bits(g["k_pool"])[pages.numpy(), slots.numpy()], kp_bits[pages.numpy(), slots.numpy()])
    # a chunk longer than its sequence is refused on the device, nothing written
    g2 = to_cuda(dict(inp, seq_lens=torch.tensor([30, 50], dtype=torch.int32)))
    k0 = g2["k_pool"].clone()
    api.paged_kv_append(g2["k_new"], g2["v_new"], g2["k_pool"], g2["v_pool"], g2["block_table"],
                        g2["cu_seqlens_q"], g2["seq_lens"])
    assert api.device_status() & ERR_PAGED_TABLE
    changed = (bits(g2["k_pool"]) != bits(k0)).any(axis=(2, 3))
    assert changed.sum() == 10                   # only sequence 1's ten new tokens
    del before
