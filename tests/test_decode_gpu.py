"""Paged-KV decode parity: the CUDA split pass + merge (through the C ABI)
against the fp64 oracle, plus exactness probes of the block-table indexing."""

import numpy as np
import pytest
import torch

import oracle
from attention_flashattention_fwd_04_b200 import api
from attention_flashattention_fwd_04_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_TOL = 2e-2
LSE_TOL = 1e-3


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def to_cuda(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run_gpu(inp, workspace=None):
    g = to_cuda(inp)
    o, lse = api.paged_attn_decode(g["q"], g["k_pool"], g["v_pool"], g["block_table"], g["seq_lens"],
                                   inp["scale"], workspace=workspace)
    assert api.device_status() == 0
    return o.cpu(), lse.cpu()


def oracle_decode(inp):
    kp = inp["k_pool"].float().numpy()
    vp = inp["v_pool"].float().numpy()
    return oracle.paged_decode(f64(inp["q"]), kp, vp, inp["block_table"].numpy(),
                               inp["seq_lens"].numpy(), inp["page_size"], inp["scale"])


def assert_close(o, lse, ro, rl):
    o = f64(o)
    lse = f64(lse)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    eo = np.abs(o - ro)
    el = np.abs(lse - rl)
    assert eo.max() <= O_TOL, f"O err {eo.max()} at {np.unravel_index(eo.argmax(), eo.shape)}"
    assert el.max() <= LSE_TOL, f"LSE err {el.max()} at {np.unravel_index(el.argmax(), el.shape)}"


def test_paged_decode_config_full():
    cfg = W.DECODE_CONFIGS["paged_decode"]
    inp = W.make_decode_inputs(cfg)
    o, lse = run_gpu(inp)
    ro, rl = oracle_decode(inp)
    assert_close(o, lse, ro, rl)


CASES = [
    # num_seqs, Hq, Hkv, d, page_size, lens
    (8, 32, 8, 128, 16, [1, 15, 16, 17, 255, 256, 257, 1000]),
    (5, 8, 8, 128, 32, [1, 31, 32, 33, 700]),
    (4, 16, 1, 64, 64, [63, 64, 65, 1500]),
    (3, 12, 4, 128, 16, [513, 2, 4097]),
    (6, 4, 2, 64, 16, [16, 48, 80, 256, 512, 777]),
    (2, 64, 4, 128, 256, [255, 3000]),
]


@pytest.mark.parametrize("S,Hq,Hkv,d,ps,lens", CASES)
def test_small_cases_with_nan_poisoned_tails(S, Hq, Hkv, d, ps, lens):
    cfg = W.DecodeConfig("t", S, Hq, Hkv, d, ps, 1, max(lens), seed=sum(lens) % 997)
    inp = W.make_decode_inputs(cfg, poison_tail=True, seq_lens=lens)
    o, lse = run_gpu(inp)
    ro, rl = oracle_decode(inp)
    assert_close(o, lse, ro, rl)


def test_garbage_workspace_and_table_padding_do_not_matter():
    cfg = W.DecodeConfig("t", 4, 8, 2, 128, 16, 1, 600, seed=21)
    inp = W.make_decode_inputs(cfg, poison_tail=True, seq_lens=[600, 1, 300, 17])
    need = api.paged_attn_decode_workspace_bytes(4, 8, 128, inp["max_pages"], 16)
    ws = torch.full(((need + 3) // 4,), float("nan"), device="cuda")
    table = inp["block_table"].clone()
    table[table < 0] = 123456  # never read: past every sequence's pages
    inp2 = dict(inp, block_table=table)
    o1, l1 = run_gpu(inp, workspace=ws)
    o2, l2 = run_gpu(inp2, workspace=ws)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ro, rl = oracle_decode(inp)
    assert_close(o1, l1, ro, rl)


def test_shared_prefix_pages():
    """Sequences may share physical pages (a common prefix)."""
    cfg = W.DecodeConfig("t", 3, 8, 2, 128, 16, 1, 400, seed=22)
    inp = W.make_decode_inputs(cfg, seq_lens=[400, 390, 64])
    table = inp["block_table"].clone()
    table[1, :20] = table[0, :20]
    table[2, :4] = table[0, :4]
    inp = dict(inp, block_table=table)
    o, lse = run_gpu(inp)
    ro, rl = oracle_decode(inp)
    assert_close(o, lse, ro, rl)
    # sequence 2's 64 tokens are exactly sequence 0's first 64: same keys, same values
    inp3 = dict(inp, q=inp["q"][[0, 0, 0]].clone())
    o3, l3 = run_gpu(inp3)
    ro3, rl3 = oracle_decode(inp3)
    assert_close(o3, l3, ro3, rl3)


@pytest.mark.parametrize("t_star", [0, 15, 16, 17, 255, 256, 257, 511, 512, 999, 1000])
def test_onehot_block_table_indexing_is_exact(t_star):
    """Make logical token t* score ~255 (log2 units) above every other token:
    all other exponentials underflow to 0, so O must equal V[t*] bit for bit.
    Sweeps t* across page and split boundaries and into the last, partial
    page (length 1001, 16-token pages, NaN-poisoned tail slots)."""
    L, Hq, Hkv, d, ps = 1001, 8, 2, 128, 16
    cfg = W.DecodeConfig("t", 2, Hq, Hkv, d, ps, 1, L, seed=23)
    inp = W.make_decode_inputs(cfg, poison_tail=True, seq_lens=[L, 37])
    kp = inp["k_pool"].float()
    table = inp["block_table"]
    live = ~torch.isnan(kp)
    kp = torch.where(live, kp * 0.01, kp)
    page, slot = int(table[0, t_star // ps]), t_star % ps
    kp[page, slot, :, 0] = 2000.0
    q = torch.zeros(2, Hq, d)
    q[..., 0] = 1.0
    inp = dict(inp, k_pool=kp.to(torch.bfloat16), q=q.to(torch.bfloat16))
    o, lse = run_gpu(inp)
    vrow = inp["v_pool"][page, slot]  # [Hkv, d]
    want = vrow.repeat_interleave(Hq // Hkv, dim=0)
    assert torch.equal(o[0], want)
    s_star = 2000.0 * inp["scale"]
    assert torch.allclose(lse[0].double(), torch.full((Hq,), s_star, dtype=torch.float64), atol=1e-3, rtol=0)


def test_invalid_table_entry_is_reported_not_faulted():
    """A table entry outside the pool is a caller error: the kernel keeps
    every copy inside the pool and records the error for attn_device_status."""
    cfg = W.DecodeConfig("t", 2, 8, 2, 128, 16, 1, 100, seed=24)
    inp = W.make_decode_inputs(cfg, seq_lens=[100, 50])
    table = inp["block_table"].clone()
    table[0, 2] = inp["num_pages"] + 7
    g = to_cuda(dict(inp, block_table=table))
    api.paged_attn_decode(g["q"], g["k_pool"], g["v_pool"], g["block_table"], g["seq_lens"], inp["scale"])
    bits = api.device_status()
    assert bits & (1 << 11)
    assert api.device_status() == 0  # reading clears it
    # a zero length is reported the same way and yields O = 0, LSE = -inf
    g2 = to_cuda(dict(inp, seq_lens=torch.tensor([100, 0], dtype=torch.int32)))
    o, lse = api.paged_attn_decode(g2["q"], g2["k_pool"], g2["v_pool"], g2["block_table"], g2["seq_lens"],
                                   inp["scale"])
    assert api.device_status() & (1 << 11)
    assert torch.all(o[1] == 0) and torch.all(torch.isinf(lse[1]))


def test_decode_graph_replays_and_follows_in_place_updates():
    """The captured split + merge gives the eager result, and picks up new
    contents written into the same buffers between launches."""
    cfg = W.DecodeConfig("t", 6, 16, 4, 128, 16, 1, 900, seed=31)
    a = to_cuda(W.make_decode_inputs(cfg, poison_tail=True, seq_lens=[900, 1, 17, 256, 511, 64]))
    graph = api.DecodeGraph(a["q"], a["k_pool"], a["v_pool"], a["block_table"], a["seq_lens"], a["scale"])
    try:
        go, gl = graph.launch()
        eo, el = api.paged_attn_decode(a["q"], a["k_pool"], a["v_pool"], a["block_table"], a["seq_lens"],
                                       a["scale"])
        torch.cuda.synchronize()
        assert torch.equal(go, eo) and torch.equal(gl, el)
        # new step: new query, shorter/longer lengths, permuted pages -- same buffers
        b = W.make_decode_inputs(W.DecodeConfig("t", 6, 16, 4, 128, 16, 1, 900, seed=32),
                                 seq_lens=[3, 880, 100, 17, 16, 700])
        nb = b["block_table"].shape[1]
        a["q"].copy_(b["q"].cuda())
        a["seq_lens"].copy_(b["seq_lens"].cuda())
        a["block_table"].fill_(-1)
        a["block_table"][:, :nb].copy_(b["block_table"].cuda()[:, :a["block_table"].shape[1]])
        npg = b["num_pages"]
        a["k_pool"][:npg].copy_(b["k_pool"].cuda())
        a["v_pool"][:npg].copy_(b["v_pool"].cuda())
        go, gl = graph.launch()
        torch.cuda.synchronize()
        assert api.device_status() == 0
        host = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in a.items()}
        ro, rl = oracle_decode(host)
        assert_close(go.cpu(), gl.cpu(), ro, rl)
    finally:
        graph.close()
