"""Additive M: the CUDA path (through the C ABI) against the fp64 oracle given
the same bf16 values of M.  Tolerances as the dense kernel (max |O - O_ref|
<= 2e-2, max |LSE - LSE_ref| <= 1e-3); rows whose scores are all -inf must
come back as exact zeros with LSE = -inf."""

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


def run(cfg, bias_view, causal):
    q, k, v = W.make_prefill_inputs(cfg)
    o = torch.full((cfg.B, cfg.Hq, cfg.N, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((cfg.B, cfg.Hq, cfg.N), float("nan"), device="cuda")
    api.attn_fwd_bias(q.cuda(), k.cuda(), v.cuda(), bias_view, causal, cfg.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return (q, k, v), f64(o), f64(lse)


def oracle_bias(bias_view, N):
    b = f64(bias_view)
    return np.broadcast_to(b, b.shape[:2] + (N, N))


def check(o, lse, ro, rl):
    empty = np.isneginf(rl)
    assert np.all(o[empty] == 0.0) and np.all(np.isneginf(lse[empty]))
    live = ~empty
    assert np.all(np.isfinite(o[live])) and np.all(np.isfinite(lse[live]))
    eo = np.abs(o[live] - ro[live])
    el = np.abs(lse[live] - rl[live])
    assert eo.max(initial=0) <= O_TOL, eo.max()
    assert el.max(initial=0) <= LSE_TOL, el.max()


CASES = [
    # B, Hq, Hkv, N, d, causal, bias batch, bias heads, kind, -inf fraction
    (1, 2, 2, 300, 128, False, 1, 2, "normal", 0.0),
    (1, 2, 2, 300, 128, True, 1, 1, "normal", 0.1),
    (2, 4, 2, 777, 64, True, 2, 4, "alibi", 0.0),
    (1, 3, 3, 1000, 128, False, 1, 3, "normal", 0.3),
    (2, 8, 2, 513, 128, True, 1, 8, "alibi", 0.0),
    (1, 2, 1, 129, 64, False, 1, 1, "normal", 0.0),
    (1, 2, 2, 1, 128, False, 1, 1, "normal", 0.0),
    (1, 2, 2, 7, 64, True, 1, 2, "normal", 0.0),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,bb,bh,kind,ninf", CASES)
def test_bias_matches_oracle(B, Hq, Hkv, N, d, causal, bb, bh, kind, ninf):
    cfg = W.PrefillConfig("t", B, Hq, Hkv, N, d, causal, seed=800 + N)
    _, view = W.make_bias_inputs((bb, bh, N, N), kind, seed=N, sigma=2.0, neg_inf_frac=ninf, device="cuda")
    (q, k, v), o, lse = run(cfg, view, causal)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), causal, cfg.scale, bias=oracle_bias(view, N))
    check(o, lse, ro, rl)


def test_fully_masked_rows_give_zeros():
    cfg = W.PrefillConfig("t", 1, 2, 2, 400, 128, True, seed=81)
    buf, view = W.make_bias_inputs((1, 2, 400, 400), "normal", seed=81, device="cpu")
    buf[0, 0, 5] = float("-inf")      # a row with no finite score
    buf[0, 1, 300:390] = float("-inf")  # a run of rows, crossing query tiles
    view = buf.cuda()[..., :400]
    (q, k, v), o, lse = run(cfg, view, True)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), True, cfg.scale, bias=oracle_bias(view, 400))
    assert np.isneginf(rl[0, 0, 5]) and np.isneginf(rl[0, 1, 300:390]).all()
    check(o, lse, ro, rl)


def test_key_padding_row_broadcast():
    """One row of M per batch entry (row stride 0): -inf on padded keys."""
    cfg = W.PrefillConfig("t", 2, 4, 2, 600, 128, False, seed=82)
    buf = torch.zeros((2, 1, 1, 600), dtype=torch.bfloat16)
    buf[0, 0, 0, 450:] = float("-inf")
    buf[1, 0, 0, 123:] = float("-inf")
    view = buf.cuda()
    (q, k, v), o, lse = run(cfg, view, False)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), False, cfg.scale, bias=oracle_bias(view, 600))
    check(o, lse, ro, rl)


def test_padding_contents_are_ignored():
    """The padding after each row's N values is read but never used: NaN or
    +inf there changes nothing, bit for bit."""
    cfg = W.PrefillConfig("t", 1, 2, 2, 301, 128, True, seed=83)
    _, clean = W.make_bias_inputs((1, 2, 301, 301), "normal", seed=83, pad_fill=0.0, device="cuda")
    _, dirty = W.make_bias_inputs((1, 2, 301, 301), "normal", seed=83, pad_fill=float("nan"), device="cuda")
    _, o1, l1 = run(cfg, clean, True)
    _, o2, l2 = run(cfg, dirty, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_constant_shift_moves_only_lse():
    """M = c everywhere: O as without M, LSE shifted by c."""
    cfg = W.PrefillConfig("t", 1, 4, 2, 700, 128, True, seed=84)
    c = 3.0
    view = torch.full((1, 1, 1, 704), c, dtype=torch.bfloat16, device="cuda")[..., :700]
    (q, k, v), o, lse = run(cfg, view, True)
    od, ld = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, cfg.scale)
    assert np.abs(o - f64(od)).max() <= O_TOL
    assert np.abs(lse - (f64(ld) + c)).max() <= LSE_TOL


def test_causal_as_m_equals_causal_flag():
    cfg = W.PrefillConfig("t", 1, 2, 2, 520, 64, False, seed=85)
    tri = torch.triu(torch.full((520, 520), float("-inf")), diagonal=1)
    buf = torch.zeros((1, 1, 520, 520), dtype=torch.bfloat16)
    buf[0, 0] = tri.to(torch.bfloat16)
    (q, k, v), o, lse = run(cfg, buf.cuda(), False)
    od, ld = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, cfg.scale)
    assert np.abs(o - f64(od)).max() <= O_TOL
    assert np.abs(lse - f64(ld)).max() <= LSE_TOL


def test_alibi_full_size_sampled():
    """A per-head linear distance penalty on the 8192-token GQA workload,
    checked on sampled rows."""
    cfg = W.PREFILL_CONFIGS["causal_gqa"]
    N = cfg.N
    _, view = W.make_bias_inputs((1, cfg.Hq, N, N), "alibi", seed=86, device="cuda")
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = api.attn_fwd_bias(q.cuda(), k.cuda(), v.cuda(), view, True, cfg.scale)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    o, lse = o.float().cpu(), lse.cpu()
    qf, kf, vf = q.float(), k.float(), v.float()
    rows = [0, 127, 128, 255, 4000, 8191]
    for h in (0, 9, 31):
        mb = view[:, h:h + 1].float().cpu().numpy()  # the oracle widens only the sampled rows
        ro, rl = oracle.attention_rows(qf, kf, vf, True, cfg.scale, 0, h, rows, bias=mb)
        check(o[0, h, rows].numpy().astype(np.float64), lse[0, h, rows].numpy().astype(np.float64), ro, rl)
