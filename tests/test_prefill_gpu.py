"""Prefill parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation): max |O - O_ref| <= 2e-2,
max |LSE - LSE_ref| <= 1e-3.  Small shapes are compared element by element;
the full-size workloads run in the launch configuration the bench times and
are compared on sampled rows, each computed exactly by the oracle.
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


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_gpu(q, k, v, causal, scale):
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal, scale)
    assert api.device_status() == 0
    return f64(o), f64(lse)


def assert_close(o, lse, ro, rl):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    err_o = np.abs(o - ro)
    err_l = np.abs(lse - rl)
    assert err_o.max() <= O_TOL, f"O err {err_o.max()} at {np.unravel_index(err_o.argmax(), err_o.shape)}"
    assert err_l.max() <= LSE_TOL, f"LSE err {err_l.max()} at {np.unravel_index(err_l.argmax(), err_l.shape)}"


SMALL = [
    # B, Hq, Hkv, N, d, causal
    (1, 1, 1, 1, 64, True),
    (1, 1, 1, 2, 128, False),
    (1, 2, 2, 64, 64, True),
    (1, 2, 1, 127, 128, True),
    (1, 2, 2, 128, 128, False),
    (2, 2, 2, 129, 64, True),
    (1, 4, 2, 255, 128, True),
    (1, 4, 4, 256, 64, False),
    (2, 4, 1, 300, 128, False),
    (1, 8, 2, 513, 128, True),
    (1, 3, 3, 700, 64, True),
    (1, 2, 2, 1000, 128, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", SMALL)
def test_small_shapes(B, Hq, Hkv, N, d, causal):
    cfg = W.PrefillConfig("t", B, Hq, Hkv, N, d, causal, seed=100 + N + d)
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = run_gpu(q, k, v, causal, cfg.scale)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), causal, cfg.scale)
    assert_close(o, lse, ro, rl)


def test_tiny_config_full():
    cfg = W.PREFILL_CONFIGS["tiny"]
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = run_gpu(q, k, v, cfg.causal, cfg.scale)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), cfg.causal, cfg.scale)
    assert_close(o, lse, ro, rl)


def _sampled(cfg, heads, rows, seed):
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), cfg.causal, cfg.scale)
    assert api.device_status() == 0
    o = o.float().cpu()
    lse = lse.cpu()
    q, k, v = q.float(), k.float(), v.float()  # exact; numpy has no bf16
    rng = np.random.default_rng(seed)
    for (b, h) in heads:
        rr = sorted(set(rows) | set(rng.integers(0, cfg.N, 12).tolist()))
        ro, rl = oracle.attention_rows(q, k, v, cfg.causal, cfg.scale, b, h, rr)
        got_o = o[b, h, rr].numpy().astype(np.float64)
        got_l = lse[b, h, rr].numpy().astype(np.float64)
        assert_close(got_o, got_l, ro, rl)


def test_causal_mha_full_size_sampled():
    cfg = W.PREFILL_CONFIGS["causal_mha"]
    _sampled(cfg, [(0, 0), (1, 7), (3, 15)], [0, 1, 127, 128, 129, 1023, 2047], 2)


def test_causal_gqa_full_size_sampled():
    cfg = W.PREFILL_CONFIGS["causal_gqa"]
    _sampled(cfg, [(0, 0), (0, 3), (0, 4), (0, 31)], [0, 1, 127, 128, 4095, 8190, 8191], 3)


def test_long_causal_full_size_sampled():
    cfg = W.PREFILL_CONFIGS["long_causal"]
    _sampled(cfg, [(0, 0), (0, 7)], [0, 1, 128, 16383, 32766, 32767], 5)


def test_causal_mha_whole_heads():
    """Two whole heads of the bench workload, every row."""
    cfg = W.PREFILL_CONFIGS["causal_mha"]
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, cfg.scale)
    assert api.device_status() == 0
    for b, h in [(0, 5), (2, 11)]:
        ro, rl = oracle.attention_forward(f64(q[b:b + 1, h:h + 1]), f64(k[b:b + 1, h:h + 1]),
                                          f64(v[b:b + 1, h:h + 1]), True, cfg.scale)
        assert_close(f64(o[b:b + 1, h:h + 1]), f64(lse[b:b + 1, h:h + 1]), ro, rl)


def test_onehot_rows_are_exact():
    """A key scoring ~255 (log2 units) above all others takes all the weight:
    every other exponential underflows to 0, so each output row equals that
    value row bit for bit (non-causal, key index 77 visible to every row)."""
    N, d = 256, 128
    q = torch.zeros(1, 2, N, d)
    q[..., 0] = 1.0
    g = torch.Generator().manual_seed(7)
    k = torch.randn(1, 2, N, d, generator=g) * 0.01
    k[..., 77, 0] = 2000.0
    v = torch.randn(1, 2, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), False, scale)
    assert torch.equal(o.cpu(), v[:, :, 77:78, :].expand(1, 2, N, d))


def test_output_does_not_depend_on_launch_history():
    cfg = W.PrefillConfig("t", 1, 4, 2, 640, 128, True, 9)
    q, k, v = (t.cuda() for t in W.make_prefill_inputs(cfg))
    a = api.attn_fwd(q, k, v, True, cfg.scale)
    b = api.attn_fwd(q, k, v, True, cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_memory_does_not_scale_with_n_squared():
    """The pages' diagnostic for a lost fused path: memory that grows with
    the square of the sequence length.  With outputs preallocated, a call
    must not take any device memory at N=4096 or N=8192."""
    free = []
    for N in (4096, 8192):
        cfg = W.PrefillConfig("t", 1, 8, 8, N, 128, True, 11)
        q, k, v = (t.cuda() for t in W.make_prefill_inputs(cfg))
        o = torch.empty_like(q)
        lse = torch.empty(1, 8, N, device="cuda")
        torch.cuda.synchronize()
        before = torch.cuda.mem_get_info()[0]
        api.attn_fwd(q, k, v, True, cfg.scale, out=o, lse=lse)
        torch.cuda.synchronize()
        free.append(before - torch.cuda.mem_get_info()[0])
    assert max(free) <= 2 * 1024 * 1024, free
