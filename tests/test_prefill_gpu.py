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


def run_gpu(q, k, v, causal, scale, window_left=None):
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal, scale, window_left=window_left)
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
    wl = cfg.window_left if cfg.window_left >= 0 else None
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), cfg.causal, cfg.scale, window_left=wl)
    assert api.device_status() == 0
    o = o.float().cpu()
    lse = lse.cpu()
    q, k, v = q.float(), k.float(), v.float()  # exact; numpy has no bf16
    rng = np.random.default_rng(seed)
    for (b, h) in heads:
        rr = sorted(set(rows) | set(rng.integers(0, cfg.N, 12).tolist()))
        ro, rl = oracle.attention_rows(q, k, v, cfg.causal, cfg.scale, b, h, rr, window_left=wl)
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


def test_long_window_full_size_sampled():
    cfg = W.PREFILL_CONFIGS["long_window"]
    _sampled(cfg, [(0, 0), (0, 5)], [0, 1, 4095, 4096, 4097, 8191, 8192, 20000, 32767], 7)


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


# -- sliding window ----------------------------------------------------------------

WINDOW = [
    # B, Hq, Hkv, N, d, causal, W (query i sees keys i-W .. i, or i-W .. N-1 when not causal)
    (1, 2, 2, 1, 64, True, 0),
    (1, 2, 1, 300, 128, True, 0),
    (1, 2, 2, 300, 128, True, 1),
    (1, 4, 2, 513, 128, True, 127),
    (1, 4, 2, 513, 64, True, 128),
    (2, 2, 2, 700, 128, True, 129),
    (1, 2, 2, 1000, 128, True, 255),
    (1, 8, 2, 1300, 128, True, 500),
    (1, 3, 3, 129, 128, False, 0),
    (1, 2, 2, 1000, 64, False, 300),
    (1, 2, 1, 640, 128, False, 129),
    (1, 2, 2, 777, 128, True, 776),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,wl", WINDOW)
def test_sliding_window_small_shapes(B, Hq, Hkv, N, d, causal, wl):
    cfg = W.PrefillConfig("t", B, Hq, Hkv, N, d, causal, seed=300 + N + wl)
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = run_gpu(q, k, v, causal, cfg.scale, window_left=wl)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), causal, cfg.scale, window_left=wl)
    assert_close(o, lse, ro, rl)


@pytest.mark.parametrize("causal", [True, False])
def test_window_covering_every_key_is_no_window(causal):
    """W >= N - 1 hides nothing: the result is the unwindowed one, bit for bit."""
    cfg = W.PrefillConfig("t", 1, 4, 2, 384, 128, causal, seed=41)
    q, k, v = (t.cuda() for t in W.make_prefill_inputs(cfg))
    a = api.attn_fwd(q, k, v, causal, cfg.scale)
    for wl in (383, 10 ** 6):
        b = api.attn_fwd(q, k, v, causal, cfg.scale, window_left=wl)
        torch.cuda.synchronize()
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("j0,wl", [(77, 0), (127, 128), (200, 129), (383, 255), (5, 600)])
def test_window_edges_are_exact(j0, wl, causal):
    """Key j0 scores ~255 (log2 units) above every other key, so a row that
    sees it returns V[j0] bit for bit and a row that does not cannot.  Row
    j0 + W is the last to see it (the left edge is inclusive); row j0 + W + 1
    is the first that does not; with causal, rows before j0 do not either."""
    N, d = 1024, 128
    q = torch.zeros(1, 2, N, d)
    q[..., 0] = 1.0
    g = torch.Generator().manual_seed(8)
    k = torch.randn(1, 2, N, d, generator=g) * 0.01
    k[..., j0, 0] = 2000.0
    v = torch.randn(1, 2, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    o, lse = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal, scale, window_left=wl)
    assert api.device_status() == 0
    o = o.cpu()
    first_row = j0 if causal else 0
    last_row = min(N - 1, j0 + wl)
    want = v[:, :, j0:j0 + 1, :].expand(1, 2, last_row - first_row + 1, d)
    assert torch.equal(o[:, :, first_row:last_row + 1], want)
    outside = [r for r in (first_row - 1, last_row + 1) if 0 <= r < N]
    for r in outside:
        assert not torch.equal(o[0, 0, r], v[0, 0, j0])
    ro, rl = oracle.attention_rows(f64(q), f64(k), f64(v), causal, scale, 0, 1, outside + [last_row],
                                   window_left=wl)
    assert_close(f64(o[0, 1, outside + [last_row]]), f64(lse[0, 1, outside + [last_row]]), ro, rl)
