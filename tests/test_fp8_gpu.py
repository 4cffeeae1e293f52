"""FP8 (e4m3) prefill: the CUDA path (through the C ABI) against the fp64
oracle over the decoded, descaled inputs.

Tolerance, from the arithmetic.  The kernel computes S and P V exactly in
fp32 from the e4m3 inputs, except that the weights P' = 2^8 * 2^(s - m) are
rounded to e4m3 before P V (m: the running max, at most 0.5 below the true
one, so P' <= 362 stays in range).  Rounding to nearest e4m3 errs by at most
2^-4 * P' for normal values and 2^-10 below 2^-6, and the row sum l' (fp32,
unrounded) is at least 2^8, so per output element
    |O - O_ref| <= 2^-4 * sum_j P_j |v_j| + 2^-18 * sum_j |v_j|
plus the bf16 rounding of O (2^-8 |O| with margin) and fp32 noise.  The test
checks every element against this bound computed from the oracle (sum_j P_j
|v_j| is the oracle's attention over |V|).  LSE is computed from unrounded
weights, so it keeps the bf16 path's 1e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from attention_flashattention_fwd_04_b200 import api
from attention_flashattention_fwd_04_b200 import workloads as W

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def decoded(codes, descale):
    return oracle.fp8_e4m3_decode(codes.cpu().numpy()) * descale


def check(cfg, causal=None, rows=None, heads=None):
    causal = cfg.causal if causal is None else causal
    (q8, k8, v8), (qd, kd, vd) = W.make_prefill_inputs_fp8(cfg)
    o, lse = api.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), causal, cfg.scale, qd, kd, vd)
    assert api.device_status() == 0
    o, lse = f64(o), f64(lse)
    q, k, v = decoded(q8, qd), decoded(k8, kd), decoded(v8, vd)
    if rows is None:
        ro, rl = oracle.attention_forward(q, k, v, causal, cfg.scale)
        ra, _ = oracle.attention_forward(q, k, np.abs(v), causal, cfg.scale)
        cum = np.cumsum(np.abs(v), axis=2) if causal else np.broadcast_to(np.abs(v).sum(2, keepdims=True), v.shape)
        g = cfg.Hq // cfg.Hkv
        sum_abs = np.repeat(cum, g, axis=1)
        got_o, got_l = o, lse
    else:
        ros, rls, ras, sas, gos, gls = [], [], [], [], [], []
        for (b, h) in heads:
            ro_, rl_ = oracle.attention_rows(q, k, v, causal, cfg.scale, b, h, rows)
            ra_, _ = oracle.attention_rows(q, k, np.abs(v), causal, cfg.scale, b, h, rows)
            hk = oracle.gqa_kv_head(h, cfg.Hq, cfg.Hkv)
            av = np.abs(v[b, hk])
            sa = np.array([av[: r + 1].sum(0) if causal else av.sum(0) for r in rows])
            ros.append(ro_); rls.append(rl_); ras.append(ra_); sas.append(sa)
            gos.append(o[b, h, rows]); gls.append(lse[b, h, rows])
        ro, rl, ra, sum_abs = map(np.stack, (ros, rls, ras, sas))
        got_o, got_l = np.stack(gos), np.stack(gls)
    bound = 2.0 ** -4 * ra + 2.0 ** -18 * sum_abs + 2.0 ** -8 * np.abs(ro) + 1e-5
    err = np.abs(got_o - ro)
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_l))
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), f"O err {err[worst]} > bound {bound[worst]} at {worst}"
    assert np.abs(got_l - rl).max() <= LSE_TOL
    # the bound is a worst case; typical errors are far below it
    assert np.sqrt(np.mean(err ** 2)) <= 0.25 * np.sqrt(np.mean(bound ** 2))
    return err, bound


SMALL = [
    # B, Hq, Hkv, N, causal
    (1, 1, 1, 1, True),
    (1, 2, 2, 64, True),
    (1, 2, 1, 127, False),
    (2, 2, 2, 129, True),
    (1, 4, 2, 255, True),
    (1, 4, 4, 256, False),
    (1, 8, 2, 513, True),
    (1, 2, 2, 1000, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,causal", SMALL)
def test_fp8_small_shapes(B, Hq, Hkv, N, causal):
    check(W.PrefillConfig("t", B, Hq, Hkv, N, 128, causal, seed=500 + N))


def test_fp8_peaked_scores():
    """Scores spread over many units (a K offset per key): most weights are
    far below the max, so the e4m3 subnormal range and the lazy-rescale
    limit are exercised."""
    check(W.PrefillConfig("t", 1, 4, 2, 700, 128, True, seed=77, k_offset_sigma=3.0))


def test_fp8_causal_gqa_full_size_sampled():
    cfg = W.PREFILL_CONFIGS["causal_gqa"]
    check(cfg, rows=[0, 1, 127, 128, 4095, 8190, 8191], heads=[(0, 0), (0, 5), (0, 31)])


def test_fp8_long_causal_full_size_sampled():
    """The benchmarked e4m3 long-context workload at full size (N = 32768, a
    per-key K offset with sigma 2): work items of up to 256 KV tiles, where
    the running max rises past the 0.5 lazy-rescale limit again and again and
    most weights fall deep into the e4m3 subnormal range.  Fixed rows at the
    start, the middle and the end of the sequence plus seeded random rows, on
    the first and last head."""
    cfg = W.PREFILL_CONFIGS["long_causal"]
    rng = np.random.default_rng(5)
    rows = sorted(set([0, 1, 128, 16383, 32766, 32767] + rng.integers(0, cfg.N, 6).tolist()))
    check(cfg, rows=rows, heads=[(0, 0), (0, 7)])


def test_fp8_descales_scale_the_result():
    """Doubling the V descale doubles O (bit for bit in fp32 before the bf16
    rounding, and bf16 doubling is exact); Q/K descales act through the
    scores only."""
    cfg = W.PrefillConfig("t", 1, 2, 2, 300, 128, True, seed=78)
    (q8, k8, v8), (qd, kd, vd) = W.make_prefill_inputs_fp8(cfg)
    q8, k8, v8 = q8.cuda(), k8.cuda(), v8.cuda()
    o1, l1 = api.attn_fwd_fp8(q8, k8, v8, True, cfg.scale, qd, kd, vd)
    o2, l2 = api.attn_fwd_fp8(q8, k8, v8, True, cfg.scale, qd, kd, 2 * vd)
    o3, l3 = api.attn_fwd_fp8(q8, k8, v8, True, cfg.scale * 4, qd / 2, kd / 2, vd)
    torch.cuda.synchronize()
    assert torch.equal(o2, o1 * 2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)
