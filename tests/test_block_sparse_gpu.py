"""Block-sparse prefill: the CUDA path (through the C ABI) against the fp64
oracle with the same 128 x 128 block mask.  Tolerances as the dense kernel
(max |O - O_ref| <= 2e-2, max |LSE - LSE_ref| <= 1e-3); rows that see no key
must come back as exact zeros with LSE = -inf."""

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


def run(cfg, keep, causal):
    q, k, v = W.make_prefill_inputs(cfg)
    o = torch.full((cfg.B, cfg.Hq, cfg.N, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((cfg.B, cfg.Hq, cfg.N), float("nan"), device="cuda")
    api.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), torch.as_tensor(keep).cuda(), causal, cfg.scale,
                              out=o, lse=lse)
    assert api.device_status() == 0
    return (q, k, v), f64(o), f64(lse)


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
    # B, Hq, Hkv, N, d, causal, density
    (1, 2, 2, 300, 128, True, 0.5),
    (1, 4, 2, 640, 128, False, 0.4),
    (2, 2, 1, 777, 64, True, 0.6),
    (1, 3, 3, 1000, 128, True, 0.25),
    (1, 2, 2, 129, 64, False, 0.5),
    (1, 8, 2, 1300, 128, True, 0.8),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,density", CASES)
def test_random_block_masks(B, Hq, Hkv, N, d, causal, density):
    cfg = W.PrefillConfig("t", B, Hq, Hkv, N, d, causal, seed=700 + N)
    nb = -(-N // 128)
    rng = np.random.default_rng(N)
    keep = rng.random((B, Hq, nb, nb)) < density
    keep[0, 0, min(1, nb - 1), :] = False          # a query block that sees nothing
    (q, k, v), o, lse = run(cfg, keep, causal)
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), causal, cfg.scale, block_mask=keep)
    check(o, lse, ro, rl)


def test_all_ones_is_the_dense_kernel_bit_for_bit():
    cfg = W.PrefillConfig("t", 1, 4, 2, 700, 128, True, seed=71)
    keep = np.ones((1, 1, 6, 6), dtype=bool)       # broadcast over batch and heads
    (q, k, v), o, lse = run(cfg, keep, True)
    od, ld = api.attn_fwd(q.cuda(), k.cuda(), v.cuda(), True, cfg.scale)
    assert np.array_equal(o, f64(od)) and np.array_equal(lse, f64(ld))


def test_all_zeros_gives_zero_rows():
    cfg = W.PrefillConfig("t", 1, 2, 2, 300, 64, False, seed=72)
    (q, k, v), o, lse = run(cfg, np.zeros((1, 2, 3, 3), dtype=bool), False)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))


def test_longformer_pattern_full_size_sampled():
    """Sliding-window blocks (the diagonal block and the one before it) plus
    a global first key block, on the 8192-token GQA workload."""
    cfg = W.PREFILL_CONFIGS["causal_gqa"]
    nb = cfg.N // 128
    keep = np.zeros((1, 1, nb, nb), dtype=bool)
    for i in range(nb):
        keep[0, 0, i, max(0, i - 1): i + 1] = True
        keep[0, 0, i, 0] = True
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = api.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(keep).cuda(), True,
                                       cfg.scale)
    assert api.device_status() == 0
    o, lse = o.float().cpu(), lse.cpu()
    full = np.broadcast_to(keep, (1, cfg.Hq, nb, nb))
    qf, kf, vf = q.float(), k.float(), v.float()
    for h in (0, 9, 31):
        rows = [0, 127, 128, 255, 4000, 8191]
        ro, rl = oracle.attention_rows(qf, kf, vf, True, cfg.scale, 0, h, rows, block_mask=full)
        check(o[0, h, rows].numpy().astype(np.float64), lse[0, h, rows].numpy().astype(np.float64), ro, rl)


def test_packed_mask_equals_boolean_mask():
    """The binding takes the mask already packed (int64 words, packed once by
    the caller) as well as boolean: the same words reach the kernel."""
    cfg = W.PrefillConfig("t", 2, 4, 2, 900, 128, True, seed=73)
    nb = -(-cfg.N // 128)
    keep = torch.from_numpy(np.random.default_rng(5).random((2, 1, nb, nb)) < 0.5)
    q, k, v = (t.cuda() for t in W.make_prefill_inputs(cfg))
    o1, l1 = api.attn_fwd_block_sparse(q, k, v, keep.cuda(), True, cfg.scale)
    o2, l2 = api.attn_fwd_block_sparse(q, k, v, api.pack_block_mask(keep).cuda(), True, cfg.scale)
    assert api.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("N,causal", [(32768, True), (20000, False)])
def test_multi_word_masks_sampled(N, causal):
    """More than 64 key blocks: the mask rows span several uint64 words (four
    at N = 32768, the limit), so every lane of the tile lister and every word
    of each set is used.  Sampled rows against the oracle."""
    cfg = W.PrefillConfig("t", 1, 2, 1, N, 128, causal, seed=74)
    nb = -(-N // 128)
    rng = np.random.default_rng(N)
    keep = rng.random((1, 2, nb, nb)) < 0.15
    keep[0, 0, :, nb - 1] = True                   # the last key block (top bits of the last word)
    keep[0, 1, :, 63:65] = True                    # blocks on both sides of the first word boundary
    keep[0, 1, 100, :] = False                     # a query block that sees nothing
    q, k, v = W.make_prefill_inputs(cfg)
    o, lse = api.attn_fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(keep).cuda(), causal,
                                       cfg.scale)
    assert api.device_status() == 0
    o, lse = o.float().cpu(), lse.cpu()
    rows = [0, 127, 128, 8191, 8192, 100 * 128 + 5, 16384, N - 129, N - 1]
    for h in (0, 1):
        ro, rl = oracle.attention_rows(q.float(), k.float(), v.float(), causal, cfg.scale, 0, h, rows,
                                       block_mask=keep[0:1])
        check(o[0, h, rows].numpy().astype(np.float64), lse[0, h, rows].numpy().astype(np.float64), ro, rl)
