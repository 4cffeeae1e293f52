"""Seeded input generators: determinism, shapes, block-table structure (CPU)."""

import math

import torch

from attention_flashattention_fwd_04_b200 import workloads as W


def test_prefill_inputs_are_seeded_and_shaped():
    cfg = W.PREFILL_CONFIGS["tiny"]
    a = W.make_prefill_inputs(cfg)
    b = W.make_prefill_inputs(cfg)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    assert a[0].shape == (1, 2, 128, 64)
    assert a[1].shape == (1, 2, 128, 64)


def test_scale_is_fp32_rounded_inverse_sqrt():
    for cfg in W.PREFILL_CONFIGS.values():
        s = cfg.scale
        assert s == float(torch.tensor(1 / math.sqrt(cfg.d), dtype=torch.float32))
    assert W.PREFILL_CONFIGS["tiny"].scale == 0.125


def test_gqa_config_shapes_and_value_scale():
    cfg = W.PrefillConfig("t", 1, 8, 2, 256, 128, True, 3, value_scale=0.5)
    q, k, v = W.make_prefill_inputs(cfg)
    assert q.shape == (1, 8, 256, 128) and k.shape == (1, 2, 256, 128)
    assert 0.4 < q.float().std().item() < 0.6


def test_k_offset_is_per_position_and_shared_across_heads():
    cfg = W.PrefillConfig("t", 1, 2, 2, 512, 128, True, 5, k_offset_sigma=2.0)
    q, k, v = W.make_prefill_inputs(cfg)
    row_means = k.float().mean(dim=-1)  # [1, 2, N]
    # the offset dominates the row mean and is the same for both heads
    assert torch.corrcoef(torch.stack([row_means[0, 0], row_means[0, 1]]))[0, 1] > 0.95
    assert 1.5 < row_means[0, 0].std().item() < 2.5


def test_decode_block_table_is_a_permutation_with_padding():
    cfg = W.DecodeConfig("t", 7, 8, 2, 64, 16, 1, 300, 9)
    inp = W.make_decode_inputs(cfg)
    L = inp["seq_lens"].long()
    table = inp["block_table"]
    ps = inp["page_size"]
    pages = (L + ps - 1) // ps
    assert int(pages.sum()) == inp["num_pages"]
    assert inp["k_pool"].shape == (inp["num_pages"], ps, 2, 64)
    ids = []
    for s in range(cfg.num_seqs):
        n = int(pages[s])
        ids += table[s, :n].tolist()
        assert bool((table[s, n:] == -1).all())
    assert sorted(ids) == list(range(inp["num_pages"]))
    assert int(L.min()) >= 1 and int(L.max()) <= 300
    again = W.make_decode_inputs(cfg)
    assert torch.equal(again["block_table"], table)
    assert torch.equal(again["k_pool"], inp["k_pool"])


def test_decode_poison_fills_only_unused_tail_slots():
    cfg = W.DecodeConfig("t", 4, 4, 2, 32, 16, 1, 100, 10)
    inp = W.make_decode_inputs(cfg, poison_tail=True, seq_lens=[1, 16, 17, 33])
    kp = inp["k_pool"].float()
    table = inp["block_table"]
    for s, L in enumerate([1, 16, 17, 33]):
        n = -(-L // 16)
        for p in range(n):
            page = kp[int(table[s, p])]
            for slot in range(16):
                t = p * 16 + slot
                assert bool(torch.isnan(page[slot]).all()) == (t >= L)


def test_paged_decode_default_config_sizes():
    cfg = W.DECODE_CONFIGS["paged_decode"]
    assert cfg.table_width == 512
    g = torch.Generator().manual_seed(cfg.seed)
    L = torch.randint(cfg.min_len, cfg.max_len + 1, (cfg.num_seqs,), generator=g)
    assert 512 <= int(L.min()) and int(L.max()) <= 8192
    b = W.decode_kv_bytes(L, cfg.Hkv, cfg.d, cfg.Hq)
    assert b > float(L.sum()) * 4096


def test_flop_convention():
    c2 = W.PREFILL_CONFIGS["causal_mha"]
    assert abs(W.prefill_flops(c2) - 68.72e9) / 68.72e9 < 1e-3
    c3 = W.PREFILL_CONFIGS["causal_gqa"]
    assert abs(W.prefill_flops(c3) - 549.76e9) / 549.76e9 < 1e-3


def test_visible_pairs_match_the_oracle_mask():
    """The windowed FLOP count equals the number of finite scores the oracle's
    mask leaves, on small shapes (including windows past either end)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(0)
    for N in (1, 5, 130, 257):
        q = rng.standard_normal((N, 4))
        for causal in (True, False):
            for wl in (-1, 0, 1, 3, 127, 128, N - 1, N + 5):
                s = oracle.attention_scores(q, q, 1.0, causal, 0, None if wl < 0 else wl)
                assert W.visible_pairs(N, causal, wl) == int(np.isfinite(s).sum()), (N, causal, wl)


def test_window_flops():
    lw = W.PREFILL_CONFIGS["long_window"]
    N, Wl = lw.N, lw.window_left
    pairs = (Wl + 1) * (Wl + 2) // 2 + (N - Wl - 1) * (Wl + 1)  # ramp, then full windows
    assert W.prefill_flops(lw) == 4.0 * lw.B * lw.Hq * lw.d * pairs


def test_bias_inputs_layout_and_values():
    buf, view = W.make_bias_inputs((1, 4, 5, 13), "alibi", pad_fill=float("nan"))
    assert buf.shape == (1, 4, 5, 16) and view.shape == (1, 4, 5, 13)
    assert view.stride(2) == 16 and view.stride(3) == 1
    assert torch.isnan(buf[..., 13:]).all()
    # head 0 of 4: slope 2^-2; entry (i, j) = -|i - j| / 4
    assert float(view[0, 0, 4, 1]) == -0.75 and float(view[0, 0, 2, 2]) == 0.0
    _, v2 = W.make_bias_inputs((2, 1, 3, 20), "normal", seed=3, neg_inf_frac=0.5)
    frac = torch.isneginf(v2.float()).float().mean().item()
    assert 0.2 < frac < 0.8


def test_block_sparse_pairs_brute_force():
    """Visible pairs under a block mask (and causality) against a count over
    the expanded element mask."""
    import numpy as np
    rng = np.random.default_rng(3)
    for N, causal in ((300, True), (300, False), (129, True), (1000, True)):
        nb = -(-N // 128)
        keep = rng.random((nb, nb)) < 0.5
        elem = keep[np.arange(N)[:, None] // 128, np.arange(N)[None, :] // 128]
        if causal:
            elem &= np.arange(N)[None, :] <= np.arange(N)[:, None]
        assert W.block_sparse_pairs(keep, N, causal) == int(elem.sum())
    # all ones and causal: every pair with j <= i
    assert W.block_sparse_pairs(np.ones((3, 3), bool), 300, True) == 300 * 301 // 2


def test_longformer_keep_pattern():
    keep = W.longformer_keep(5)
    assert keep.dtype == torch.bool and keep.shape == (5, 5)
    assert keep[:, 0].all()                                   # global first block
    assert all(keep[i, i] and keep[i, i - 1] for i in range(1, 5))
    assert int(keep.sum()) == 1 + 2 + 3 + 3 + 3               # row 0: {0}; row 1: {0,1}; rows 2+: {0,i-1,i}


def test_alibi_rows_match_the_full_generator():
    buf, view = W.make_bias_inputs((1, 3, 40, 37), "alibi")
    for h in range(3):
        assert torch.equal(W.alibi_rows(3, h, 5, 40, 37), view[0, h, 5:])


def test_bench_mask_work_accounting():
    """FLOPs and bytes bench.py credits the mask workloads with."""
    import bench
    c = W.PREFILL_CONFIGS["causal_gqa"]
    f, b = bench.mask_work("longformer", c)
    assert b == 0.0
    assert f == 4.0 * c.d * W.block_sparse_pairs(W.longformer_keep(c.N // 128), c.N, True) * c.B * c.Hq
    f, b = bench.mask_work("alibi", c)
    pairs = c.N * (c.N + 1) // 2
    assert f == W.prefill_flops(c) == 4.0 * c.d * c.N * c.N / 2 * c.Hq   # the dense lines' convention
    m_bytes = 2.0 * pairs * c.Hq                                  # every head its own M
    qkvo = 2.0 * c.N * c.d * (2 * c.Hq + 2 * c.Hkv) + 4.0 * c.Hq * c.N
    assert b == m_bytes + qkvo
    # the per-head M makes this prefill HBM-bound at the measured peaks
    peaks = bench.load_peaks()
    assert b / (peaks["hbm_gbs"] * 1e9) > f / (peaks["bf16_tflops"] * 1e12)


def test_traffic_records_follow_each_kernels_sources(tmp_path, monkeypatch):
    """A traffic record counts only while its kernel's own sources are
    unchanged: records whose hash does not match are dropped."""
    import bench
    good = bench.kernel_source_hash("decode_split_kernel")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.txt").write_text(
        "# comment\n"
        f"kernel=decode_split_kernel bench=paged_decode sha={good} dram_bytes_per_launch=123 read=100 write=23\n"
        "kernel=prefill_fwd_kernel bench=causal_mha sha=0000000000000000 dram_bytes_per_launch=5 read=4 write=1\n"
        f"kernel=unknown_kernel bench=x sha={good} dram_bytes_per_launch=7 read=7 write=0\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda k=None: good if k == "decode_split_kernel" else "ffffffffffffffff")
    t = bench.load_traffic()
    assert t == {("decode_split_kernel", "paged_decode"): 123.0}
    # every kernel the bench reports has a source set, and every listed file exists
    for k, files in bench.KERNEL_SOURCE_SETS.items():
        assert set(files) <= set(bench.KERNEL_SOURCES)


def test_clock_window_picks_the_samples_of_a_region():
    """bench.ClockSampler.window: the samples inside the host-time window plus
    the nearest one on each side if it lies within 20 ms; reasons from those
    samples only."""
    import bench
    s = object.__new__(bench.ClockSampler)
    s.max_mhz = 1965
    ms = 1e-3
    s.samples = [(0.0, 1000, 0x1), (10 * ms, 1965, 0x0), (11 * ms, 1965, 0x4), (12 * ms, 1800, 0x0),
                 (30 * ms, 1965, 0x0), (900 * ms, 500, 0x40)]
    w = s.window(10.5 * ms, 12.5 * ms)
    assert w["samples"] == 2 and w["samples_with_neighbours"] == 4   # 10 ms and 30 ms are neighbours
    assert w["sm_mhz"] == 1965 and w["reasons"] == ["sw_power_cap"]  # 0x40 at 900 ms is too far away
    short = s.window(11.2 * ms, 11.3 * ms)                            # shorter than one sample period
    assert short["samples"] == 0 and short["samples_with_neighbours"] == 2 and short["sm_mhz"] == 1882.5
    assert s.window(500 * ms, 600 * ms)["sm_mhz"] is None              # nothing near
