"""The CPU oracle against its pins, and planted mistakes against the pins.

CPU only.  The second half copies the oracle module, plants one plausible
mistake in the copy (dropped scale, shifted mask, transposed operand, wrong
GQA mapping, wrong log base, wrong softmax axis, wrong page arithmetic ...)
and checks that at least one pin fails, so the pins are known to have teeth.
"""

from __future__ import annotations

import importlib.util
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as oracle_attention
from tests import oracle_pins

ORACLE_FILE = oracle_attention.__file__


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle_attention)


def test_attention_rows_and_row_chunks_agree():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, 4, 70, 8)) for _ in range(3))
    k, v = k[:, :2], v[:, :2]
    full_o, full_l = oracle.attention_forward(q, k, v, True, 0.3)
    chunk_o, chunk_l = oracle.attention_forward(q, k, v, True, 0.3, row_chunk=16)
    assert np.array_equal(full_o, chunk_o) or np.max(np.abs(full_o - chunk_o)) < 1e-13
    assert np.max(np.abs(full_l - chunk_l)) < 1e-13
    rows = [0, 5, 63, 69]
    ro, rl = oracle.attention_rows(q, k, v, True, 0.3, 0, 3, rows)
    assert np.max(np.abs(ro - full_o[0, 3, rows])) < 1e-13
    assert np.max(np.abs(rl - full_l[0, 3, rows])) < 1e-13


def test_split_merge_identity():
    """The reading behind split-KV decode: attention over a key set equals the
    LSE-weighted merge of attention over a partition of it, with
    lse = log sum_t exp(lse_t) and O = sum_t exp(lse_t - lse) O_t.  This is the
    rescaling identity behind the online softmax ("Five things", second point,
    on the anylearn.cc lesson)."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 16))
    k = rng.standard_normal((100, 16))
    v = rng.standard_normal((100, 16))
    o_full, l_full = oracle.attention_head(q, k, v, 0.25, False)
    bounds = [0, 7, 40, 41, 100]
    parts = [oracle.attention_head(q, k[a:b], v[a:b], 0.25, False) for a, b in zip(bounds, bounds[1:])]
    lses = np.array([p[1][0] for p in parts])
    lse = lses.max() + math.log(np.exp(lses - lses.max()).sum())
    o = sum(np.exp(l - lse) * p[0][0] for p, l in zip(parts, lses))
    assert abs(lse - l_full[0]) < 1e-12
    assert np.max(np.abs(o - o_full[0])) < 1e-12


def test_gqa_mapping_rejects_bad_group():
    with pytest.raises(ValueError):
        oracle.gqa_kv_head(0, 6, 4)


# -- planted mistakes ------------------------------------------------------------

def _fresh_oracle():
    spec = importlib.util.spec_from_file_location("_oracle_mutant", ORACLE_FILE)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_drop_scale(m):
    orig = m.attention_scores
    m.attention_scores = lambda q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None: orig(
        q, k, 1.0, causal, row_offset, window_left, keep, bias)


def _mut_mask_includes_diagonal(m):
    def scores(q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        s = float(scale) * (np.asarray(q, float) @ np.asarray(k, float).T)
        if causal:
            rows = np.arange(row_offset, row_offset + s.shape[0])[:, None]
            cols = np.arange(s.shape[1])[None, :]
            s = np.where(cols >= rows, -np.inf, s)
        return s
    m.attention_scores = scores


def _mut_mask_off_by_one_late(m):
    def scores(q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        s = float(scale) * (np.asarray(q, float) @ np.asarray(k, float).T)
        if causal:
            rows = np.arange(row_offset, row_offset + s.shape[0])[:, None]
            cols = np.arange(s.shape[1])[None, :]
            s = np.where(cols > rows + 1, -np.inf, s)
        return s
    m.attention_scores = scores


def _mut_no_mask(m):
    orig = m.attention_scores
    m.attention_scores = lambda q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None: orig(
        q, k, scale, False, row_offset, window_left, keep, bias)


def _mut_transposed_scores(m):
    def scores(q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        q = np.asarray(q, float)
        k = np.asarray(k, float)
        s = float(scale) * (k @ q.T)
        if s.shape != (q.shape[0], k.shape[0]):
            s = float(scale) * (q @ k.T)[:, ::-1]
        if causal:
            rows = np.arange(row_offset, row_offset + s.shape[0])[:, None]
            cols = np.arange(s.shape[1])[None, :]
            s = np.where(cols > rows, -np.inf, s)
        return s
    m.attention_scores = scores


def _mut_gqa_modulo(m):
    m.gqa_kv_head = lambda h, Hq, Hkv: h % Hkv


def _mut_lse_log2(m):
    orig = m.softmax_with_lse
    def f(s):
        p, lse = orig(s)
        return p, lse / math.log(2.0)
    m.softmax_with_lse = f


def _mut_softmax_wrong_axis(m):
    def f(s):
        s = np.asarray(s, float)
        mx = np.max(s, axis=0, keepdims=True)
        lse = mx + np.log(np.sum(np.exp(s - mx), axis=0, keepdims=True))
        p = np.exp(s - lse)
        p = np.nan_to_num(p)
        return p, np.nan_to_num(np.max(s, axis=-1))
    m.softmax_with_lse = f


def _mut_pv_transposed(m):
    def head(q, k, v, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        s = m.attention_scores(q, k, scale, causal, row_offset, window_left, keep, bias)
        p, lse = m.softmax_with_lse(s)
        v = np.asarray(v, float)
        if p.shape[0] == p.shape[1]:
            return p.T @ v, lse
        return p @ v[::-1], lse
    m.attention_head = head


def _mut_page_slot_swapped(m):
    def gather(pool, row, L, ps):
        pool = np.asarray(pool)
        t = np.arange(int(L))
        return pool[np.asarray(row)[t % ps % len(row)], (t // ps) % ps]
    m.gather_paged_kv = gather


def _mut_page_no_table(m):
    def gather(pool, row, L, ps):
        pool = np.asarray(pool)
        t = np.arange(int(L))
        return pool[t // ps, t % ps]
    m.gather_paged_kv = gather


def _mut_scale_squared(m):
    orig = m.attention_scores
    m.attention_scores = lambda q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None: orig(
        q, k, scale * scale, causal, row_offset, window_left, keep, bias)


def _mut_window_off_by_one(m):
    orig = m.attention_scores
    def scores(q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        w = None if window_left is None or window_left < 0 else window_left + 1
        return orig(q, k, scale, causal, row_offset, w, keep, bias)
    m.attention_scores = scores


def _mut_window_ignored(m):
    orig = m.attention_scores
    m.attention_scores = lambda q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None: orig(
        q, k, scale, causal, row_offset, None, keep, bias)


def _mut_append_shifted(m):
    orig = m.paged_append
    def f(kp, vp, kn, vn, table, cu, lens, ps):
        return orig(kp, vp, kn, vn, table, cu, np.asarray(lens) + 1, ps)  # writes one slot late
    m.paged_append = f


def _mut_append_ignores_table(m):
    def f(kp, vp, kn, vn, table, cu, lens, ps):
        kp, vp = np.array(kp, copy=True), np.array(vp, copy=True)
        for s in range(len(lens)):
            q0, ql = int(cu[s]), int(cu[s + 1]) - int(cu[s])
            ctx = int(lens[s]) - ql
            for i in range(ql):
                t = ctx + i
                kp[t // ps, t % ps] = np.asarray(kn)[q0 + i]
                vp[t // ps, t % ps] = np.asarray(vn)[q0 + i]
        return kp, vp
    m.paged_append = f


def _mut_prefill_no_offset(m):
    orig = m.attention_head
    def head(q, k, v, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        return orig(q, k, v, scale, causal, 0, window_left, keep, bias)
    m.attention_head = head


def _mut_prefill_queries_from_start(m):
    """Takes the new queries as tokens 0..q_len-1 (top-left alignment)."""
    orig = m.paged_prefill
    def f(q, kp, vp, table, cu, lens, ps, scale, causal=True):
        cu = np.asarray(cu)
        ql = np.diff(cu)
        o_, l_ = orig(q, kp, vp, table, cu, ql, ps, scale, causal)
        return o_, l_
    m.paged_prefill = f


def _mut_fp8_bias8(m):
    orig = m.fp8_e4m3_decode
    m.fp8_e4m3_decode = lambda c: orig(c) / 2.0


def _mut_fp8_no_subnormals(m):
    orig = m.fp8_e4m3_decode
    def f(c):
        c = np.asarray(c, dtype=np.uint8)
        v = orig(c)
        e = (c.astype(np.int64) >> 3) & 0xF
        mm = c.astype(np.int64) & 7
        sign = np.where(c & 0x80, -1.0, 1.0)
        return np.where(e == 0, sign * (1 + mm / 8.0) * 2.0 ** -7, v)
    m.fp8_e4m3_decode = f


def _mut_fp8_v_descale_ignored(m):
    orig = m.attention_forward_fp8
    m.attention_forward_fp8 = lambda q8, k8, v8, qd, kd, vd, causal, scale, row_chunk=None: orig(
        q8, k8, v8, qd, kd, 1.0, causal, scale, row_chunk)


def _mut_block_mask_transposed(m):
    orig = m.block_keep
    def f(bm, rows, n_keys, block=128):
        bm = np.asarray(bm, dtype=bool)
        return orig(np.swapaxes(bm, -1, -2), rows, n_keys, block)
    m.block_keep = f


def _mut_block_mask_ignored(m):
    m.block_keep = lambda bm, rows, n_keys, block=128: np.ones((len(np.atleast_1d(rows)), int(n_keys)), dtype=bool)


def _mut_empty_rows_nan(m):
    def f(s):
        s = np.asarray(s, float)
        mx = np.max(s, axis=-1, keepdims=True)
        with np.errstate(all="ignore"):
            lse = mx + np.log(np.sum(np.exp(s - mx), axis=-1, keepdims=True))
            return np.exp(s - lse), lse[..., 0]
    m.softmax_with_lse = f


def _mut_bias_before_scale(m):
    orig = m.attention_scores
    def scores(q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        if bias is None:
            return orig(q, k, scale, causal, row_offset, window_left, keep, None)
        return orig(q, k, scale, causal, row_offset, window_left, keep, np.asarray(bias) * scale)
    m.attention_scores = scores


def _mut_bias_transposed(m):
    orig = m.attention_scores
    def scores(q, k, scale, causal, row_offset=0, window_left=None, keep=None, bias=None):
        b = None if bias is None else (np.asarray(bias).T if np.asarray(bias).shape[0] == np.asarray(bias).shape[1]
                                       else np.asarray(bias)[:, ::-1])
        return orig(q, k, scale, causal, row_offset, window_left, keep, b)
    m.attention_scores = scores


MUTANTS = [
    _mut_drop_scale,
    _mut_scale_squared,
    _mut_mask_includes_diagonal,
    _mut_mask_off_by_one_late,
    _mut_no_mask,
    _mut_transposed_scores,
    _mut_gqa_modulo,
    _mut_lse_log2,
    _mut_softmax_wrong_axis,
    _mut_pv_transposed,
    _mut_page_slot_swapped,
    _mut_page_no_table,
    _mut_window_off_by_one,
    _mut_window_ignored,
    _mut_append_shifted,
    _mut_append_ignores_table,
    _mut_prefill_no_offset,
    _mut_prefill_queries_from_start,
    _mut_fp8_bias8,
    _mut_fp8_no_subnormals,
    _mut_fp8_v_descale_ignored,
    _mut_block_mask_transposed,
    _mut_block_mask_ignored,
    _mut_empty_rows_nan,
    _mut_bias_before_scale,
    _mut_bias_transposed,
]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__)
def test_planted_mistake_is_caught(mutate):
    mod = _fresh_oracle()
    mutate(mod)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except Exception:  # AssertionError or a crash both count as caught
            failed.append(pin.__name__)
    assert failed, f"no pin catches {mutate.__name__}"
