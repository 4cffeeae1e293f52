"""The C-ABI library: it loads, exports every declared symbol, and rejects bad
arguments on the host before touching the GPU.  CPU only (no kernel runs:
every call below fails validation before any CUDA call)."""

import ctypes

import pytest

from attention_flashattention_fwd_04_b200 import api
from attention_flashattention_fwd_04_b200.build import build


@pytest.fixture(scope="module")
def lib():
    build()
    return api.lib()


def test_every_declared_function_is_exported(lib):
    names = api.header_functions()
    assert set(names) == set(api.SIGNATURES), names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.attn_abi_version() == 1
    for code in range(8):
        s = api.status_string(code)
        assert s and s != "unknown status"
    assert api.status_string(99) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned non-null value; never dereferenced


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=16, d=64, causal=1,
         scale=0.125):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(o=None), 1), (dict(lse=None), 1),
    (dict(B=0), 2), (dict(Hq=0), 2), (dict(Hkv=0), 2), (dict(N=0), 2), (dict(N=-5), 2),
    (dict(d=96), 2), (dict(d=256), 2), (dict(Hq=6, Hkv=4), 2), (dict(causal=2), 2),
    (dict(scale=0.0), 2), (dict(scale=-1.0), 2), (dict(scale=float("inf")), 2), (dict(scale=float("nan")), 2),
    (dict(B=1 << 16, Hq=1 << 16, Hkv=1 << 16), 2),
    (dict(q=FAKE + 8), 3), (dict(o=FAKE + 2), 3), (dict(lse=FAKE + 2), 3),
])
def test_attn_fwd_rejects(lib, kw, code):
    assert _fwd(lib, **kw) == code


@pytest.mark.parametrize("wl,code", [(-2, 2), (-100, 2)])
def test_attn_fwd_window_rejects(lib, wl, code):
    assert lib.attn_fwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 16, 64, 1, wl, 0.125, None) == code
    assert lib.attn_fwd_window(None, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 16, 64, 1, 4, 0.125, None) == 1
    assert lib.attn_fwd_window(FAKE + 8, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 16, 64, 1, 4, 0.125, None) == 3


def _dec(lib, q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, ps=16, o=FAKE, lse=FAKE, S=2, Hq=8, Hkv=2,
         d=128, max_pages=4, num_pages=8, scale=0.1, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.paged_attn_decode_workspace_bytes(S, Hq, d, max_pages, ps) if ps > 0 else 0
    return lib.paged_attn_decode(q, kp, vp, bt, sl, ps, o, lse, S, Hq, Hkv, d, max_pages, num_pages,
                                 scale, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(kp=None), 1), (dict(vp=None), 1), (dict(bt=None), 1), (dict(sl=None), 1),
    (dict(o=None), 1), (dict(lse=None), 1),
    (dict(S=0), 2), (dict(Hq=0), 2), (dict(d=80), 2), (dict(Hq=6, Hkv=4), 2), (dict(max_pages=0), 2),
    (dict(num_pages=0), 2), (dict(ps=0), 2), (dict(scale=0.0), 2), (dict(S=70000), 2),
    (dict(ps=8), 5), (dict(ps=24), 5), (dict(ps=512), 5), (dict(Hq=34, Hkv=2), 5),
    (dict(ws=None), 4), (dict(ws_bytes=16), 4),
    (dict(q=FAKE + 4), 3), (dict(ws=FAKE + 8), 3), (dict(bt=FAKE + 2), 3),
])
def test_paged_decode_rejects(lib, kw, code):
    assert _dec(lib, **kw) == code


def test_workspace_formula(lib):
    S, Hq, d, max_pages, ps = 64, 32, 128, 512, 16
    split = lib.paged_attn_decode_split_tokens(S, 8, max_pages, ps)
    assert split % 16 == 0 and split > 0
    splits = -(-max_pages * ps // split)
    rows = S * Hq * splits
    o_bytes = rows * d * 4
    lse_off = (o_bytes + 255) // 256 * 256
    assert lib.paged_attn_decode_workspace_bytes(S, Hq, d, max_pages, ps) == lse_off + rows * 4
    assert lib.paged_attn_decode_workspace_bytes(0, Hq, d, max_pages, ps) == 0
    assert lib.paged_attn_decode_workspace_bytes(S, Hq, 96, max_pages, ps) == 0


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.attn_fwd(q, q, q)


def _decode_tensors(**bad):
    import torch
    S, Hq, Hkv, d, pages, ps, mp = 3, 8, 2, 128, 10, 16, 4
    t = dict(q=torch.zeros(S, Hq, d, dtype=torch.bfloat16),
             k_pool=torch.zeros(pages, ps, Hkv, d, dtype=torch.bfloat16),
             v_pool=torch.zeros(pages, ps, Hkv, d, dtype=torch.bfloat16),
             block_table=torch.zeros(S, mp, dtype=torch.int32),
             seq_lens=torch.ones(S, dtype=torch.int32))
    t.update(bad)
    return t


@pytest.mark.parametrize("wrapper", ["paged_attn_decode", "paged_attn_decode_noalloc", "DecodeGraph"])
@pytest.mark.parametrize("bad, what", [
    ("v_pool", "v_pool shape"), ("block_table", "one row per sequence"), ("seq_lens", "one row per sequence"),
    ("k_pool", "head dim")])
def test_decode_wrappers_refuse_mismatched_shapes_before_any_launch(lib, wrapper, bad, what):
    # The C layer sees only pointers: a short v_pool, block_table or seq_lens
    # would be read past its end.  The binding's shape checks come before its
    # device checks, so they show here on CPU tensors.
    import torch
    good = _decode_tensors()
    shrunk = {"v_pool": good["v_pool"][:-1].contiguous(), "block_table": good["block_table"][:-1].contiguous(),
              "seq_lens": good["seq_lens"][:-1].contiguous(),
              "k_pool": torch.zeros(10, 16, 2, 64, dtype=torch.bfloat16)}[bad]
    t = _decode_tensors(**{bad: shrunk})
    fn = getattr(api, wrapper)
    with pytest.raises(ValueError, match=what):
        fn(t["q"], t["k_pool"], t["v_pool"], t["block_table"], t["seq_lens"], 0.1)
    with pytest.raises(ValueError, match="CUDA tensor"):  # consistent shapes: then the device check
        fn(good["q"], good["k_pool"], good["v_pool"], good["block_table"], good["seq_lens"], 0.1)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="missing"):
        api.lib()


def test_decode_graph_rejects_bad_arguments_on_the_host(lib):
    import ctypes
    h = ctypes.c_void_p(123)
    args = [FAKE] * 5 + [16, FAKE, FAKE, 2, 8, 2, 128, 4, 8, 0.1, FAKE,
                         lib.paged_attn_decode_workspace_bytes(2, 8, 128, 4, 16)]
    assert lib.paged_attn_decode_graph_create(*args, None) == 1          # no handle slot
    bad = list(args)
    bad[11] = 96                                                          # d
    assert lib.paged_attn_decode_graph_create(*bad, ctypes.byref(h)) == 2
    assert h.value is None                                                # cleared on failure
    bad = list(args)
    bad[0] = None
    assert lib.paged_attn_decode_graph_create(*bad, ctypes.byref(h)) == 1
    bad = list(args)
    bad[-1] = 8                                                           # workspace too small
    assert lib.paged_attn_decode_graph_create(*bad, ctypes.byref(h)) == 4
    assert lib.paged_attn_decode_graph_launch(None, None) == 1
    assert lib.paged_attn_decode_graph_destroy(None) == 0


def _app(lib, kn=FAKE, vn=FAKE, kp=FAKE, vp=FAKE, cu=FAKE, sl=FAKE, bt=FAKE, S=2, total_q=5, Hkv=2, d=128,
         ps=16, max_pages=4, num_pages=8):
    return lib.paged_kv_append(kn, vn, kp, vp, cu, sl, bt, S, total_q, Hkv, d, ps, max_pages, num_pages, None)


@pytest.mark.parametrize("kw,code", [
    (dict(kn=None), 1), (dict(vn=None), 1), (dict(kp=None), 1), (dict(vp=None), 1), (dict(cu=None), 1),
    (dict(sl=None), 1), (dict(bt=None), 1),
    (dict(S=0), 2), (dict(total_q=-1), 2), (dict(Hkv=0), 2), (dict(d=96), 2), (dict(max_pages=0), 2),
    (dict(num_pages=0), 2), (dict(ps=0), 2), (dict(num_pages=1 << 28, ps=16), 2),
    (dict(ps=8), 5), (dict(ps=48), 5), (dict(ps=512), 5),
    (dict(kn=FAKE + 8), 3), (dict(kp=FAKE + 2), 3), (dict(cu=FAKE + 2), 3), (dict(bt=FAKE + 1), 3),
])
def test_paged_kv_append_rejects(lib, kw, code):
    assert _app(lib, **kw) == code


def test_paged_kv_append_with_no_new_tokens_is_a_no_op(lib):
    # nothing to copy: no kernel is launched, the new-row pointers are not needed
    assert _app(lib, kn=None, vn=None, total_q=0) == 0


def _pp(lib, q=FAKE, kp=FAKE, vp=FAKE, cu=FAKE, sl=FAKE, bt=FAKE, o=FAKE, lse=FAKE, S=2, total_q=5, Hq=8, Hkv=2,
        d=128, ps=16, max_pages=4, num_pages=8, causal=1, scale=0.1, fn="paged_prefill"):
    if fn == "paged_prefill":
        return lib.paged_prefill(q, kp, vp, cu, sl, bt, o, lse, S, total_q, Hq, Hkv, d, ps, max_pages, num_pages,
                                 causal, scale, None)
    return lib.paged_prefill_append(q, FAKE, FAKE, kp, vp, cu, sl, bt, o, lse, S, total_q, Hq, Hkv, d, ps,
                                    max_pages, num_pages, causal, scale, None)


@pytest.mark.parametrize("fn", ["paged_prefill", "paged_prefill_append"])
@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(lse=None), 1), (dict(kp=None), 1), (dict(bt=None), 1),
    (dict(S=0), 2), (dict(Hq=0), 2), (dict(Hq=6, Hkv=4), 2), (dict(d=80), 2), (dict(causal=2), 2),
    (dict(scale=0.0), 2), (dict(scale=float("nan")), 2), (dict(total_q=1 << 30, Hq=8), 2),
    (dict(ps=24), 5), (dict(S=1025), 5), (dict(total_q=600000, Hq=2, Hkv=2), 5),
    (dict(q=FAKE + 8), 3), (dict(o=FAKE + 4), 3), (dict(lse=FAKE + 2), 3), (dict(sl=FAKE + 2), 3),
])
def test_paged_prefill_rejects(lib, fn, kw, code):
    assert _pp(lib, fn=fn, **kw) == code


def test_paged_prefill_with_no_new_tokens_is_a_no_op(lib):
    assert _pp(lib, total_q=0) == 0


def _fp8(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=16, d=128, causal=1, scale=0.1,
         qd=1.0, kd=1.0, vd=1.0):
    return lib.attn_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, qd, kd, vd, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(v=None), 1), (dict(lse=None), 1),
    (dict(B=0), 2), (dict(N=0), 2), (dict(d=96), 2), (dict(Hq=6, Hkv=4), 2), (dict(causal=3), 2),
    (dict(scale=0.0), 2), (dict(qd=0.0), 2), (dict(kd=-1.0), 2), (dict(vd=float("inf")), 2),
    (dict(qd=1e30, kd=1e30), 2),
    (dict(d=64), 5),
    (dict(q=FAKE + 8), 3), (dict(o=FAKE + 2), 3),
])
def test_attn_fwd_fp8_rejects(lib, kw, code):
    assert _fp8(lib, **kw) == code


def _bs(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=300, d=128, causal=1, scale=0.1,
        mask=FAKE, bs=0, hs=0):
    return lib.attn_fwd_block_sparse(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, mask, bs, hs, None)


@pytest.mark.parametrize("kw,code", [
    (dict(mask=None), 1), (dict(q=None), 1),
    (dict(N=0), 2), (dict(d=96), 2), (dict(causal=2), 2), (dict(scale=0.0), 2), (dict(bs=-1), 2),
    (dict(hs=-5), 2),
    (dict(N=32769), 5),
    (dict(mask=FAKE + 4), 3), (dict(q=FAKE + 8), 3),
])
def test_attn_fwd_block_sparse_rejects(lib, kw, code):
    assert _bs(lib, **kw) == code


def _bias(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=300, d=128, causal=0, scale=0.1,
          bias=FAKE, bs=0, hs=0, rs=304):
    return lib.attn_fwd_bias(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, bias, bs, hs, rs, None)


@pytest.mark.parametrize("kw,code", [
    (dict(bias=None), 1), (dict(o=None), 1),
    (dict(N=0), 2), (dict(d=96), 2), (dict(Hq=3), 2), (dict(causal=2), 2), (dict(scale=float("nan")), 2),
    (dict(bs=-8), 2), (dict(hs=-8), 2), (dict(rs=-8), 2), (dict(rs=296), 2), (dict(rs=300), 2),
    (dict(bias=FAKE + 8), 3), (dict(q=FAKE + 4), 3), (dict(bs=12), 3), (dict(hs=4), 3), (dict(rs=305), 3),
    (dict(lse=FAKE + 2), 3),
])
def test_attn_fwd_bias_rejects(lib, kw, code):
    assert _bias(lib, **kw) == code


def test_pack_block_mask_bit_layout():
    """The binding's packer (marshalling only, runs wherever the tensor is):
    bit j % 64 of word j / 64 set iff key block j is kept, bit 63 included."""
    import numpy as np
    import torch
    from attention_flashattention_fwd_04_b200 import api
    rng = np.random.default_rng(9)
    for nb in (1, 63, 64, 65, 130, 256):
        keep = torch.from_numpy(rng.random((2, 3, 4, nb)) < 0.5)
        keep[0, 0, 0, nb - 1] = True
        words = api.pack_block_mask(keep)
        assert words.dtype == torch.int64 and words.shape == (2, 3, 4, -(-nb // 64))
        u = words.numpy().view(np.uint64)
        for idx in np.ndindex(2, 3, 4):
            for j in range(nb):
                bit = (int(u[idx + (j // 64,)]) >> (j % 64)) & 1
                assert bit == int(keep[idx + (j,)])
            for j in range(nb, 64 * u.shape[-1]):          # bits past the last block stay clear
                assert (int(u[idx + (j // 64,)]) >> (j % 64)) & 1 == 0


def test_bias_span_check():
    """The binding refuses an M whose padded rows would reach past its storage."""
    import torch
    from attention_flashattention_fwd_04_b200 import api
    ok = torch.zeros(1, 2, 5, 16, dtype=torch.bfloat16)[..., :13]          # rows padded to 16
    assert api.bias_span_ok(ok, [0, ok.stride(1), ok.stride(2)])
    tight = torch.zeros(1, 2, 5, 13, dtype=torch.bfloat16)                 # 13-element rows, no padding
    assert not api.bias_span_ok(tight, [0, tight.stride(1), tight.stride(2)])
    row = torch.zeros(2, 1, 1, 601, dtype=torch.bfloat16)                  # key-padding row, 601 not padded
    assert not api.bias_span_ok(row, [row.stride(0), 0, 0])
    row = torch.zeros(2, 1, 1, 608, dtype=torch.bfloat16)[..., :601]
    assert api.bias_span_ok(row, [row.stride(0), 0, 0])
    mult8 = torch.zeros(1, 1, 7, 64, dtype=torch.bfloat16)                 # N a multiple of 8: no padding needed
    assert api.bias_span_ok(mult8, [0, 0, mult8.stride(2)])
    off = torch.zeros(1, 1, 1, 24, dtype=torch.bfloat16)[..., 8:]          # a view ending exactly at the storage end
    assert api.bias_span_ok(off, [0, 0, 0])
