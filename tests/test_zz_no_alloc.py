"""paged_attn_decode_noalloc: the decode entry point for callers that must not
allocate device memory (a plug-in inside a host program that owns all device
memory, a serving loop that cannot afford a cudaMalloc that may synchronise
the device).  It keeps its split partials in a scratch array built into the
library instead of a caller workspace.

The GPU test calls it twice in a row, once through the C ABI and once
through the Python binding, and compares each result with the regular,
workspace-taking entry point on the same inputs.  Both run the same kernels
with the same split plan, so the results must be identical bit for bit: a
tolerance would hide a partial overwrite of the shared scratch.  This file is
named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

from attention_flashattention_fwd_04_b200 import api
from attention_flashattention_fwd_04_b200 import workloads as W
from attention_flashattention_fwd_04_b200.build import build

FAKE = 1 << 20  # aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build()
    return api.lib()


def _noalloc(lib, ptrs, sizes, scale, stream):
    q, kp, vp, bt, sl, o, lse = ptrs
    S, Hq, Hkv, d, max_pages, num_pages, ps = sizes
    return lib.paged_attn_decode_noalloc(q, kp, vp, bt, sl, ps, o, lse, S, Hq, Hkv, d, max_pages, num_pages,
                                         scale, stream)


def test_noalloc_refuses_oversized_and_null_before_any_cuda_call(lib):
    # 4096 sequences x 64 heads x 2048 pages of 16 tokens needs far more than 48 MiB
    big = (4096, 64, 8, 128, 2048, 1 << 20, 16)
    assert lib.paged_attn_decode_workspace_bytes(4096, 64, 128, 2048, 16) > api.NOALLOC_SCRATCH_BYTES
    assert _noalloc(lib, [FAKE] * 7, big, 0.1, None) == 4
    assert _noalloc(lib, [None] + [FAKE] * 6, (2, 8, 2, 128, 4, 8, 16), 0.1, None) == 1


def test_noalloc_reports_a_bad_argument_as_itself_even_when_oversized(lib):
    # The regular entry point's checks come before the scratch-size check:
    # an oversized call with a bad argument names the argument, not the size.
    S, Hq, d, mp, ps = 4096, 64, 128, 2048, 16
    assert lib.paged_attn_decode_workspace_bytes(S, Hq, d, mp, ps) > api.NOALLOC_SCRATCH_BYTES
    assert _noalloc(lib, [FAKE] * 7, (S, Hq, 7, d, mp, 1 << 20, ps), 0.1, None) == 2     # Hq % Hkv != 0
    assert _noalloc(lib, [FAKE] * 7, (S, Hq, 8, 96, mp, 1 << 20, ps), 0.1, None) == 2    # d not 64 / 128
    assert _noalloc(lib, [FAKE] * 7, (S, Hq, 8, d, mp, 1 << 20, 24), 0.1, None) == 5     # page size
    assert _noalloc(lib, [FAKE + 8] + [FAKE] * 6, (S, Hq, 8, d, mp, 1 << 20, ps), 0.1, None) == 3  # alignment
    assert _noalloc(lib, [FAKE] * 7, (S, Hq, 8, d, mp, 1 << 20, ps), -1.0, None) == 2    # scale


def test_declared_scratch_size_matches_binding():
    with open(api.os.path.join(api.INCLUDE, "attn_b200.h")) as f:
        text = f.read()
    assert "#define ATTN_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)" in text
    assert api.NOALLOC_SCRATCH_BYTES == 48 * 1024 * 1024


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice(lib):
    cfg = W.DECODE_CONFIGS["paged_decode"]  # the bench workload: 33.8 MB of partials
    inp = W.make_decode_inputs(cfg, poison_tail=True)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    S, Hq, d = g["q"].shape
    num_pages, ps, Hkv, _ = g["k_pool"].shape
    max_pages = g["block_table"].shape[1]
    assert api.paged_attn_decode_workspace_bytes(S, Hq, d, max_pages, ps) <= api.NOALLOC_SCRATCH_BYTES

    ref_o, ref_lse = api.paged_attn_decode(g["q"], g["k_pool"], g["v_pool"], g["block_table"], g["seq_lens"],
                                           inp["scale"])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for call in ("c_abi", "binding"):
        o = torch.full_like(g["q"], float("nan"))
        lse = torch.full((S, Hq), float("nan"), device="cuda")
        if call == "c_abi":
            rc = _noalloc(lib, [g["q"].data_ptr(), g["k_pool"].data_ptr(), g["v_pool"].data_ptr(),
                                g["block_table"].data_ptr(), g["seq_lens"].data_ptr(), o.data_ptr(),
                                lse.data_ptr()],
                          (S, Hq, Hkv, d, max_pages, num_pages, ps), inp["scale"], stream)
            assert rc == 0, api.status_string(rc)
        else:
            api.paged_attn_decode_noalloc(g["q"], g["k_pool"], g["v_pool"], g["block_table"], g["seq_lens"],
                                          inp["scale"], out=o, lse=lse)
        bits = ctypes.c_uint(0)
        assert lib.attn_device_status(stream, ctypes.byref(bits)) == 0, bits.value
        assert torch.equal(o, ref_o), (o.float() - ref_o.float()).abs().max().item()
        assert torch.equal(lse, ref_lse), (lse - ref_lse).abs().max().item()
