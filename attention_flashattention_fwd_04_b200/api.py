"""ctypes binding over the C ABI in ``include/attn_b200.h``.

Argument marshalling only: every step of the attention runs in the CUDA
kernels of ``libattn_b200.so``.  PyTorch supplies device memory (outputs,
workspace) and the current stream.  There is no CPU or PyTorch fallback: if
the library is missing or a call fails, this module raises.
"""

from __future__ import annotations

import ctypes
import functools
import os
import re

import torch

from .build import INCLUDE, LIB_PATH

ATTN_OK = 0
_STATUS_NAMES = {
    0: "ATTN_OK",
    1: "ATTN_ERR_NULL",
    2: "ATTN_ERR_SHAPE",
    3: "ATTN_ERR_ALIGN",
    4: "ATTN_ERR_WORKSPACE",
    5: "ATTN_ERR_UNSUPPORTED",
    6: "ATTN_ERR_LAUNCH",
    7: "ATTN_ERR_DEVICE",
}

_c_p = ctypes.c_void_p
_c_i = ctypes.c_int
_c_f = ctypes.c_float
_c_sz = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/attn_b200.h
SIGNATURES = {
    "attn_abi_version": (_c_i, []),
    "attn_status_string": (ctypes.c_char_p, [_c_i]),
    "attn_last_cuda_error": (_c_i, []),
    "attn_fwd": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p]),
    "attn_fwd_window": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f,
                               _c_p]),
    "paged_attn_decode_split_tokens": (_c_i, [_c_i, _c_i, _c_i, _c_i]),
    "paged_attn_decode_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i]),
    "paged_attn_decode": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i,
                                 _c_i, _c_i, _c_f, _c_p, _c_sz, _c_p]),
    "paged_attn_decode_noalloc": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_p, _c_p, _c_i, _c_i, _c_i,
                                         _c_i, _c_i, _c_i, _c_f, _c_p]),
    "paged_attn_decode_graph_create": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_p, _c_p, _c_i, _c_i, _c_i,
                                              _c_i, _c_i, _c_i, _c_f, _c_p, _c_sz,
                                              ctypes.POINTER(ctypes.c_void_p)]),
    "paged_attn_decode_graph_launch": (_c_i, [_c_p, _c_p]),
    "paged_attn_decode_graph_destroy": (_c_i, [_c_p]),
    "attn_device_status": (_c_i, [_c_p, ctypes.POINTER(ctypes.c_uint)]),
    "attn_fwd_block_sparse": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p,
                                     ctypes.c_longlong, ctypes.c_longlong, _c_p]),
    "attn_fwd_bias": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p,
                             ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, _c_p]),
    "attn_fwd_fp8": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f, _c_f, _c_f, _c_f,
                            _c_p]),
    "paged_kv_append": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i,
                               _c_i, _c_p]),
    "paged_prefill": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i,
                             _c_i, _c_i, _c_i, _c_f, _c_p]),
    "paged_prefill_append": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i,
                                    _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p]),
}

# Size of the scratch array built into the library for paged_attn_decode_noalloc.
NOALLOC_SCRATCH_BYTES = 48 * 1024 * 1024

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        name = _STATUS_NAMES.get(status, str(status))
        msg = f"{what}: {name} ({status_string(status)})"
        if status == 6:
            msg += f"; cudaError {lib().attn_last_cuda_error()}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded C library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m attention_flashattention_fwd_04_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/attn_b200.h."""
    with open(os.path.join(INCLUDE, "attn_b200.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != ATTN_OK:
        raise AttnError(rc, what)


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _require(t: torch.Tensor, name: str, dtype, ndim: int, cuda: bool = True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_first_tensor_device(fn):
    """Runs a wrapper with its first tensor argument's CUDA device current, so
    that the stream it takes and any output it allocates belong to that
    device (the kernels run on the current device)."""
    @functools.wraps(fn)
    def wrapped(*args, **kwargs):
        first = next((a for a in args if isinstance(a, torch.Tensor)), None)
        if first is None or not first.is_cuda:
            return fn(*args, **kwargs)  # the wrapper's own checks reject it
        with torch.cuda.device(first.device):
            return fn(*args, **kwargs)
    return wrapped


@_on_first_tensor_device
def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
             scale: float | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, stream=None, window_left: int | None = None):
    """Fused attention forward.  q [B,Hq,N,d], k/v [B,Hkv,N,d] bf16 CUDA.

    ``window_left`` = W restricts query i to keys j >= i - W (sliding window).
    Returns (o [B,Hq,N,d] bf16, lse [B,Hq,N] fp32).
    """
    _require(q, "q", torch.bfloat16, 4)
    _require(k, "k", torch.bfloat16, 4)
    _require(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} do not match q {tuple(q.shape)}")
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.bfloat16, 4)
    _require(lse, "lse", torch.float32, 3)
    if window_left is None:
        rc = lib().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                            B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream_handle(stream))
        _check(rc, "attn_fwd")
    else:
        rc = lib().attn_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                   B, Hq, Hkv, N, d, int(bool(causal)), int(window_left), float(scale),
                                   _stream_handle(stream))
        _check(rc, "attn_fwd_window")
    return out, lse


def paged_attn_decode_split_tokens(num_seqs: int, Hkv: int, max_pages: int, page_size: int) -> int:
    return int(lib().paged_attn_decode_split_tokens(num_seqs, Hkv, max_pages, page_size))


def paged_attn_decode_workspace_bytes(num_seqs: int, Hq: int, d: int, max_pages: int, page_size: int) -> int:
    return int(lib().paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_pages, page_size))


def _decode_args(q, k_pool, v_pool, block_table, seq_lens, out=None, lse=None):
    """Checks shared by the paged-decode wrappers, made before any CUDA call
    (the C layer sees only pointers, so a short v_pool, block_table or
    seq_lens would be read past its end): dtypes, ranks, contiguity and
    consistent shapes first, then that every tensor is on q's CUDA device.
    Returns (S, Hq, d, num_pages, page_size, Hkv, max_pages)."""
    named = [(q, "q", torch.bfloat16, 3), (k_pool, "k_pool", torch.bfloat16, 4),
             (v_pool, "v_pool", torch.bfloat16, 4), (block_table, "block_table", torch.int32, 2),
             (seq_lens, "seq_lens", torch.int32, 1)]
    if out is not None:
        named.append((out, "out", torch.bfloat16, 3))
    if lse is not None:
        named.append((lse, "lse", torch.float32, 2))
    for t, name, dt, nd in named:
        _require(t, name, dt, nd, cuda=False)
    S, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_pool.shape
    if dk != d:
        raise ValueError(f"k_pool's head dim {dk} does not match q's {d}")
    if v_pool.shape != k_pool.shape:
        raise ValueError(f"v_pool shape {tuple(v_pool.shape)} differs from k_pool's {tuple(k_pool.shape)}")
    if block_table.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError(f"block_table {tuple(block_table.shape)} / seq_lens {tuple(seq_lens.shape)} do not "
                         f"have one row per sequence ({S})")
    if out is not None and out.shape != q.shape:
        raise ValueError(f"out shape {tuple(out.shape)} differs from q's {tuple(q.shape)}")
    if lse is not None and lse.shape != (S, Hq):
        raise ValueError(f"lse shape {tuple(lse.shape)} is not ({S}, {Hq})")
    for t, name, _, _ in named:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")
    return S, Hq, d, num_pages, page_size, Hkv, block_table.shape[1]


def paged_attn_decode(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                      block_table: torch.Tensor, seq_lens: torch.Tensor, scale: float | None = None,
                      workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, stream=None):
    """Decode attention over a paged KV cache.

    q [S,Hq,d] bf16; k_pool/v_pool [num_pages,page_size,Hkv,d] bf16;
    block_table [S,max_pages] int32; seq_lens [S] int32 (all on the GPU).
    Returns (o [S,Hq,d] bf16, lse [S,Hq] fp32).
    """
    S, Hq, d, num_pages, page_size, Hkv, max_pages = _decode_args(q, k_pool, v_pool, block_table, seq_lens,
                                                                  out, lse)
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    with torch.cuda.device(q.device):
        need = paged_attn_decode_workspace_bytes(S, Hq, d, max_pages, page_size)
        if workspace is None:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        elif not workspace.is_cuda or workspace.device != q.device:
            raise ValueError(f"workspace must be on {q.device}")
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
        rc = lib().paged_attn_decode(
            q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(),
            page_size, out.data_ptr(), lse.data_ptr(), S, Hq, Hkv, d, max_pages, num_pages, float(scale),
            workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check(rc, "paged_attn_decode")
    return out, lse


def paged_attn_decode_noalloc(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                              block_table: torch.Tensor, seq_lens: torch.Tensor, scale: float | None = None,
                              out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """paged_attn_decode without a workspace, for callers that may not
    allocate device memory (the outputs still come from the caller; pass
    ``out``/``lse`` to avoid any allocation here too).  The split partials go
    to a 48 MiB array built into the library, shared by all calls on a
    device: calls that can overlap on the GPU must not use it concurrently.
    """
    S, Hq, d, num_pages, page_size, Hkv, max_pages = _decode_args(q, k_pool, v_pool, block_table, seq_lens,
                                                                  out, lse)
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    with torch.cuda.device(q.device):
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
        rc = lib().paged_attn_decode_noalloc(
            q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(),
            page_size, out.data_ptr(), lse.data_ptr(), S, Hq, Hkv, d, max_pages, num_pages,
            float(scale), _stream_handle(stream))
    if rc == 4:
        need = paged_attn_decode_workspace_bytes(S, Hq, d, max_pages, page_size)
        raise AttnError(rc, f"paged_attn_decode_noalloc: needs {need} bytes of scratch, "
                            f"more than the built-in {NOALLOC_SCRATCH_BYTES}")
    _check(rc, "paged_attn_decode_noalloc")
    return out, lse


class DecodeGraph:
    """One paged-decode step (split pass + merge) captured as a CUDA graph.

    Construct it with the same tensors as :func:`paged_attn_decode`; then
    change their contents in place (same shapes) and call :meth:`launch` for
    each step.  The tensors, the workspace and the outputs are kept alive by
    this object; ``out`` and ``lse`` hold the results after each launch.
    """

    def __init__(self, q, k_pool, v_pool, block_table, seq_lens, scale=None, workspace=None, out=None, lse=None):
        self._handle = None
        S, Hq, d, num_pages, page_size, Hkv, max_pages = _decode_args(q, k_pool, v_pool, block_table, seq_lens,
                                                                      out, lse)
        if scale is None:
            scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
        self.device = q.device
        with torch.cuda.device(q.device):
            need = paged_attn_decode_workspace_bytes(S, Hq, d, max_pages, page_size)
            if workspace is not None and (not workspace.is_cuda or workspace.device != q.device):
                raise ValueError(f"workspace must be on {q.device}")
            self.workspace = workspace if workspace is not None else torch.empty(
                max(need, 16), dtype=torch.uint8, device=q.device)
            self.out = out if out is not None else torch.empty_like(q)
            self.lse = lse if lse is not None else torch.empty((S, Hq), dtype=torch.float32, device=q.device)
            self._keep = (q, k_pool, v_pool, block_table, seq_lens)
            handle = ctypes.c_void_p()
            rc = lib().paged_attn_decode_graph_create(
                q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(),
                page_size, self.out.data_ptr(), self.lse.data_ptr(), S, Hq, Hkv, d, max_pages, num_pages,
                float(scale), self.workspace.data_ptr(), self.workspace.numel() * self.workspace.element_size(),
                ctypes.byref(handle))
        _check(rc, "paged_attn_decode_graph_create")
        self._handle = handle

    def launch(self, stream=None):
        if self._handle is None:
            raise RuntimeError("DecodeGraph is closed")
        with torch.cuda.device(self.device):
            rc = lib().paged_attn_decode_graph_launch(self._handle, _stream_handle(stream))
        _check(rc, "paged_attn_decode_graph_launch")
        return self.out, self.lse

    def close(self):
        h, self._handle = getattr(self, "_handle", None), None
        if h is not None:
            _check(lib().paged_attn_decode_graph_destroy(h), "paged_attn_decode_graph_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    bits = ctypes.c_uint(0)
    rc = lib().attn_device_status(_stream_handle(stream), ctypes.byref(bits))
    if rc not in (ATTN_OK, 7):
        raise AttnError(rc, "attn_device_status")
    return int(bits.value)


def _paged_chunk_args(k_pool, v_pool, block_table, cu_seqlens_q, seq_lens):
    _require(k_pool, "k_pool", torch.bfloat16, 4)
    _require(v_pool, "v_pool", torch.bfloat16, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _require(seq_lens, "seq_lens", torch.int32, 1)
    if v_pool.shape != k_pool.shape:
        raise ValueError("k_pool and v_pool differ in shape")
    S = seq_lens.shape[0]
    if cu_seqlens_q.shape[0] != S + 1 or block_table.shape[0] != S:
        raise ValueError("cu_seqlens_q / block_table do not match the number of sequences")
    num_pages, page_size, Hkv, d = k_pool.shape
    return S, num_pages, page_size, Hkv, d, block_table.shape[1]


@_on_first_tensor_device
def paged_kv_append(k_new: torch.Tensor, v_new: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                    block_table: torch.Tensor, cu_seqlens_q: torch.Tensor, seq_lens: torch.Tensor, stream=None):
    """Write each sequence's new K/V rows (packed [total_q, Hkv, d] bf16,
    rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1) into the paged pools at
    logical tokens seq_lens[s] - q_len .. seq_lens[s] - 1.  In place."""
    S, num_pages, page_size, Hkv, d, max_pages = _paged_chunk_args(k_pool, v_pool, block_table, cu_seqlens_q,
                                                                   seq_lens)
    _require(k_new, "k_new", torch.bfloat16, 3)
    _require(v_new, "v_new", torch.bfloat16, 3)
    total_q = k_new.shape[0]
    if k_new.shape != (total_q, Hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new / v_new do not match the pools")
    rc = lib().paged_kv_append(k_new.data_ptr(), v_new.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                               cu_seqlens_q.data_ptr(), seq_lens.data_ptr(), block_table.data_ptr(), S, total_q,
                               Hkv, d, page_size, max_pages, num_pages, _stream_handle(stream))
    _check(rc, "paged_kv_append")


def _prefill_outputs(q, out, lse):
    total_q, Hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((total_q, Hq), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.bfloat16, 3)
    _require(lse, "lse", torch.float32, 2)
    return out, lse


@_on_first_tensor_device
def paged_prefill(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, block_table: torch.Tensor,
                  cu_seqlens_q: torch.Tensor, seq_lens: torch.Tensor, causal: bool = True,
                  scale: float | None = None, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                  stream=None):
    """Chunked prefill over a paged cache: q [total_q, Hq, d] bf16 packed by
    sequence; new query i of sequence s is token seq_lens[s] - q_len + i.
    Returns (o [total_q, Hq, d] bf16, lse [total_q, Hq] fp32)."""
    S, num_pages, page_size, Hkv, d, max_pages = _paged_chunk_args(k_pool, v_pool, block_table, cu_seqlens_q,
                                                                   seq_lens)
    _require(q, "q", torch.bfloat16, 3)
    total_q, Hq, dq = q.shape
    if dq != d:
        raise ValueError("q and the pools differ in head dim")
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    out, lse = _prefill_outputs(q, out, lse)
    rc = lib().paged_prefill(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), cu_seqlens_q.data_ptr(),
                             seq_lens.data_ptr(), block_table.data_ptr(), out.data_ptr(), lse.data_ptr(), S, total_q,
                             Hq, Hkv, d, page_size, max_pages, num_pages, int(bool(causal)), float(scale),
                             _stream_handle(stream))
    _check(rc, "paged_prefill")
    return out, lse


@_on_first_tensor_device
def paged_prefill_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_pool: torch.Tensor,
                         v_pool: torch.Tensor, block_table: torch.Tensor, cu_seqlens_q: torch.Tensor,
                         seq_lens: torch.Tensor, causal: bool = True, scale: float | None = None,
                         out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """paged_kv_append then paged_prefill in one call (the pools are
    updated in place).  Returns (o, lse) as paged_prefill does."""
    S, num_pages, page_size, Hkv, d, max_pages = _paged_chunk_args(k_pool, v_pool, block_table, cu_seqlens_q,
                                                                   seq_lens)
    _require(q, "q", torch.bfloat16, 3)
    _require(k_new, "k_new", torch.bfloat16, 3)
    _require(v_new, "v_new", torch.bfloat16, 3)
    total_q, Hq, dq = q.shape
    if dq != d or k_new.shape != (total_q, Hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("q / k_new / v_new do not match the pools")
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    out, lse = _prefill_outputs(q, out, lse)
    rc = lib().paged_prefill_append(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_pool.data_ptr(),
                                    v_pool.data_ptr(), cu_seqlens_q.data_ptr(), seq_lens.data_ptr(),
                                    block_table.data_ptr(), out.data_ptr(), lse.data_ptr(), S, total_q, Hq, Hkv, d,
                                    page_size, max_pages, num_pages, int(bool(causal)), float(scale),
                                    _stream_handle(stream))
    _check(rc, "paged_prefill_append")
    return out, lse


@_on_first_tensor_device
def attn_fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, scale: float | None = None,
                 q_descale: float = 1.0, k_descale: float = 1.0, v_descale: float = 1.0,
                 out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Fused attention forward with e4m3 inputs: q [B,Hq,N,128], k/v
    [B,Hkv,N,128] as torch.float8_e4m3fn (or their uint8 codes); the
    attention is over q*q_descale, k*k_descale, v*v_descale.
    Returns (o [B,Hq,N,128] bf16, lse [B,Hq,N] fp32)."""
    def codes(t, name):
        if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
            t = t.view(torch.uint8)
        _require(t, name, torch.uint8, 4)
        return t
    q, k, v = codes(q, "q"), codes(k, "k"), codes(v, "v")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} do not match q {tuple(q.shape)}")
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.bfloat16, 4)
    _require(lse, "lse", torch.float32, 3)
    rc = lib().attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N,
                            d, int(bool(causal)), float(scale), float(q_descale), float(k_descale), float(v_descale),
                            _stream_handle(stream))
    _check(rc, "attn_fwd_fp8")
    return out, lse


def pack_block_mask(keep: torch.Tensor) -> torch.Tensor:
    """Boolean block mask [B', H', q_blocks, k_blocks] (B' in {1, B}, H' in
    {1, Hq}; block = 128 rows / keys) -> the uint64 rows attn_fwd_block_sparse
    reads: bit j % 64 of word j / 64 set iff keep[..., j].  Returned as int64
    words [B', H', q_blocks, ceil(k_blocks / 64)] on keep's device."""
    if keep.dim() != 4:
        raise ValueError("keep must be [B, H, q_blocks, k_blocks]")
    nw = -(-keep.shape[-1] // 64)
    pad = torch.zeros(*keep.shape[:-1], nw * 64, dtype=torch.int64, device=keep.device)
    pad[..., : keep.shape[-1]] = keep.to(torch.int64)
    bits = pad.view(*keep.shape[:-1], nw, 64)
    weights = torch.ones(64, dtype=torch.int64, device=keep.device) << torch.arange(64, device=keep.device)
    return (bits * weights).sum(-1)  # bit 63 wraps to the sign bit: the same 64 bits


@_on_first_tensor_device
def attn_fwd_block_sparse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, keep: torch.Tensor,
                          causal: bool = True, scale: float | None = None, out: torch.Tensor | None = None,
                          lse: torch.Tensor | None = None, stream=None):
    """attn_fwd with a block-sparse mask: ``keep`` boolean [B or 1, Hq or 1,
    ceil(N/128), ceil(N/128)] (1 = the 128x128 block is computed), or the
    same mask already packed by ``pack_block_mask`` (int64 words [B or 1,
    Hq or 1, ceil(N/128), ceil(ceil(N/128)/64)], on q's device; a caller
    that reuses one mask packs it once).  Rows that see no key give O = 0,
    LSE = -inf."""
    _require(q, "q", torch.bfloat16, 4)
    _require(k, "k", torch.bfloat16, 4)
    _require(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} do not match q {tuple(q.shape)}")
    nb = -(-N // 128)
    nw = -(-nb // 64)
    if keep.dtype == torch.int64:
        if (keep.dim() != 4 or keep.shape[2:] != (nb, nw) or keep.shape[0] not in (1, B)
                or keep.shape[1] not in (1, Hq) or keep.device != q.device or not keep.is_contiguous()):
            raise ValueError(f"packed mask must be contiguous int64 [1 or {B}, 1 or {Hq}, {nb}, {nw}] on q's "
                             f"device, got {tuple(keep.shape)}")
        words = keep
    else:
        if (keep.dim() != 4 or keep.shape[2:] != (nb, nb) or keep.shape[0] not in (1, B)
                or keep.shape[1] not in (1, Hq)):
            raise ValueError(f"keep must be [1 or {B}, 1 or {Hq}, {nb}, {nb}], got {tuple(keep.shape)}")
        words = pack_block_mask(keep.to(q.device)).contiguous()
    h_stride = 0 if keep.shape[1] == 1 else nb * nw
    b_stride = 0 if keep.shape[0] == 1 else keep.shape[1] * nb * nw
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.bfloat16, 4)
    _require(lse, "lse", torch.float32, 3)
    rc = lib().attn_fwd_block_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq,
                                     Hkv, N, d, int(bool(causal)), float(scale), words.data_ptr(), b_stride, h_stride,
                                     _stream_handle(stream))
    _check(rc, "attn_fwd_block_sparse")
    return out, lse


def bias_span_ok(bias: torch.Tensor, strides) -> bool:
    """Whether every element the additive-M kernel reads lies in ``bias``'s
    storage: each row is read in 16-byte vectors up to the next multiple of 8
    elements, so the last row's padding must be there too (the C ABI takes a
    plain pointer and cannot check this)."""
    N = bias.shape[3]
    padded = -(-N // 8) * 8
    last = sum((bias.shape[i] - 1) * strides[i] for i in range(3)) + padded - 1
    end_bytes = (bias.storage_offset() + last + 1) * bias.element_size()
    return end_bytes <= bias.untyped_storage().nbytes()


@_on_first_tensor_device
def attn_fwd_bias(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bias: torch.Tensor, causal: bool = False,
                  scale: float | None = None, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                  stream=None):
    """attn_fwd with an additive mask M: softmax(scale * q k^T + M) v.

    ``bias`` is bf16 [B or 1, Hq or 1, N or 1, N] (natural-log units, -inf
    allowed), a strided view whose last dimension is contiguous and whose
    other strides are multiples of 8 elements: e.g. a slice ``[..., :N]`` of a
    buffer whose rows are padded to a multiple of 8.  Size-1 dimensions
    broadcast (stride 0 is passed).  Rows whose scores are all -inf give
    O = 0, LSE = -inf."""
    _require(q, "q", torch.bfloat16, 4)
    _require(k, "k", torch.bfloat16, 4)
    _require(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} do not match q {tuple(q.shape)}")
    if bias.dtype != torch.bfloat16 or bias.device != q.device or bias.dim() != 4:
        raise ValueError("bias must be a 4-d bf16 tensor on q's device")
    if (bias.shape[0] not in (1, B) or bias.shape[1] not in (1, Hq) or bias.shape[2] not in (1, N)
            or bias.shape[3] != N):
        raise ValueError(f"bias must be [1 or {B}, 1 or {Hq}, 1 or {N}, {N}], got {tuple(bias.shape)}")
    if N > 1 and bias.stride(3) != 1:
        raise ValueError("bias rows must be contiguous")
    strides = [0 if bias.shape[i] == 1 else bias.stride(i) for i in range(3)]
    if not bias_span_ok(bias, strides):
        raise ValueError("bias rows must be padded to a multiple of 8 elements within the tensor's storage "
                         "(e.g. a [..., :N] view of a buffer whose last dimension is rounded up to 8)")
    if scale is None:
        scale = float(torch.tensor(d ** -0.5, dtype=torch.float32))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.bfloat16, 4)
    _require(lse, "lse", torch.float32, 3)
    rc = lib().attn_fwd_bias(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N,
                             d, int(bool(causal)), float(scale), bias.data_ptr(), strides[0], strides[1], strides[2],
                             _stream_handle(stream))
    _check(rc, "attn_fwd_bias")
    return out, lse
