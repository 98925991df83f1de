"""MLA decode over a paged latent KV cache, B200-native (sm_100a).

Thin Python binding of ``libmla_decode.so`` (C ABI in ``include/mla_decode.h``).
PyTorch supplies device memory and streams only; every step of the decode runs
in the library's CUDA kernels. Names mirror the C ABI:

    nbytes, max_splits = workspace_size(batch, max_pages, q_len, heads)
    plan(seqlens, max_pages, q_len, heads, workspace)
    run(q, kv_cache, block_table, seqlens, out, lse, workspace, scale=...)

``MlaDecoder`` bundles a workspace for a fixed shape.
"""

from __future__ import annotations

import ctypes
import math

from . import _lib
from ._lib import (  # noqa: F401
    FLAG_BAD_PAGE, FLAG_BAD_PREFIX, FLAG_BAD_SEQLEN, FLAG_PLAN_MISMATCH, FLAG_TIMEOUT, MLA_KV_BF16, MLA_KV_FP8_E4M3,
    PHASE_ATTEND, PHASE_COMBINE, MlaError)

DEFAULT_SCALE = 1.0 / math.sqrt(192.0)
PAGE = 64
D_QK = 576
D_V = 512

_KV = {"bf16": MLA_KV_BF16, "fp8": MLA_KV_FP8_E4M3, MLA_KV_BF16: MLA_KV_BF16, MLA_KV_FP8_E4M3: MLA_KV_FP8_E4M3}


def _kv(kv_dtype) -> int:
    try:
        return _KV[kv_dtype]
    except KeyError:
        raise ValueError(f"kv_dtype must be 'bf16' or 'fp8', got {kv_dtype!r}") from None


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def version() -> str:
    return _lib.load().mla_version().decode()


def workspace_size(batch: int, max_pages: int, q_len: int, heads: int, kv_dtype="bf16"):
    """(bytes, max_splits) of the workspace for this shape (host-only query)."""
    lib = _lib.load()
    nbytes = ctypes.c_size_t(0)
    splits = ctypes.c_int(0)
    _lib.check(lib.mla_decode_plan(None, None, 0, batch, max_pages, q_len, heads, _kv(kv_dtype), 0, None,
                                   ctypes.byref(nbytes), ctypes.byref(splits), None))
    return int(nbytes.value), int(splits.value)


def plan(seqlens, max_pages: int, q_len: int, heads: int, workspace, kv_dtype="bf16", sm_budget: int = 0,
         stream=None, block_table=None, num_pages: int = 0) -> None:
    """Enqueue the device-side split-KV planner for this step. With
    ``block_table`` (and the pool's ``num_pages``) the planner also
    range-checks the page ids the step will read."""
    lib = _lib.load()
    nbytes = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    splits = ctypes.c_int(0)
    _lib.check(lib.mla_decode_plan(_ptr(seqlens), _ptr(block_table), int(num_pages), int(seqlens.shape[0]),
                                   max_pages, q_len, heads, _kv(kv_dtype), sm_budget, _ptr(workspace),
                                   ctypes.byref(nbytes), ctypes.byref(splits), _stream(stream)))


def run(q, kv_cache, block_table, seqlens, out, lse, workspace, kv_dtype="bf16", scale: float = DEFAULT_SCALE,
        num_pages=None, stream=None, phases=None) -> None:
    """Enqueue the decode attention. q [B, T, H, 576] bf16, out [B, T, H, 512]
    bf16 and lse [B, T, H] fp32 are device tensors; kv_cache is the page pool.
    ``phases`` (PHASE_ATTEND | PHASE_COMBINE) selects mla_decode_run_phases."""
    lib = _lib.load()
    B, T, H, _ = q.shape
    if num_pages is None:
        num_pages = int(kv_cache.shape[0])
    args = (_ptr(q), _ptr(kv_cache), int(num_pages), _kv(kv_dtype), _ptr(block_table), _ptr(seqlens), _ptr(out),
            _ptr(lse), B, int(block_table.shape[1]), T, H, float(scale), _ptr(workspace),
            workspace.numel() * workspace.element_size())
    if phases is None:
        _lib.check(lib.mla_decode_run(*args, _stream(stream)))
    else:
        _lib.check(lib.mla_decode_run_phases(*args, int(phases), _stream(stream)))


def decode_noalloc(q, kv_cache, block_table, seqlens, out, lse, kv_dtype="bf16", scale: float = DEFAULT_SCALE,
                   num_pages=None, stream=None) -> None:
    """One decode step (plan + run) on the library's built-in scratch, for
    callers that cannot supply a workspace. Calls share that scratch: keep them
    ordered on one stream. The first call on a device must precede any stream
    capture. Shapes needing more than NOALLOC_SCRATCH_BYTES are rejected."""
    lib = _lib.load()
    B, T, H, _ = q.shape
    if num_pages is None:
        num_pages = int(kv_cache.shape[0])
    _lib.check(lib.mla_decode_noalloc(_ptr(q), _ptr(kv_cache), int(num_pages), _kv(kv_dtype), _ptr(block_table),
                                      _ptr(seqlens), _ptr(out), _ptr(lse), B, int(block_table.shape[1]), T, H,
                                      float(scale), _stream(stream)))


def append(kv_new, kv_cache, block_table, seqlens, kv_dtype="bf16", num_pages=None, flag=None,
           stream=None) -> None:
    """Enqueue the latent-cache append: the q_len new tokens' rows kv_new
    [B, T, 576] bf16 go to positions L_b - T .. L_b - 1 of each sequence,
    through the block table (fp8 caches: quantised with a per-token scale).
    ``flag`` is an optional device int32 tensor for bad-length / bad-page bits."""
    lib = _lib.load()
    B, T, _ = kv_new.shape
    if num_pages is None:
        num_pages = int(kv_cache.shape[0])
    _lib.check(lib.mla_cache_append(_ptr(kv_new), _ptr(kv_cache), int(num_pages), _kv(kv_dtype),
                                    _ptr(block_table), _ptr(seqlens), B, int(block_table.shape[1]), T,
                                    _ptr(flag), _stream(stream)))


def cascade_workspace_size(batch: int, max_pages: int, q_len: int, heads: int, kv_dtype="bf16") -> int:
    """Bytes of workspace mla_decode_cascade needs for this shape (host-only query)."""
    nbytes = ctypes.c_size_t(0)
    _lib.check(_lib.load().mla_decode_cascade(None, None, 1, _kv(kv_dtype), None, None, 0, None, None, batch,
                                              max_pages, q_len, heads, 1.0, None, ctypes.byref(nbytes), None))
    return int(nbytes.value)


def cascade(q, kv_cache, block_table, seqlens, prefix_len: int, out, lse, workspace, kv_dtype="bf16",
            scale: float = DEFAULT_SCALE, num_pages=None, stream=None) -> None:
    """Enqueue a prefix-shared (cascade) decode step: the first prefix_len
    tokens (pages shared by every sequence) are attended by all query rows of
    the batch at once, the rest per sequence, and the two are merged. Same
    shapes as run(); ``workspace`` from cascade_workspace_size()."""
    B, T, H, _ = q.shape
    if num_pages is None:
        num_pages = int(kv_cache.shape[0])
    nbytes = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _lib.check(_lib.load().mla_decode_cascade(_ptr(q), _ptr(kv_cache), int(num_pages), _kv(kv_dtype),
                                              _ptr(block_table), _ptr(seqlens), int(prefix_len), _ptr(out),
                                              _ptr(lse), B, int(block_table.shape[1]), T, H, float(scale),
                                              _ptr(workspace), ctypes.byref(nbytes), _stream(stream)))


def absorb_q(q, w_uk, q_out, flag=None, stream=None) -> None:
    """q_out[n, h] = [W_UK[h]^T q[n, h, :128] | q[n, h, 128:]]: q [N, H, 192],
    w_uk [H, 128, 512], q_out [N, H, 576], all bf16 device tensors."""
    N, H, _ = q.shape
    _lib.check(_lib.load().mla_absorb_q(_ptr(q), _ptr(w_uk), _ptr(q_out), N, H, _ptr(flag), _stream(stream)))


def project_out(o, w_uv, y, flag=None, stream=None) -> None:
    """y[n, h] = W_UV[h] o[n, h]: o [N, H, 512], w_uv [H, 128, 512], y [N, H, 128],
    all bf16 device tensors."""
    N, H, _ = o.shape
    _lib.check(_lib.load().mla_project_out(_ptr(o), _ptr(w_uv), _ptr(y), N, H, _ptr(flag), _stream(stream)))


def read_device_flag(workspace, stream=None) -> int:
    """Device flag bits of the last planned/run step (synchronises the stream)."""
    lib = _lib.load()
    flag = ctypes.c_int(0)
    status = lib.mla_read_device_flag(_ptr(workspace), ctypes.byref(flag), _stream(stream))
    if status not in (_lib.MLA_OK, _lib.MLA_ERR_DEVICE_FLAG):
        _lib.check(status)
    return int(flag.value)


def set_wait_timeout_ns(ns: int) -> None:
    _lib.check(_lib.load().mla_set_wait_timeout_ns(int(ns)))


class MlaDecoder:
    """Workspace + output buffers for one fixed decode shape on one device."""

    def __init__(self, batch: int, max_pages: int, q_len: int, heads: int, kv_dtype="bf16", device=None,
                 sm_budget: int = 0):
        import torch
        self.batch, self.max_pages, self.q_len, self.heads = batch, max_pages, q_len, heads
        self.kv_dtype = kv_dtype
        self.sm_budget = sm_budget
        self.device = torch.device(device if device is not None else "cuda")
        nbytes, self.max_splits = workspace_size(batch, max_pages, q_len, heads, kv_dtype)
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        self.out = torch.empty((batch, q_len, heads, D_V), dtype=torch.bfloat16, device=self.device)
        self.lse = torch.empty((batch, q_len, heads), dtype=torch.float32, device=self.device)

    def plan(self, seqlens, stream=None, block_table=None, num_pages: int = 0):
        plan(seqlens, self.max_pages, self.q_len, self.heads, self.workspace, self.kv_dtype, self.sm_budget, stream,
             block_table, num_pages)

    def run(self, q, kv_cache, block_table, seqlens, scale: float = DEFAULT_SCALE, stream=None):
        run(q, kv_cache, block_table, seqlens, self.out, self.lse, self.workspace, self.kv_dtype, scale,
            stream=stream)
        return self.out, self.lse

    def __call__(self, q, kv_cache, block_table, seqlens, scale: float = DEFAULT_SCALE, stream=None):
        self.plan(seqlens, stream, block_table, int(kv_cache.shape[0]))
        return self.run(q, kv_cache, block_table, seqlens, scale, stream)

    def device_flag(self, stream=None) -> int:
        return read_device_flag(self.workspace, stream)
