"""mla_decode_noalloc: the decode step for callers that cannot supply a
workspace (it runs on scratch built into the library) must give the same
results as the ordinary plan + run with a caller-owned workspace, and match
the fp64 oracle within the usual tolerance.

Collected last on purpose: the scratch array is shared by every call, so this
file also checks that results stay right after other tests have run."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import _lib, inputs
from parity_util import assert_close, to_device

pytestmark = pytest.mark.gpu


def _workspace_path(w, tensors):
    q, cache, bt, sl = tensors
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    out, lse = dec(q, cache, bt, sl, scale=w.scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _noalloc_path(w, tensors):
    q, cache, bt, sl = tensors
    out = torch.full((w.batch, w.q_len, w.heads, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.batch, w.q_len, w.heads), float("nan"), dtype=torch.float32, device="cuda")
    mla.decode_noalloc(q, cache, bt, sl, out, lse, scale=w.scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def test_noalloc_matches_the_workspace_path_on_two_calls_in_a_row():
    # Two different steps back to back: the second must not see the first's leftovers.
    steps = [
        inputs.make_workload("na1", batch=3, heads=64, q_len=2, seqlens=[1500, 700, 90], seed=41),
        inputs.make_workload("na2", batch=2, heads=128, q_len=1, seqlens=[5000, 333], seed=42),
    ]
    for w in steps:
        tensors = to_device(w)
        ref_out, ref_lse = _workspace_path(w, tensors)
        out, lse = _noalloc_path(w, tensors)
        assert_close(out, lse, ref_out, ref_lse, what=f"noalloc {w.name}")
        o_ref, l_ref = oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, w.scale)
        assert_close(out, lse, o_ref, l_ref, what=f"noalloc {w.name} vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = _lib.load()
    st = lib.mla_decode_noalloc(None, None, 1, 0, None, None, None, None, 4096, 1024, 1, 128, 0.07, None)
    assert st == _lib.MLA_ERR_WORKSPACE_TOO_SMALL
    msg = lib.mla_get_last_error().decode()
    assert "MLA_NOALLOC_SCRATCH_BYTES" in msg and str(_lib.NOALLOC_SCRATCH_BYTES) in msg
