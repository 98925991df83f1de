"""Failure detection on the device without a fault: every wait in the decode
kernel is bounded. With the bound set to 1 ns the first wait that is not
already satisfied runs out; the kernel then drains its in-flight copies and
MMAs, frees its tensor memory, sets MLA_FLAG_TIMEOUT in the workspace and
returns. The host reads the flag, and the same CUDA context then runs a normal
step correctly.

Every kernel variant is exercised (bf16 and fp8 caches, 64- and 128-row
tiles). The two softmax warps of a lane quarter meet on bounded mbarrier waits,
so a warp that gives up cannot strand its partner."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import assert_close, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,T,kv", [(64, 1, "bf16"), (128, 2, "bf16"), (64, 1, "fp8"), (128, 1, "fp8")])
def test_wait_timeout_sets_flag_and_context_recovers(H, T, kv):
    w = inputs.make_workload("tmo", batch=2, heads=H, q_len=T, seqlens=[4096, 700], kv_dtype=kv, seed=31)
    mla.set_wait_timeout_ns(1)
    try:
        _, _, flag = run_gpu(w)
    finally:
        mla.set_wait_timeout_ns(10 ** 9)
    assert flag & mla.FLAG_TIMEOUT
    out, lse, flag = run_gpu(w)
    assert flag == 0
    ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, kv, w.block_table, w.seqlens)
    assert_close(out, lse, ro, rl, kv_dtype=kv, what=f"after timeout H{H} T{T} {kv}")
