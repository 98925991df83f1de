"""GPU: the split-KV plan and the launches that derive it on the device.

- Both device planners (the one-warp planner of small 64-row steps and the
  block-wide one, one-pass and chunked) against the host restatement of the
  plan (tests/plan_ref.py), word for word.
- A decode launch of a small batch derives the plan itself and does not wait
  for the planner kernel: two attention launches in a row on one workspace must
  still leave the second one's result, and a plan that differs from the
  planner's must be reported (MLA_FLAG_PLAN_MISMATCH), not used silently.
"""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import assert_close, to_device
import plan_ref

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,T,lens,budget", [
    (1, 64, 1, [50_000], 0),                     # one-warp planner, one long sequence
    (3, 16, 4, [5000, 64, 9000], 0),             # one-warp planner, 64 rows
    (5, 64, 1, [3, 70_000, 700, 0, 4096], 12),   # one-warp planner, one invalid length, a budget
    (32, 32, 2, None, 0),                        # one-warp planner, a full warp of sequences
    (2, 128, 2, [20_000, 7000], 0),              # block-wide planner (128-row tiles)
    (40, 16, 1, None, 0),                        # block-wide planner, more than a warp
    (1100, 16, 1, None, 30),                     # chunked planner (more than 1,024 sequences)
])
def test_device_plan_matches_host_restatement(B, H, T, lens, budget):
    rng = np.random.default_rng(B * 1000 + H)
    if lens is None:
        lens = rng.integers(1, 3000, size=B).tolist()
    max_pages = max((max(lens) + 63) // 64, 1)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    nbytes, max_splits = mla.workspace_size(B, max_pages, T, H)
    c_max = max_splits - B
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
    mla.plan(sl, max_pages, T, H, ws, sm_budget=budget)
    torch.cuda.synchronize()
    c_use = plan_ref.c_use_of(budget, c_max, T, H)
    want = plan_ref.plan(lens, T, H, max_pages, c_use, c_max)
    got = plan_ref.read_plan(ws.cpu().numpy(), B, c_max, len(want["list"]))
    assert got["hdr"] == want["hdr"]
    assert got["seq"] == want["seq"]
    assert got["list"] == want["list"] and got["vcp"] == want["vcp"]
    assert got["first_b"] == want["first_b"]
    flag = int(ws[:4].view(torch.int32).cpu()[0])
    bad_len = any(not (T <= L <= 64 * max_pages) for L in lens)
    assert flag == (mla.FLAG_BAD_SEQLEN if bad_len else 0)


@pytest.mark.parametrize("H,T", [(64, 1), (64, 4)])
def test_two_attention_launches_in_a_row(H, T):
    """plan, attention with q1, attention with q2 (same workspace, no planner in
    between), combine: the result is q2's. The second attention launch derives
    its plan itself and may start while the first runs; it must not store before
    the first is done."""
    w = inputs.make_workload("twice", batch=1, heads=H, q_len=T, seqlens=[40_000], seed=31 + T)
    q, cache, bt, sl = to_device(w)
    q1 = torch.randn_like(q.float()).to(torch.bfloat16)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    out, lse = dec.out, dec.lse
    for _ in range(3):
        dec.plan(sl)
        mla.run(q1, cache, bt, sl, out, lse, dec.workspace, phases=mla.PHASE_ATTEND)
        mla.run(q, cache, bt, sl, out, lse, dec.workspace, phases=mla.PHASE_ATTEND)
        mla.run(q, cache, bt, sl, out, lse, dec.workspace, phases=mla.PHASE_COMBINE)
        torch.cuda.synchronize()
        assert dec.device_flag() == 0
        ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, w.scale)
        assert_close(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ro, rl,
                     what=f"H{H} T{T}")


def test_plan_mismatch_is_reported():
    """A captured plan replayed after a later plan call with another SM budget:
    the decode launch uses the later (recorded) plan, the planner kernel wrote
    the captured one, and the flag says so."""
    w = inputs.make_workload("mismatch", batch=1, heads=64, q_len=1, seqlens=[30_000], seed=41)
    q, cache, bt, sl = to_device(w)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        mla.plan(sl, w.max_pages, w.q_len, w.heads, dec.workspace, stream=stream)   # set-up outside capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            mla.plan(sl, w.max_pages, w.q_len, w.heads, dec.workspace, stream=stream)           # all SMs
        mla.plan(sl, w.max_pages, w.q_len, w.heads, dec.workspace, sm_budget=16, stream=stream)  # recorded
        g.replay()                                                                              # planner: all SMs
        mla.run(q, cache, bt, sl, dec.out, dec.lse, dec.workspace, stream=stream)
        stream.synchronize()
    assert dec.device_flag() & mla.FLAG_PLAN_MISMATCH
    # planned and run consistently again: no flag, and the right result
    dec.plan(sl)
    dec.run(q, cache, bt, sl)
    torch.cuda.synchronize()
    assert dec.device_flag() == 0
    ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, w.scale)
    assert_close(dec.out.float().cpu().numpy().astype(np.float64), dec.lse.cpu().numpy().astype(np.float64), ro, rl,
                 what="after a consistent plan")


@pytest.mark.parametrize("B,H,T", [(32, 64, 1), (33, 64, 1), (32, 16, 4), (33, 128, 2)])
def test_self_planning_batch_boundary(B, H, T):
    """32 sequences: the decode kernel plans itself; 33: it reads the planner's
    plan. Both against the oracle, with a mix of lengths that splits some."""
    rng = np.random.default_rng(B * 7 + H + T)
    lens = [int(x) for x in rng.integers(T, 2500, size=B)]
    lens[0] = 20_000                                   # one long sequence, cut into many pieces
    w = inputs.make_workload("boundary", batch=B, heads=H, q_len=T, seqlens=lens, seed=B + H)
    q, cache, bt, sl = to_device(w)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    out, lse = dec(q, cache, bt, sl)
    torch.cuda.synchronize()
    assert dec.device_flag() == 0
    ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, w.scale)
    assert_close(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ro, rl,
                 what=f"B{B} H{H} T{T}")


def test_small_batch_on_a_workspace_planned_elsewhere():
    """A workspace this process never planned (here: a device copy of a planned
    one) has no host record, so its decode kernel reads the planner's plan from
    the workspace instead of deriving it: same result."""
    w = inputs.make_workload("copied", batch=2, heads=64, q_len=1, seqlens=[30_000, 900], seed=43)
    q, cache, bt, sl = to_device(w)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    dec.plan(sl)
    ws2 = dec.workspace.clone()
    out2, lse2 = torch.empty_like(dec.out), torch.empty_like(dec.lse)
    mla.run(q, cache, bt, sl, out2, lse2, ws2)
    torch.cuda.synchronize()
    assert mla.read_device_flag(ws2) == 0
    ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, w.scale)
    assert_close(out2.float().cpu().numpy().astype(np.float64), lse2.cpu().numpy().astype(np.float64), ro, rl,
                 what="workspace planned elsewhere")
    # and the self-planned run on the original workspace gives the same bits
    dec.run(q, cache, bt, sl)
    torch.cuda.synchronize()
    assert torch.equal(dec.out, out2) and torch.equal(dec.lse, lse2)
