"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import assert_close, run_gpu, to_device

pytestmark = pytest.mark.gpu


def ref(w):
    return oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, w.scale)


def test_tiny_config():
    w = inputs.tiny()
    out, lse, flag = run_gpu(w)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, what="tiny")


@pytest.mark.parametrize("B,H,T,lens", [
    (1, 64, 1, [1000]),
    (2, 64, 1, [1000, 333]),
    (1, 64, 4, [300]),
    (3, 128, 2, [700, 64, 129]),
    (2, 16, 3, [200, 77]),
    (1, 128, 4, [190]),
    (4, 32, 2, [1, 2, 3, 63]) ,
])
def test_small_shapes(B, H, T, lens):
    lens = [max(L, T) for L in lens]
    w = inputs.make_workload("small", batch=B, heads=H, q_len=T, seqlens=lens, seed=sum(lens) + H + T)
    out, lse, flag = run_gpu(w)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, what=f"B{B} H{H} T{T} L{lens}")


@pytest.mark.parametrize("L", [1, 2, 4, 63, 64, 65, 127, 128, 129, 4095, 4097])
@pytest.mark.parametrize("T", [1, 4])
def test_context_edges(L, T):
    if L < T:
        pytest.skip("L < q_len is invalid")
    w = inputs.make_workload("edge", batch=1, heads=64, q_len=T, seqlens=[L], seed=L * 7 + T)
    out, lse, flag = run_gpu(w)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, what=f"L{L} T{T}")


@pytest.mark.parametrize("sm_budget", [2, 4, 10, 0])
def test_forced_split_counts_agree(sm_budget):
    w = inputs.make_workload("split", batch=2, heads=64, q_len=2, seqlens=[3000, 1500], seed=11)
    out, lse, flag = run_gpu(w, sm_budget=sm_budget)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, what=f"sm_budget={sm_budget}")


def test_shared_prefix_pages():
    w = inputs.make_workload("prefix", batch=4, heads=128, q_len=2, seqlens=[900, 1400, 640, 2000], seed=12,
                             shared_prefix_tokens=640)
    out, lse, flag = run_gpu(w)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, what="shared prefix")


def test_deterministic_and_page_scramble_bitwise():
    w = inputs.make_workload("det", batch=2, heads=64, q_len=2, seqlens=[2500, 777], seed=13)
    q, cache, bt, sl = to_device(w)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    o1, l1 = [x.clone() for x in dec(q, cache, bt, sl)]
    o2, l2 = [x.clone() for x in dec(q, cache, bt, sl)]
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    perm = torch.randperm(cache.shape[0], generator=torch.Generator().manual_seed(5)).to(cache.device)
    cache2 = torch.empty_like(cache)
    cache2[perm] = cache
    bt2 = perm[bt.long()].to(torch.int32)
    o3, l3 = [x.clone() for x in dec(q, cache2, bt2, sl)]
    torch.cuda.synchronize()
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_bad_seqlen_sets_flag_and_nan_rows():
    w = inputs.make_workload("bad", batch=3, heads=64, q_len=2, seqlens=[500, 300, 200], seed=14)
    q, cache, bt, sl = to_device(w)
    sl[1] = 1                                  # < q_len: invalid
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    out, lse = dec(q, cache, bt, sl)
    flag = dec.device_flag()
    assert flag & mla.FLAG_BAD_SEQLEN
    o = out.float().cpu().numpy()
    assert np.all(np.isnan(o[1]))
    ro, rl = oracle.mla_decode_ref(w.q_bits[[0, 2]], w.cache, "bf16", w.block_table[[0, 2]], w.seqlens[[0, 2]])
    assert_close(o[[0, 2]].astype(np.float64), lse.cpu().numpy()[[0, 2]].astype(np.float64), ro, rl,
                 what="valid rows next to a bad one")


def test_bad_page_id_sets_flag():
    w = inputs.make_workload("badpage", batch=1, heads=64, q_len=1, seqlens=[300], seed=15)
    q, cache, bt, sl = to_device(w)
    bt[0, 2] = cache.shape[0] + 5             # outside the pool: must not be read
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    dec(q, cache, bt, sl)
    assert dec.device_flag() & mla.FLAG_BAD_PAGE


def _plan_flag(w, bt, sl, cache, with_table):
    """Flag word after the planner alone (no decode kernel): the block-table
    check of mla_decode_plan reports through the decode kernel, so read the
    check words the planner left in the workspace header."""
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    if with_table:
        dec.plan(sl, block_table=bt, num_pages=int(cache.shape[0]))
    else:
        dec.plan(sl)
    torch.cuda.synchronize()
    hdr = dec.workspace[:64 * 4].view(torch.int32).cpu().numpy()
    return dec, hdr


def test_planner_checks_the_block_table():
    # 70 pages used by sequence 0, 3 by sequence 1; bad ids planted in the used
    # range of sequence 0 (found) and past the used range of sequence 1 (never
    # read, so not reported).
    w = inputs.make_workload("plancheck", batch=2, heads=64, q_len=1, seqlens=[70 * 64 - 5, 150], seed=16,
                             max_pages=80)
    q, cache, bt, sl = to_device(w)
    dec, hdr = _plan_flag(w, bt, sl, cache, with_table=True)
    n_chk = int(hdr[7])
    assert n_chk >= 1 and not any(hdr[8:8 + n_chk])              # a good table: nothing found
    bt[1, 10] = -3                                               # past sequence 1's 3 pages
    dec, hdr = _plan_flag(w, bt, sl, cache, with_table=True)
    assert not any(hdr[8:8 + int(hdr[7])])
    bt[0, 69] = cache.shape[0]                                   # sequence 0's last page: out of range
    dec, hdr = _plan_flag(w, bt, sl, cache, with_table=True)
    assert any(hdr[8:8 + int(hdr[7])])
    dec.run(q, cache, bt, sl)
    assert dec.device_flag() & mla.FLAG_BAD_PAGE
    # without a table the planner checks nothing (and records that)
    dec, hdr = _plan_flag(w, bt, sl, cache, with_table=False)
    assert int(hdr[7]) == 0


# ---------------------------------------------------------------- fp8-e4m3 cache

@pytest.mark.parametrize("B,H,T,lens", [
    (1, 16, 1, [256]),
    (2, 64, 1, [1000, 333]),
    (1, 64, 4, [300]),
    (3, 128, 1, [700, 64, 129]),
    (2, 128, 2, [513, 4097]),
    (4, 32, 2, [2, 3, 63, 65]),
])
def test_fp8_cache_small_shapes(B, H, T, lens):
    w = inputs.make_workload("fp8s", batch=B, heads=H, q_len=T, seqlens=lens, kv_dtype="fp8",
                             seed=sum(lens) + 3 * H + T)
    out, lse, flag = run_gpu(w)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, kv_dtype="fp8", what=f"fp8 B{B} H{H} T{T} L{lens}")


@pytest.mark.parametrize("sm_budget", [2, 6, 0])
def test_fp8_forced_splits(sm_budget):
    w = inputs.make_workload("fp8split", batch=3, heads=128, q_len=1, seqlens=[2000, 900, 64], kv_dtype="fp8",
                             seed=17)
    out, lse, flag = run_gpu(w, sm_budget=sm_budget)
    ro, rl = ref(w)
    assert flag == 0
    assert_close(out, lse, ro, rl, kv_dtype="fp8", what=f"fp8 sm_budget={sm_budget}")


def test_large_batch_general_planner():
    """More sequences than the planner's one-thread-per-sequence pass holds
    (1,024): the chunked planner path, checked on sampled rows of every tenth
    sequence plus the first and last."""
    rng = np.random.default_rng(77)
    lens = rng.integers(1, 300, size=1030).tolist()
    w = inputs.make_workload("bigbatch", batch=1030, heads=16, q_len=1, seqlens=lens, seed=78)
    out, lse, flag = run_gpu(w)
    assert flag == 0
    pick = sorted(set(list(range(0, 1030, 10)) + [1029]))
    ro, rl = oracle.mla_decode_ref(w.q_bits[pick], w.cache, "bf16", w.block_table[pick], w.seqlens[pick])
    assert_close(out[pick], lse[pick], ro, rl, what="batch 1030")


def test_many_listed_sequences():
    """600 sequences for the combine kernel to visit (split or invalid): 560 get an
    invalid length (NaN rows, flag set); the 40 valid ones are long enough to be
    split across clusters, and their items sit far apart in the combine list."""
    B = 600
    rng = np.random.default_rng(91)
    valid = np.arange(0, B, 15)
    lens = np.full(B, 64, dtype=np.int64)
    lens[valid] = rng.integers(500, 2000, size=valid.size)
    w = inputs.make_workload("listed", batch=B, heads=16, q_len=1, seqlens=lens, seed=92)
    q, cache, bt, sl = to_device(w)
    bad = np.setdiff1d(np.arange(B), valid)
    sl[torch.from_numpy(bad).to(sl.device)] = 0                 # < q_len: invalid
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads)
    out, lse = dec(q, cache, bt, sl)
    torch.cuda.synchronize()
    assert dec.device_flag() & mla.FLAG_BAD_SEQLEN
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(o[bad])) and np.all(np.isnan(l[bad]))
    ro, rl = oracle.mla_decode_ref(w.q_bits[valid], w.cache, "bf16", w.block_table[valid], w.seqlens[valid])
    assert_close(o[valid], l[valid], ro, rl, what="valid rows among 560 invalid ones")
