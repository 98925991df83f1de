"""GPU parity of the latent-cache append (mla_cache_append, through the C ABI)
against the oracle's append: bit-exact pages for bf16 and fp8-e4m3 caches
(codes and per-token scales), then append followed by decode, end to end,
against the fp64 decode oracle on the appended cache."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import assert_close, run_gpu

pytestmark = pytest.mark.gpu

D = 576


def _bf16_rows(rng, shape, std=0.5):
    return inputs.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _pool(rng, kv_dtype, pages):
    if kv_dtype == "bf16":
        return rng.integers(0, 1 << 16, size=(pages, 64, D), dtype=np.uint16)
    return rng.integers(0, 256, size=(pages, inputs.FP8_PAGE_BYTES), dtype=np.uint8)


def _to_dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(a.copy()).cuda()


def _from_dev(t, like):
    if like.dtype == np.uint16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_append_matches_oracle_bitwise(kv_dtype, T):
    rng = np.random.default_rng(100 + T + (7 if kv_dtype == "fp8" else 0))
    lens = np.array([T, 63, 64, 65, 128 + T, 1000, 4095, 4096], dtype=np.int64)
    lens = np.maximum(lens, T)
    B, max_pages = len(lens), 70
    pages = 1 + B * max_pages
    bt = rng.permutation(pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    cache = _pool(rng, kv_dtype, pages)
    new = _bf16_rows(rng, (B, T, D))
    new[0, 0, :7] = 0                                      # zeros and
    new[1, 0] = 0                                          # an all-zero row (sigma = 1)
    new[2, T - 1, 3] = inputs.f32_to_bf16_bits(np.float32(-0.0))
    ref = oracle.cache_append_ref(cache, kv_dtype, new, bt, lens)
    c_d = _to_dev(cache)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.append(_to_dev(new), c_d, torch.from_numpy(bt).cuda(), torch.from_numpy(lens.astype(np.int32)).cuda(),
               kv_dtype, flag=flag)
    torch.cuda.synchronize()
    got = _from_dev(c_d, cache)
    assert int(flag.item()) == 0
    assert np.array_equal(got, ref)


def test_append_flags_bad_rows_and_writes_nothing_for_them():
    rng = np.random.default_rng(9)
    B, T, max_pages, pages = 3, 2, 4, 20
    bt = rng.permutation(pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    bt[2, 1] = pages + 3                                   # sequence 2's new rows land in page 1
    lens = np.array([100, 1, 70], dtype=np.int32)          # sequence 1: L < q_len
    cache = _pool(rng, "bf16", pages)
    new = _bf16_rows(rng, (B, T, D))
    c_d = _to_dev(cache)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.append(_to_dev(new), c_d, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), "bf16", flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == (mla.FLAG_BAD_SEQLEN | mla.FLAG_BAD_PAGE)
    ref = oracle.cache_append_ref(cache, "bf16", new, bt, lens)   # writes sequence 0 only
    assert np.array_equal(_from_dev(c_d, cache), ref)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_append_then_decode_matches_the_oracle(kv_dtype):
    # A decode step as a serving loop runs it: the cache holds every token but
    # the T new ones (their slots hold NaN), append writes them, decode reads.
    T, H = 2, 64
    lens = [1000, 129, 4097]
    wb = inputs.make_workload("appdec", batch=3, heads=H, q_len=T, seqlens=lens, seed=31)
    rows = wb.cache                                        # bf16 [pages, 64, 576]
    new = np.empty((3, T, D), dtype=np.uint16)
    for b, L in enumerate(lens):
        for t in range(T):
            j = L - T + t
            new[b, t] = rows[wb.block_table[b, j // 64], j % 64]
    if kv_dtype == "bf16":
        stale = rows.copy()
        for b, L in enumerate(lens):
            for t in range(T):
                j = L - T + t
                stale[wb.block_table[b, j // 64], j % 64] = inputs.BF16_NAN
    else:
        stale = inputs.encode_fp8_pages(rows)
        for b, L in enumerate(lens):
            for t in range(T):
                j = L - T + t
                pg = stale[wb.block_table[b, j // 64]]
                pg[(j % 64) * D:(j % 64 + 1) * D] = inputs.E4M3_NAN
                pg[inputs.FP8_DATA_BYTES + 4 * (j % 64):inputs.FP8_DATA_BYTES + 4 * (j % 64) + 4] = 0xFF
    expect = oracle.cache_append_ref(stale, kv_dtype, new, wb.block_table, wb.seqlens)
    c_d = _to_dev(stale)
    bt = torch.from_numpy(wb.block_table).cuda()
    sl = torch.from_numpy(wb.seqlens).cuda()
    mla.append(_to_dev(new), c_d, bt, sl, kv_dtype)
    q = torch.from_numpy(wb.q_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    out, lse, flag = run_gpu(wb, tensors=(q, c_d, bt, sl), decoder=mla.MlaDecoder(3, wb.max_pages, T, H, kv_dtype))
    assert flag == 0
    assert np.array_equal(_from_dev(c_d, stale), expect)
    ro, rl = oracle.mla_decode_ref(wb.q_bits, expect, kv_dtype, wb.block_table, wb.seqlens, wb.scale)
    assert_close(out, lse, ro, rl, kv_dtype=kv_dtype, what=f"append + decode ({kv_dtype})")


def test_bulk_append_full_pages():
    # A large append (64 sequences x 4 tokens into an fp8 pool of 2,000 pages):
    # bit-exact against the oracle, and equal to the input generator's torch
    # writer on every written slot.
    rng = np.random.default_rng(12)
    B, T, max_pages, pages = 64, 4, 30, 2000
    bt = rng.permutation(pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    lens = rng.integers(T, max_pages * 64 + 1, size=B).astype(np.int32)
    cache = _pool(rng, "fp8", pages)
    new = _bf16_rows(rng, (B, T, D), std=3.0)
    c_d = _to_dev(cache)
    mla.append(_to_dev(new), c_d, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), "fp8")
    torch.cuda.synchronize()
    got = _from_dev(c_d, cache)
    assert np.array_equal(got, oracle.cache_append_ref(cache, "fp8", new, bt, lens))
    ref_pages = inputs.encode_fp8_pages(np.broadcast_to(new.reshape(B * T, 1, D), (B * T, 64, D)).copy())
    for i in range(B * T):
        b, t = divmod(i, T)
        j = int(lens[b]) - T + t
        pg, slot = got[bt[b, j // 64]], j % 64
        assert np.array_equal(pg[slot * D:(slot + 1) * D], ref_pages[i, slot * D:(slot + 1) * D])
        assert np.array_equal(pg[inputs.FP8_DATA_BYTES + 4 * slot:inputs.FP8_DATA_BYTES + 4 * slot + 4],
                              ref_pages[i, inputs.FP8_DATA_BYTES + 4 * slot:inputs.FP8_DATA_BYTES + 4 * slot + 4])


@pytest.mark.parametrize("std", [1e-30, 1e-3, 0.5, 40.0, 3e30])
def test_fp8_quantiser_is_exact_over_many_rows(std):
    # 32,768 rows over magnitudes from tiny (scales near the fp32 subnormal
    # range) to huge: every code and scale equals the fp32-division rule.
    rng = np.random.default_rng(int(np.log10(std) + 50))
    B, T = 8192, 4
    x = rng.standard_normal((B, T, D)).astype(np.float32) * np.float32(std)
    x[:, :, ::7] *= np.float32(1e-3)                      # spread within rows too
    new = inputs.f32_to_bf16_bits(x)
    bt = np.arange(B, dtype=np.int32).reshape(B, 1)
    lens = np.full(B, 64, dtype=np.int32)                 # rows to slots 60..63 of page b
    cache = np.zeros((B, inputs.FP8_PAGE_BYTES), dtype=np.uint8)
    c_d = _to_dev(cache)
    mla.append(_to_dev(new), c_d, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), "fp8")
    torch.cuda.synchronize()
    got = c_d.cpu().numpy()
    codes, sigma = oracle.quantise_rows_fp8(new.reshape(-1, D))
    got_codes = got[:, 60 * D:64 * D].reshape(-1, D)
    got_sigma = got[:, inputs.FP8_DATA_BYTES + 240:inputs.FP8_DATA_BYTES + 256].copy().view("<f4").reshape(-1)
    assert np.array_equal(got_sigma, sigma)
    bad = np.argwhere(got_codes != codes)
    assert bad.size == 0, (bad[:5], got_codes[tuple(bad[0])], codes[tuple(bad[0])])
