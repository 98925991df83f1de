"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test targets a mistake the oracle could plausibly contain (wrong gather
index, wrong causal offset, wrong scale, dropped rope term, wrong lse base,
mis-decoded element formats, mis-applied fp8 scale) and fails if it is there.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import D_QK, D_V, PAGE, FP8_PAGE_BYTES
from mla_paged_kv_05_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
S192 = 1.0 / math.sqrt(192.0)


def bf16_bits(x):
    return inputs.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def paged(rows_bits, rng, extra=1):
    """Scatter logical rows [L, 576] (uint16) into a shuffled page pool."""
    L = rows_bits.shape[0]
    n = (L + PAGE - 1) // PAGE
    pool = n + extra
    perm = rng.permutation(pool)
    cache = np.full((pool, PAGE, D_QK), inputs.BF16_NAN, dtype=np.uint16)
    bt = np.zeros((1, n), dtype=np.int32)
    for i in range(n):
        bt[0, i] = perm[i]
        seg = rows_bits[i * PAGE:(i + 1) * PAGE]
        cache[perm[i], :seg.shape[0]] = seg
    return cache, bt


# ---------------------------------------------------------------- decoders

def test_bf16_decode_known_encodings():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x7F80, 0x4049, 0x0001], dtype=np.uint16)
    v = oracle.decode_bf16(bits)
    assert v[0] == 1.0 and v[1] == -2.0 and v[2] == 0.0 and math.copysign(1, v[3]) < 0
    assert math.isinf(v[4]) and v[5] == 3.140625 and v[6] == 2.0 ** -133


def test_bf16_decode_matches_torch_on_all_finite_patterns():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_e4m3_decode_matches_ocp_table():
    with open(os.path.join(GOLDEN, "e4m3_ocp_table.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            code, val = line.split()
            got = oracle.decode_e4m3(np.array([int(code, 16)], dtype=np.uint8))[0]
            if val == "nan":
                assert math.isnan(got), code
            else:
                assert got == float(val), (code, got, val)
                assert math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode_e4m3(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


# ---------------------------------------------------------------- gather + causal mask

@pytest.mark.parametrize("L,T", [(1, 1), (5, 1), (63, 2), (64, 4), (65, 3), (200, 4), (130, 1)])
def test_one_hot_rows_identify_the_visible_tokens(L, T):
    """q = 0 makes every visible token weigh 1/|vis|. Row j's V is the one-hot
    e_(j mod 512) (plus a marker in column j // 512 + 1 style), so the output
    names exactly which logical tokens were gathered for each query t."""
    rng = np.random.default_rng(L * 10 + T)
    rows = np.zeros((L, D_QK), dtype=np.float32)
    for j in range(L):
        rows[j, j % D_V] = 1.0
        rows[j, D_V + (j % 64)] = rng.standard_normal()      # rope part: must not matter
    cache, bt = paged(bf16_bits(rows), rng)
    H = 2
    q = np.zeros((1, T, H, D_QK), dtype=np.uint16)
    out, lse = oracle.mla_decode_ref(q, cache, "bf16", bt, np.array([L]))
    for t in range(T):
        nvis = L - T + t + 1
        expect = np.zeros(D_V)
        for j in range(nvis):
            expect[j % D_V] += 1.0 / nvis
        for h in range(H):
            np.testing.assert_allclose(out[0, t, h], expect, rtol=0, atol=1e-15)
            assert abs(lse[0, t, h] - math.log(nvis)) < 1e-13


def test_two_token_closed_form_scores_scale_and_rope():
    """z_j = s <q, k_j> with s = 1/sqrt(192); the rope columns count."""
    a, b = 3.0, -1.0                 # latent contributions
    ra, rb = 0.5, 2.0                # rope contributions
    rows = np.zeros((2, D_QK), dtype=np.float32)
    rows[0, 7] = a; rows[0, D_V + 3] = ra; rows[0, 100] = 5.0
    rows[1, 7] = b; rows[1, D_V + 3] = rb; rows[1, 200] = -4.0
    qv = np.zeros((1, 1, 1, D_QK), dtype=np.float32)
    qv[0, 0, 0, 7] = 2.0
    qv[0, 0, 0, D_V + 3] = 4.0
    rng = np.random.default_rng(7)
    cache, bt = paged(bf16_bits(rows), rng)
    out, lse = oracle.mla_decode_ref(bf16_bits(qv), cache, "bf16", bt, np.array([2]))
    z0 = S192 * (2.0 * a + 4.0 * ra)
    z1 = S192 * (2.0 * b + 4.0 * rb)
    w0 = 1.0 / (1.0 + math.exp(z1 - z0))
    w1 = 1.0 - w0
    expect = np.zeros(D_V)
    expect[7] = w0 * a + w1 * b
    expect[100] = w0 * 5.0
    expect[200] = w1 * -4.0
    np.testing.assert_allclose(out[0, 0, 0], expect, rtol=1e-14, atol=1e-14)
    assert abs(lse[0, 0, 0] - math.log(math.exp(z0) + math.exp(z1))) < 1e-14


def test_constant_v_gives_v():
    rng = np.random.default_rng(11)
    L, T, H = 150, 3, 4
    v = rng.standard_normal(D_V).astype(np.float32)
    rows = rng.standard_normal((L, D_QK)).astype(np.float32)
    rows[:, :D_V] = v
    # the latent also feeds the scores; make scores vary through the rope part only
    cache, bt = paged(bf16_bits(rows), rng)
    q = bf16_bits(rng.standard_normal((1, T, H, D_QK)))
    out, _ = oracle.mla_decode_ref(q, cache, "bf16", bt, np.array([L]))
    vb = inputs.bf16_bits_to_f32(bf16_bits(v)).astype(np.float64)
    for t in range(T):
        for h in range(H):
            np.testing.assert_allclose(out[0, t, h], vb, rtol=1e-12, atol=1e-12)


def test_single_token_context_returns_its_v_and_score():
    rng = np.random.default_rng(12)
    row = rng.standard_normal((1, D_QK)).astype(np.float32)
    qv = rng.standard_normal((1, 1, 3, D_QK)).astype(np.float32)
    cache, bt = paged(bf16_bits(row), rng)
    qb = bf16_bits(qv)
    out, lse = oracle.mla_decode_ref(qb, cache, "bf16", bt, np.array([1]))
    rk = inputs.bf16_bits_to_f32(bf16_bits(row)).astype(np.float64)[0]
    qf = inputs.bf16_bits_to_f32(qb).astype(np.float64)
    for h in range(3):
        np.testing.assert_array_equal(out[0, 0, h], rk[:D_V])
        z = S192 * float(np.dot(qf[0, 0, h], rk))
        assert abs(lse[0, 0, h] - z) < 1e-12


def test_page_scramble_is_bitwise_invariant():
    w = inputs.make_workload("t", batch=3, heads=4, q_len=2, seqlens=[130, 64, 7], seed=3)
    out1, lse1 = oracle.mla_decode_ref(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens)
    rng = np.random.default_rng(99)
    pi = rng.permutation(w.num_pages)
    cache2 = np.empty_like(w.cache)
    cache2[pi] = w.cache
    bt2 = pi[w.block_table].astype(np.int32)
    out2, lse2 = oracle.mla_decode_ref(w.q_bits, cache2, "bf16", bt2, w.seqlens)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_causal_rows_equal_shorter_single_query_contexts():
    w = inputs.make_workload("t", batch=1, heads=3, q_len=4, seqlens=[131], seed=5)
    out, lse = oracle.mla_decode_ref(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens)
    for t in range(4):
        Lp = 131 - 4 + t + 1
        q1 = w.q_bits[:, t:t + 1]
        o1, l1 = oracle.mla_decode_ref(q1, w.cache, "bf16", w.block_table, np.array([Lp]))
        np.testing.assert_allclose(out[0, t], o1[0, 0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[0, t], l1[0, 0], rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- absorbed == un-absorbed

def test_absorbed_form_matches_unabsorbed_mla():
    """With integer W_UK and q_nope the absorbed query W_UK^T q_nope is exact in
    bf16, so the public oracle (bf16 inputs) can be compared with explicit
    per-head up-projection (fp64)."""
    rng = np.random.default_rng(21)
    H, T, L = 3, 2, 97
    W_UK = rng.integers(-1, 2, size=(H, 128, D_V)).astype(np.float64)
    W_UV = rng.standard_normal((H, 128, D_V))
    q_nope = rng.integers(-2, 3, size=(T, H, 128)).astype(np.float64)
    q_rope = inputs.bf16_bits_to_f32(bf16_bits(rng.standard_normal((T, H, 64)))).astype(np.float64)
    c = inputs.bf16_bits_to_f32(bf16_bits(rng.standard_normal((L, D_V)) * 0.05)).astype(np.float64)
    k_rope = inputs.bf16_bits_to_f32(bf16_bits(rng.standard_normal((L, 64)))).astype(np.float64)
    q_abs = np.zeros((1, T, H, D_QK))
    for t in range(T):
        for h in range(H):
            q_abs[0, t, h, :D_V] = W_UK[h].T @ q_nope[t, h]
            q_abs[0, t, h, D_V:] = q_rope[t, h]
    assert np.abs(q_abs).max() < 256           # integers below 256 are exact in bf16
    qb = bf16_bits(q_abs)
    assert np.array_equal(inputs.bf16_bits_to_f32(qb), q_abs.astype(np.float32))
    cache, bt = paged(bf16_bits(np.concatenate([c, k_rope], axis=1)), rng)
    out, lse = oracle.mla_decode_ref(qb, cache, "bf16", bt, np.array([L]))
    for h in range(H):
        vis = [L - T + t + 1 for t in range(T)]
        o_un, l_un = oracle.unabsorbed_mla(q_nope[:, h], q_rope[:, h], W_UK[h], W_UV[h], c, k_rope, vis)
        for t in range(T):
            np.testing.assert_allclose(W_UV[h] @ out[0, t, h], o_un[t], rtol=1e-10, atol=1e-12)
            assert abs(lse[0, t, h] - l_un[t]) < 1e-11


def test_unabsorbed_reference_against_hand_computed_two_tokens():
    """Pins the un-absorbed helper itself (so the absorption pin is not circular)."""
    W_UK = np.zeros((128, D_V)); W_UK[0, 0] = 1.0
    W_UV = np.zeros((128, D_V)); W_UV[5, 0] = 2.0
    c = np.zeros((2, D_V)); c[0, 0] = 1.0; c[1, 0] = -1.0
    k_rope = np.zeros((2, 64)); k_rope[1, 0] = 3.0
    q_nope = np.zeros((1, 128)); q_nope[0, 0] = 2.0
    q_rope = np.zeros((1, 64)); q_rope[0, 0] = 1.0
    o, l = oracle.unabsorbed_mla(q_nope, q_rope, W_UK, W_UV, c, k_rope, [2])
    z0, z1 = S192 * 2.0, S192 * (-2.0 + 3.0)
    w0 = math.exp(z0) / (math.exp(z0) + math.exp(z1))
    assert abs(o[0, 5] - (w0 * 2.0 + (1 - w0) * -2.0)) < 1e-14
    assert abs(l[0] - math.log(math.exp(z0) + math.exp(z1))) < 1e-14


# ---------------------------------------------------------------- fp8 cache

def test_fp8_with_power_of_two_scales_equals_bf16_path():
    """Codes x 2^k are exact in bf16, so the fp8 oracle must equal the bf16
    oracle on the decoded cache, bit for bit."""
    rng = np.random.default_rng(31)
    L, T, H = 100, 2, 2
    n = (L + PAGE - 1) // PAGE
    codes = rng.integers(0, 256, size=(n, PAGE, D_QK)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3A                    # no NaN codes
    exps = rng.integers(-6, 3, size=(n, PAGE))
    scales = np.ldexp(1.0, exps).astype(np.float32)
    fp8 = np.zeros((n, FP8_PAGE_BYTES), dtype=np.uint8)
    fp8[:, :PAGE * D_QK] = codes.reshape(n, -1)
    fp8[:, PAGE * D_QK:] = scales.astype("<f4").view(np.uint8).reshape(n, -1)
    vals = oracle.decode_e4m3(codes) * scales[..., None].astype(np.float64)
    bf = bf16_bits(vals.astype(np.float32))
    assert np.array_equal(inputs.bf16_bits_to_f32(bf).astype(np.float64), vals)
    bt = rng.permutation(n).astype(np.int32)[None, :]
    fp8 = fp8[np.argsort(bt[0])]                 # physical page bt[0,i] holds logical page i
    bf = bf[np.argsort(bt[0])]
    q = bf16_bits(rng.standard_normal((1, T, H, D_QK)))
    o8, l8 = oracle.mla_decode_ref(q, fp8, "fp8", bt, np.array([L]))
    ob, lb = oracle.mla_decode_ref(q, bf, "bf16", bt, np.array([L]))
    assert np.array_equal(o8, ob) and np.array_equal(l8, lb)


def test_fp8_scale_multiplies_the_token_row():
    """Doubling one token's scale doubles that token's V in a q=0 average."""
    rng = np.random.default_rng(32)
    L = 10
    codes = np.zeros((1, PAGE, D_QK), dtype=np.uint8)
    codes[0, :L, 0] = 0x38                                  # 1.0
    scales = np.ones((1, PAGE), dtype=np.float32)
    scales[0, 3] = 0.75
    fp8 = np.zeros((1, FP8_PAGE_BYTES), dtype=np.uint8)
    fp8[0, :PAGE * D_QK] = codes.reshape(-1)
    fp8[0, PAGE * D_QK:] = scales.view(np.uint8).reshape(-1)
    q = np.zeros((1, 1, 1, D_QK), dtype=np.uint16)
    out, _ = oracle.mla_decode_ref(q, fp8, "fp8", np.zeros((1, 1), np.int32), np.array([L]))
    assert abs(out[0, 0, 0, 0] - (9 * 1.0 + 0.75) / 10) < 1e-15


# ---------------------------------------------------------------- row sampler

def test_row_sampler_matches_whole_batch_oracle():
    w = inputs.make_workload("t", batch=2, heads=4, q_len=3, seqlens=[300, 129], seed=8)
    out, lse = oracle.mla_decode_ref(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens)
    rows = [(0, 0, 0), (0, 2, 3), (1, 1, 2), (1, 2, 0)]
    o, l = oracle.mla_decode_ref_rows(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens,
                                      rows, chunk_tokens=100)
    for i, (b, t, h) in enumerate(rows):
        np.testing.assert_allclose(o[i], out[b, t, h], rtol=1e-12, atol=1e-13)
        assert abs(l[i] - lse[b, t, h]) < 1e-12


def test_generated_fp8_cache_decodes_near_its_bf16_source():
    """The cache writer's e4m3 encoding stays within half an e4m3 ulp (2^-4
    relative) of the bf16 row it encodes."""
    w = inputs.make_workload("t", batch=1, heads=1, q_len=1, seqlens=[64], seed=9, poison=False)
    src = inputs.bf16_bits_to_f32(w.cache).astype(np.float64)
    enc = inputs.encode_fp8_pages(w.cache)
    codes = enc[:, :PAGE * D_QK].reshape(-1, PAGE, D_QK)
    sc = enc[:, PAGE * D_QK:].copy().view("<f4").reshape(-1, PAGE).astype(np.float64)
    dec = oracle.decode_e4m3(codes) * sc[..., None]
    err = np.abs(dec - src)
    bound = np.maximum(np.abs(src) * 2.0 ** -4, sc[..., None] * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-9))


# ---------------------------------------------------------------- cache append (fp8 quantise-on-write)

def _all_finite_e4m3_codes():
    c = np.arange(256, dtype=np.uint8)
    return c[(c & 0x7F) != 0x7F]


def test_e4m3_encode_round_trips_every_finite_code():
    codes = _all_finite_e4m3_codes()
    vals = oracle.decode_e4m3(codes).astype(np.float32)
    assert np.array_equal(oracle.encode_e4m3(vals), codes)


def test_e4m3_encode_ties_go_to_the_even_code_and_others_to_the_nearer():
    pos = oracle.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)   # midpoints are exact in fp32
    lo = np.arange(0x7E)
    got = oracle.encode_e4m3(mids)
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, lo + 1))
    below = np.nextafter(mids, np.float32(-np.inf))
    above = np.nextafter(mids, np.float32(np.inf))
    assert np.array_equal(oracle.encode_e4m3(below), lo)
    assert np.array_equal(oracle.encode_e4m3(above), lo + 1)


def test_e4m3_encode_saturates_and_keeps_the_sign():
    got = oracle.encode_e4m3(np.array([448.0, 460.0, 464.0, 1e30, -1000.0, -0.0, 0.0], dtype=np.float32))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x00]


def test_e4m3_encode_matches_torch_conversion():
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 10.0, 150.0)]).astype(np.float32)
    y = np.clip(y, -448.0, 448.0)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_e4m3(y), ref)


def test_fp8_row_quantiser_hand_computed_row():
    x = np.zeros(D_QK, dtype=np.float32)
    x[:4] = [3.5, 1.75, -0.5, 0.0]
    x[100] = -2.0 ** -20            # far below one code step: rounds to -0
    codes, sigma = oracle.quantise_rows_fp8(bf16_bits(x)[None, :])
    assert sigma[0] == np.float32(3.5 / 448.0) == np.float32(2.0 ** -7)
    # 3.5 / 2^-7 = 448 -> 0x7E; 224 = 1.75 * 2^7 -> 0x76; -64 = -(2^6) -> 0xE8; 0 -> 0x00
    assert list(codes[0, :4]) == [0x7E, 0x76, 0xE8, 0x00]
    assert codes[0, 100] == 0x80 and not codes[0, 4:100].any() and not codes[0, 101:].any()
    z_codes, z_sigma = oracle.quantise_rows_fp8(np.zeros((1, D_QK), dtype=np.uint16))
    assert z_sigma[0] == 1.0 and not z_codes.any()


def test_fp8_row_quantiser_matches_the_torch_cache_writer():
    # The input generator's fp8 writer (torch ops) and the oracle (own encoder)
    # implement the same rule independently.
    rng = np.random.default_rng(4)
    rows = bf16_bits(rng.standard_normal((3, PAGE, D_QK)).astype(np.float32) * 0.5)
    rows[0, 5] = 0                                          # a zero row: sigma 1
    pages = inputs.encode_fp8_pages(rows)
    codes, sigma = oracle.quantise_rows_fp8(rows.reshape(-1, D_QK))
    assert np.array_equal(pages[:, :PAGE * D_QK].reshape(-1, D_QK), codes)
    assert np.array_equal(pages[:, PAGE * D_QK:].copy().view("<f4").reshape(-1), sigma)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_cache_append_writes_the_last_positions_through_the_block_table(kv_dtype):
    # L = 66, T = 3: tokens 63, 64, 65 -> page bt[0] slot 63, page bt[1] slots 0 and 1.
    rng = np.random.default_rng(5)
    if kv_dtype == "bf16":
        cache = rng.integers(0, 1 << 16, size=(5, PAGE, D_QK), dtype=np.uint16)
    else:
        cache = rng.integers(0, 256, size=(5, FP8_PAGE_BYTES), dtype=np.uint8)
    bt = np.array([[3, 1, 4]], dtype=np.int32)
    new = bf16_bits(rng.standard_normal((1, 3, D_QK)).astype(np.float32))
    out = oracle.cache_append_ref(cache, kv_dtype, new, bt, np.array([66]))
    written = [(3, 63), (1, 0), (1, 1)]
    for t, (page, slot) in enumerate(written):
        if kv_dtype == "bf16":
            assert np.array_equal(out[page, slot], new[0, t])
        else:
            codes, sigma = oracle.quantise_rows_fp8(new[0, t][None, :])
            assert np.array_equal(out[page, slot * D_QK:(slot + 1) * D_QK], codes[0])
            assert out[page, PAGE * D_QK:].copy().view("<f4")[slot] == sigma[0]
    # everything else is untouched
    mask = np.ones(out.shape[:2] if kv_dtype == "bf16" else out.shape, dtype=bool)
    for page, slot in written:
        if kv_dtype == "bf16":
            mask[page, slot] = False
        else:
            mask[page, slot * D_QK:(slot + 1) * D_QK] = False
            mask[page, PAGE * D_QK + 4 * slot:PAGE * D_QK + 4 * slot + 4] = False
    assert np.array_equal(out[mask], cache[mask])
    # a sequence shorter than q_len is invalid and writes nothing
    assert np.array_equal(oracle.cache_append_ref(cache, kv_dtype, new, bt, np.array([2])), cache)


def test_decoded_fp8_append_is_within_one_code_step_of_the_row():
    rng = np.random.default_rng(6)
    row = bf16_bits(rng.standard_normal((1, D_QK)).astype(np.float32))
    codes, sigma = oracle.quantise_rows_fp8(row)
    back = oracle.decode_e4m3(codes[0]) * float(sigma[0])
    x = oracle.decode_bf16(row[0])
    # e4m3 has 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    big = np.abs(x) >= 2.0 ** -6 * float(sigma[0])
    assert np.all(np.abs(back[big] - x[big]) <= 2.0 ** -4 * np.abs(x[big]) + 1e-12)


# ---------------------------------------------------------------- absorbed projections

def test_absorb_and_project_hand_computed():
    # one token, one head, integer entries: q_nope = e_0 + 2 e_1, W_UK rows 0/1 known
    q = np.zeros((1, 1, 192))
    q[0, 0, 0], q[0, 0, 1] = 1.0, 2.0
    q[0, 0, 128:192] = np.arange(64)
    w_uk = np.zeros((1, 128, 512))
    w_uk[0, 0, 3], w_uk[0, 1, 3], w_uk[0, 1, 7] = 5.0, -1.0, 4.0
    qt = oracle.absorb_q(q, w_uk)
    expect = np.zeros(576)
    expect[3] = 1 * 5 + 2 * (-1)
    expect[7] = 2 * 4
    expect[512:] = np.arange(64)
    assert np.array_equal(qt[0, 0], expect)
    o = np.zeros((1, 1, 512))
    o[0, 0, 3], o[0, 0, 7] = 2.0, -3.0
    w_uv = np.zeros((1, 128, 512))
    w_uv[0, 10, 3], w_uv[0, 10, 7], w_uv[0, 11, 7] = 1.0, 1.0, 2.0
    y = oracle.project_out(o, w_uv)
    expect_y = np.zeros(128)
    expect_y[10] = 2.0 - 3.0
    expect_y[11] = -6.0
    assert np.array_equal(y[0, 0], expect_y)


def test_absorbed_pipeline_equals_unabsorbed_attention():
    # absorb -> decode oracle on the latent cache -> project == per-head un-absorbed MLA
    rng = np.random.default_rng(21)
    H, T, L = 3, 2, 150
    c = rng.standard_normal((L, 512)) * 0.5
    k_rope = rng.standard_normal((L, 64)) * 0.5
    q = rng.standard_normal((T, H, 192))
    w_uk = rng.standard_normal((H, 128, 512)) * 0.05
    w_uv = rng.standard_normal((H, 128, 512)) * 0.05
    qt = oracle.absorb_q(q, w_uk)                                   # [T, H, 576]
    K = np.concatenate([c, k_rope], axis=1)
    vis = np.repeat(np.array([L - T + t + 1 for t in range(T)]), H)
    o, lse = oracle.attend_rows(qt.reshape(T * H, 576), K, vis, S192)
    y = oracle.project_out(o.reshape(T, H, 512), w_uv)
    for h in range(H):
        ref_o, ref_lse = oracle.unabsorbed_mla(q[:, h, :128], q[:, h, 128:], w_uk[h], w_uv[h], c, k_rope,
                                               vis[h::H], S192)
        assert np.allclose(y[:, h], ref_o, rtol=1e-11, atol=1e-12)
        assert np.allclose(lse.reshape(T, H)[:, h], ref_lse, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- cascade (prefix-shared) decode

@pytest.mark.parametrize("prefix", [0, 64, 128, 320])
def test_cascade_merge_equals_whole_sequence_attention(prefix):
    # two disjoint token sets merged by their lse == the decode oracle over the union
    w = inputs.make_workload("casc", batch=3, heads=8, q_len=2, seqlens=[400, 330, 520], seed=31,
                             shared_prefix_tokens=320)
    ref_o, ref_l = oracle.mla_decode_ref(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens, w.scale)
    o, l = oracle.cascade_decode_ref(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens, prefix, w.scale)
    assert np.allclose(o, ref_o, rtol=1e-12, atol=1e-13) and np.allclose(l, ref_l, rtol=1e-13, atol=1e-12)


def test_merge_states_closed_forms():
    a = np.array([[1.0, 2.0]]); b = np.array([[3.0, -1.0]])
    # equal lse: the plain average, lse + ln 2
    o, l = oracle.merge_states(a, np.array([0.5]), b, np.array([0.5]))
    assert np.allclose(o, [[2.0, 0.5]]) and np.isclose(l[0], 0.5 + math.log(2.0))
    # a set the row does not see (lse = -inf) has weight 0
    o, l = oracle.merge_states(a, np.array([-np.inf]), b, np.array([1.25]))
    assert np.array_equal(o, b) and l[0] == 1.25
    # weights e^(lse - lse*): lse_a = ln 3, lse_b = 0 -> 3/4 and 1/4
    o, l = oracle.merge_states(a, np.array([math.log(3.0)]), b, np.array([0.0]))
    assert np.allclose(o, 0.75 * a + 0.25 * b) and np.isclose(l[0], math.log(4.0))
