"""Every e4m3 code through the fp8 cache path, exactly.

A one-token context gives that token softmax weight 1, so each output row is
the token's V row (first 512 latent columns) times its scale. With scale 1 the
output must equal the decoded codes bit for bit: every finite e4m3 value is a
bf16 value. The 512 V columns hold the 254 finite codes (twice, the second
copy reversed); NaN codes stand in the 63 masked tail tokens of the page,
whose scales are NaN too, and must not reach the result. Both tile heights
(16 heads: 64-row tiles, 128 heads: 128-row tiles) are checked against the
OCP E4M3 definition as decoded by the oracle and the golden table.
"""

from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp_table.txt")


def _finite_codes():
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def _page_with_all_codes():
    codes = _finite_codes()                                # 254 codes
    v = np.concatenate([codes, codes[::-1], np.zeros(4, np.uint8)])   # 512 columns
    page = np.full((inputs.PAGE, 576), 0x7F, dtype=np.uint8)         # tail tokens: NaN codes
    page[0, :512] = v
    page[0, 512:] = 0x38                                   # rope columns: 1.0
    scales = np.full(inputs.PAGE, np.nan, dtype="<f4")
    scales[0] = 1.0
    out = np.empty((2, inputs.FP8_PAGE_BYTES), dtype=np.uint8)
    for p in range(2):   # page 1 is never referenced; all NaN
        out[p, : inputs.PAGE * 576] = page.reshape(-1) if p == 0 else 0xFF
        out[p, inputs.PAGE * 576:] = scales.view(np.uint8) if p == 0 else 0xFF
    return out, v


def _golden_values():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                code, val = line.split()[:2]
                vals[int(code, 16)] = float(val)
    return vals


@pytest.mark.gpu
@pytest.mark.parametrize("heads", [16, 128])
def test_every_e4m3_code_exact(heads):
    pages, v_codes = _page_with_all_codes()
    rng = np.random.default_rng(heads)
    q_bits = inputs.f32_to_bf16_bits(rng.standard_normal((1, 1, heads, 576)).astype(np.float32) * 0.01)
    bt = np.zeros((1, 1), dtype=np.int32)
    sl = np.array([1], dtype=np.int32)
    scale = 1.0 / np.sqrt(192.0)

    q = torch.from_numpy(q_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    cache = torch.from_numpy(pages).cuda()
    dec = mla.MlaDecoder(1, 1, 1, heads, "fp8")
    out, lse = dec(q, cache, torch.from_numpy(bt).cuda(), torch.from_numpy(sl).cuda(), scale=scale)
    torch.cuda.synchronize()
    assert dec.device_flag() == 0
    got = out.float().cpu().numpy().astype(np.float64)[0, 0]          # [heads, 512]

    ref_out, ref_lse = oracle.mla_decode_ref(q_bits, pages, "fp8", bt, sl, scale)
    expect = oracle.decode_e4m3(v_codes)
    assert np.array_equal(ref_out[0, 0], np.broadcast_to(expect, (heads, 512)))
    # bit-exact against the definition, every head
    assert np.array_equal(got, np.broadcast_to(expect, (heads, 512))), (
        np.argwhere(got != expect)[:8], got[got != expect][:8])
    # and against the printed table entries that occur
    gold = _golden_values()
    for col, c in enumerate(v_codes[:508]):
        if int(c) in gold:
            assert got[0, col] == gold[int(c)] or (gold[int(c)] == 0.0 and got[0, col] == 0.0)
    assert np.abs(lse.cpu().numpy()[0, 0] - ref_lse[0, 0]).max() <= 1e-3
