"""GPU parity of the prefix-shared (cascade) decode (mla_decode_cascade,
through the C ABI) against the fp64 decode oracle over the whole sequences:
the prefix pass (all query rows of the batch over the shared pages), the
suffix pass and the LSE merge together must give the ordinary decode's
result within the bf16 tolerance."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import LSE_TOL, TOL, assert_close, to_device

pytestmark = pytest.mark.gpu


def run_cascade(w, prefix_len, tensors=None):
    q, cache, bt, sl = tensors if tensors is not None else to_device(w)
    out = torch.full((w.batch, w.q_len, w.heads, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.batch, w.q_len, w.heads), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = mla.cascade_workspace_size(w.batch, w.max_pages, w.q_len, w.heads, w.kv_dtype)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    mla.cascade(q, cache, bt, sl, prefix_len, out, lse, ws, w.kv_dtype, scale=w.scale)
    torch.cuda.synchronize()
    flag = mla.read_device_flag(ws)
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), flag


@pytest.mark.parametrize("B,H,T,lens,prefix,kv", [
    (4, 64, 2, [1000, 1400, 900, 2000], 640, "bf16"),
    (8, 16, 1, [700, 650, 900, 1300, 641, 1100, 2000, 777], 640, "bf16"),   # 8 sequences per row tile
    (3, 128, 4, [800, 1200, 900], 768, "bf16"),
    (5, 32, 3, [300, 500, 700, 260, 1000], 256, "fp8"),
    (2, 64, 1, [130, 200], 64, "bf16"),
    (2, 64, 2, [500, 600], 0, "bf16"),                                       # no prefix: an ordinary step
])
def test_cascade_matches_oracle(B, H, T, lens, prefix, kv):
    w = inputs.make_workload("cascade", batch=B, heads=H, q_len=T, seqlens=lens, kv_dtype=kv,
                             shared_prefix_tokens=max(prefix, 64), seed=sum(lens) + H)
    out, lse, flag = run_cascade(w, prefix)
    assert flag == 0
    ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, kv, w.block_table, w.seqlens, w.scale)
    assert_close(out, lse, ro, rl, kv_dtype=kv, what=f"cascade B{B} H{H} T{T} P{prefix} {kv}")
    # and the oracle's own cascade form agrees (prefix / suffix / merge)
    if prefix:
        co, cl = oracle.cascade_decode_ref(w.q_bits, w.cache, kv, w.block_table, w.seqlens, prefix, w.scale)
        assert np.allclose(co, ro, atol=1e-12) and np.allclose(cl, rl, atol=1e-12)


def test_cascade_flags_unshared_prefix_and_short_sequences():
    w = inputs.make_workload("cflags", batch=4, heads=16, q_len=2, seqlens=[900, 1000, 700, 800],
                             shared_prefix_tokens=640, seed=5)
    q, cache, bt, sl = to_device(w)
    bt_bad = bt.clone()
    bt_bad[2, 3] = bt[2, 12]                                   # sequence 2's prefix page 3 is not shared
    _, _, flag = run_cascade(w, 640, (q, cache, bt_bad, sl))
    assert flag & mla.FLAG_BAD_PREFIX
    sl_short = sl.clone()
    sl_short[1] = 641                                          # 641 < 640 + q_len
    out, lse, flag = run_cascade(w, 640, (q, cache, bt, sl_short))
    assert flag & mla.FLAG_BAD_SEQLEN and not (flag & mla.FLAG_BAD_PREFIX)
    assert np.all(np.isnan(out[1]))
    keep = [0, 2, 3]
    ro, rl = oracle.mla_decode_ref(w.q_bits[keep], w.cache, "bf16", w.block_table[keep], w.seqlens[keep], w.scale)
    assert_close(out[keep], lse[keep], ro, rl, what="rows next to a too-short sequence")


@pytest.mark.parametrize("name", ["agentic", "prefix_h16"])
def test_full_size_cascade(name):
    # the batch's own shared prefix (page-aligned, short of every sequence's new tokens); every
    # sequence's first and last rows, the tile-boundary rows and random rows against the oracle
    w = inputs.WORKLOADS[name]()
    prefix = inputs.cascade_prefix_len(w)
    assert prefix >= 20 * 1024
    out, lse, flag = run_cascade(w, prefix)
    assert flag == 0 and np.all(np.isfinite(out))
    rng = np.random.default_rng(3)
    rows = set()
    n = w.q_len * w.heads
    for b in range(w.batch):
        picks = {0, n - 1} | {int(x) for x in rng.integers(0, n, size=4)}
        rows.update((b, r // w.heads, r % w.heads) for r in picks)
    rows = sorted(rows)
    ro, rl = oracle.mla_decode_ref_rows(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, rows, w.scale)
    got = np.stack([out[b, t, h] for (b, t, h) in rows])
    gl = np.array([lse[b, t, h] for (b, t, h) in rows])
    atol, rl2 = TOL[w.kv_dtype]
    d = got - ro
    assert np.abs(d).max() <= atol and np.linalg.norm(d) / np.linalg.norm(ro) <= rl2
    assert np.abs(gl - rl).max() <= LSE_TOL
