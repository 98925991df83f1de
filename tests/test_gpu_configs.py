"""Full-size workloads (the shapes the benchmark and the decode targets use):
the CUDA path, in the launch configuration bench.py times (device planner with
the block-table check, all SMs), against the fp64 oracle on sampled (b, t, h)
rows, plus whole-tensor properties.

Row samples: every row where the oracle is cheap (the 50K step, the 128K
speculative step); elsewhere, for EVERY sequence, its first and last query
rows, the rows on each side of every 128-row tile boundary, and random rows.
A row's result depends on every split piece of its sequence, so a compared row
also checks that sequence's split/combine path at full size."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import LSE_TOL, TOL, to_device

pytestmark = pytest.mark.gpu

# (b, t, h) rows compared per sequence on the batched/long workloads (beyond
# the fixed ones), and workloads compared on every row.
RANDOM_ROWS_PER_SEQ = {"spec_256k": 24, "spec_1m": 8, "agentic": 6, "fp8": 3}
ALL_ROWS = {"tiny", "kimi_50k", "spec_128k"}


def sample_rows(w, name, seed=0):
    T, H = w.q_len, w.heads
    rows_per_seq = T * H
    if name in ALL_ROWS:
        return [(b, t, h) for b in range(w.batch) for t in range(T) for h in range(H)]
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(w.batch):
        picks = {0, rows_per_seq - 1}
        for edge in range(128, rows_per_seq, 128):   # both sides of each row-tile boundary
            picks.update({edge - 1, edge})
        picks.update(int(x) for x in rng.integers(0, rows_per_seq, size=RANDOM_ROWS_PER_SEQ[name]))
        rows.update((b, r // H, r % H) for r in picks)
    return sorted(rows)


@pytest.mark.parametrize("name", ["tiny", "kimi_50k", "spec_128k", "spec_256k", "spec_1m", "agentic", "fp8"])
def test_full_size_workload(name):
    w = inputs.WORKLOADS[name]()
    q, cache, bt, sl = to_device(w)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads, w.kv_dtype)
    out, lse = dec(q, cache, bt, sl, scale=w.scale)
    torch.cuda.synchronize()
    assert dec.device_flag() == 0
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
    rows = sample_rows(w, name)
    assert {b for (b, _, _) in rows} == set(range(w.batch))   # every sequence is compared
    ro, rl = oracle.mla_decode_ref_rows(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, rows, w.scale)
    got = np.stack([o[b, t, h] for (b, t, h) in rows])
    gl = np.array([l[b, t, h] for (b, t, h) in rows])
    atol, rl2 = TOL[w.kv_dtype]
    d = got - ro
    max_abs = float(np.abs(d).max())
    rel = float(np.linalg.norm(d) / np.linalg.norm(ro))
    lse_err = float(np.abs(gl - rl).max())
    # per-sequence relative error too, so that one bad sequence cannot hide in a batch's norm
    worst_seq = 0.0
    for b in range(w.batch):
        idx = [i for i, r in enumerate(rows) if r[0] == b]
        worst_seq = max(worst_seq, float(np.linalg.norm(d[idx]) / np.linalg.norm(ro[idx])))
    assert max_abs <= atol and rel <= rl2 and worst_seq <= rl2 and lse_err <= LSE_TOL, (
        name, len(rows), max_abs, rel, worst_seq, lse_err)
    # Property at any size: every output row is a convex combination of the
    # sequence's V rows (values ~N(0, 0.5), |x| < 4 in practice; fp8 codes x
    # sigma likewise).
    assert np.abs(o).max() <= 8.0
