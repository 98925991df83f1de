"""Full-size workloads (the shapes the benchmark and the decode targets use):
the CUDA path, in the launch configuration bench.py times, against the fp64
oracle on sampled (b, t, h) rows, plus whole-tensor properties."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import LSE_TOL, TOL, to_device

pytestmark = pytest.mark.gpu


def sample_rows(w, n=10, seed=0):
    rng = np.random.default_rng(seed)
    rows = {(0, 0, 0), (w.batch - 1, w.q_len - 1, w.heads - 1), (0, w.q_len - 1, w.heads // 2)}
    while len(rows) < n:
        rows.add((int(rng.integers(w.batch)), int(rng.integers(w.q_len)), int(rng.integers(w.heads))))
    return sorted(rows)


@pytest.mark.parametrize("name", ["tiny", "kimi_50k", "spec_128k", "spec_1m", "agentic", "fp8"])
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
    rows = sample_rows(w)
    ro, rl = oracle.mla_decode_ref_rows(w.q_bits, w.cache, w.kv_dtype, w.block_table, w.seqlens, rows, w.scale)
    got = np.stack([o[b, t, h] for (b, t, h) in rows])
    gl = np.array([l[b, t, h] for (b, t, h) in rows])
    atol, rl2 = TOL[w.kv_dtype]
    d = got - ro
    max_abs = float(np.abs(d).max())
    rel = float(np.linalg.norm(d) / np.linalg.norm(ro))
    lse_err = float(np.abs(gl - rl).max())
    assert max_abs <= atol and rel <= rl2 and lse_err <= LSE_TOL, (name, max_abs, rel, lse_err)
    # Property at any size: |out| is bounded by the largest |V| entry of the sequence's visible rows
    # (a convex combination); checked against a loose global bound.
    assert np.abs(o).max() <= 8.0
