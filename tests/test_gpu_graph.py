"""CUDA-graph capture of plan + run: replays with new seqlens / block-table
contents (same shapes) stay correct and are bitwise deterministic."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import assert_close, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,T", [(64, 1), (128, 2)])
def test_graph_replay_with_changed_contents(H, T):
    w1 = inputs.make_workload("g1", batch=3, heads=H, q_len=T, seqlens=[1500, 700, 90], seed=21, extra_pages=20)
    q, cache, bt, sl = to_device(w1)
    dec = mla.MlaDecoder(w1.batch, w1.max_pages, T, H)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        dec(q, cache, bt, sl)              # warm-up outside capture
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        dec(q, cache, bt, sl, stream=stream)
    for seed, lens in [(22, [1500, 700, 90]), (23, [64, 1501, 1000]), (24, [T, 33, 1536])]:
        w = inputs.make_workload("g", batch=3, heads=H, q_len=T, seqlens=lens, seed=seed,
                                 max_pages=w1.max_pages)
        q2, cache2, bt2, sl2 = to_device(w)
        assert cache2.shape[0] <= cache.shape[0]
        cache[:cache2.shape[0]].copy_(cache2)
        q.copy_(q2)
        bt.copy_(bt2)
        sl.copy_(sl2)
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        o1, l1 = dec.out.clone(), dec.lse.clone()
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        assert torch.equal(o1, dec.out) and torch.equal(l1, dec.lse)
        assert dec.device_flag(stream) == 0
        ro, rl = oracle.mla_decode_ref(w.q_bits, w.cache, "bf16", w.block_table, w.seqlens)
        assert_close(o1.float().cpu().numpy().astype(np.float64), l1.cpu().numpy().astype(np.float64), ro, rl,
                     what=f"replay lens={lens}")
