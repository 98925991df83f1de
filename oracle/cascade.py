"""Plain CPU oracle for the prefix-shared (cascade) decode: attention over a
shared prefix and over each sequence's own suffix, merged by their
log-sum-exp weights.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). The pages describe
multi-turn agentic serving with prefix reuse across KV pages (zubnet.ai,
"LightSeek TokenSpeed 580 TPS ... B200", second paragraph: hybrid prefix
caching; 24-ai.news "TokenSpeed ... 580 token/s", optimisations list: prefix
caching with a KV hit rate above 90%). Splitting a row's visible tokens into
two disjoint sets A (the shared prefix) and B (the rest) and attending to
each gives (out_A, lse_A) and (out_B, lse_B); the attention over A u B is

    lse = log(exp(lse_A) + exp(lse_B))
    out = exp(lse_A - lse) out_A + exp(lse_B - lse) out_B

(a set a row does not see has lse = -inf and weight 0). Pinned by
``tests/test_oracle_pins.py``: the merge of two disjoint token sets equals
the decode oracle over their union, for several split points.
"""

from __future__ import annotations

import numpy as np

from .mla_oracle import PAGE, attend_rows, decode_bf16, gather_latent


def merge_states(out_a, lse_a, out_b, lse_b):
    """LSE-weighted merge of two partial attention results over disjoint token sets."""
    out_a, out_b = np.asarray(out_a, np.float64), np.asarray(out_b, np.float64)
    lse_a, lse_b = np.asarray(lse_a, np.float64), np.asarray(lse_b, np.float64)
    m = np.maximum(lse_a, lse_b)
    m = np.where(np.isfinite(m), m, 0.0)
    wa = np.exp(lse_a - m)
    wb = np.exp(lse_b - m)
    den = wa + wb
    lse = m + np.log(den)
    out = (wa[..., None] * out_a + wb[..., None] * out_b) / den[..., None]
    return out, lse


def cascade_decode_ref(q_bits, cache, kv_dtype, block_table, seqlens, prefix_len, scale=1.0 / np.sqrt(192.0)):
    """Cascade form of the decode oracle: every row attends to the first
    ``prefix_len`` tokens of its sequence (the shared prefix, all of it
    visible) and, separately, to tokens prefix_len .. L_b - 1 under the causal
    rule; the two are merged. Requires L_b >= prefix_len + T. Equals
    ``mla_decode_ref`` up to rounding. Returns out [B, T, H, 512], lse [B, T, H]."""
    q = decode_bf16(q_bits)
    B, T, H, _ = q.shape
    out = np.empty((B, T, H, 512))
    lse = np.empty((B, T, H))
    for b in range(B):
        L = int(seqlens[b])
        if L < prefix_len + T:
            raise ValueError(f"sequence {b}: length {L} < prefix {prefix_len} + q_len {T}")
        K = gather_latent(cache, kv_dtype, block_table, b, L)
        rows = q[b].reshape(T * H, 576)
        vis_pre = np.full(T * H, prefix_len)
        vis_suf = np.repeat(np.array([L - T + t + 1 - prefix_len for t in range(T)]), H)
        if prefix_len > 0:
            oa, la = attend_rows(rows, K[:prefix_len], vis_pre, scale)
        else:
            oa, la = np.zeros((T * H, 512)), np.full(T * H, -np.inf)
        ob, lb = attend_rows(rows, K[prefix_len:], vis_suf, scale)
        o, l = merge_states(oa, la, ob, lb)
        out[b] = o.reshape(T, H, 512)
        lse[b] = l.reshape(T, H)
    return out, lse


__all__ = ["merge_states", "cascade_decode_ref", "PAGE"]
