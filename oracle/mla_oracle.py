"""Plain, slow, obviously-correct fp64 oracle for absorbed-MLA decode attention
over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). Written from the pages'
description, not from any kernel:

* evermx.com, "TokenSpeed: speed-of-light LLM inference engine for agentic
  workloads", section "Pluggable Kernel Registry": the subject is an MLA
  (Multi-head Latent Attention) decode kernel, used under speculative decoding.
* zubnet.ai (es/fr), "LightSeek TokenSpeed 580 TPS ... B200", second paragraph:
  KV lives in pages and decode reads them through index indirection instead of
  copies; the whole decode step is CUDA-graph captured.

The pages give no formula, so the oracle is the textbook definition of
absorbed MLA decode (DeepSeek-V2/V3 style), with these readings:

* one latent row per token, 576 wide = 512 compressed latent + 64 RoPE dims,
  shared by every head; V is the first 512 columns of the same row;
* the query rows are already absorbed: q~ = [W_UK^T q_nope | q_rope] (576 wide);
* score scale s = 1/sqrt(192) (the un-absorbed per-head QK width 128 + 64);
* pages of 64 tokens; token j of sequence b sits in physical page
  ``block_table[b, j // 64]`` at slot ``j % 64``;
* the T query tokens of a step are the last T positions of the sequence
  (already counted in ``seqlens``): query t sees tokens j <= L_b - T + t;
* lse is the natural log of the softmax denominator of the scaled scores.

For every b, t, h::

    K_b[j]  = cache[block_table[b, j // 64], j % 64]          (j < L_b)
    z_j     = s * <q[b,t,h], K_b[j]>                            (j visible)
    lse     = log sum_j exp(z_j)
    out     = sum_j exp(z_j - lse) * K_b[j, :512]

Every function below is pinned by ``tests/test_oracle_pins.py`` to closed
forms, invariants, an independent decoder (torch) and the OCP FP8 table.
"""

from __future__ import annotations

import numpy as np

D_QK = 576          # latent (512) + rope (64) width of one cache row
D_V = 512           # V = first 512 columns of the row
PAGE = 64           # tokens per page
# fp8 page: 64 x 576 e4m3 codes, then 64 little-endian fp32 per-token scales.
FP8_DATA_BYTES = PAGE * D_QK
FP8_PAGE_BYTES = FP8_DATA_BYTES + PAGE * 4


# ---------------------------------------------------------------------------
# Element decoders (format definitions)
# ---------------------------------------------------------------------------

def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64.

    bfloat16 is the upper half of an IEEE-754 binary32 word: placing the 16
    bits in the high half of a 32-bit word gives the same value as binary32.
    """
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 codes (uint8) -> float64, from the format definition.

    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0
    encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there are no infinities.
    (OCP 8-bit Floating Point Specification, v1.0, section 5.3.)
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = (m / 8.0) * 2.0 ** -6
    val = np.where(e == 0, subnormal, normal)
    val = np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)
    return sign * val


# ---------------------------------------------------------------------------
# Paged gather
# ---------------------------------------------------------------------------

def _page_rows(cache: np.ndarray, kv_dtype: str, page: int) -> np.ndarray:
    """One physical page as float64 [64, 576] (fp8: code value x token scale)."""
    if kv_dtype == "bf16":
        return decode_bf16(cache[page])
    if kv_dtype == "fp8":
        raw = np.asarray(cache[page], dtype=np.uint8)
        codes = raw[:FP8_DATA_BYTES].reshape(PAGE, D_QK)
        scales = raw[FP8_DATA_BYTES:FP8_PAGE_BYTES].copy().view("<f4").astype(np.float64)
        return decode_e4m3(codes) * scales[:, None]
    raise ValueError(f"unknown kv_dtype {kv_dtype!r}")


def gather_latent(cache, kv_dtype, block_table, b, L, j0=0, j1=None) -> np.ndarray:
    """Latent rows K_b[j] for j in [j0, j1) as float64 [j1 - j0, 576].

    Token j lives in physical page block_table[b, j // 64], slot j % 64.
    """
    if j1 is None:
        j1 = L
    rows = np.empty((j1 - j0, D_QK), dtype=np.float64)
    j = j0
    while j < j1:
        logical_page = j // PAGE
        slot = j % PAGE
        take = min(PAGE - slot, j1 - j)
        phys = int(block_table[b, logical_page])
        rows[j - j0:j - j0 + take] = _page_rows(cache, kv_dtype, phys)[slot:slot + take]
        j += take
    return rows


# ---------------------------------------------------------------------------
# Attention core: softmax(q K^T s) V for rows with their own visible length
# ---------------------------------------------------------------------------

def attend_rows(qrows: np.ndarray, K: np.ndarray, vis: np.ndarray, scale: float):
    """fp64 attention of query rows over a shared key/value row set.

    qrows: [R, 576] float64; K: [L, 576] float64 (V = K[:, :512]);
    vis[r]: number of leading rows of K that query r sees (1 <= vis[r] <= L).
    Returns out [R, 512] and natural-log lse [R].
    """
    qrows = np.asarray(qrows, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    z = (qrows @ K.T) * scale                              # [R, L]
    j = np.arange(K.shape[0])[None, :]
    visible = j < np.asarray(vis)[:, None]
    z = np.where(visible, z, -np.inf)
    zmax = z.max(axis=1, keepdims=True)
    w = np.exp(z - zmax)                                   # 0 where masked
    denom = w.sum(axis=1, keepdims=True)
    lse = (zmax + np.log(denom))[:, 0]
    out = (w / denom) @ K[:, :D_V]
    return out, lse


# ---------------------------------------------------------------------------
# Public oracle entry points
# ---------------------------------------------------------------------------

def _visible_lengths(L: int, T: int) -> np.ndarray:
    """Query t of T sees tokens j <= L - T + t, i.e. L - T + t + 1 of them."""
    return np.array([L - T + t + 1 for t in range(T)], dtype=np.int64)


def mla_decode_ref(q_bits, cache, kv_dtype, block_table, seqlens, scale=1.0 / np.sqrt(192.0)):
    """Whole-batch oracle.

    q_bits: uint16 bf16 bits [B, T, H, 576]; cache: uint16 [pages, 64, 576]
    (bf16) or uint8 [pages, 37120] (fp8 page + per-token fp32 scales);
    block_table int32 [B, max_pages]; seqlens int [B].
    Returns out float64 [B, T, H, 512], lse float64 [B, T, H].
    """
    q = decode_bf16(q_bits)
    B, T, H, _ = q.shape
    out = np.empty((B, T, H, D_V), dtype=np.float64)
    lse = np.empty((B, T, H), dtype=np.float64)
    for b in range(B):
        L = int(seqlens[b])
        if L < T:
            raise ValueError(f"sequence {b}: length {L} < q_len {T}")
        K = gather_latent(cache, kv_dtype, block_table, b, L)
        vis = np.repeat(_visible_lengths(L, T), H)         # rows ordered (t, h)
        o, s = attend_rows(q[b].reshape(T * H, D_QK), K, vis, scale)
        out[b] = o.reshape(T, H, D_V)
        lse[b] = s.reshape(T, H)
    return out, lse


def mla_decode_ref_rows(q_bits, cache, kv_dtype, block_table, seqlens, rows,
                        scale=1.0 / np.sqrt(192.0), chunk_tokens=1 << 16):
    """Oracle for a sample of (b, t, h) rows at any context length.

    Same definition as ``mla_decode_ref``; the scores z_j of the sampled rows
    are formed chunk by chunk of the gathered rows (to bound host memory), then
    lse and the weighted V sum follow the definition in two plain passes.
    Returns out float64 [len(rows), 512], lse float64 [len(rows)].
    """
    q = decode_bf16(q_bits)
    T = q.shape[1]
    rows = [tuple(int(x) for x in r) for r in rows]
    out = np.empty((len(rows), D_V), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    by_b = {}
    for i, (b, t, h) in enumerate(rows):
        by_b.setdefault(b, []).append((i, t, h))
    for b, items in by_b.items():
        L = int(seqlens[b])
        if L < T:
            raise ValueError(f"sequence {b}: length {L} < q_len {T}")
        qsel = np.stack([q[b, t, h] for (_, t, h) in items])           # [R, 576]
        vis = np.array([L - T + t + 1 for (_, t, _) in items])
        z = np.empty((len(items), L), dtype=np.float64)
        for j0 in range(0, L, chunk_tokens):
            j1 = min(L, j0 + chunk_tokens)
            K = gather_latent(cache, kv_dtype, block_table, b, L, j0, j1)
            z[:, j0:j1] = (qsel @ K.T) * scale
        z = np.where(np.arange(L)[None, :] < vis[:, None], z, -np.inf)
        zmax = z.max(axis=1, keepdims=True)
        w = np.exp(z - zmax)
        denom = w.sum(axis=1, keepdims=True)
        p = w / denom
        acc = np.zeros((len(items), D_V), dtype=np.float64)
        for j0 in range(0, L, chunk_tokens):
            j1 = min(L, j0 + chunk_tokens)
            K = gather_latent(cache, kv_dtype, block_table, b, L, j0, j1)
            acc += p[:, j0:j1] @ K[:, :D_V]
        for k, (i, _, _) in enumerate(items):
            out[i] = acc[k]
            lse[i] = zmax[k, 0] + np.log(denom[k, 0])
    return out, lse


def unabsorbed_mla(q_nope, q_rope, W_UK, W_UV, c, k_rope, vis, scale=1.0 / np.sqrt(192.0)):
    """Un-absorbed MLA for one head, used only to pin the absorbed form.

    q_nope [R, 128], q_rope [R, 64] (R query rows of one head), W_UK, W_UV
    [128, 512] up-projections of that head, c [L, 512] latents, k_rope [L, 64].
    Per-head key k_j = [W_UK c_j | k_rope_j] (192 wide), value v_j = W_UV c_j
    (128 wide); z_j = s <[q_nope | q_rope], k_j>; out = sum_j softmax(z)_j v_j.
    Returns out [R, 128], lse [R].
    """
    k = np.concatenate([c @ W_UK.T, k_rope], axis=1)       # [L, 192]
    v = c @ W_UV.T                                         # [L, 128]
    qq = np.concatenate([q_nope, q_rope], axis=1)          # [R, 192]
    z = (qq @ k.T) * scale
    z = np.where(np.arange(c.shape[0])[None, :] < np.asarray(vis)[:, None], z, -np.inf)
    zmax = z.max(axis=1, keepdims=True)
    w = np.exp(z - zmax)
    denom = w.sum(axis=1, keepdims=True)
    return (w / denom) @ v, (zmax + np.log(denom))[:, 0]
