"""Seeded synthetic inputs for MLA decode over a paged latent cache.

This module only draws and lays out inputs: random normals rounded to bf16,
random page permutations, block tables, sequence lengths, and the fp8-e4m3
cache encoding (the cache *writer*). It holds none of the decode arithmetic,
and it serves both the CUDA path and the CPU oracle, which share nothing else.

Shapes and distributions follow the decode workloads this library targets:
q ~ N(0, 1); latent cache rows ~ N(0, std) (std 1.0 for the tiny case, 0.5
elsewhere); pages of 64 tokens drawn from a randomly permuted physical pool
that holds extra never-referenced pages; optional shared-prefix pages across
sequences (multi-turn prefix reuse, zubnet.ai "LightSeek TokenSpeed 580 TPS"
second paragraph; 24-ai.news "TokenSpeed ... 580 token/s", optimisations list).
Slots past a sequence's end in its last page, and the extra pool pages, are
filled with NaN so that any read of them that leaks into a result shows up.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

PAGE = 64
D_QK = 576
D_V = 512
FP8_DATA_BYTES = PAGE * D_QK            # 36,864
FP8_PAGE_BYTES = FP8_DATA_BYTES + PAGE * 4   # + 64 fp32 token scales = 37,120
E4M3_MAX = 448.0
BF16_NAN = 0x7FC0
E4M3_NAN = 0x7F

K = 1024   # "128K" = 131,072 tokens etc.


@dataclasses.dataclass
class Workload:
    name: str
    batch: int
    heads: int
    q_len: int
    kv_dtype: str                 # "bf16" or "fp8"
    seqlens: np.ndarray           # int32 [B]
    block_table: np.ndarray       # int32 [B, max_pages]
    q_bits: np.ndarray            # uint16 (bf16 bits) [B, T, H, 576]
    cache: np.ndarray             # uint16 [P, 64, 576] or uint8 [P, 37120]
    scale: float = 1.0 / math.sqrt(192.0)
    shared_prefix_tokens: int = 0
    seed: int = 0

    @property
    def num_pages(self) -> int:
        return int(self.cache.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def rows(self) -> int:
        return self.q_len * self.heads

    def describe(self) -> dict:
        return {
            "workload": self.name, "batch": self.batch, "heads": self.heads,
            "q_len": self.q_len, "kv_dtype": self.kv_dtype,
            "sum_context": int(self.seqlens.astype(np.int64).sum()),
            "max_context": int(self.seqlens.max()) if self.batch else 0,
            "page": PAGE, "num_pages": self.num_pages, "seed": self.seed,
            "shared_prefix_tokens": self.shared_prefix_tokens,
        }


# ---------------------------------------------------------------------------
# element encodings used to store the draws
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest-even, returning the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def encode_fp8_pages(rows_bits: np.ndarray) -> np.ndarray:
    """Write bf16 latent rows into fp8-e4m3 pages with a per-token fp32 scale.

    rows_bits: uint16 [P, 64, 576]. Per token: sigma = amax|x| / 448 (1 when
    the row is all zero), code = e4m3(x / sigma) rounded to nearest even and
    saturated to +-448. Page layout: 64 x 576 codes, then 64 fp32 sigmas.
    """
    x = torch.from_numpy(bf16_bits_to_f32(rows_bits).copy())          # [P, 64, 576]
    amax = x.abs().amax(dim=-1)                                        # [P, 64]
    sigma = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / sigma[..., None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    P = rows_bits.shape[0]
    out = np.empty((P, FP8_PAGE_BYTES), dtype=np.uint8)
    out[:, :FP8_DATA_BYTES] = codes.reshape(P, FP8_DATA_BYTES)
    out[:, FP8_DATA_BYTES:] = sigma.numpy().astype("<f4").view(np.uint8).reshape(P, PAGE * 4)
    return out


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------

def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def _cache_pages(seed: int, num_pages: int, std: float, chunk: int = 512) -> np.ndarray:
    """num_pages x 64 x 576 bf16 normals, drawn chunk by chunk from child seeds."""
    out = np.empty((num_pages, PAGE, D_QK), dtype=np.uint16)
    children = np.random.SeedSequence([seed, 0xCAC4E]).spawn((num_pages + chunk - 1) // chunk)
    for i, ss in enumerate(children):
        p0 = i * chunk
        p1 = min(num_pages, p0 + chunk)
        out[p0:p1] = _normal_bf16(np.random.default_rng(ss), (p1 - p0, PAGE, D_QK), std)
    return out


def make_workload(name: str, *, batch: int, heads: int, q_len: int, seqlens,
                  kv_dtype: str = "bf16", cache_std: float = 0.5, seed: int = 0,
                  shared_prefix_tokens: int = 0, extra_pages: int = 2,
                  max_pages: Optional[int] = None, poison: bool = True) -> Workload:
    """Build one seeded workload.

    Logical pages of every sequence are mapped to physical pages drawn from a
    random permutation of the pool. With ``shared_prefix_tokens`` > 0 the first
    ceil(min(L_b, prefix)/64) pages of every sequence are the same physical
    pages (prefix reuse); the rest are private.
    """
    seqlens = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    assert seqlens.shape[0] == batch
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x5EED]))
    n_pages = [(int(L) + PAGE - 1) // PAGE for L in seqlens]
    if max_pages is None:
        max_pages = max([1] + n_pages)
    shared_pages = (shared_prefix_tokens + PAGE - 1) // PAGE
    if shared_prefix_tokens:
        assert shared_prefix_tokens % PAGE == 0
        private = [max(0, n - shared_pages) for n in n_pages]
        used_shared = min(shared_pages, max(n_pages) if n_pages else 0)
        needed = used_shared + sum(private)
    else:
        needed = sum(n_pages)
    pool = needed + extra_pages
    perm = rng.permutation(pool).astype(np.int32)
    block_table = np.zeros((batch, max_pages), dtype=np.int32)
    # unused block-table entries point at a poisoned extra page: never read
    poison_page = perm[needed] if extra_pages else 0
    block_table[:] = poison_page
    cursor = 0
    if shared_prefix_tokens:
        shared_ids = perm[:used_shared]
        cursor = used_shared
        for b in range(batch):
            k = min(n_pages[b], shared_pages)
            block_table[b, :k] = shared_ids[:k]
            r = n_pages[b] - k
            block_table[b, k:k + r] = perm[cursor:cursor + r]
            cursor += r
    else:
        for b in range(batch):
            block_table[b, :n_pages[b]] = perm[cursor:cursor + n_pages[b]]
            cursor += n_pages[b]
    q_bits = _normal_bf16(np.random.default_rng(np.random.SeedSequence([seed, 0x0])),
                          (batch, q_len, heads, D_QK), 1.0)
    cache = _cache_pages(seed, pool, cache_std)
    if poison:
        for b in range(batch):
            L = int(seqlens[b])
            tail = L % PAGE
            if tail and not (shared_prefix_tokens and L <= shared_prefix_tokens):
                cache[block_table[b, n_pages[b] - 1], tail:, :] = BF16_NAN
        for p in perm[needed:]:
            cache[p] = BF16_NAN
    if kv_dtype == "fp8":
        fp8 = encode_fp8_pages(cache)
        if poison:
            for b in range(batch):
                L = int(seqlens[b])
                tail = L % PAGE
                if tail and not (shared_prefix_tokens and L <= shared_prefix_tokens):
                    page = block_table[b, n_pages[b] - 1]
                    data = fp8[page, :FP8_DATA_BYTES].reshape(PAGE, D_QK)
                    data[tail:, :] = E4M3_NAN
                    sc = fp8[page, FP8_DATA_BYTES:].view("<f4")
                    sc[tail:] = np.float32("nan")
            for p in perm[needed:]:
                fp8[p, :] = 0xFF
        cache = fp8
    elif kv_dtype != "bf16":
        raise ValueError(kv_dtype)
    return Workload(name=name, batch=batch, heads=heads, q_len=q_len, kv_dtype=kv_dtype,
                    seqlens=seqlens.astype(np.int32), block_table=block_table, q_bits=q_bits,
                    cache=cache, shared_prefix_tokens=shared_prefix_tokens, seed=seed)


# ---------------------------------------------------------------------------
# the five decode workloads (and their scaled-down parity twins)
# ---------------------------------------------------------------------------

def tiny(seed: int = 0) -> Workload:
    """Batch 1, 16 heads, q_len 1, 256 tokens in 4 shuffled pages, N(0,1)."""
    return make_workload("tiny_b1_h16_t1_L256", batch=1, heads=16, q_len=1, seqlens=[256],
                         cache_std=1.0, seed=seed)


def kimi_50k(seed: int = 1, context: int = 50_000) -> Workload:
    """Kimi-K2.5-shaped single-user decode: batch 1, 64 heads, q_len 1."""
    return make_workload(f"kimi_b1_h64_t1_L{context}", batch=1, heads=64, q_len=1,
                         seqlens=[context], seed=seed)


def spec_decode(context: int, seed: int = 2) -> Workload:
    """Speculative decode: batch 1, 64 heads, q_len 4 (1 verified + 3 drafts)."""
    return make_workload(f"spec_b1_h64_t4_L{context}", batch=1, heads=64, q_len=4,
                         seqlens=[context], seed=seed)


def agentic_batch(seed: int = 4, batch: int = 16, lo: int = 20 * K, hi: int = 60 * K,
                  prefix: int = 40 * K) -> Workload:
    """Multi-turn agentic batch: 128 heads, q_len 2, L ~ U[lo, hi], shared prefix."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x1E7]))
    seqlens = rng.integers(lo, hi + 1, size=batch)
    return make_workload(f"agentic_b{batch}_h128_t2", batch=batch, heads=128, q_len=2,
                         seqlens=seqlens, seed=seed, shared_prefix_tokens=prefix)


def fp8_batch(seed: int = 5, batch: int = 64, median: int = 8 * K, sigma_ln: float = 1.0,
              lo: int = 1 * K, hi: int = 64 * K, heads: int = 128) -> Workload:
    """fp8-e4m3 cache throughput: 128 heads, q_len 1, lognormal contexts."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x109]))
    seqlens = np.clip(np.rint(np.exp(rng.normal(math.log(median), sigma_ln, size=batch))),
                      lo, hi).astype(np.int64)
    return make_workload(f"fp8_b{batch}_h{heads}_t1", batch=batch, heads=heads, q_len=1,
                         seqlens=seqlens, kv_dtype="fp8", seed=seed)


def prefix_batch(seed: int = 6, batch: int = 16, heads: int = 16, q_len: int = 1, prefix: int = 40 * K,
                 hi: int = 60 * K) -> Workload:
    """The agentic batch's prefix sharing at 16 heads and q_len 1 (a memory-bound
    step): contexts U[prefix + 64, hi], so every sequence shares the whole
    40,960-token prefix and has its new tokens past it."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x9F1]))
    seqlens = rng.integers(prefix + PAGE, hi + 1, size=batch)
    return make_workload(f"prefix_b{batch}_h{heads}_t{q_len}", batch=batch, heads=heads, q_len=q_len,
                         seqlens=seqlens, seed=seed, shared_prefix_tokens=prefix)


def cascade_prefix_len(w: Workload) -> int:
    """The longest page-aligned prefix a cascade step can share over the whole
    batch: within the shared pages and short of every sequence's new tokens."""
    if not w.shared_prefix_tokens:
        return 0
    p = min(w.shared_prefix_tokens, int(w.seqlens.min()) - w.q_len)
    return max(0, p // PAGE * PAGE)


WORKLOADS = {
    "tiny": tiny,
    "kimi_50k": kimi_50k,
    "spec_128k": lambda seed=2: spec_decode(128 * K, seed),
    "spec_256k": lambda seed=2: spec_decode(256 * K, seed),
    "spec_1m": lambda seed=3: spec_decode(1024 * K, seed),
    "agentic": agentic_batch,
    "fp8": fp8_batch,
    "prefix_h16": prefix_batch,
    # the fp8 batch at 64 heads: the 64-row fp8 kernel variant (profiling and parity)
    "fp8_h64": lambda seed=7: fp8_batch(seed=seed, heads=64),
}
