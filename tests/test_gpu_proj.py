"""GPU parity of the absorbed-MLA projections (mla_absorb_q, mla_project_out,
through the C ABI) against the fp64 oracle, and the whole absorbed step
(absorb -> decode -> project) against the un-absorbed attention.

Tolerance of one projection: the kernel multiplies bf16 operands exactly, sums
in fp32 and rounds the result to bf16 (nearest-even), so each output is within
2^-9 of its magnitude plus the fp32 summation error (at most ~512 * 2^-24 of
the sum of |terms|); the test allows 2^-8 |ref| + 1e-4 max|ref|."""

import numpy as np
import pytest
import torch

import oracle
import mla_paged_kv_05_b200 as mla
from mla_paged_kv_05_b200 import inputs
from parity_util import run_gpu

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, std):
    return inputs.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def _host(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _close(got_bits, ref, what):
    got = oracle.decode_bf16(got_bits)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max()
    bad = np.argwhere(np.abs(got - ref) > bound)
    assert bad.size == 0, (what, bad[:4], got[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("N,H", [(1, 1), (4, 64), (64, 128), (128, 16), (200, 8), (300, 3)])
def test_absorb_matches_oracle(N, H):
    rng = np.random.default_rng(N * 131 + H)
    q = _bf16(rng, (N, H, 192), 1.0)
    w = _bf16(rng, (H, 128, 512), 0.05)
    out = torch.full((N, H, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.absorb_q(_dev(q), _dev(w), out, flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    got = _host(out)
    ref = oracle.absorb_q(q, w)
    _close(got[..., :512], ref[..., :512], f"absorb N{N} H{H}")
    assert np.array_equal(got[..., 512:], q[..., 128:])         # RoPE part passes through bit for bit


@pytest.mark.parametrize("N,H", [(1, 1), (4, 64), (64, 128), (128, 16), (200, 8), (300, 3)])
def test_project_matches_oracle(N, H):
    rng = np.random.default_rng(N * 171 + H)
    o = _bf16(rng, (N, H, 512), 0.3)
    w = _bf16(rng, (H, 128, 512), 0.05)
    y = torch.full((N, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    mla.project_out(_dev(o), _dev(w), y)
    torch.cuda.synchronize()
    _close(_host(y), oracle.project_out(o, w), f"project N{N} H{H}")


def test_projections_leave_other_memory_alone():
    # outputs of n_tokens rows only: a guard row after the output stays untouched
    rng = np.random.default_rng(3)
    N, H = 5, 4
    q = _bf16(rng, (N, H, 192), 1.0)
    w = _bf16(rng, (H, 128, 512), 0.05)
    buf = torch.full((N + 1, H, 576), 7.0, dtype=torch.bfloat16, device="cuda")
    mla.absorb_q(_dev(q), _dev(w), buf[:N])
    torch.cuda.synchronize()
    assert torch.all(buf[N] == 7.0)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_absorbed_step_matches_unabsorbed_attention(kv_dtype):
    # q (un-absorbed, per head 128 + 64) -> absorb -> decode over the latent cache
    # -> project, against the un-absorbed attention in fp64 on the same cache.
    B, T, H = 2, 2, 16
    lens = [700, 129]
    w_ = inputs.make_workload("absorbed", batch=B, heads=H, q_len=T, seqlens=lens, seed=61, kv_dtype=kv_dtype)
    rng = np.random.default_rng(62)
    q = _bf16(rng, (B * T, H, 192), 1.0)
    w_uk = _bf16(rng, (H, 128, 512), 0.05)
    w_uv = _bf16(rng, (H, 128, 512), 0.05)
    q_abs = torch.empty((B * T, H, 576), dtype=torch.bfloat16, device="cuda")
    mla.absorb_q(_dev(q), _dev(w_uk), q_abs)
    cache = (torch.from_numpy(w_.cache.view(np.int16)).view(torch.bfloat16) if kv_dtype == "bf16"
             else torch.from_numpy(w_.cache)).cuda()
    bt = torch.from_numpy(w_.block_table).cuda()
    sl = torch.from_numpy(w_.seqlens).cuda()
    dec = mla.MlaDecoder(B, w_.max_pages, T, H, kv_dtype)
    out, lse = dec(q_abs.view(B, T, H, 576), cache, bt, sl, scale=w_.scale)
    y = torch.empty((B * T, H, 128), dtype=torch.bfloat16, device="cuda")
    mla.project_out(out.view(B * T, H, 512), _dev(w_uv), y)
    torch.cuda.synchronize()
    assert dec.device_flag() == 0
    got = oracle.decode_bf16(_host(y)).reshape(B, T, H, 128)
    got_lse = lse.cpu().numpy().astype(np.float64)
    qf = oracle.decode_bf16(q).reshape(B, T, H, 192)
    wk, wv = oracle.decode_bf16(w_uk), oracle.decode_bf16(w_uv)
    for b, L in enumerate(lens):
        K = oracle.gather_latent(w_.cache, kv_dtype, w_.block_table, b, L)
        vis = [L - T + t + 1 for t in range(T)]
        for h in range(H):
            ref, ref_lse = oracle.unabsorbed_mla(qf[b, :, h, :128], qf[b, :, h, 128:], wk[h], wv[h], K[:, :512],
                                                 K[:, 512:], vis, w_.scale)
            d = got[b, :, h] - ref
            rel = np.linalg.norm(d) / np.linalg.norm(ref)
            # two more bf16 roundings than the decode alone (q~ and y): 1e-2 relative, lse 3e-3
            assert rel <= 1e-2 and np.abs(got_lse[b, :, h] - ref_lse).max() <= 3e-3, (b, h, rel)
