"""Helpers shared by the GPU parity tests: upload a seeded workload, run the
CUDA path through the C ABI, and compare with the fp64 oracle."""

from __future__ import annotations

import numpy as np
import torch

import mla_paged_kv_05_b200 as mla

# Tolerances for the bf16 output against the fp64 oracle (max-abs, rel-L2) and
# for lse (abs). fp8 caches get the wider pair; lse stays at 1e-3.
TOL = {"bf16": (1e-2, 5e-3), "fp8": (3e-2, 1.5e-2)}
LSE_TOL = 1e-3


def to_device(w, device="cuda"):
    q = torch.from_numpy(w.q_bits.view(np.int16).copy()).view(torch.bfloat16).to(device)
    if w.kv_dtype == "bf16":
        cache = torch.from_numpy(w.cache.view(np.int16)).view(torch.bfloat16).to(device)
    else:
        cache = torch.from_numpy(w.cache).to(device)
    bt = torch.from_numpy(w.block_table).to(device)
    sl = torch.from_numpy(w.seqlens).to(device)
    return q, cache, bt, sl


def run_gpu(w, sm_budget=0, tensors=None, decoder=None):
    q, cache, bt, sl = tensors if tensors is not None else to_device(w)
    dec = decoder or mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads, w.kv_dtype, sm_budget=sm_budget)
    out, lse = dec(q, cache, bt, sl, scale=w.scale)
    torch.cuda.synchronize()
    flag = dec.device_flag()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), flag


def assert_close(out, lse, ref_out, ref_lse, kv_dtype="bf16", what=""):
    atol, rtol_l2 = TOL[kv_dtype]
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    d = out - ref_out
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel_l2 = float(np.linalg.norm(d) / max(np.linalg.norm(ref_out), 1e-30)) if d.size else 0.0
    lse_err = float(np.abs(lse - ref_lse).max()) if lse.size else 0.0
    assert max_abs <= atol and rel_l2 <= rtol_l2 and lse_err <= LSE_TOL, (
        f"{what}: max_abs={max_abs:.3e} (<= {atol}) rel_l2={rel_l2:.3e} (<= {rtol_l2}) "
        f"lse_err={lse_err:.3e} (<= {LSE_TOL})")
    return max_abs, rel_l2, lse_err
