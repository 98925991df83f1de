"""Plain CPU oracle for the absorbed-MLA projections around the decode
attention: the query absorption before it and the value up-projection after
it.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). The pages name an MLA
(Multi-head Latent Attention) decode kernel (evermx.com, "TokenSpeed:
speed-of-light LLM inference engine for agentic workloads", section
"Pluggable Kernel Registry") without giving its algebra; this is the textbook
absorbed form, the same reading as ``mla_oracle.unabsorbed_mla``: per head h,
a 128-wide no-RoPE query part and a 64-wide RoPE part, up-projections
W_UK[h], W_UV[h] of shape [128, 512] from the shared 512-wide latent c_j, so

    k_nope_j = W_UK[h] c_j        q . k_nope_j = (W_UK[h]^T q_nope) . c_j
    v_j      = W_UV[h] c_j        sum_j p_j v_j = W_UV[h] (sum_j p_j c_j)

Absorption: q~[n, h] = [W_UK[h]^T q[n, h, :128] | q[n, h, 128:192]] (576
wide, the decode kernel's query row). Projection: y[n, h] = W_UV[h] o[n, h]
with o the decode output (512 wide). Both in fp64 on the bf16 inputs. Pinned
by ``tests/test_oracle_pins.py`` against hand-computed integer products and
against the un-absorbed attention through the decode oracle.
"""

from __future__ import annotations

import numpy as np

from .mla_oracle import decode_bf16

D_NOPE = 128
D_ROPE = 64
D_LATENT = 512


def _f64(x):
    x = np.asarray(x)
    return decode_bf16(x) if x.dtype == np.uint16 else x.astype(np.float64)


def absorb_q(q, w_uk) -> np.ndarray:
    """q [N, H, 192] (bf16 bits or float), w_uk [H, 128, 512] -> q~ [N, H, 576] float64."""
    q = _f64(q)
    w = _f64(w_uk)
    N, H, _ = q.shape
    out = np.empty((N, H, D_LATENT + D_ROPE), dtype=np.float64)
    for h in range(H):
        out[:, h, :D_LATENT] = q[:, h, :D_NOPE] @ w[h]          # (W_UK[h]^T q_nope)^T
        out[:, h, D_LATENT:] = q[:, h, D_NOPE:D_NOPE + D_ROPE]
    return out


def project_out(o, w_uv) -> np.ndarray:
    """o [N, H, 512] (bf16 bits or float), w_uv [H, 128, 512] -> y [N, H, 128] float64."""
    o = _f64(o)
    w = _f64(w_uv)
    N, H, _ = o.shape
    out = np.empty((N, H, D_NOPE), dtype=np.float64)
    for h in range(H):
        out[:, h, :] = o[:, h, :] @ w[h].T                     # W_UV[h] o
    return out
