"""Host restatement of the split-KV planner's output, for tests of the device
planner (test infrastructure: the planner is scheduling, not part of the
attention the oracle defines).

Cost model: sequence b with L_b tokens (valid when q_len <= L_b <= 64 *
max_pages) has n_b = ceil(L_b / 64) pages and costs n_b + 2 units; the batch's
costs are laid end to end; cluster c takes the units [c * P, (c + 1) * P) with
P = max(4, ceil(total / c_use)). A sequence whose pages fall in more than one
cluster is split; the combine kernel visits every sequence with splits != 1.
"""

import numpy as np

SEQ_OVERHEAD = 2
MIN_PAYLOAD = 4
HDR_WORDS = 64
SEQ_WORDS = 8


def _align(x, a):
    return (x + a - 1) // a * a


def tile_rows(q_len, heads):
    return 64 if q_len * heads <= 64 else 128


def row_tiles(q_len, heads):
    tr = tile_rows(q_len, heads)
    return (q_len * heads + tr - 1) // tr


def c_use_of(sm_budget, c_max, q_len, heads):
    if sm_budget <= 0:
        return c_max
    return min(c_max, max(1, (sm_budget // 2) // row_tiles(q_len, heads)))


def layout(batch, c_max):
    """Byte offsets of the plan's parts in the workspace."""
    off = HDR_WORDS * 4
    first_b = off
    off = _align(off + 4 * c_max, 16)
    seq = off
    off = _align(off + 4 * SEQ_WORDS * batch, 16)
    lst = off
    off = _align(off + 4 * batch, 16)
    vcp = off
    return {"first_b": first_b, "seq": seq, "list": lst, "vcp": vcp}


def combine_items(splits, rows):
    warps = 1 if splits <= 8 else 2 if splits <= 16 else 4 if splits <= 32 else 8
    return (rows * 4 * warps + 8 - 1) // 8


def plan(seqlens, q_len, heads, max_pages, c_use, c_max):
    """The plan as dicts of python ints: header words, per-sequence records,
    the combine list with its inclusive item prefix, and each cluster's first
    sequence."""
    rows = q_len * heads
    B = len(seqlens)
    L = [int(x) for x in seqlens]
    n = [(l + 63) // 64 if q_len <= l <= 64 * max_pages else 0 for l in L]
    cost = [k + SEQ_OVERHEAD if k > 0 else 0 for k in n]
    start = [0] * B
    for b in range(1, B):
        start[b] = start[b - 1] + cost[b - 1]
    total = sum(cost)
    payload = max(MIN_PAYLOAD, -(-total // c_use))
    clusters = -(-total // payload) if total > 0 else 0
    first, splits = [0] * B, [0] * B
    for b in range(B):
        if n[b] > 0:
            ps = start[b] + SEQ_OVERHEAD
            first[b] = ps // payload
            splits[b] = (ps + n[b] - 1) // payload - first[b] + 1
    slot, s = [0] * B, 0
    for b in range(B):
        slot[b] = s
        s += splits[b] if splits[b] > 1 else 0
    listed = [b for b in range(B) if splits[b] != 1]
    vcp, acc = [], 0
    for b in listed:
        acc += combine_items(splits[b], rows)
        vcp.append(acc)
    ends = [start[b] + cost[b] for b in range(B)]
    first_b = []
    for c in range(c_max):
        fb = B
        if c < clusters:
            x0 = c * payload
            fb = next((b for b in range(B) if ends[b] > x0), B)
        first_b.append(fb)
    hdr = {1: clusters, 2: payload, 3: total, 4: s, 5: len(listed), 6: acc}
    seq = [(start[b], n[b], first[b], splits[b], slot[b], L[b]) for b in range(B)]
    return {"hdr": hdr, "seq": seq, "list": listed, "vcp": vcp, "first_b": first_b}


def read_plan(ws_bytes, batch, c_max, listed):
    """The same parts read back from a workspace (numpy uint8 array)."""
    w32 = ws_bytes.view(np.int32)
    lay = layout(batch, c_max)
    hdr = {k: int(w32[k]) for k in range(1, 7)}
    seq_words = w32[lay["seq"] // 4: lay["seq"] // 4 + SEQ_WORDS * batch].reshape(batch, SEQ_WORDS)
    seq = [tuple(int(v) for v in seq_words[b, :6]) for b in range(batch)]
    lst = [int(v) for v in w32[lay["list"] // 4: lay["list"] // 4 + listed]]
    vcp = [int(v) for v in w32[lay["vcp"] // 4: lay["vcp"] // 4 + listed]]
    first_b = [int(v) for v in w32[lay["first_b"] // 4: lay["first_b"] // 4 + c_max]]
    return {"hdr": hdr, "seq": seq, "list": lst, "vcp": vcp, "first_b": first_b}
