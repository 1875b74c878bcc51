"""Brute-force single-query attention over a contiguous cache, in pure
Python (oracle self-check only; tiny inputs).

The contiguous per-request cache is the layout the pages contrast paging
with ("PagedAttention 与 vLLM 推理加速" §2.2).  Here each sequence's keys and
values are plain Python lists in logical order; no block table, slot or
page is involved, so agreement with ``attention.paged_decode`` pins the
oracle's gather through the table.
"""
import math


def contiguous_decode(q_row, keys, values, scale):
    """q_row: list[float]; keys/values: list of rows (list[float]) in order."""
    if not keys:
        return [0.0] * len(values[0]) if values else []
    logits = []
    for k in keys:
        dot = 0.0
        for a, b in zip(q_row, k):
            dot += a * b
        logits.append(scale * dot)
    top = max(logits)
    weights = [math.exp(x - top) for x in logits]
    total = math.fsum(weights)
    out = []
    for d in range(len(values[0])):
        out.append(math.fsum(w * v[d] for w, v in zip(weights, values)) / total)
    return out
