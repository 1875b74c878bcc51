"""Test-side helpers shared by the oracle pins and the GPU parity tests."""
import numpy as np

import oracle


def logical_token_ids(wl):
    """For each step sequence, the ids of its tokens in logical order.

    An id is an index into the prefill arrays (k_tokens/v_tokens) or
    ('new', b) for the step's token of batch entry b.  Worked out from the
    op log alone -- no allocator, slot or block table is involved.
    """
    seqs = {}
    cursor = 0
    for op in wl.ops:
        if op[0] == "add":
            seqs[op[1]] = []
        elif op[0] == "append":
            seqs[op[1]] = seqs[op[1]] + list(range(cursor, cursor + op[2]))
            cursor += op[2]
        elif op[0] == "fork":
            seqs[op[2]] = list(seqs[op[1]])
        elif op[0] == "free":
            del seqs[op[1]]
    out = []
    for b, sid in enumerate(wl.step_seqs):
        ids = list(seqs[int(sid)])
        if wl.step_append_mask[b]:
            ids.append(("new", b))
        out.append(ids)
    return out


def logical_rows(wl, values, b, kv_head, widen):
    """(keys, values) float64 rows of step sequence b, kv-head ``kv_head``."""
    ids = logical_token_ids(wl)[b]
    ks, vs = [], []
    for t in ids:
        if isinstance(t, tuple):
            ks.append(values["k_new"][t[1], kv_head])
            vs.append(values["v_new"][t[1], kv_head])
        else:
            ks.append(values["k_tokens"][t, kv_head])
            vs.append(values["v_tokens"][t, kv_head])
    if not ks:
        return np.zeros((0, wl.D)), np.zeros((0, wl.D))
    return widen(np.stack(ks), wl.dtype), widen(np.stack(vs), wl.dtype)


def relabel_blocks(cache_k, cache_v, tables, context_lens, perm, block_size=16):
    """Move every physical block i to perm[i]; rewrite the tables to match."""
    k2 = np.empty_like(cache_k)
    v2 = np.empty_like(cache_v)
    k2[perm] = cache_k
    v2[perm] = cache_v
    t2 = tables.copy()
    for b, n in enumerate(context_lens):
        pages = -(-int(n) // block_size)
        t2[b, :pages] = perm[tables[b, :pages]]
    return k2, v2, t2


def privatise(cache_k, cache_v, tables, context_lens, block_size=16):
    """Give every sequence its own copy of every block its table names.

    Returns a larger pool where no block is shared, and the new tables.
    """
    pages = [-(-int(n) // block_size) for n in context_lens]
    nb0 = cache_k.shape[0]
    total = nb0 + sum(pages)
    k2 = np.empty((total,) + cache_k.shape[1:], dtype=cache_k.dtype)
    v2 = np.empty_like(k2)
    k2[:nb0] = cache_k
    v2[:nb0] = cache_v
    t2 = tables.copy()
    nxt = nb0
    for b, p in enumerate(pages):
        for j in range(p):
            src = tables[b, j]
            k2[nxt] = cache_k[src]
            v2[nxt] = cache_v[src]
            t2[b, j] = nxt
            nxt += 1
    return k2, v2, t2


def make_multi_case(ctx, nq, Hq, Hkv, D, dtype, seed, v_scale=1.0):
    """Pool, tables and values for sequences of lengths ``ctx`` (the last
    ``nq[b]`` tokens being the new ones); blocks placed by a permutation.
    V is drawn N(0, v_scale^2)."""
    rng = np.random.default_rng(seed)
    pages = [-(-c // 16) for c in ctx]
    nb = sum(pages) + 5
    perm = rng.permutation(nb)
    store = {"f32": np.float32, "f16": np.float16, "bf16": np.float32}[dtype]
    k = oracle.nan_fill((nb, Hkv, 16, D), dtype)
    v = oracle.nan_fill((nb, Hkv, 16, D), dtype)
    W = max(pages) + 2
    tables = np.full((len(ctx), W), nb + 100, dtype=np.int32)
    rows_k, rows_v = [], []
    used = 0
    for b, c in enumerate(ctx):
        tables[b, :pages[b]] = perm[used:used + pages[b]]
        used += pages[b]
        kk = rng.standard_normal((c, Hkv, D)).astype(store)
        vv = (rng.standard_normal((c, Hkv, D)) * v_scale).astype(store)
        if dtype == "bf16":  # keep the upper half: exact bf16 values
            kk = (kk.view(np.uint32) >> 16).astype(np.uint16)
            vv = (vv.view(np.uint32) >> 16).astype(np.uint16)
        for j in range(c):
            k[tables[b, j // 16], :, j % 16] = kk[j]
            v[tables[b, j // 16], :, j % 16] = vv[j]
        rows_k.append(kk)
        rows_v.append(vv)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), Hq, D)).astype(store)
    if dtype == "bf16":
        q = (q.view(np.uint32) >> 16).astype(np.uint16)
    return dict(q=q, k=k, v=v, tables=tables, ctx=np.array(ctx, dtype=np.int32), qs=qs, rows_k=rows_k,
                rows_v=rows_v, dtype=dtype, G=Hq // Hkv)


# Mantissa bits of the 16-bit output formats and their smallest normal
# exponent (below it the spacing stays that of the smallest binade).
_FMT = {"f16": (10, -14), "bf16": (7, -126)}


def half_ulp(x, dtype):
    """Half the spacing of the output format ``dtype`` at |x| (elementwise):
    the error of rounding the exact value to that format once."""
    bits, emin = _FMT[dtype]
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.where(a > 0, np.floor(np.log2(np.where(a > 0, a, 1.0))), emin)
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - bits - 1).astype(np.int64))


def ulp_aware_bound(ref, dtype, tol):
    """Elementwise bound for a 16-bit output of a kernel that computes in
    fp32 and rounds once: the stated max-abs tolerance, or -- where the
    output's magnitude makes the format's own rounding larger -- half an ulp
    of the fp64 reference in the output format plus a fp32-level slack of
    2^-14 |ref| (far below the 16-bit formats' precision)."""
    ref = np.asarray(ref, dtype=np.float64)
    return np.maximum(tol, half_ulp(ref, dtype) + np.ldexp(np.abs(ref), -14))
