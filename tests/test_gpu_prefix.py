"""GPU parity of the shared-prefix (cascade) decode against the fp64 oracle.

The cascade reads the shared prefix once per kv-head for all sequences, then
each sequence's suffix, and merges; the oracle is the plain definition over
each sequence's whole context.  Sequences that do not start with the given
prefix (a relabelled block, a context shorter than the prefix) must still
come out right: the kernel checks each table on the device and decodes such
a sequence over its whole context.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


def prepared(wl):
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200.replay import build_step
    vals = workloads.draw_values(wl)
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    pkv.copy_blocks(c.k, c.v, st["cow_pairs"])
    pkv.kv_append(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"])
    ref = oracle.replay(wl, vals)
    return vals, st, ref


def cascade(st, wl, bt=None, cl=None, prefix_pages=None):
    import paged_kv_cache_365_b200 as pkv
    c = st["cache"]
    tables = st["host"]["block_tables"]
    lens = st["host"]["context_lens"]
    pp = pkv.common_prefix_pages(tables, lens) if prefix_pages is None else prefix_pages
    assert pp > 0
    prefix = torch.from_numpy(np.ascontiguousarray(tables[0, :pp])).cuda()
    out = pkv.paged_attention_decode_prefix(st["q"], c.k, c.v, st["block_tables"] if bt is None else bt,
                                            st["context_lens"] if cl is None else cl, st["max_context_len"],
                                            prefix, wl.scale)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    return out.float().cpu().numpy().astype(np.float64), pp


CASES = [
    workloads.prefix13b(seed=31, B=12, prefix_tokens=256, suffix_range=(1, 100), Hq=8, Hkv=8, D=128,
                        dtype="f16", name="pfx_f16_mha"),
    workloads.prefix13b(seed=32, B=20, prefix_tokens=512, suffix_range=(0, 700), Hq=16, Hkv=2, D=128,
                        dtype="bf16", name="pfx_bf16_gqa8"),
    workloads.prefix13b(seed=33, B=9, prefix_tokens=160, suffix_range=(3, 40), Hq=8, Hkv=2, D=64,
                        dtype="bf16", name="pfx_bf16_d64"),
    workloads.prefix13b(seed=34, B=140, prefix_tokens=64, suffix_range=(1, 30), Hq=2, Hkv=2, D=128,
                        dtype="f16", name="pfx_f16_many_seqs"),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_cascade_matches_oracle(wl):
    vals, st, ref = prepared(wl)
    got, pp = cascade(st, wl)
    assert pp * 16 == {"pfx_f16_mha": 256, "pfx_bf16_gqa8": 512, "pfx_bf16_d64": 160,
                       "pfx_f16_many_seqs": 64}[wl.name]
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype)
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= TOL[wl.dtype]


def test_cascade_full_size_prefix_workload():
    wl = workloads.named("prefix13b", 0)
    vals, st, ref = prepared(wl)
    got, pp = cascade(st, wl)
    assert pp == 64
    seqs = list(range(0, wl.B, 9)) + [wl.B - 1]
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"],
                               ref["context_lens"], wl.scale, wl.dtype, seqs=seqs)
    assert np.abs(got[seqs] - want[seqs]).max() <= TOL[wl.dtype]


def test_non_conforming_sequences_fall_back_to_their_whole_context():
    import paged_kv_cache_365_b200 as pkv
    wl = CASES[0]
    vals, st, ref = prepared(wl)
    c = st["cache"]
    tables = st["host"]["block_tables"].copy()
    lens = st["host"]["context_lens"].copy()
    pp = pkv.common_prefix_pages(tables, lens)
    # sequence 3: its third prefix page moved to a private copy (same data)
    free = sorted(set(range(wl.num_blocks)) - set(int(x) for x in tables[:, :].ravel() if x < wl.num_blocks))
    src, dst = int(tables[3, 2]), int(free[0])
    pkv.copy_blocks(c.k, c.v, torch.tensor([[src, dst]], dtype=torch.int32, device="cuda"))
    tables[3, 2] = dst
    # sequence 5: a context shorter than the prefix
    lens[5] = 37
    bt = torch.from_numpy(tables).cuda()
    cl = torch.from_numpy(lens).cuda()
    got, _ = cascade(st, wl, bt=bt, cl=cl, prefix_pages=pp)
    ref_tables = ref["block_tables"].copy()
    ref_tables[3, 2] = dst
    ref["cache"].copy_blocks([(src, dst)])
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref_tables, lens, wl.scale, wl.dtype)
    assert np.abs(got - want).max() <= TOL[wl.dtype]


def test_sequence_with_empty_suffix():
    """A sequence whose context is exactly the prefix: all of it comes from
    the prefix pass."""
    wl = CASES[0]
    vals, st, ref = prepared(wl)
    lens = st["host"]["context_lens"].copy()
    import paged_kv_cache_365_b200 as pkv
    pp = pkv.common_prefix_pages(st["host"]["block_tables"], lens)
    lens[0] = pp * 16
    got, _ = cascade(st, wl, cl=torch.from_numpy(lens).cuda(), prefix_pages=pp)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"], lens, wl.scale,
                               wl.dtype)
    assert np.abs(got - want).max() <= TOL[wl.dtype]


def test_cascade_agrees_with_plain_decode():
    import paged_kv_cache_365_b200 as pkv
    wl = CASES[1]
    vals, st, ref = prepared(wl)
    got, _ = cascade(st, wl)
    c = st["cache"]
    plain = pkv.paged_attention_decode(st["q"], c.k, c.v, st["block_tables"], st["context_lens"],
                                       st["max_context_len"], wl.scale).float().cpu().numpy()
    assert np.abs(got - plain).max() <= TOL[wl.dtype]


@pytest.mark.parametrize("wl", CASES[:2], ids=lambda w: w.name)
def test_phases_on_two_streams_are_bit_identical(wl):
    """Prefix pass on a second stream, suffix pass and merge on the first:
    the same bits as the one-launch cascade."""
    import paged_kv_cache_365_b200 as pkv
    vals, st, ref = prepared(wl)
    want, pp = cascade(st, wl)
    c = st["cache"]
    tables = st["host"]["block_tables"]
    prefix = torch.from_numpy(np.ascontiguousarray(tables[0, :pp])).cuda()
    B, hq, d = st["q"].shape
    ws = torch.empty(pkv.decode_prefix_workspace_bytes(B, hq, d, st["max_context_len"], pp), dtype=torch.uint8,
                     device="cuda")
    out = torch.full_like(st["q"], float("nan"))
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    args = (st["q"], c.k, c.v, st["block_tables"], st["context_lens"], st["max_context_len"], prefix, wl.scale)
    fork.record(main)
    side.wait_event(fork)
    with torch.cuda.stream(side):
        pkv.paged_attention_decode_prefix(*args, out=out, workspace=ws, stream=side, phase=0)
        join.record(side)
    pkv.paged_attention_decode_prefix(*args, out=out, workspace=ws, stream=main, phase=1)
    main.wait_event(join)
    pkv.paged_attention_decode_prefix(*args, out=out, workspace=ws, stream=main, phase=2)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    assert np.array_equal(out.float().cpu().numpy().astype(np.float64), want)
    with pytest.raises(ValueError):  # the phases need the caller's workspace
        pkv.paged_attention_decode_prefix(*args, phase=0)


def test_cache_step_on_a_shared_prefix_batch():
    """PagedKVCache.step on a shared-prefix batch (copy-on-write copies,
    append, the cascade) against the oracle."""
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200.replay import replay_ops, to_torch
    wl = workloads.prefix13b(seed=41, B=16, prefix_tokens=256, suffix_range=(1, 60), Hq=8, Hkv=4, D=128,
                             dtype="f16", name="pfx_step")
    vals = workloads.draw_values(wl)
    cache = pkv.PagedKVCache(wl.num_blocks, wl.Hkv, wl.D, torch.float16, "cuda", wl.free_order)
    replay_ops(cache, wl.ops, to_torch(vals["k_tokens"], "f16", "cuda"), to_torch(vals["v_tokens"], "f16", "cuda"))
    ids = [int(s) for s in wl.step_seqs]
    out = cache.step(ids, torch.from_numpy(vals["q"]), torch.from_numpy(vals["k_new"]),
                     torch.from_numpy(vals["v_new"]), scale=wl.scale)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    ref = oracle.replay(wl, vals)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"], ref["context_lens"],
                               wl.scale, "f16")
    assert np.abs(out.float().numpy() - want).max() <= TOL["f16"]


def test_partial_copy_append_matches_oracle_on_every_token():
    """The shared-prefix step with its copy-on-write copies cut to the rows
    that hold tokens, fused with the append: every token row of every
    sequence bit-exact against the oracle's full copy + append, the decode
    within tolerance."""
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200.replay import build_step
    wl = workloads.prefix13b(seed=51, B=24, prefix_tokens=128, suffix_range=(1, 90), Hq=8, Hkv=8, D=128,
                             dtype="f16", name="pfx_rows_gpu")
    vals = workloads.draw_values(wl)
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    copies = pkv.cow_copy_rows(st["host"]["cow_pairs"], st["host"]["step_slots"])
    assert len(copies) and (copies[:, 2] < 16).all()
    pkv.kv_append_copy(st["k_new"], st["v_new"], c.k, c.v, st["slot_mapping"], torch.from_numpy(copies).cuda())
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    ref = oracle.replay(wl, vals)
    gk, gv = c.k.cpu().view(torch.int16).numpy(), c.v.cpu().view(torch.int16).numpy()
    tables, lens = ref["block_tables"], ref["context_lens"]
    for b in range(wl.B):
        tok = np.arange(int(lens[b]))
        blk, off = tables[b, tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], ref["cache"].k[blk, :, off].view(np.int16))
        assert np.array_equal(gv[blk, :, off], ref["cache"].v[blk, :, off].view(np.int16))
    got, _ = cascade(st, wl)
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, tables, lens, wl.scale, wl.dtype)
    assert np.abs(got - want).max() <= TOL["f16"]


FUSED_CASES = [
    (workloads.prefix13b(seed=61, B=24, prefix_tokens=128, suffix_range=(1, 90), Hq=8, Hkv=8, D=128,
                         dtype="f16", name="fused_f16"), True, 0),
    (workloads.prefix13b(seed=62, B=20, prefix_tokens=512, suffix_range=(0, 700), Hq=16, Hkv=2, D=128,
                         dtype="bf16", name="fused_bf16_gqa"), True, 0),
    (workloads.prefix13b(seed=63, B=20, prefix_tokens=512, suffix_range=(0, 700), Hq=16, Hkv=2, D=128,
                         dtype="bf16", name="fused_bf16_plain"), False, 0),
    (workloads.prefix13b(seed=64, B=12, prefix_tokens=256, suffix_range=(1, 300), Hq=8, Hkv=4, D=64,
                         dtype="f16", name="fused_f16_split"), False, 64),
    (workloads.prefix13b(seed=65, B=12, prefix_tokens=256, suffix_range=(1, 300), Hq=8, Hkv=4, D=128,
                         dtype="bf16", name="fused_bf16_cascade_split"), True, 64),
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: c[0].name)
def test_fused_step_matches_separate_calls(case):
    """pkv_decode_step (the copy-on-write copies, the append and the decode
    in one launch: the CTA that reads a sequence's last page writes its
    token first) against kv_append_copy followed by the decode on the same
    state: every token row of the pool and the output bit-identical, and
    the output within tolerance of the oracle.  Cascade and plain decode,
    with and without several partitions per sequence."""
    import paged_kv_cache_365_b200 as pkv
    from paged_kv_cache_365_b200.replay import build_step
    wl, use_cascade, partition = case
    vals = workloads.draw_values(wl)
    st = build_step(wl, vals, "cuda")
    c = st["cache"]
    copies = pkv.cow_copy_rows(st["host"]["cow_pairs"], st["host"]["step_slots"])
    assert len(copies) > 0
    dcopies = torch.from_numpy(copies).cuda()
    tables, lens = st["host"]["block_tables"], st["host"]["context_lens"]
    prefix = None
    if use_cascade:
        pp = pkv.cascade_prefix_pages(tables, lens, c.k.dtype)
        assert pp > 0
        prefix = torch.from_numpy(np.ascontiguousarray(tables[0, :pp])).cuda()
    k2, v2 = c.k.clone(), c.v.clone()
    # separate launches on the copy of the pool
    pkv.kv_append_copy(st["k_new"], st["v_new"], k2, v2, st["slot_mapping"], dcopies)
    if use_cascade:
        sep = pkv.paged_attention_decode_prefix(st["q"], k2, v2, st["block_tables"], st["context_lens"],
                                                st["max_context_len"], prefix, wl.scale, partition=partition)
    else:
        sep = pkv.paged_attention_decode(st["q"], k2, v2, st["block_tables"], st["context_lens"],
                                         st["max_context_len"], wl.scale, partition=partition)
    fused = pkv.decode_step(st["q"], c.k, c.v, st["k_new"], st["v_new"], st["slot_mapping"], dcopies,
                            st["block_tables"], st["context_lens"], st["max_context_len"], wl.scale,
                            prefix_blocks=prefix, partition=partition)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    assert torch.equal(fused.view(torch.int16), sep.view(torch.int16))
    gk, gv = c.k.cpu().view(torch.int16).numpy(), c.v.cpu().view(torch.int16).numpy()
    sk, sv = k2.cpu().view(torch.int16).numpy(), v2.cpu().view(torch.int16).numpy()
    for b in range(wl.B):
        tok = np.arange(int(lens[b]))
        blk, off = tables[b, tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], sk[blk, :, off])
        assert np.array_equal(gv[blk, :, off], sv[blk, :, off])
    ref = oracle.replay(wl, vals)
    for b in range(wl.B):
        tok = np.arange(int(lens[b]))
        blk, off = tables[b, tok // 16], tok % 16
        assert np.array_equal(gk[blk, :, off], ref["cache"].k[blk, :, off].view(np.int16))
    want = oracle.paged_decode(vals["q"], ref["cache"].k, ref["cache"].v, ref["block_tables"], ref["context_lens"],
                               wl.scale, wl.dtype)
    assert np.abs(fused.float().cpu().numpy() - want).max() <= TOL[wl.dtype]
