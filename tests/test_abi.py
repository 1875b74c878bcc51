"""The C-ABI library loads, exports every entry point include/pkv.h
declares, and rejects bad arguments before touching the GPU (no compute
calls here: these run without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_365_b200 import _lib
    return _lib.lib


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 20
    raw = ctypes.CDLL(os.path.join(ROOT, "paged_kv_cache_365_b200", "libpkv.so"))
    for n in names:
        assert hasattr(raw, n), n


def test_binding_prototypes_cover_the_header():
    from paged_kv_cache_365_b200 import _lib
    assert sorted(_lib.PROTOTYPES) == header_functions()


def test_status_strings(lib):
    assert lib.pkv_status_string(0) == b"ok"
    assert lib.pkv_status_string(2) == b"block pool exhausted"
    assert lib.pkv_abi_version() == 1


FAKE = ctypes.c_void_p(1 << 20)  # 16-byte aligned; never dereferenced (rejected first)
ODD = ctypes.c_void_p((1 << 20) + 8)


def decode(lib, **kw):
    args = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, mb=8, cl=FAKE, maxctx=100, B=2, Hq=8, Hkv=2,
                D=128, NB=64, scale=0.1, part=0, dt=1, ws=FAKE, wsb=1 << 30, stream=None)
    args.update(kw)
    return lib.pkv_paged_attention_decode(args["out"], args["q"], args["k"], args["v"], args["bt"], args["mb"],
                                          args["cl"], args["maxctx"], args["B"], args["Hq"], args["Hkv"],
                                          args["D"], args["NB"], args["scale"], args["part"], args["dt"],
                                          args["ws"], args["wsb"], args["stream"])


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(D=256), dict(Hq=6, Hkv=2), dict(Hq=7, Hkv=2), dict(Hq=32, Hkv=2), dict(part=17),
    dict(part=4096), dict(part=8), dict(dt=3), dict(NB=0), dict(mb=0), dict(maxctx=8 * 16 + 1),
    dict(maxctx=-1), dict(B=-1), dict(B=70000), dict(out=ODD), dict(k=ODD), dict(q=None),
    dict(scale=float("nan")), dict(maxctx=1000, mb=100, ws=None), dict(maxctx=1000, mb=100, wsb=100),
])
def test_decode_rejects_bad_arguments(lib, bad):
    assert decode(lib, **bad) == 1


def test_decode_workspace_bytes(lib):
    # one partition: nothing needed
    assert lib.pkv_decode_workspace_bytes(4, 8, 128, 512, 0) == 0
    # 3 partitions of 512: B*Hq*P*(D+2)*4
    assert lib.pkv_decode_workspace_bytes(4, 8, 128, 1025, 0) == 4 * 8 * 3 * 130 * 4
    assert lib.pkv_decode_workspace_bytes(4, 8, 64, 100, 16) == 4 * 8 * 7 * 66 * 4
    assert lib.pkv_decode_workspace_bytes(4, 8, 96, 1000, 0) == 0  # unsupported -> 0
    # auto past 4096 tokens: 1024-token partitions
    assert lib.pkv_decode_workspace_bytes(2, 8, 128, 8192, 0) == 2 * 8 * 8 * 130 * 4
    assert lib.pkv_decode_workspace_bytes(2, 8, 128, 4096, 0) == 2 * 8 * 8 * 130 * 4
    assert lib.pkv_decode_workspace_bytes(2, 8, 128, 4097, 0) == 2 * 8 * 5 * 130 * 4
    assert lib.pkv_decode_workspace_bytes(4, 8, 128, 1000, 17) == 0


def test_zero_sized_calls_are_no_ops(lib):
    assert decode(lib, B=0, out=None, q=None) == 0
    assert lib.pkv_kv_append(None, None, None, None, None, 0, 2, 64, 16, 0, None) == 0
    assert lib.pkv_copy_blocks(None, None, None, 0, 2, 64, 16, 0, None) == 0


@pytest.mark.parametrize("args", [
    (FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 80, 16, 1, None),     # head_dim
    (FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0, 64, 16, 1, None),     # Hkv
    (FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 64, 16, 1, None),    # num_tokens
    (FAKE, FAKE, ODD, FAKE, FAKE, 4, 2, 64, 16, 1, None),      # alignment
    (FAKE, FAKE, FAKE, FAKE, None, 4, 2, 64, 16, 1, None),     # slots
    (FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 7, None),     # dtype
])
def test_append_rejects_bad_arguments(lib, args):
    assert lib.pkv_kv_append(*args) == 1


def test_copy_rejects_bad_arguments(lib):
    assert lib.pkv_copy_blocks(FAKE, FAKE, FAKE, 70000, 2, 64, 16, 1, None) == 1
    assert lib.pkv_copy_blocks(FAKE, FAKE, None, 3, 2, 64, 16, 1, None) == 1
    assert lib.pkv_copy_blocks(ODD, FAKE, FAKE, 3, 2, 64, 16, 1, None) == 1


@pytest.mark.parametrize("pairs,ok", [
    ([[0, 1], [2, 3]], True),
    ([], True),
    ([[0, 1], [2, 1]], False),   # duplicate dst
    ([[0, 1], [1, 2]], False),   # dst 1 is also a src
    ([[0, 16]], False),          # out of range
    ([[-1, 3]], False),
])
def test_copy_pairs_host_check(pairs, ok):
    from paged_kv_cache_365_b200 import PkvError, copy_blocks_check
    p = np.array(pairs, dtype=np.int32).reshape(-1, 2)
    if ok:
        copy_blocks_check(p, 16)
    else:
        with pytest.raises(PkvError):
            copy_blocks_check(p, 16)


def test_kv_cache_bytes_matches_page_example():
    import json
    from paged_kv_cache_365_b200 import kv_cache_bytes
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "kv_size_example.json")))
    n = kv_cache_bytes(g["layers"], g["heads"], g["head_dim"], g["seq_len"], g["dtype_bytes"])
    assert n == g["expected_bytes"]
    assert abs(n / 1e9 - g["page_figure_gb"]) / g["page_figure_gb"] < g["page_figure_rel_tol"]


def test_prefix_workspace_and_rejections(lib):
    up = lambda x: (x + 15) // 16 * 16
    B, Hq, D, ctx, pp = 4, 8, 128, 1100, 20
    # auto partition: the longest suffix 1100 - 320 = 780 rounded up to 784
    P, C = 2, 1  # ceil(1100/784), ceil(20/64)
    want = up(up(up(up(up(B * Hq * P * D * 4) + B * Hq * P * 8) + B * Hq * C * D * 4) + B * Hq * C * 8) + B * 4)
    assert lib.pkv_decode_prefix_workspace_bytes(B, Hq, D, ctx, pp, 0) == want
    assert lib.pkv_decode_prefix_workspace_bytes(B, Hq, D, ctx, 0, 0) == 0
    # explicit partition 512: P = 3
    want512 = up(up(up(up(up(B * Hq * 3 * D * 4) + B * Hq * 3 * 8) + B * Hq * C * D * 4) + B * Hq * C * 8) + B * 4)
    assert lib.pkv_decode_prefix_workspace_bytes(B, Hq, D, ctx, pp, 512) == want512
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 100, FAKE, 1100, FAKE, 20, 4, 8, 2, 128, 64, ctypes.c_float(0.1), 0,
            1, FAKE, 1 << 30, None]
    for idx, bad in ((17, 0), (9, 0), (9, 101), (8, None), (18, None), (19, 16)):
        a = list(args)
        a[idx] = bad
        assert lib.pkv_paged_attention_decode_prefix(*a) == 1, (idx, bad)
    for phase in (-1, 3):
        assert lib.pkv_paged_attention_decode_prefix_phase(*args[:-1], phase, None) == 1


def multi_ws(T, Hq, D, P):
    """Partials T*Hq*P*D*4 (rounded to 16) + T*Hq*P*8 when P > 1, then the
    tcgen05 kernel's counter (16) and work list (2*T*P entries of 8)."""
    part = 0
    if P > 1:
        o = T * Hq * P * D * 4
        part = (o + 15) // 16 * 16 + T * Hq * P * 8
    return (part + 15) // 16 * 16 + 16 + 2 * T * P * 8


def test_multi_workspace_and_rejections(lib):
    assert lib.pkv_multi_workspace_bytes(10, 8, 128, 512, 512) == multi_ws(10, 8, 128, 1)
    assert lib.pkv_multi_workspace_bytes(10, 8, 128, 1100, 512) == multi_ws(10, 8, 128, 3)
    assert lib.pkv_multi_workspace_bytes(10, 8, 96, 1100, 512) == 0
    # auto partition: 2048 tokens (one partition here), 1024 past 4096 tokens
    assert lib.pkv_multi_workspace_bytes(10, 8, 128, 2048, 0) == multi_ws(10, 8, 128, 1)
    assert lib.pkv_multi_workspace_bytes(10, 8, 128, 5000, 0) == multi_ws(10, 8, 128, 5)
    # 512-token partitions: 1100 tokens split, so the workspace is checked
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 100, FAKE, 1100, FAKE, 8, 40, 4, 8, 2, 128, 64, ctypes.c_float(0.1), 512,
            1, FAKE, 1 << 30, None]
    for idx, bad in ((18, 0), (18, 3), (14, 96), (12, 6), (9, -1), (10, -1), (8, None), (19, None), (20, 16),
                     (7, 100 * 16 + 1), (16, ctypes.c_float(float("inf")))):
        a = list(args)
        a[idx] = bad
        assert lib.pkv_paged_attention_multi(*a) == 1, (idx, bad)
    # grid limit of the kernels below the tcgen05 one: num_seqs * (row tiles
    # per sequence) <= 65535 (8 tokens x G 4 = 32 rows: one tile)
    a = list(args)
    a[11] = 65536
    assert lib.pkv_paged_attention_multi(*a) == 1
    # the tcgen05 kernel's work list: at most 32767 tiles of 128 rows per
    # sequence (2^20 tokens x G 4 = 32768 tiles)
    a = list(args)
    a[9], a[10] = 1 << 20, 1 << 20
    assert lib.pkv_paged_attention_multi(*a) == 1
    # nothing to do
    a = list(args)
    a[10] = 0
    assert lib.pkv_paged_attention_multi(*a) == 0


def test_fp8_rejections(lib):
    f = ctypes.c_float
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 1, f(0.1), f(0.1), None]
    for idx, bad in ((9, 0), (9, 3), (7, 96), (10, f(0.0)), (11, f(-1.0)), (10, f(float("nan"))), (4, None),
                     (2, ODD)):
        a = list(ok)
        a[idx] = bad
        assert lib.pkv_kv_append_fp8(*a) == 1, (idx, bad)
    a = list(ok)
    a[5] = 0
    assert lib.pkv_kv_append_fp8(*a) == 0
    dec = [FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 100, 2, 8, 2, 128, 64, f(0.1), f(0.1), f(0.1), 0, 1, FAKE,
           1 << 30, None]
    for idx, bad in ((17, 0), (17, 3), (14, f(0.0)), (15, f(float("inf"))), (11, 96), (9, 6)):
        a = list(dec)
        a[idx] = bad
        assert lib.pkv_paged_attention_decode_fp8(*a) == 1, (idx, bad)


def test_append_copy_rejections(lib):
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, 2, 2, 64, 16, 1, None]
    for idx, bad in ((11, 7), (9, 80), (8, 0), (5, -1), (7, -1), (2, ODD), (4, None), (6, None)):
        a = list(ok)
        a[idx] = bad
        assert lib.pkv_kv_append_copy(*a) == 1, (idx, bad)
    a = list(ok)
    a[5], a[7] = 0, 0
    assert lib.pkv_kv_append_copy(*a) == 0


def test_cow_copy_rows():
    from paged_kv_cache_365_b200 import cow_copy_rows
    rows = cow_copy_rows(np.array([[3, 7], [4, 9], [5, 11]]), np.array([7 * 16 + 5, 9 * 16 + 15, -1, 9 * 16 + 3]))
    assert rows.tolist() == [[3, 7, 5], [4, 9, 3], [5, 11, 16]]


def test_selftest_bounded_wait_rejects_limits(lib):
    for bad in (0, -5, (1 << 32) + 1):
        assert lib.pkv_selftest_bounded_wait(bad, None) == 1, bad


def test_decode_step_rejections(lib):
    """pkv_decode_step checks its own arguments (the step's writes) before
    anything is launched, then those of the decode it fuses."""
    f = ctypes.c_float
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE, 8, FAKE, 100, None, 0, 4, 8, 2, 128, 64, f(0.1),
          0, 1, None, 0, None]
    for idx, bad in ((22, 0), (22, 3), (8, -1), (8, 5), (7, None), (4, None), (5, ODD), (6, None), (14, -1),
                     (18, 96), (17, 3), (12, 8 * 16 + 1)):
        a = list(ok)
        a[idx] = bad
        assert lib.pkv_decode_step(*a) == 1, (idx, bad)
    # the cascade form needs its prefix blocks and workspace
    a = list(ok)
    a[14] = 4
    assert lib.pkv_decode_step(*a) == 1


def test_decode_step_fp8_rejections(lib):
    """pkv_decode_step_fp8 checks the step's writes, the two scales and the
    FP8 decode's arguments before anything is launched."""
    f = ctypes.c_float
    ok = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE, 8, FAKE, 100, None, 0, 4, 8, 2, 128, 64, f(0.1),
          f(0.05), f(0.05), 0, 1, None, 0, None]
    for idx, bad in ((24, 0), (24, 3), (8, -1), (8, 5), (7, None), (4, None), (5, ODD), (6, None), (18, 96),
                     (17, 3), (12, 8 * 16 + 1), (21, f(0.0)), (22, f(float("inf"))), (22, f(float("nan"))),
                     (21, f(-1.0)), (14, -1)):
        a = list(ok)
        a[idx] = bad
        assert lib.pkv_decode_step_fp8(*a) == 1, (idx, bad)
    # a context past one partition needs the workspace; so does the cascade,
    # which also needs its prefix blocks
    a = list(ok)
    a[10], a[12] = 128, 2000
    assert lib.pkv_decode_step_fp8(*a) == 1
    a = list(ok)
    a[14] = 4
    assert lib.pkv_decode_step_fp8(*a) == 1
    a[13] = FAKE
    assert lib.pkv_decode_step_fp8(*a) == 1


def test_multi_fp8_rejections(lib):
    """pkv_paged_attention_multi_fp8: the multi-token argument checks plus
    the two scales (finite, > 0), all before any CUDA call."""
    f = ctypes.c_float
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 100, FAKE, 1100, FAKE, 8, 40, 4, 8, 2, 128, 64, f(0.1), f(0.05), f(0.05),
            512, 1, FAKE, 1 << 30, None]
    for idx, bad in ((20, 0), (20, 3), (14, 96), (12, 6), (9, -1), (8, None), (21, None), (22, 16),
                     (7, 100 * 16 + 1), (16, f(float("inf"))), (17, f(0.0)), (18, f(-1.0)), (17, f(float("nan"))),
                     (18, f(float("inf")))):
        a = list(args)
        a[idx] = bad
        assert lib.pkv_paged_attention_multi_fp8(*a) == 1, (idx, bad)
    # every shape takes 128-row tiles, at most 32767 a sequence
    a = list(args)
    a[9], a[10] = 1 << 20, 1 << 20
    assert lib.pkv_paged_attention_multi_fp8(*a) == 1
    a = list(args)
    a[10] = 0
    assert lib.pkv_paged_attention_multi_fp8(*a) == 0
