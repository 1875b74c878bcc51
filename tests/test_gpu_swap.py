"""GPU parity of preemption by swapping: the library's allocator plans the
swap, pkv_swap_blocks moves the blocks between the device pool and a pinned
host pool, and the oracle (RefAllocator + RefCache + swap_blocks) does the
same on the CPU.  Bit-exact: copy pairs, every held block of both pools;
attention after the round trip within the decode tolerance of the fp64
oracle.  The device pool starts as NaN, so a block the copy missed shows."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def pkv():
    import paged_kv_cache_365_b200 as m
    return m


def bits(t):
    return t.cpu().view(torch.int16).numpy()


def obits(a):
    return a.view(np.int16)


def draw(rng, n, Hkv, D):
    return rng.standard_normal((2, n, Hkv, D)).astype(np.float16)


@pytest.mark.parametrize("Hkv,D", [(4, 128), (2, 64)])
def test_swap_round_trip_matches_oracle(Hkv, D):
    m = pkv()
    rng = np.random.default_rng(11)
    nb, nh = 40, 48
    order = rng.permutation(nb).astype(np.int32)
    cache = m.PagedKVCache(nb, Hkv, D, torch.float16, free_order=order)
    cache.enable_swap(nh)
    ref = oracle.RefAllocator(nb, order, num_host_blocks=nh)
    dev = oracle.RefCache(nb, Hkv, D, "f16")
    host = oracle.RefCache(nh, Hkv, D, "f16")

    def write(sid, n):
        vals = draw(rng, n, Hkv, D)
        slots, cows = ref.append_tokens(sid, n)
        dev.copy_blocks(cows)
        dev.append(vals[0], vals[1], np.array(slots))
        gs = cache.prefill(sid, torch.from_numpy(vals[0]), torch.from_numpy(vals[1]))
        assert list(gs) == list(slots)

    for sid in (0, 1, 2):
        ref.add_seq(sid)
        cache.add_seq(sid)
    write(0, 70)
    ref.fork(0, 3)
    cache.fork(0, 3)
    write(3, 9)          # copy-on-write of the shared partial block
    write(1, 33)
    write(2, 100)

    out_pairs = ref.swap_out([0, 3, 1])
    oracle.swap_blocks(host, dev, out_pairs)
    g_pairs = cache.swap_out([0, 3, 1])
    assert [tuple(int(x) for x in p) for p in g_pairs] == out_pairs
    # a new sequence takes (and overwrites) the released device blocks
    ref.add_seq(9)
    cache.add_seq(9)
    write(9, 150)
    in_pairs = ref.swap_in([1, 3, 0])
    oracle.swap_blocks(dev, host, in_pairs)
    g_pairs = cache.swap_in([1, 3, 0])
    assert [tuple(int(x) for x in p) for p in g_pairs] == in_pairs
    torch.cuda.synchronize()
    assert m.get_error() == 0
    assert cache.alloc.state() == ref.state() and cache.alloc.host_state() == ref.host_state()

    held = sorted({b for t in ref.tables.values() for b in t})
    assert np.array_equal(bits(cache.k)[held], obits(dev.k)[held])
    assert np.array_equal(bits(cache.v)[held], obits(dev.v)[held])
    written = sorted({h for _, h in out_pairs})
    assert np.array_equal(bits(cache.host_k)[written], obits(host.k)[written])
    assert np.array_equal(bits(cache.host_v)[written], obits(host.v)[written])

    # attention over the swapped-back sequences and the newcomer
    sids = [0, 1, 2, 3, 9]
    tables = [ref.block_table(s)[0] for s in sids]
    lens = np.array([ref.block_table(s)[1] for s in sids], dtype=np.int32)
    w = max(len(t) for t in tables)
    bt = np.array([t + [nb + 7] * (w - len(t)) for t in tables], dtype=np.int32)
    q = rng.standard_normal((len(sids), 2 * Hkv, D)).astype(np.float16)
    want = oracle.paged_decode(q, dev.k, dev.v, bt, lens, D ** -0.5, "f16")
    got = m.paged_attention_decode(torch.from_numpy(q).cuda(), cache.k, cache.v, torch.from_numpy(bt).cuda(),
                                   torch.from_numpy(lens).cuda(), int(lens.max()), D ** -0.5)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    assert np.abs(got.float().cpu().numpy() - want).max() <= 2e-3


def test_swap_blocks_large_and_direct():
    """7B-shaped blocks (32 kv-heads, D 128, bf16: 128 KiB of K per block):
    300 scattered blocks out to pinned memory and back into other blocks,
    bit for bit; pairs given in pinned host memory work too."""
    m = pkv()
    g = torch.Generator(device="cuda").manual_seed(5)
    nb, nh, n = 700, 400, 300
    shape = (nb, 32, 16, 128)
    k = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
    hk = torch.empty((nh,) + shape[1:], dtype=torch.bfloat16, pin_memory=True)
    hv = torch.empty((nh,) + shape[1:], dtype=torch.bfloat16, pin_memory=True)
    rng = np.random.default_rng(3)
    src = rng.choice(nb, n, replace=False)
    hdst = rng.choice(nh, n, replace=False)
    out_pairs = np.stack([src, hdst], 1).astype(np.int32)
    m.swap_blocks_check(out_pairs, nb, nh)
    m.swap_blocks(hk, hv, k, v, torch.from_numpy(out_pairs).cuda())
    back = rng.choice(np.setdiff1d(np.arange(nb), src), n, replace=False)
    in_pairs = np.stack([hdst, back], 1).astype(np.int32)
    k2, v2 = k.clone(), v.clone()
    m.swap_blocks(k2, v2, hk, hv, torch.from_numpy(in_pairs).pin_memory())
    torch.cuda.synchronize()
    assert m.get_error() == 0
    s, b = torch.from_numpy(src).cuda(), torch.from_numpy(back).cuda()
    assert torch.equal(k2[b].view(torch.int16), k[s].view(torch.int16))
    assert torch.equal(v2[b].view(torch.int16), v[s].view(torch.int16))
    untouched = torch.from_numpy(np.setdiff1d(np.arange(nb), back)).cuda()
    assert torch.equal(k2[untouched].view(torch.int16), k[untouched].view(torch.int16))


def test_swap_range_flags_and_rejections():
    m = pkv()
    shape = (8, 2, 16, 64)
    k = torch.zeros(shape, dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    hk = torch.ones(shape, dtype=torch.float16, pin_memory=True)
    hv = torch.ones(shape, dtype=torch.float16, pin_memory=True)
    # one good pair, one naming a block past the destination pool
    pairs = torch.tensor([[1, 2], [3, 8]], dtype=torch.int32, device="cuda")
    m.swap_blocks(k, v, hk, hv, pairs)
    torch.cuda.synchronize()
    assert m.get_error() == m.ERR_COPY_RANGE
    assert torch.equal(k[2], hk[1].cuda()) and k.sum().item() == 16 * 64 * 2
    # pageable host memory is refused before anything is launched
    pageable = torch.ones(shape, dtype=torch.float16)
    with pytest.raises(ValueError):
        m.swap_blocks(k, v, pageable, pageable, pairs)
    lib = m._lib.lib
    st = lib.pkv_swap_blocks(k.data_ptr(), v.data_ptr(), 8, pageable.data_ptr(), pageable.data_ptr(), 8,
                             pairs.data_ptr(), 2, 2, 64, 1, None)
    assert st == 1
    torch.cuda.synchronize()
    assert m.get_error() == 0
