"""The kernels' failure path on a B200 without a fault: their waits on
staged copies are bounded, give up with PKV_ERR_TIMEOUT in the device error
word, and leave the context usable (a decode right after still matches the
oracle).  The wait is made to run out on a barrier that nothing completes."""
import numpy as np
import pytest
import torch

import oracle
from helpers import make_multi_case

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_flags_timeout():
    import paged_kv_cache_365_b200 as m
    assert m.get_error() == 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    m.selftest_bounded_wait(2_000_000)  # ~1 ms at 2 GHz
    end.record()
    torch.cuda.synchronize()
    assert m.get_error() & m.ERR_TIMEOUT
    assert m.get_error() == 0  # read and cleared
    assert start.elapsed_time(end) < 1000.0


def test_context_usable_after_a_timeout():
    import paged_kv_cache_365_b200 as m
    m.selftest_bounded_wait(100_000)
    torch.cuda.synchronize()
    assert m.get_error() == m.ERR_TIMEOUT
    c = make_multi_case([5, 40, 300], [1, 1, 1], 8, 2, 128, "f16", seed=11)  # one query per sequence
    scale = 128 ** -0.5
    want = oracle.paged_decode(c["q"], c["k"], c["v"], c["tables"], c["ctx"], scale, "f16")
    out = m.paged_attention_decode(torch.from_numpy(c["q"]).cuda(), torch.from_numpy(c["k"]).cuda(),
                                   torch.from_numpy(c["v"]).cuda(), torch.from_numpy(c["tables"]).cuda(),
                                   torch.from_numpy(c["ctx"]).cuda(), int(c["ctx"].max()), scale)
    torch.cuda.synchronize()
    assert m.get_error() == 0
    assert np.abs(out.float().cpu().numpy() - want).max() <= 2e-3
