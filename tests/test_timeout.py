"""Bounded waits of the decode step (GPU).

The step's work items wait for one another by polling counters; every wait gives up after a
bounded number of polls, raises TWL_FLAG_TIMEOUT, aborts the launch and returns, so the host reads
the error and the context stays usable.  The test makes a wait run out without any device fault:
through the library's test hook the INT4-estimate items wait for a count that nothing reaches,
with a short poll limit.  The next launch on the same workspace must then be exact (the aborted
launch leaves no stale synchronisation words or page masks behind).
"""
import numpy as np
import pytest
import torch

from workloads import synth

from twl_checks import check_step_group

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from adaptive_top_sparse_b200 import twl
    from adaptive_top_sparse_b200.layer import DecodeLayer


def test_decode_step_wait_gives_up_and_the_next_launch_is_exact():
    wl = synth.make_decode("timeout", 2, 8, 2, [700, 300], seed=33, temperature=True)
    layer = DecodeLayer.from_workload(wl)
    layer.build_aux()
    assert layer.status(clear=True)[0] == twl.TWL_OK
    q = torch.from_numpy(wl.q).cuda()
    try:
        twl.twl_test_set_waits(4096, True)
        layer.decode(q, wl.p, wl.eps)
        torch.cuda.synchronize()
    finally:
        twl.twl_test_set_waits(0, False)
    status, flags = layer.status(clear=True)
    assert status == twl.TWL_ERR_TIMEOUT and flags & twl.TWL_FLAG_TIMEOUT
    # the context and the workspace stay usable: the next launches are exact
    for _ in range(2):
        stats = layer.alloc_stats()
        o, lse = layer.decode(q, wl.p, wl.eps, stats)
        st = {k: v.cpu().numpy() for k, v in stats.items()}
        o, lse = o.cpu().numpy(), lse.cpu().numpy()
        for b in range(wl.batch):
            for kvh in range(wl.num_kv_heads):
                check_step_group(wl, b, kvh, st, o, lse)
        assert layer.status()[0] == twl.TWL_OK
    assert np.all(np.isfinite(o))
