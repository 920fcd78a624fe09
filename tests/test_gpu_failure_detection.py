"""Failure detection without a GPU fault: a bounded wait that nothing completes
must give up, report through the device status word and leave the context
usable (no trap, no endless loop, no bad address)."""
import time

import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from workloads import gen

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    import torch
    st = int(torch.cuda.current_stream().cuda_stream)
    svdq.svdq_clear_device_status(st)
    assert svdq.svdq_get_device_status(st) == 0
    t0 = time.perf_counter()
    svdq.svdq_selftest_wait_timeout(20_000_000, st)          # 20 ms limit
    word = svdq.svdq_get_device_status(st)                    # synchronises
    elapsed = time.perf_counter() - t0
    assert word & 1, "timeout bit"
    assert (word >> 8) & 0xFF == 4 and (word >> 16) & 0xFF == 1, hex(word)
    assert 0.015 < elapsed < 5.0, elapsed
    svdq.svdq_clear_device_status(st)
    assert svdq.svdq_get_device_status(st) == 0
    # the context is still usable: a small layer runs and reports no timeout
    rng = np.random.default_rng(3)
    M, K, N = 64, 256, 128
    X = gen.random_bf16(rng, (M, K))
    W = gen.random_bf16(rng, (N, K), 0.02)
    lam = gen.calibrate_lambda(X, W)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()  # noqa: E731
    lin = svdq.SvdqLinear(dev(W), torch.from_numpy(lam).cuda(), None, r=16)
    Y = lin.forward(dev(X).view(torch.bfloat16))
    torch.cuda.synchronize()
    assert torch.isfinite(Y.float()).all()
    assert svdq.svdq_get_device_status(st) == 0
