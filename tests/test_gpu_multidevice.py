"""Two devices driven from one process: every kernel's shared-memory opt-in
and every per-device resource must be set up on each device it runs on.
Skipped with fewer than two GPUs."""
import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import check_y, torch

pytestmark = pytest.mark.gpu


def test_forward_on_two_devices_in_one_process():
    t = torch()
    if t.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    spec = gen.workload("small")
    d = gen.make_linear(spec)
    outs = []
    for dev in (0, 1):
        with t.cuda.device(dev):
            to = lambda a: t.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda(dev)  # noqa: E731
            lin = svdq.SvdqLinear(to(d["W"]), t.from_numpy(d["lam"]).cuda(dev), to(d["bias"]), r=spec.r)
            Y = lin.forward(to(d["X"]).view(t.bfloat16))
            t.cuda.synchronize(dev)
            outs.append((Y.view(t.int16).cpu().numpy().view(np.uint16), lin.export()))
    assert np.array_equal(outs[0][0], outs[1][0])
    exp = outs[1][1]
    prep = dict(inv_lambda=exp["inv_lambda"], L1=exp["L1"], L2t=exp["L2t"], w_codes=exp["w_codes"],
                w_scales=exp["w_scales"], bias=d["bias"])
    check_y(outs[1][0], ref.linear_forward(d["X"], prep)["Y64"], "device 1")
