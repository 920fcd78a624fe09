"""GPU test of svdq_linear_forward_noalloc, the forward for callers that cannot
allocate device memory (plugin hosts that own the allocator, latency-critical
loops where cudaMalloc would synchronise): its output must match
svdq_linear_forward's on two calls in a row, and oversized shapes must be
refused.  This file is collected last so that a run stopping at the first
failure has run every other test; it also passes on its own."""
import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from workloads import gen

pytestmark = pytest.mark.gpu


def _linear(M, K, N, r, seed):
    import torch
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    x[:, rng.choice(K, 4, replace=False)] *= 40
    w = rng.standard_normal((N, K)) * 0.02
    X, W = gen.to_bf16_bits(x), gen.to_bf16_bits(w)
    B = gen.to_bf16_bits(rng.standard_normal(N) * 0.01)
    lam = gen.calibrate_lambda(X, W)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()  # noqa: E731
    lin = svdq.SvdqLinear(dev(W), torch.from_numpy(lam).cuda(), dev(B), r=r)
    return lin, dev(X)


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


def _close(a_bits, b_bits):
    """The parity bar of the other tests: 4e-3 rms + 2 bf16 ulps per element."""
    a = (a_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = (b_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rms = np.sqrt(np.mean(b ** 2))
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    assert np.all(np.abs(a - b) <= 4e-3 * rms + 2 * ulp)


def test_noalloc_matches_workspace_forward_on_two_calls():
    import torch
    st = int(torch.cuda.current_stream().cuda_stream)
    for seed, (M, K, N, r) in enumerate([(300, 512, 384, 32), (1000, 1024, 640, 16)]):
        lin, X = _linear(M, K, N, r, 100 + seed)
        Y_ref = torch.empty((M, N), dtype=torch.int16, device="cuda")
        nb = lin.workspace_bytes(M)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        svdq.svdq_linear_forward(X.data_ptr(), M, lin.w, Y_ref.data_ptr(), ws.data_ptr(), nb, st)
        Y = torch.full((M, N), -1, dtype=torch.int16, device="cuda")
        svdq.svdq_linear_forward_noalloc(X.data_ptr(), M, lin.w, Y.data_ptr(), st)
        torch.cuda.synchronize()
        _close(_bits(Y), _bits(Y_ref))
        # a second call in a row, on new inputs, reuses the same scratch
        lin2, X2 = _linear(M, K, N, r, 200 + seed)
        Y2_ref = torch.empty((M, N), dtype=torch.int16, device="cuda")
        svdq.svdq_linear_forward(X2.data_ptr(), M, lin2.w, Y2_ref.data_ptr(), ws.data_ptr(), nb, st)
        Y2 = torch.full((M, N), -1, dtype=torch.int16, device="cuda")
        svdq.svdq_linear_forward_noalloc(X2.data_ptr(), M, lin2.w, Y2.data_ptr(), st)
        torch.cuda.synchronize()
        _close(_bits(Y2), _bits(Y2_ref))
    assert svdq.svdq_get_device_status(st) == 0


def test_noalloc_refuses_shapes_beyond_its_scratch():
    import torch
    st = int(torch.cuda.current_stream().cuda_stream)
    lin, X = _linear(64, 512, 256, 32, 7)
    M_big = 200000                    # codes + scales + D of 200000 rows exceed 64 MiB
    need = svdq.svdq_forward_workspace_bytes(M_big, 256, 512, 32)
    assert need > (64 << 20)
    with pytest.raises(svdq.SvdqError, match="WORKSPACE_TOO_SMALL.*fixed scratch"):
        svdq.svdq_linear_forward_noalloc(X.data_ptr(), M_big, lin.w, X.data_ptr(), st)
