"""Head-major output (the QKV layout for attention consumers): the GEMM and the
whole layer write Y[h][m][d] = Y[m][h * head_dim + d], bit for bit the values
of the row-major path."""
import numpy as np
import pytest

from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import check_y, dev_f32, dev_u16, gpu_d, stream, to_np_u16, torch, y_with_d

pytestmark = pytest.mark.gpu

svdq = pytest.importorskip("w4a4_rank_corrected_act_b200")


def _layer(M, K, N, r, seed):
    spec = gen.LinearSpec("heads", M, K, N, r, seed)
    d = gen.make_linear(spec)
    lin = svdq.SvdqLinear(dev_u16(d["W"]), dev_f32(d["lam"]), dev_u16(d["bias"]), r=r)
    torch().cuda.synchronize()
    return lin, d


def _to_heads(Y, head_dim):
    M, N = Y.shape
    return np.ascontiguousarray(Y.reshape(M, N // head_dim, head_dim).transpose(1, 0, 2))


# (M, K, N, r, head_dim): ragged M, r = 0 / 16 / 32, and one shape with more
# tiles than SMs so that CTAs store tiles through both epilogue paths
@pytest.mark.parametrize("act_kernel", [0, 2], ids=["auto", "act128"])
@pytest.mark.parametrize("M,K,N,r,hd", [(300, 512, 768, 32, 128), (129, 1024, 512, 16, 64),
                                         (40, 768, 384, 0, 32), (2048, 256, 2048, 32, 128)])
def test_heads_layout_matches_row_major(M, K, N, r, hd, act_kernel):
    """act_kernel 2 forces the 128-row activation kernel (D on the tensor cores)."""
    with svdq.override(svdq.SVDQ_OVERRIDE_ACT_KERNEL, act_kernel):
        _heads_case(M, K, N, r, hd)


def _heads_case(M, K, N, r, hd):
    t = torch()
    lin, d = _layer(M, K, N, r, seed=M + K + N + hd)
    X = dev_u16(d["X"])
    nb = lin.workspace_bytes(M)
    ws = t.empty(max(nb, 256), dtype=t.uint8, device="cuda")
    Y = t.empty((M, N), dtype=t.int16, device="cuda")
    Yh = t.full((N // hd, M, hd), 0x5A5A, dtype=t.int16, device="cuda")
    svdq.svdq_linear_forward(X.data_ptr(), M, lin.w, Y.data_ptr(), ws.data_ptr(), nb, stream())
    svdq.svdq_linear_forward_heads(X.data_ptr(), M, lin.w, hd, Yh.data_ptr(), ws.data_ptr(), nb, stream())
    t.cuda.synchronize()
    yr = to_np_u16(Y)
    assert np.array_equal(to_np_u16(Yh), _to_heads(yr, hd))
    # and against the oracle through the row-major view
    exp = lin.export()
    prep = dict(inv_lambda=exp["inv_lambda"], L1=exp["L1"], L2t=exp["L2t"], w_codes=exp["w_codes"],
                w_scales=exp["w_scales"], bias=d["bias"])
    o = ref.linear_forward(d["X"], prep)
    back = to_np_u16(Yh).transpose(1, 0, 2).reshape(M, N)
    yd = y_with_d(o["Y64"], o["D"], gpu_d(lin, X, M), exp["L2t"]) if r else None
    check_y(back, o["Y64"], "heads", y_given_gpu_d=yd)


def test_gemm_heads_16_byte_aligned_output():
    """Only 16-byte-aligned Y: the last tiles' direct stores take two 16-byte stores."""
    t = torch()
    M, K, N, r, hd = 200, 512, 512, 32, 64
    lin, d = _layer(M, K, N, r, seed=5)
    X = dev_u16(d["X"])
    codes = t.empty(svdq.svdq_act_codes_bytes(M, K), dtype=t.uint8, device="cuda")
    scales = t.empty(svdq.svdq_act_scales_bytes(M, K), dtype=t.uint8, device="cuda")
    D = t.empty((M, r), dtype=t.int16, device="cuda")
    svdq.svdq_quantize_act(X.data_ptr(), M, lin.w, codes.data_ptr(), scales.data_ptr(), D.data_ptr(), stream())
    Y = t.empty((M, N), dtype=t.int16, device="cuda")
    svdq.svdq_gemm(codes.data_ptr(), scales.data_ptr(), D.data_ptr(), M, lin.w, Y.data_ptr(), stream())
    guard = 0x5A5A
    buf = t.full((M * N + 64,), guard, dtype=t.int16, device="cuda")
    Yh = buf[8:8 + M * N]
    assert Yh.data_ptr() % 32 == 16
    svdq.svdq_gemm_heads(codes.data_ptr(), scales.data_ptr(), D.data_ptr(), M, lin.w, hd, Yh.data_ptr(),
                         stream())
    t.cuda.synchronize()
    assert np.array_equal(to_np_u16(Yh).reshape(N // hd, M, hd), _to_heads(to_np_u16(Y), hd))
    rest = to_np_u16(buf)
    assert np.all(rest[:8] == guard) and np.all(rest[8 + M * N:] == guard)


def test_heads_rejects_bad_head_dim():
    t = torch()
    lin, d = _layer(64, 256, 384, 16, seed=7)
    ws = t.empty(max(lin.workspace_bytes(64), 256), dtype=t.uint8, device="cuda")
    Y = t.empty((64, 384), dtype=t.int16, device="cuda")
    X = dev_u16(d["X"])
    for hd in (24, 256, 0):                 # not a multiple of 16 / does not divide N / zero
        with pytest.raises(svdq.SvdqError, match="INVALID_ARG"):
            svdq.svdq_linear_forward_heads(X.data_ptr(), 64, lin.w, hd, Y.data_ptr(), ws.data_ptr(),
                                           lin.workspace_bytes(64), stream())
