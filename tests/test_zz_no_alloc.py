"""rt_qgemm_noalloc, called through the C ABI, against rt_qgemm_q4/q8.

The entry point runs the same kernels as the workspace entry points on the
same inputs, with the activation scratch in a fixed device array instead of
the workspace, so the two must agree bit for bit.  Checked here:
  - two calls in a row (a weight-streamed q8 GEMM, then an
    activation-resident q4 GEMM that reads less scratch than the first one
    left behind) give exactly the workspace entry point's results, and so
    does the same pair run again over the stale array;
  - those later calls change the free device memory by nothing;
  - the other kernels (SIMT, weight-stationary, weight-streamed q4) agree too;
  - a weight-streamed problem above the scratch limit is rejected and Y is
    left untouched, while the CTA-pair activation-resident kernel, which
    rounds the activations inside the kernel, runs at a size above it.
The file runs alone in a fresh process as well as after the other tests.
"""
import pytest

import int8_dequant_gemm_b200 as rtq
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module", autouse=True)
def rtq_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from int8_dequant_gemm_b200 import build
    build.build()
    return rtq.lib()


def _problem(fmt, M, N, K, seed):
    X = torch.from_numpy(wl.activations(M, K, seed=seed)).cuda()
    W = wl.weights(N, K, seed=seed + 1)
    if fmt == 4:
        Wq, sm = rtq.quantize_q4_g32(W)
        return X, torch.from_numpy(Wq).cuda(), torch.from_numpy(sm).cuda()
    Wq, s = rtq.quantize_q8_row(W)
    return X, torch.from_numpy(Wq).cuda(), torch.from_numpy(s).cuda()


def _reference(fmt, X, Wq, S, path):
    f = rtq.qgemm_q4 if fmt == 4 else rtq.qgemm_q8
    return f(X, Wq, S, path=path)


def _same(Y, Yref):
    """Same kernels, same inputs, same order of operations: the same bits."""
    assert torch.equal(Y, Yref), (Y - Yref).abs().max().item()


def test_two_calls_in_a_row_match_the_workspace_entry_point():
    A = (8, 1000, 700, 2048)     # weight-streamed, 4 MB of scratch
    B = (4, 2048, 1024, 512)     # activation-resident, 2 MB of scratch
    assert rtq.plan(*A) == "tc_w_streamed" and rtq.plan(*B) == "tc_x_resident"
    pa = _problem(*A, seed=501)
    pb = _problem(*B, seed=502)
    ref_a = _reference(A[0], *pa, "auto")
    ref_b = _reference(B[0], *pb, "auto")
    Ya = torch.full_like(ref_a, float("nan"))
    Yb = torch.full_like(ref_b, float("nan"))
    torch.cuda.synchronize()

    rtq.qgemm_noalloc(A[0], *pa, Ya)
    rtq.qgemm_noalloc(B[0], *pb, Yb)
    torch.cuda.synchronize()
    _same(Ya, ref_a)
    _same(Yb, ref_b)

    # the same pair again, over whatever the first pair left in the array
    free_before = torch.cuda.mem_get_info()[0]
    Ya.fill_(float("nan"))
    Yb.fill_(float("nan"))
    rtq.qgemm_noalloc(A[0], *pa, Ya)
    rtq.qgemm_noalloc(B[0], *pb, Yb)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    _same(Ya, ref_a)
    _same(Yb, ref_b)
    assert rtq.device_status() == rtq.OK


@pytest.mark.parametrize("fmt,M,N,K,path", [
    (4, 4, 512, 512, "auto"),        # SIMT
    (8, 80, 512, 512, "auto"),       # weight-stationary tcgen05
    (4, 300, 640, 1024, "tc"),       # weight-streamed q4
    (8, 4096, 512, 512, "tc"),       # activation-resident
    (4, 20000, 256, 512, "auto"),    # CTA pairs, no scratch; M * K * 2 above the scratch size
])
def test_other_kernels_match(fmt, M, N, K, path):
    X, Wq, S = _problem(fmt, M, N, K, seed=510 + M)
    ref = _reference(fmt, X, Wq, S, path)
    Y = torch.full_like(ref, float("nan"))
    rtq.qgemm_noalloc(fmt, X, Wq, S, Y, path=path)
    torch.cuda.synchronize()
    _same(Y, ref)


def test_scratch_limit_rejects_and_leaves_y_untouched():
    M, N, K = 4100, 256, 2048      # M * K * 2 just above 16 MiB
    assert M * K * 2 > rtq.NOALLOC_SCRATCH_BYTES
    assert rtq.plan(8, M, N, K) == "tc_w_streamed"
    X, Wq, S = _problem(8, M, N, K, seed=520)
    Y = torch.full((M, N), 7.0, device="cuda")
    with pytest.raises(rtq.RtqError) as e:
        rtq.qgemm_noalloc(8, X, Wq, S, Y)
    assert e.value.status == rtq.RT_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all())
