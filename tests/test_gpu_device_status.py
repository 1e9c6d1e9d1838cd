"""The device status word on a GPU: bounded waits that run out, and
activations outside the fp16 operand range.

Failure path (no GPU fault, no hang): rt_debug_inject(1, 2 ms) makes the first
producer arrival of every CTA go missing -- in the weight-stationary kernels a
converter thread skips its arrival on the first stage, in the TMA-fed kernels
the weight TMA thread never requests its first box -- so a consumer's wait,
bounded to 2 ms, runs out.  The kernel must then wind down (drain its issued
MMAs and copies, release TMEM, pass every cluster barrier), latch
RT_ERR_DEVICE_TIMEOUT, and leave the context usable: after
rt_debug_inject(0, 0) the same call gives the oracle's result again.

Range: the tensor-core path rounds activations to fp16; an activation that
rounds to infinity latches RT_ERR_OPERAND_RANGE (the SIMT path keeps fp32 and
reports nothing).
"""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

TC_TOL = 4e-3
WAIT_NS = 2_000_000     # 2 ms bound while a failure is injected


@pytest.fixture(scope="module", autouse=True)
def rtq_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from int8_dequant_gemm_b200 import build
    build.build()
    import int8_dequant_gemm_b200 as rtq
    rtq.lib()
    torch.cuda.synchronize()
    assert rtq.device_status() == rtq.OK
    yield rtq
    rtq.debug_inject(0, 0)
    torch.cuda.synchronize()
    assert rtq.device_status() == rtq.OK


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rel_err(Y, Yref):
    return float(np.max(np.abs(np.asarray(Y, np.float64) - Yref)) / np.max(np.abs(Yref)))


def _problem(fmt, M, N, K, seed):
    X = wl.activations(M, K, seed)
    W = wl.weights(N, K, seed + 1)
    q = oracle.quant_q4_g32(W) if fmt == 4 else oracle.quant_q8_row(W)
    ref = (oracle.gemm_q4 if fmt == 4 else oracle.gemm_q8)(X, *q)
    return X, q, ref


# (fmt, M, N, K, kernel): one launch of each tensor-core kernel family
CASES = [
    (4, 80, 256, 64, "tc_w_stationary"),      # one CTA per tile, no split (one K step)
    (4, 80, 256, 128, "tc_w_stationary"),     # K split over clusters of 2 CTAs
    (8, 80, 512, 2048, "tc_w_stationary"),    # K split over clusters of 8 CTAs
    (4, 300, 512, 512, "tc_x_resident"),
    (4, 16500, 384, 256, "tc_x_resident_pair"),
    (8, 300, 512, 1024, "tc_w_streamed"),
    (4, 700, 384, 768, "tc_w_streamed"),
]


@pytest.mark.parametrize("fmt,M,N,K,kernel", CASES)
def test_injected_missing_arrival_times_out_and_recovers(rtq_lib, fmt, M, N, K, kernel):
    assert rtq_lib.plan(fmt, M, N, K) == kernel
    X, q, ref = _problem(fmt, M, N, K, seed=900 + M + K)
    Xd, Wd, Sd = dev(X), dev(q[0]), dev(q[1])
    fn = rtq_lib.qgemm_q4 if fmt == 4 else rtq_lib.qgemm_q8
    rtq_lib.debug_inject(1, WAIT_NS)
    try:
        fn(Xd, Wd, Sd)                           # enqueued fine; the device gives up
        assert rtq_lib.device_status() == rtq_lib.RT_ERR_DEVICE_TIMEOUT
    finally:
        rtq_lib.debug_inject(0, 0)
    assert rtq_lib.device_status() == rtq_lib.OK   # the word was cleared by the read
    Y = fn(Xd, Wd, Sd).cpu().numpy()
    assert rtq_lib.device_status() == rtq_lib.OK
    assert rel_err(Y, ref) <= TC_TOL


def test_injected_timeout_in_grouped_block_launch(rtq_lib):
    """The block driver's grouped launch at M = 80: four projections in
    clusters with per-projection K splits; no cluster stores a tile."""
    M = 80
    assert rtq_lib.block_fused(M, 512, 2048) == 1
    host = {}
    for i, name in enumerate(("qkvg", "wo", "w13", "w2")):
        spec = wl.BLOCK_PROJECTIONS[name]
        W = wl.weights(spec["N"], spec["K"], 950 + i)
        host[name] = oracle.quant_q4_g32(W) if spec["fmt"] == "q4" else oracle.quant_q8_row(W)
        host["x_" + name] = wl.activations(M, spec["K"], 960 + i)
    blk = rtq_lib.QBlock(*(dev(a) for n in ("qkvg", "wo", "w13", "w2") for a in host[n]))
    X = [dev(host["x_" + n]) for n in ("qkvg", "wo", "w13", "w2")]
    Y = [torch.full((M, wl.BLOCK_PROJECTIONS[n]["N"]), 7.0, device="cuda")
         for n in ("qkvg", "wo", "w13", "w2")]
    rtq_lib.debug_inject(1, WAIT_NS)
    try:
        rtq_lib.qblock_project(blk, *X, *Y)
        assert rtq_lib.device_status() == rtq_lib.RT_ERR_DEVICE_TIMEOUT
    finally:
        rtq_lib.debug_inject(0, 0)
    # every CTA timed out, so no tile passed the cluster's all-finished check
    for y in Y:
        assert bool((y == 7.0).all())
    rtq_lib.qblock_project(blk, *X, *Y)
    assert rtq_lib.device_status() == rtq_lib.OK
    for n, y in zip(("qkvg", "wo", "w13", "w2"), Y):
        gemm = oracle.gemm_q4 if wl.BLOCK_PROJECTIONS[n]["fmt"] == "q4" else oracle.gemm_q8
        assert rel_err(y.cpu().numpy(), gemm(host["x_" + n], *host[n])) <= TC_TOL, n


@pytest.mark.parametrize("M,kernel", [(80, "tc_w_stationary"), (80, "tc_w_stationary_split"),
                                      (300, "tc_x_resident"), (16500, "tc_x_resident_pair")])
def test_activation_outside_fp16_range_is_reported(rtq_lib, M, kernel):
    N, K = {"tc_w_stationary": (256, 64), "tc_w_stationary_split": (512, 2048),
            "tc_x_resident": (256, 512), "tc_x_resident_pair": (256, 256)}[kernel]
    X, q, _ = _problem(8, M, N, K, seed=970 + M)
    X[M // 2, 3] = 1.0e5                         # rounds to +inf in fp16
    Xd, Wd, Sd = dev(X), dev(q[0]), dev(q[1])
    Y = rtq_lib.qgemm_q8(Xd, Wd, Sd, path="tc")
    assert rtq_lib.device_status() == rtq_lib.RT_ERR_OPERAND_RANGE
    assert not bool(torch.isfinite(Y[M // 2]).all())
    assert bool(torch.isfinite(Y[: M // 2]).all())
    # the fp32 SIMT path holds the value and has nothing to report
    Ys = rtq_lib.qgemm_q8(Xd, Wd, Sd, path="simt")
    assert rtq_lib.device_status() == rtq_lib.OK
    assert bool(torch.isfinite(Ys).all())
    # in range again: nothing reported
    X[M // 2, 3] = 1.0
    rtq_lib.qgemm_q8(dev(X), Wd, Sd, path="tc")
    assert rtq_lib.device_status() == rtq_lib.OK


def test_injected_timeout_in_list_kernel(rtq_lib):
    """The projection-list kernel: the first weight slot of every CTA never
    completes, so its dequantizers' waits run out; the weight producers
    still drain their copies and the CTA releases TMEM."""
    M = 80
    shapes = [(4, 2048, 512), (8, 512, 2048), (4, 1024, 512)]
    host = [_problem(f, M, n, k, seed=990 + i) for i, (f, n, k) in enumerate(shapes)]
    projs = [rtq_lib.Proj(f, dev(X), dev(q[0]), dev(q[1]), torch.full((M, n), 7.0, device="cuda"))
             for (f, n, k), (X, q, _) in zip(shapes, host)]
    assert rtq_lib.batch_plan(projs, path="tc") == "tc_list"
    rtq_lib.debug_inject(1, WAIT_NS)
    try:
        rtq_lib.qgemm_batch(projs, path="tc")
        assert rtq_lib.device_status() == rtq_lib.RT_ERR_DEVICE_TIMEOUT
    finally:
        rtq_lib.debug_inject(0, 0)
    rtq_lib.qgemm_batch(projs, path="tc")
    assert rtq_lib.device_status() == rtq_lib.OK
    for p, (_, _, ref) in zip(projs, host):
        assert rel_err(p.Y.cpu().numpy(), ref) <= TC_TOL


def test_activation_outside_fp16_range_in_list_kernel(rtq_lib):
    M = 48
    X, q, _ = _problem(4, M, 1024, 512, seed=995)
    X[5, 100] = -7.0e4
    Y = torch.empty((M, 1024), device="cuda")
    rtq_lib.qgemm_batch([rtq_lib.Proj(4, dev(X), dev(q[0]), dev(q[1]), Y)], path="tc")
    assert rtq_lib.device_status() == rtq_lib.RT_ERR_OPERAND_RANGE
    assert not bool(torch.isfinite(Y[5]).all()) and bool(torch.isfinite(Y[6:]).all())
