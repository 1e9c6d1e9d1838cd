"""The fp32 bias fused into the GEMM epilogue (rt_qgemm, list entries, block
recipes) on a GPU: Y = X W^T + b, the bias added to every output row of the
projection ("biases ... stay fp32": int4 card, "Quantization format").
Expected values: the oracle's product plus the bias in double."""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

TOL = {"simt": 1e-5, "tc": 4e-3}


@pytest.fixture(scope="module", autouse=True)
def rtq_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from int8_dequant_gemm_b200 import build
    build.build()
    import int8_dequant_gemm_b200 as rtq
    rtq.lib()
    yield rtq
    torch.cuda.synchronize()
    assert rtq.device_status() == rtq.OK


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rel_err(Y, Yref):
    return float(np.max(np.abs(np.asarray(Y, np.float64) - Yref)) / np.max(np.abs(Yref)))


def problem(fmt, M, N, K, seed):
    X = wl.activations(M, K, seed)
    W = wl.weights(N, K, seed + 1)
    b = (0.5 * wl.activations(1, N, seed + 2)[0]).astype(np.float32)
    if fmt == 4:
        q = oracle.quant_q4_g32(W)
        ref = oracle.gemm_q4(X, *q)
    elif fmt == 8:
        q = oracle.quant_q8_row(W)
        ref = oracle.gemm_q8(X, *q)
    else:
        q = (oracle.quant_e4m3(W), None)
        ref = oracle.gemm_e4m3(X, q[0])
    return X, q, b, ref + b.astype(np.float64)[None, :]


# (fmt, M, N, K, path, kernel)
CASES = [(4, 5, 640, 512, "simt", "simt"), (8, 3, 300, 256, "simt", "simt"),
         (4, 80, 2048, 512, "tc", "tc_w_stationary"), (8, 80, 512, 2048, "tc", "tc_w_stationary"),
         (3, 48, 1001, 512, "tc", "tc_w_stationary"), (4, 300, 1000, 512, "tc", "tc_x_resident"),
         (8, 700, 384, 576, "tc", "tc_w_streamed"), (3, 2048, 512, 2048, "tc", "tc_w_streamed"),
         (4, 16400, 640, 128, "tc", "tc_x_resident_pair")]


@pytest.mark.parametrize("fmt,M,N,K,path,kernel", CASES)
def test_bias_on_every_kernel(rtq_lib, fmt, M, N, K, path, kernel):
    assert rtq_lib.plan(fmt, M, N, K, path) == kernel
    X, q, b, ref = problem(fmt, M, N, K, seed=800 + M + N)
    Y = rtq_lib.qgemm(fmt, dev(X), dev(q[0]), None if q[1] is None else dev(q[1]), dev(b),
                      path=path).cpu().numpy()
    assert rel_err(Y, ref) <= TOL[path]
    # without the bias the same call gives the plain product
    Y0 = rtq_lib.qgemm(fmt, dev(X), dev(q[0]), None if q[1] is None else dev(q[1]), None,
                       path=path).cpu().numpy()
    assert rel_err(Y0, ref - b.astype(np.float64)[None, :]) <= TOL[path]


def test_bias_in_list_entries(rtq_lib):
    M = 80
    specs = [(4, 2048, 512), (8, 512, 2048), (3, 1024, 512), (8, 512, 512)]
    projs, refs = [], []
    for i, (f, N, K) in enumerate(specs):
        X, q, b, ref = problem(f, M, N, K, seed=850 + i)
        bias = dev(b) if i % 2 == 0 else None
        projs.append(rtq_lib.Proj(f, dev(X), dev(q[0]), None if q[1] is None else dev(q[1]),
                                  torch.empty((M, N), device="cuda"), bias))
        refs.append(ref if bias is not None else ref - b.astype(np.float64)[None, :])
    rtq_lib.qgemm_batch(projs, path="tc")
    for p, ref in zip(projs, refs):
        assert rel_err(p.Y.cpu().numpy(), ref) <= TOL["tc"]


@pytest.mark.parametrize("M", [80, 2048])
def test_bias_in_block_recipe(rtq_lib, M):
    names = ("qkvg", "wo", "w13", "w2")
    fmts = (4, 8, 4, 8)
    host, ws = {}, []
    for i, (n, f) in enumerate(zip(names, fmts)):
        spec = wl.BLOCK_PROJECTIONS[n]
        X, q, b, ref = problem(f, M, spec["N"], spec["K"], seed=870 + i)
        host[n] = (X, ref)
        ws.append((f, dev(q[0]), dev(q[1]), dev(b)))
    blk = rtq_lib.QBlockFmt(*ws)
    Y = [torch.empty((M, wl.BLOCK_PROJECTIONS[n]["N"]), device="cuda") for n in names]
    rtq_lib.qblock_project_fmt(blk, *(dev(host[n][0]) for n in names), *Y)
    rows = None if M <= 128 else wl.sample_rows(M, 64, seed=3)
    for n, y in zip(names, Y):
        got = y.cpu().numpy() if rows is None else y.cpu().numpy()[rows]
        ref = host[n][1] if rows is None else host[n][1][rows]
        assert rel_err(got, ref) <= TOL["tc"], n
