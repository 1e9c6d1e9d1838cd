"""FP8 E4M3 weights ("RT-J -- FP8 E4M3 checkpoints", "FP8 Format": weight
matrices hold float8_e4m3fn values, no scale) on a GPU, through the C ABI.

  - dequantization exports: every finite code to its exact value, in fp32
    and in fp16 (the tensor-core operand), bit for bit against the oracle;
  - X = I gives the weights transposed, bit for bit, on both paths;
  - GEMM parity on every kernel (SIMT <= 1e-5; weight-stationary with and
    without split K, activation-resident, weight-streamed, the projection
    list and the grouped block launch <= 4e-3 and within the fp16 rounding
    bound of the activations; e4m3 weights are exact in fp16).
Weights are N(0, 0.02^2) rounded by the oracle's e4m3 encoder.
"""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

SIMT_TOL = 1e-5
TC_TOL = 4e-3


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


def weights(N, K, seed, outliers=True):
    W = wl.weights(N, K, seed)
    if outliers:
        W = wl.with_outliers(W, seed + 1)
    return oracle.quant_e4m3(W)


def within_bound(Y, X, What):
    """Only the activations are rounded (to fp16, relative 2^-11) and the sum
    is fp32; fp16-subnormal activations carry an absolute 2^-25 instead."""
    u = 2.0 ** -11
    A = np.abs(X.astype(np.float64)) @ np.abs(What).T
    slack = 2.0 ** -25 * np.abs(What).sum(axis=1)[None, :]
    bound = (u + (X.shape[1] + 1) * 2.0 ** -23) * A + slack
    return not (np.abs(np.asarray(Y, np.float64) - X.astype(np.float64) @ What.T) > bound).any()


def test_dequant_exports_bit_exact(rtq_lib):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    g = np.random.default_rng(3)
    Wq = np.concatenate([np.resize(codes, 16 * 64), g.choice(codes, 48 * 64)]).reshape(64, 64)
    exact = oracle.dequant_e4m3(Wq)
    got32 = rtq_lib.dequant_e4m3_f32(dev(Wq)).cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), exact.astype(np.float32).view(np.uint32))
    got16 = rtq_lib.dequant_e4m3_f16(dev(Wq)).cpu().numpy()
    assert np.array_equal(got16, exact.astype(np.float16).view(np.uint16))
    # every e4m3 value is exact in fp16
    assert np.array_equal(exact.astype(np.float16).astype(np.float64), exact)


@pytest.mark.parametrize("path", ["simt", "tc"])
def test_identity_input_bit_exact(rtq_lib, path):
    N, K = 256, 512
    Wq = weights(N, K, 31)
    Y = rtq_lib.gemm_e4m3(torch.eye(K, device="cuda"), dev(Wq), path=path)
    assert np.array_equal(Y.cpu().numpy(), oracle.dequant_e4m3(Wq).astype(np.float32).T)


SHAPES = [(5, 640, 1024, "simt"), (80, 512, 2048, "tc_w_stationary"),
          (1, 128, 64, "tc_w_stationary"), (300, 1000, 512, "tc_x_resident"),
          (700, 384, 576, "tc_w_streamed"), (2048, 512, 2048, "tc_w_streamed"),
          (16400, 256, 128, "tc_x_resident_pair")]


@pytest.mark.parametrize("M,N,K,kernel", SHAPES)
def test_gemm_parity(rtq_lib, M, N, K, kernel):
    path = "simt" if kernel == "simt" else "tc"
    assert rtq_lib.plan(3, M, N, K, path) == kernel
    X = wl.activations(M, K, 40 + M)
    Wq = weights(N, K, 50 + N)
    Y = rtq_lib.gemm_e4m3(dev(X), dev(Wq), path=path).cpu().numpy()
    ref = oracle.gemm_e4m3(X, Wq)
    assert rel_err(Y, ref) <= (SIMT_TOL if path == "simt" else TC_TOL)
    if path == "tc":
        assert within_bound(Y, X, oracle.dequant_e4m3(Wq))


def test_list_kernel_with_e4m3_entries(rtq_lib):
    M = 80
    specs = [(3, 2048, 512), (4, 1024, 512), (3, 512, 2048), (8, 512, 512), (3, 300, 1024)]
    projs, refs = [], []
    for i, (f, N, K) in enumerate(specs):
        X = wl.activations(M, K, 60 + i)
        W = wl.weights(N, K, 70 + i)
        if f == 3:
            q = (oracle.quant_e4m3(W), None)
            refs.append(oracle.gemm_e4m3(X, q[0]))
        elif f == 4:
            q = oracle.quant_q4_g32(W)
            refs.append(oracle.gemm_q4(X, *q))
        else:
            q = oracle.quant_q8_row(W)
            refs.append(oracle.gemm_q8(X, *q))
        projs.append(rtq_lib.Proj(f, dev(X), dev(q[0]), None if q[1] is None else dev(q[1]),
                                  torch.empty((M, N), device="cuda")))
    assert rtq_lib.batch_plan(projs, path="tc") == "tc_list"
    rtq_lib.qgemm_batch(projs, path="tc")
    for p, ref in zip(projs, refs):
        assert rel_err(p.Y.cpu().numpy(), ref) <= TC_TOL


@pytest.mark.parametrize("M", [80, 2048])
def test_all_e4m3_block(rtq_lib, M):
    """The FP8 card's recipe: every block projection in e4m3 (grouped launch
    at M = 80, one call each at M = 2048, checked on sampled rows)."""
    names = ("qkvg", "wo", "w13", "w2")
    host = {}
    for i, n in enumerate(names):
        W = wl.projection_weights(3, 0, n)
        host[n] = oracle.quant_e4m3(W)
        host["x_" + n] = wl.projection_input(3, 0, n, M)
    blk = rtq_lib.QBlockFmt(*((3, dev(host[n]), None) for n in names))
    assert rtq_lib.block_fused_fmt(blk, M) == (1 if M <= 128 else 0)
    Y = [torch.empty((M, wl.BLOCK_PROJECTIONS[n]["N"]), device="cuda") for n in names]
    rtq_lib.qblock_project_fmt(blk, *(dev(host["x_" + n]) for n in names), *Y)
    rows = None if M <= 128 else wl.sample_rows(M, 64, seed=9)
    for n, y in zip(names, Y):
        ref = oracle.gemm_e4m3(host["x_" + n], host[n], rows=rows)
        got = y.cpu().numpy() if rows is None else y.cpu().numpy()[rows]
        assert rel_err(got, ref) <= TC_TOL, n
