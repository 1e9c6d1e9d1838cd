"""The int8 card's all-int8 (Q8_0-style) block recipe through
rt_qblock_project_fmt on a GPU: every projection q8 with a per-row fp32
scale, qkvg a q8 [2048, 512] tensor and w13 a q8 [4096, 512] tensor
("RT-J -- int8 (Q8_0-style) quantized checkpoints", "Quantization format").

At M = 80 the four projections run as one grouped launch; at M = 2048 and
4096 qkvg, wo and w13 share one launch of the activation-resident kernel
(its q8 build) and w2 runs on the weight-streamed kernel (checked on sampled
rows).  A block
with the int4 card's mixed formats through the same entry point must give
the bits of rt_qblock_project.
"""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

TC_TOL = 4e-3
NAMES = ("qkvg", "wo", "w13", "w2")


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


def _block(config, M, fmts, outliers=True):
    host = {}
    for name, fmt in zip(NAMES, fmts):
        W = wl.projection_weights(config, 0, name, outliers)
        host[name] = (fmt, oracle.quant_q4_g32(W) if fmt == 4 else oracle.quant_q8_row(W))
        host["x_" + name] = wl.projection_input(config, 0, name, M)
    return host


def _run(rtq, host, M, path="auto"):
    blk = rtq.QBlockFmt(*((host[n][0], dev(host[n][1][0]), dev(host[n][1][1])) for n in NAMES))
    X = [dev(host["x_" + n]) for n in NAMES]
    Y = [torch.empty((M, wl.BLOCK_PROJECTIONS[n]["N"]), device="cuda") for n in NAMES]
    rtq.qblock_project_fmt(blk, *X, *Y, path=path)
    return blk, X, Y


@pytest.mark.parametrize("M,n_check", [(80, None), (2048, 96), (4096, 64)])
def test_all_int8_block_matches_oracle(rtq_lib, M, n_check):
    host = _block(3 if M <= 2048 else 4, M, (8, 8, 8, 8))
    blk, X, Y = _run(rtq_lib, host, M)
    assert rtq_lib.block_fused_fmt(blk, M) == (1 if M <= 128 else 0)
    rows = None if n_check is None else wl.sample_rows(M, n_check, seed=M + 1)
    for name, y in zip(NAMES, Y):
        ref = oracle.gemm_q8(host["x_" + name], *host[name][1], rows=rows)
        got = y.cpu().numpy() if rows is None else y.cpu().numpy()[rows]
        assert rel_err(got, ref) <= TC_TOL, name


def test_mixed_formats_match_rt_qblock_project_bits(rtq_lib):
    M = 80
    host = _block(3, M, (4, 8, 4, 8), outliers=False)
    _, X, Y = _run(rtq_lib, host, M)
    blk = rtq_lib.QBlock(*(dev(a) for n in NAMES for a in host[n][1]))
    Y2 = [torch.empty_like(y) for y in Y]
    rtq_lib.qblock_project(blk, *X, *Y2)
    for a, b in zip(Y, Y2):
        assert torch.equal(a, b)


def test_all_int8_block_on_the_simt_path(rtq_lib):
    M = 5
    host = _block(3, M, (8, 8, 8, 8))
    _, _, Y = _run(rtq_lib, host, M, path="simt")
    for name, y in zip(NAMES, Y):
        ref = oracle.gemm_q8(host["x_" + name], *host[name][1])
        assert rel_err(y.cpu().numpy(), ref) <= 1e-5, name
