"""GPU parity of the CUDA path against the CPU oracle, called through the C ABI.

Packed weights come from the ORACLE's quantizer (or are random bytes), inputs
from the seeded workload generator, and expected values only from oracle/.

Gates:
  - dequantization exports: bit-exact (fp32 and fp16 renderings = the exact
    value rounded once);
  - X = I turns the GEMM into W_hat^T: bit-exact on every path;
  - SIMT GEMM: max|Y - Y_ref| / max|Y_ref| <= 1e-5;
  - tensor-core GEMM (fp16 operands): <= 4e-3, and every output within the
    first-order rounding bound of its operands (below);
  - no write outside Y (NaN guard bands), deterministic repeats, device
    status word clear afterwards.
"""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

SIMT_TOL = 1e-5
TC_TOL = 4e-3
# unit roundoff (2^-11) of the fp16 operands of the tensor-core path
UNIT = {"tc": 2.0 ** -11}
MAX_REL = {"simt": SIMT_TOL, "tc": TC_TOL, "auto": TC_TOL}


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
    assert rtq.device_status() == 0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rel_err(Y, Yref):
    Y = np.asarray(Y, dtype=np.float64)
    return float(np.max(np.abs(Y - Yref)) / max(np.max(np.abs(Yref)), 1e-300))


def f16_round(x32: np.ndarray) -> np.ndarray:
    """fp32 -> nearest-even fp16 (numpy's conversion), back as fp32 values."""
    return np.asarray(x32, dtype=np.float32).astype(np.float16).astype(np.float32)


def assert_within_rounding_bound(Y, X, What, path):
    """Elementwise first-order bound of the tensor-core path: each product
    x*w carries the roundings of x and w to fp16 (relative u each) and the
    fp32 accumulation adds at most K*2^-23 relative to sum|x*w|; an fp16
    subnormal operand (below 2^-14) is rounded with an absolute error of at
    most 2^-25 instead."""
    u = UNIT[path]
    A = np.abs(X.astype(np.float64)) @ np.abs(What).T
    K = X.shape[1]
    slack = 2.0 ** -25 * (np.abs(What).sum(axis=1)[None, :] +
                          np.abs(X.astype(np.float64)).sum(axis=1)[:, None])
    bound = (2.0 * u + u * u + 2.0 ** -23 + K * 2.0 ** -23) * A + slack
    ref = X.astype(np.float64) @ What.T
    bad = np.abs(np.asarray(Y, np.float64) - ref) > bound
    assert not bad.any(), f"{bad.sum()} outputs outside the rounding bound"


def q4_weights(N, K, seed, outliers=False):
    W = wl.weights(N, K, seed)
    if outliers:
        W = wl.with_outliers(W, seed)
    return oracle.quant_q4_g32(W)


def q8_weights(N, K, seed, outliers=False):
    W = wl.weights(N, K, seed)
    if outliers:
        W = wl.with_outliers(W, seed)
    return oracle.quant_q8_row(W)


def random_q4(N, K, seed):
    """Random payload bytes and random binary16 (scale, min), both signs."""
    g = np.random.default_rng(seed)
    Wq = g.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sc = g.uniform(-0.05, 0.05, size=(N, K // 32)).astype(np.float16)
    mn = g.uniform(-0.5, 0.5, size=(N, K // 32)).astype(np.float16)
    sc[0, 0] = 0.0
    sm = np.stack([sc.view(np.uint16), mn.view(np.uint16)], axis=-1)
    return Wq, np.ascontiguousarray(sm)


# ------------------------------------------------------------ dequantization
@pytest.mark.parametrize("N,K", [(64, 32), (130, 512), (512, 2048)])
def test_dequant_q4_exports_bit_exact(rtq_lib, N, K):
    for Wq, sm in (q4_weights(N, K, seed=N + K, outliers=True), random_q4(N, K, seed=N)):
        exact = oracle.dequant_q4(Wq, sm)
        ref32 = exact.astype(np.float32)
        got32 = rtq_lib.dequant_q4_f32(dev(Wq), dev(sm)).cpu().numpy()
        assert np.array_equal(got32.view(np.uint32), ref32.view(np.uint32))
        goth = rtq_lib.dequant_q4_f16(dev(Wq), dev(sm)).cpu().numpy()
        refh = exact.astype(np.float16).view(np.uint16)
        assert np.array_equal(goth, refh)


@pytest.mark.parametrize("N,K", [(16, 16), (512, 512), (512, 2048)])
def test_dequant_q8_export_bit_exact(rtq_lib, N, K):
    Wq, s = q8_weights(N, K, seed=N * 3 + K, outliers=True)
    Wq[0, 0] = -128  # representable in the format even if the quantizer never emits it
    ref32 = oracle.dequant_q8(Wq, s).astype(np.float32)
    got = rtq_lib.dequant_q8_f32(dev(Wq), dev(s)).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref32.view(np.uint32))


# --------------------------------------------------- X = I: exact transposes
@pytest.mark.parametrize("path", ["simt", "tc"])
def test_identity_input_q4_bit_exact(rtq_lib, path):
    N, K = 384, 512
    Wq, sm = q4_weights(N, K, seed=77, outliers=True)
    Y = rtq_lib.qgemm_q4(torch.eye(K, device="cuda"), dev(Wq), dev(sm), path=path)
    exact = oracle.dequant_q4(Wq, sm)
    if path == "simt":
        ref32 = exact.astype(np.float32).T
    else:
        ref32 = exact.astype(np.float16).astype(np.float32).T
    assert np.array_equal(Y.cpu().numpy(), ref32)


@pytest.mark.parametrize("path", ["simt", "tc"])
def test_identity_input_q8_bit_exact(rtq_lib, path):
    N, K = 256, 512
    Wq, s = q8_weights(N, K, seed=78, outliers=True)
    Y = rtq_lib.qgemm_q8(torch.eye(K, device="cuda"), dev(Wq), dev(s), path=path)
    ref32 = oracle.dequant_q8(Wq, s).astype(np.float32).T
    assert np.array_equal(Y.cpu().numpy(), ref32)


# ----------------------------------------------------------- GEMM parity
SIMT_SHAPES = [(1, 2048, 512), (3, 130, 96), (17, 300, 128), (80, 2048, 512), (79, 512, 2048),
               (129, 64, 64), (8, 1, 32)]
# one activation tile splits K over a cluster of 2, 4 or 8 CTAs: (81, 130, 128)
# -> 2, (64, 5120, 256) -> 4, (80, 2048, 512) and (80, 512, 2048) -> 8; (48,
# 1001, 512) reduces into an odd N, (5, 640, 1024) leaves 2 columns per CTA
TC_SHAPES = [(16, 256, 64), (80, 2048, 512), (80, 512, 2048), (81, 130, 128), (300, 512, 512),
             (1, 128, 64), (256, 200, 192), (1000, 640, 512), (64, 5120, 256), (48, 1001, 512),
             (5, 640, 1024)]


def _run_q4(rtq_lib, M, N, K, path, seed, outliers=False):
    X = wl.activations(M, K, seed)
    Wq, sm = q4_weights(N, K, seed + 1, outliers)
    Y = rtq_lib.qgemm_q4(dev(X), dev(Wq), dev(sm), path=path).cpu().numpy()
    if path in UNIT:
        assert_within_rounding_bound(Y, X, oracle.dequant_q4(Wq, sm), path)
    return Y, oracle.gemm_q4(X, Wq, sm)


def _run_q8(rtq_lib, M, N, K, path, seed, outliers=False):
    X = wl.activations(M, K, seed)
    Wq, s = q8_weights(N, K, seed + 1, outliers)
    Y = rtq_lib.qgemm_q8(dev(X), dev(Wq), dev(s), path=path).cpu().numpy()
    if path in UNIT:
        assert_within_rounding_bound(Y, X, oracle.dequant_q8(Wq, s), path)
    return Y, oracle.gemm_q8(X, Wq, s)


@pytest.mark.parametrize("M,N,K", SIMT_SHAPES)
def test_simt_parity_q4(rtq_lib, M, N, K):
    Y, ref = _run_q4(rtq_lib, M, N, K, "simt", seed=M + N + K, outliers=True)
    assert rel_err(Y, ref) <= SIMT_TOL


@pytest.mark.parametrize("M,N,K", [s for s in SIMT_SHAPES if s[2] % 16 == 0])
def test_simt_parity_q8(rtq_lib, M, N, K):
    Y, ref = _run_q8(rtq_lib, M, N, K, "simt", seed=M * 7 + N + K, outliers=True)
    assert rel_err(Y, ref) <= SIMT_TOL


@pytest.mark.parametrize("M,N,K", TC_SHAPES)
def test_tc_parity_q4(rtq_lib, M, N, K, path="tc"):
    Y, ref = _run_q4(rtq_lib, M, N, K, path, seed=M + 3 * N + K, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


@pytest.mark.parametrize("M,N,K", TC_SHAPES)
def test_tc_parity_q8(rtq_lib, M, N, K, path="tc"):
    Y, ref = _run_q8(rtq_lib, M, N, K, path, seed=M + 5 * N + K, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


# shapes that the activation-resident kernel takes: ragged M and N, K from 64 to
# 512, a CTA run that crosses activation blocks
XS_SHAPES = [(2048, 1024, 512), (2000, 1000, 512), (1500, 2100, 256), (4096, 512, 512),
             (2048, 2048, 128), (300, 6000, 128), (150, 640, 512), (200, 384, 256),
             (500, 1002, 256)]


@pytest.mark.parametrize("M,N,K", XS_SHAPES)
def test_x_resident_parity_q4(rtq_lib, M, N, K, path="tc"):
    assert rtq_lib.plan(4, M, N, K, path) == "tc_x_resident"
    Y, ref = _run_q4(rtq_lib, M, N, K, path, seed=M + 7 * N + K, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


@pytest.mark.parametrize("M,N,K", XS_SHAPES)
def test_x_resident_parity_q8(rtq_lib, M, N, K, path="tc"):
    assert rtq_lib.plan(8, M, N, K, path) == "tc_x_resident"
    Y, ref = _run_q8(rtq_lib, M, N, K, path, seed=M + 11 * N + K, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


# shapes that the TMA-fed weight-streamed kernel takes: K above the resident
# limit; ragged M and N; q4 chunks of (scale, min) words that end inside a
# chunk (K = 640).  The launch picks the activation tile height from the tile
# count on 148 SMs: the first six shapes take 64 rows, and the
# four (M, 700, 768) shapes 96, 128, 160 and 192 rows, so every epilogue split
# (16 + 16 .. 32 + 32 + 32 columns per warp) runs
WS_SHAPES = [(2048, 512, 2048), (300, 640, 1024), (200, 512, 768), (1000, 700, 2048),
             (129, 256, 640), (300, 1002, 768), (1572, 700, 768), (2312, 700, 768),
             (3089, 700, 768), (3866, 700, 768)]


@pytest.mark.parametrize("M,N,K", WS_SHAPES)
def test_w_streamed_parity_q4(rtq_lib, M, N, K, path="tc"):
    assert rtq_lib.plan(4, M, N, K, path) == "tc_w_streamed"
    Y, ref = _run_q4(rtq_lib, M, N, K, path, seed=M + 13 * N + K, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


@pytest.mark.parametrize("M,N,K", WS_SHAPES)
def test_w_streamed_parity_q8(rtq_lib, M, N, K, path="tc"):
    assert rtq_lib.plan(8, M, N, K, path) == "tc_w_streamed"
    Y, ref = _run_q8(rtq_lib, M, N, K, path, seed=M + 17 * N + K, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


def test_w_streamed_odd_step_count_q8(rtq_lib, path="tc"):
    """q8 with K = 576: nine 64-wide K steps, so the last two-step box of
    packed codes is half past the end of each row (zero-filled by TMA)."""
    M, N, K = 700, 384, 576
    assert rtq_lib.plan(8, M, N, K, path) == "tc_w_streamed"
    Y, ref = _run_q8(rtq_lib, M, N, K, path, seed=4242, outliers=True)
    assert rel_err(Y, ref) <= MAX_REL[path]


def test_w_streamed_many_tiles_every_tile(rtq_lib):
    """Several 128 x 128 tiles per persistent CTA (M = 32768, N = 1024, q8,
    K = 2048): every tile against the fp32 SIMT path, twice."""
    M, N, K = 32768, 1024, 2048
    X = dev(wl.activations(M, K, 6010))
    Wq, s = q8_weights(N, K, 6005, outliers=True)
    Wd, Sd = dev(Wq), dev(s)
    assert rtq_lib.plan(8, M, N, K) == "tc_w_streamed"
    ys = rtq_lib.qgemm_q8(X, Wd, Sd, path="simt")
    scale = ys.abs().max()
    for _ in range(2):
        yt = rtq_lib.qgemm_q8(X, Wd, Sd, path="tc")
        tile_err = ((yt - ys).abs() / scale).view(M // 128, 128, N // 128, 128).amax(dim=(1, 3))
        assert float(tile_err.max()) <= TC_TOL, int((tile_err > TC_TOL).sum())


def test_x_resident_long_runs_every_tile(rtq_lib):
    """Many weight tiles per CTA and several activation-block reloads per run
    (M = 65536, N = 2048): every 128 x 128 output tile against the fp32 SIMT
    path on the same inputs, twice.  This is the regime in which a packed-code
    staging slot could be refilled before its reads completed."""
    M, N, K = 65536, 2048, 512
    X = dev(wl.activations(M, K, 5010))
    Wq, sm = q4_weights(N, K, 5005, outliers=True)
    Wd, Sd = dev(Wq), dev(sm)
    assert rtq_lib.plan(4, M, N, K) == "tc_x_resident_pair"
    ys = rtq_lib.qgemm_q4(X, Wd, Sd, path="simt")
    scale = ys.abs().max()
    for _ in range(2):
        yt = rtq_lib.qgemm_q4(X, Wd, Sd, path="tc")
        tile_err = ((yt - ys).abs() / scale).view(M // 128, 128, N // 128, 128).amax(dim=(1, 3))
        assert float(tile_err.max()) <= TC_TOL, int((tile_err > TC_TOL).sum())


# the CTA-pair activation-resident kernel (from M = 16384): ragged M, an odd
# number of 128-row weight tiles (the last pair's second CTA holds rows past
# N), K from 128 to 512
# ragged M (16500, 16390) and N (700, 1000, 130: rows of Y not a multiple of
# 16 bytes)
XP_SHAPES = [(16384, 640, 512), (16500, 700, 384), (17000, 256, 128), (16400, 1000, 256),
             (16390, 130, 256)]


@pytest.mark.parametrize("fmt", [4, 8])
@pytest.mark.parametrize("M,N,K", XP_SHAPES)
def test_x_resident_pair_parity(rtq_lib, fmt, M, N, K):
    """Every 128 x 128 output tile against the fp32 SIMT path on the same
    inputs, and 64 sampled rows (among them the first and last of every
    192-row activation block's two halves near the ends) against the
    oracle."""
    assert rtq_lib.plan(fmt, M, N, K) == "tc_x_resident_pair"
    Xh = wl.activations(M, K, 7100 + M + fmt)
    q = q4_weights(N, K, 7101 + N, outliers=True) if fmt == 4 else q8_weights(N, K, 7101 + N, True)
    fn = rtq_lib.qgemm_q4 if fmt == 4 else rtq_lib.qgemm_q8
    X, Wd, Sd = dev(Xh), dev(q[0]), dev(q[1])
    yt = fn(X, Wd, Sd, path="tc")
    ys = fn(X, Wd, Sd, path="simt")
    scale = ys.abs().max()
    mt, nt = (M + 127) // 128, (N + 127) // 128
    pad = torch.zeros((mt * 128, nt * 128), device="cuda")
    pad[:M, :N] = (yt - ys).abs() / scale
    tile_err = pad.view(mt, 128, nt, 128).amax(dim=(1, 3))
    assert float(tile_err.max()) <= TC_TOL, int((tile_err > TC_TOL).sum())
    rng = np.random.default_rng(M + N + K)
    rows = np.unique(np.concatenate([[0, 95, 96, 191, 192, M - 1], rng.integers(0, M, 58)]))
    gemm = oracle.gemm_q4 if fmt == 4 else oracle.gemm_q8
    ref = gemm(np.ascontiguousarray(Xh[rows]), *q)
    assert rel_err(yt[rows].cpu().numpy(), ref) <= MAX_REL["tc"]


def test_x_resident_pair_identity_bit_exact(rtq_lib):
    """X made of 16384 rows of the identity's 256 rows, over and over: every
    output is one weight rounded to fp16, in both CTAs' rows of every tile."""
    N, K = 1152, 256
    Wq, sm = q4_weights(N, K, seed=93, outliers=True)
    M = 16384
    assert rtq_lib.plan(4, M, N, K) == "tc_x_resident_pair"
    X = torch.eye(K, device="cuda").repeat(M // K, 1)
    Y = rtq_lib.qgemm_q4(X, dev(Wq), dev(sm)).cpu().numpy()
    ref = oracle.dequant_q4(Wq, sm).astype(np.float16).astype(np.float32).T
    assert np.array_equal(Y, np.tile(ref, (M // K, 1)))


def test_x_resident_identity_bit_exact(rtq_lib):
    """X = I over four activation blocks: every output is one rounded weight."""
    N, K = 12800, 512
    Wq, sm = q4_weights(N, K, seed=91, outliers=True)
    assert rtq_lib.plan(4, K, N, K) == "tc_x_resident"
    Y = rtq_lib.qgemm_q4(torch.eye(K, device="cuda"), dev(Wq), dev(sm)).cpu().numpy()
    ref = oracle.dequant_q4(Wq, sm).astype(np.float16).astype(np.float32).T
    assert np.array_equal(Y, ref)


@pytest.mark.parametrize("fmt", [4, 8])
def test_x_resident_x_16_byte_aligned(rtq_lib, fmt):
    """X that starts 16 bytes past a 32-byte boundary (the ABI asks for 16
    only): the activation-resident route must give the bits it gives for an
    aligned copy of X."""
    M, N, K = 700, 640, 384
    assert rtq_lib.plan(fmt, M, N, K) == "tc_x_resident"
    X = wl.activations(M, K, 77 + fmt)
    if fmt == 4:
        q = q4_weights(N, K, 78, outliers=True)
        fn, ref = rtq_lib.qgemm_q4, oracle.gemm_q4(X, *q)
    else:
        q = q8_weights(N, K, 78, outliers=True)
        fn, ref = rtq_lib.qgemm_q8, oracle.gemm_q8(X, *q)
    buf = torch.empty(M * K + 4, device="cuda")
    Xo = buf[4:].view(M, K)
    Xo.copy_(dev(X))
    assert Xo.data_ptr() % 32 == 16
    Wd, Sd = dev(q[0]), dev(q[1])
    Ya = fn(dev(X), Wd, Sd, path="tc")
    Yo = fn(Xo, Wd, Sd, path="tc")
    assert torch.equal(Ya, Yo)
    assert rel_err(Yo.cpu().numpy(), ref) <= MAX_REL["tc"]


def test_random_format_bytes_both_paths(rtq_lib):
    M, N, K = 96, 256, 256
    X = wl.activations(M, K, 5)
    Wq, sm = random_q4(N, K, 6)
    ref = oracle.gemm_q4(X, Wq, sm)
    for path in ("simt", "tc"):
        Y = rtq_lib.qgemm_q4(dev(X), dev(Wq), dev(sm), path=path).cpu().numpy()
        assert rel_err(Y, ref) <= MAX_REL[path], path
        if path in UNIT:
            assert_within_rounding_bound(Y, X, oracle.dequant_q4(Wq, sm), path)


# ------------------------------------------------------- edge cases, guards
@pytest.mark.parametrize("path", ["simt", "tc"])
@pytest.mark.parametrize("M", [1, 3, 17, 79, 81, 129])
def test_guard_bands_and_ragged_sizes(rtq_lib, path, M):
    N, K = 136, 128
    X = wl.activations(M, K, M)
    Wq, sm = q4_weights(N, K, 40 + M)
    guard = 1024
    nan_bits = torch.full((M * N + 2 * guard,), 0x7FC01234, dtype=torch.int32, device="cuda")
    buf = nan_bits.view(torch.float32)
    Y = buf[guard:guard + M * N].view(M, N)
    rtq_lib.qgemm_q4(dev(X), dev(Wq), dev(sm), Y=Y, path=path)
    host = nan_bits.cpu().numpy()
    assert np.all(host[:guard] == 0x7FC01234) and np.all(host[guard + M * N:] == 0x7FC01234)
    tol = SIMT_TOL if path == "simt" else TC_TOL
    assert rel_err(Y.cpu().numpy(), oracle.gemm_q4(X, Wq, sm)) <= tol


def test_zero_rows_is_a_no_op(rtq_lib):
    Wq, sm = q4_weights(128, 64, 1)
    X = torch.empty((0, 64), device="cuda")
    Y = rtq_lib.qgemm_q4(X, dev(Wq), dev(sm))
    assert Y.shape == (0, 128)


@pytest.mark.parametrize("path", ["simt", "tc"])
def test_deterministic_repeats_and_side_stream(rtq_lib, path):
    M, N, K = 200, 512, 512
    X = dev(wl.activations(M, K, 9))
    Wq, sm = q4_weights(N, K, 10)
    Wq, sm = dev(Wq), dev(sm)
    a = rtq_lib.qgemm_q4(X, Wq, sm, path=path)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = rtq_lib.qgemm_q4(X, Wq, sm, path=path, stream=s)
    s.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------- full sizes, sampled outputs
@pytest.mark.parametrize("fmt", ["q4", "q8"])
def test_full_size_m65536_sampled_rows(rtq_lib, fmt):
    """The M sweep's largest point (B=64, S=1024) with 1% x20 outlier groups,
    on the AUTO path, checked on 256 seeded rows (rows are independent)."""
    M = 65536
    if fmt == "q4":
        N, K = 2048, 512
        W = wl.with_outliers(wl.weights(N, K, wl.seed_for(5, 0, "w1")), wl.seed_for(5, 0, "w1"))
        Wq, sm = oracle.quant_q4_g32(W)
    else:
        N, K = 512, 2048
        W = wl.with_outliers(wl.weights(N, K, wl.seed_for(5, 0, "w2")), wl.seed_for(5, 0, "w2"))
        Wq, sm = oracle.quant_q8_row(W)
    X = wl.activations(M, K, wl.seed_for(5, 0, "x_ffn"))
    rows = wl.sample_rows(M, 256, seed=123)
    fn = rtq_lib.qgemm_q4 if fmt == "q4" else rtq_lib.qgemm_q8
    gemm = oracle.gemm_q4 if fmt == "q4" else oracle.gemm_q8
    ref = gemm(X, Wq, sm, rows=rows)
    Xd, Wd, Sd = dev(X), dev(Wq), dev(sm)
    for path, tol in (("auto", TC_TOL), ("simt", SIMT_TOL)):
        Y = fn(Xd, Wd, Sd, path=path)
        assert rel_err(Y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref) <= tol, path


def _block_tensors(config, block, M, outliers=False):
    host = {}
    for name in ("qkvg", "wo", "w13", "w2"):
        W = wl.projection_weights(config, block, name, outliers)
        fmt = wl.BLOCK_PROJECTIONS[name]["fmt"]
        host[name] = oracle.quant_q4_g32(W) if fmt == "q4" else oracle.quant_q8_row(W)
        host["x_" + name] = wl.projection_input(config, block, name, M)
    return host


@pytest.mark.parametrize("M,n_check", [(80, None), (2048, 96), (4096, 64)])
def test_block_driver_matches_oracle(rtq_lib, M, n_check):
    """One RT-J block's projection set through rt_qblock_project (AUTO path,
    the configuration the benchmark times); at M >= 2048 on sampled rows."""
    h = _block_tensors(4 if M == 4096 else 3, 0, M)
    blk = rtq_lib.QBlock(*(dev(a) for a in (*h["qkvg"], *h["wo"], *h["w13"], *h["w2"])))
    X = {n: dev(h["x_" + n]) for n in ("qkvg", "wo", "w13", "w2")}
    Y = {"qkvg": torch.empty((M, 2048), device="cuda"), "wo": torch.empty((M, 512), device="cuda"),
         "w13": torch.empty((M, 4096), device="cuda"), "w2": torch.empty((M, 512), device="cuda")}
    rtq_lib.qblock_project(blk, X["qkvg"], X["wo"], X["w13"], X["w2"],
                           Y["qkvg"], Y["wo"], Y["w13"], Y["w2"])
    rows = None if n_check is None else wl.sample_rows(M, n_check, seed=M)
    for name in ("qkvg", "wo", "w13", "w2"):
        fmt = wl.BLOCK_PROJECTIONS[name]["fmt"]
        gemm = oracle.gemm_q4 if fmt == "q4" else oracle.gemm_q8
        ref = gemm(h["x_" + name], *h[name], rows=rows)
        got = Y[name].cpu().numpy() if rows is None else Y[name].cpu().numpy()[rows]
        tol = TC_TOL if rtq_lib.auto_path(4 if fmt == "q4" else 8, M, 1, 512) == 2 else SIMT_TOL
        assert rel_err(got, ref) <= tol, name


def _sized_block(d_model, d_ff, M, seed):
    """A seeded block of any size: weights ~ N(0, 0.02^2) quantized by the
    oracle, activations ~ N(0, 1)."""
    shapes = {"qkvg": ("q4", 4 * d_model, d_model), "wo": ("q8", d_model, d_model),
              "w13": ("q4", 2 * d_ff, d_model), "w2": ("q8", d_model, d_ff)}
    host = {}
    for i, (name, (fmt, N, K)) in enumerate(shapes.items()):
        W = wl.weights(N, K, seed + i)
        host[name] = oracle.quant_q4_g32(W) if fmt == "q4" else oracle.quant_q8_row(W)
        host["x_" + name] = wl.activations(M, K, seed + 10 + i)
    return host, shapes


def _guarded_outputs(M, shapes, guard=64):
    """The four Y buffers as views of one NaN-filled allocation, separated by
    `guard` floats that the kernels must not write."""
    sizes = [M * shapes[n][1] for n in ("qkvg", "wo", "w13", "w2")]
    flat = torch.full((sum(sizes) + 5 * guard,), float("nan"), device="cuda")
    views, off = {}, guard
    for n, sz in zip(("qkvg", "wo", "w13", "w2"), sizes):
        views[n] = flat[off:off + sz].view(M, shapes[n][1])
        off += sz + guard
    return flat, views, sizes


# (M, d_model, d_ff, path).  The grouped launch splits each projection's K by
# its own factor inside clusters of a common size; the comments give the plan.
FUSED_CASES = [
    (80, 512, 2048, "auto"),      # RT-J block at the small-M config: qkvg, wo, w13 split by 2
                                  # (4 tiles per cluster of 8), w2 by 8; 136 CTAs of 4 K steps
    (16, 512, 2048, "tc"),        # 16-column activation tile (AUTO runs q4 on SIMT here)
    (48, 512, 2048, "auto"),
    (128, 512, 2048, "auto"),     # largest single activation tile
    (1, 512, 2048, "tc"),         # one row, tensor cores forced
    (80, 512, 2048, "tc"),
    (100, 256, 1024, "auto"),     # wo's 2 tiles half-fill a cluster: 2 CTA pairs store nothing
    (37, 1024, 4096, "auto"),     # 272 CTAs of 8 K steps
    (16, 2048, 8192, "tc"),       # clusters of 4: w2 split by 4, the others unsplit
]


@pytest.mark.parametrize("M,d_model,d_ff,path", FUSED_CASES)
def test_block_driver_grouped_launch_matches_oracle(rtq_lib, M, d_model, d_ff, path):
    """rt_qblock_project at M <= 128 runs the four projections as one grouped
    tcgen05 launch; every output element against the oracle, nothing written
    outside the outputs, and a repeat gives the same bits."""
    assert rtq_lib.block_fused(M, d_model, d_ff, path) == 1
    h, shapes = _sized_block(d_model, d_ff, M, seed=1000 + M + d_model)
    blk = rtq_lib.QBlock(*(dev(a) for a in (*h["qkvg"], *h["wo"], *h["w13"], *h["w2"])),
                         d_model=d_model, d_ff=d_ff)
    X = {n: dev(h["x_" + n]) for n in ("qkvg", "wo", "w13", "w2")}
    flat, Y, sizes = _guarded_outputs(M, shapes)
    rtq_lib.qblock_project(blk, X["qkvg"], X["wo"], X["w13"], X["w2"],
                           Y["qkvg"], Y["wo"], Y["w13"], Y["w2"], path=path)
    first = {n: Y[n].cpu().numpy().copy() for n in Y}
    for n in ("qkvg", "wo", "w13", "w2"):
        gemm = oracle.gemm_q4 if shapes[n][0] == "q4" else oracle.gemm_q8
        ref = gemm(h["x_" + n], *h[n])
        assert rel_err(first[n], ref) <= MAX_REL[path], n
    guard = torch.ones_like(flat, dtype=torch.bool)
    off = 64
    for sz in sizes:
        guard[off:off + sz] = False
        off += sz + 64
    assert torch.isnan(flat[guard]).all()
    rtq_lib.qblock_project(blk, X["qkvg"], X["wo"], X["w13"], X["w2"],
                           Y["qkvg"], Y["wo"], Y["w13"], Y["w2"], path=path)
    for n in Y:
        assert np.array_equal(Y[n].cpu().numpy(), first[n]), n


def test_block_driver_grouped_launch_shared_input(rtq_lib):
    """qkvg, wo and w13 read one activation buffer (allowed: inputs are only
    read) in the grouped launch."""
    M = 64
    h, shapes = _sized_block(512, 2048, M, seed=77)
    Xs = dev(h["x_qkvg"])
    blk = rtq_lib.QBlock(*(dev(a) for a in (*h["qkvg"], *h["wo"], *h["w13"], *h["w2"])))
    Y = {n: torch.empty((M, shapes[n][1]), device="cuda") for n in shapes}
    rtq_lib.qblock_project(blk, Xs, Xs, Xs, dev(h["x_w2"]), Y["qkvg"], Y["wo"], Y["w13"], Y["w2"])
    for n in ("qkvg", "wo", "w13"):
        gemm = oracle.gemm_q4 if shapes[n][0] == "q4" else oracle.gemm_q8
        assert rel_err(Y[n].cpu().numpy(), gemm(h["x_qkvg"], *h[n])) <= TC_TOL, n
    assert rel_err(Y["w2"].cpu().numpy(), oracle.gemm_q8(h["x_w2"], *h["w2"])) <= TC_TOL


def test_device_status_clear(rtq_lib):
    torch.cuda.synchronize()
    assert rtq_lib.device_status() == 0
