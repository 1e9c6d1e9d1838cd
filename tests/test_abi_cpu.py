"""Host-side checks of the C ABI that need no GPU.

- librtq.so loads and exports every function include/rtq.h declares.
- Argument validation returns the documented status before any CUDA call
  (the pointers below are never dereferenced).
- The library's host quantizers match the oracle's bit for bit on the
  workloads' weights, outliers included.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import int8_dequant_gemm_b200 as rtq
from int8_dequant_gemm_b200 import build as rtq_build
from int8_dequant_gemm_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RT_OK, INVALID, ALIGN, SHAPE, CUDA, TIMEOUT, RANGE = 0, 1, 2, 3, 4, 5, 6


@pytest.fixture(scope="module", autouse=True)
def built():
    rtq_build.build()
    return rtq.lib()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "rtq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(rt_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("rt_qgemm_q4", "rt_qgemm_q8", "rt_qblock_project", "rt_quantize_q4_g32",
                     "rt_quantize_q8_row", "rt_dequant_q4_f32", "rt_dequant_q8_f32",
                     "rt_device_status", "rt_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(rtq.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings_and_version():
    for s in range(11):
        assert rtq.status_string(s) and rtq.status_string(s) != "unknown status"
    assert rtq.status_string(99) == "unknown status"
    assert rtq.lib().rt_version() >= 100


# fake, well-aligned, non-overlapping device addresses (never dereferenced)
X, W, S, Y = 0x10000000, 0x20000000, 0x30000000, 0x40000000


@pytest.mark.parametrize("fn", ["rt_qgemm_q4", "rt_qgemm_q8"])
def test_validation_statuses(fn):
    f = getattr(rtq, fn)
    K = 64
    assert f(None, W, S, Y, 4, 16, K, 0, None) == INVALID          # null X with M > 0
    assert f(X, None, S, Y, 4, 16, K, 0, None) == INVALID          # null weights
    assert f(X, W, S, Y, -1, 16, K, 0, None) == INVALID            # negative M
    assert f(X, W, S, Y, 4, 0, K, 0, None) == INVALID              # N < 1
    assert f(X + 4, W, S, Y, 4, 16, K, 0, None) == ALIGN           # X not 16-byte aligned
    assert f(X, W + 8, S, Y, 4, 16, K, 0, None) == ALIGN           # Wq not 16-byte aligned
    assert f(X, W, S + 2, Y, 4, 16, K, 0, None) == ALIGN           # scales not 4-byte aligned
    assert f(X, W, S, Y + 8, 4, 16, K, 0, None) == ALIGN           # Y not 16-byte aligned
    assert f(X, W, S, X, 4, 16, K, 0, None) == INVALID             # Y overlaps X
    assert f(X, W, S, W, 4, 16, K, 0, None) == INVALID             # Y overlaps Wq
    assert f(X, W, S, Y, 4, 16, K, 7, None) == INVALID             # unknown path
    assert f(X, W, S, Y, 4, 16, K, 3, None) == INVALID             # path 3 no longer exists
    assert f(None, W, S, None, 0, 16, K, 0, None) == RT_OK         # M == 0 is a no-op
    bad_k = 40 if fn == "rt_qgemm_q4" else 24
    assert f(X, W, S, Y, 4, 16, bad_k, 0, None) == SHAPE           # K not a multiple of the granule
    assert f(X, W, S, Y, 4, 16, 96, 2, None) == SHAPE              # forced TC needs K % 64


def test_auto_path_dispatch():
    # the measured single-call crossover: q4 SIMT up to M = 16, q8 and e4m3 at M = 1
    assert rtq.auto_path(4, 16, 2048, 512) == 1 and rtq.auto_path(4, 17, 2048, 512) == 2
    assert rtq.auto_path(8, 1, 512, 2048) == 1 and rtq.auto_path(8, 2, 512, 2048) == 2
    assert rtq.auto_path(3, 1, 512, 2048) == 1 and rtq.auto_path(3, 2, 512, 2048) == 2
    assert rtq.auto_path(4, 1, 2048, 512) == 1
    assert rtq.auto_path(4, 80, 2048, 512) == 2
    assert rtq.auto_path(8, 65536, 512, 2048) == 2
    assert rtq.auto_path(4, 80, 2048, 96) == 1      # K % 64 != 0 -> SIMT
    assert rtq.auto_path(4, 80, 2048, 40) == -1     # not a q4 shape
    assert rtq.auto_path(5, 80, 2048, 512) == -1


def test_kernel_plan():
    assert rtq.plan(4, 4, 2048, 512) == "simt"
    assert rtq.plan(4, 80, 2048, 512) == "tc_w_stationary"
    assert rtq.plan(4, 4096, 4096, 512) == "tc_x_resident"
    assert rtq.plan(4, 65536, 2048, 512) == "tc_x_resident_pair"   # CTA pairs from M = 16384
    assert rtq.plan(4, 16383, 2048, 512) == "tc_x_resident"
    assert rtq.plan(8, 16384, 512, 128) == "tc_x_resident_pair"
    assert rtq.plan(3, 20000, 512, 384) == "tc_x_resident_pair"
    assert rtq.plan(8, 65536, 512, 2048) == "tc_w_streamed"
    assert rtq.plan(8, 4096, 512, 2048) == "tc_w_streamed"     # K > 512 does not fit resident
    assert rtq.plan(4, 200, 512, 512) == "tc_x_resident"       # one full block and a tail
    assert rtq.plan(4, 129, 512, 512) == "tc_x_resident"
    assert rtq.plan(4, 200, 512, 768) == "tc_w_streamed"       # K above the resident limit
    assert rtq.plan(4, 300, 512, 192) == "tc_w_stationary"     # q4 TMA needs K % 128
    assert rtq.plan(8, 4096, 512, 2048, "tc") == "tc_w_streamed"
    assert rtq.plan(8, 4096, 512, 2048, 3) == "rejected"       # no path 3 (bf16 operands removed)
    assert rtq.plan(4, 4096, 4096, 512, "simt") == "simt"
    assert rtq.plan(4, 4096, 4096, 96, "tc") == "rejected"
    assert rtq.plan(4, 4096, 4096, 40) == "rejected"


def test_workspace_sizes():
    assert rtq.workspace_bytes(4, 4096, 4096, 512) == 4096 * 512 * 2
    assert rtq.workspace_bytes(4, 65536, 2048, 512) == 0          # CTA pairs: in-kernel rounding
    assert rtq.workspace_bytes(8, 4096, 512, 2048) == 4096 * 2048 * 2
    assert rtq.workspace_bytes(4, 80, 2048, 512) == 0
    assert rtq.workspace_bytes(4, 4, 2048, 512) == 0
    assert rtq.workspace_bytes(4, 80, 2048, 40) == -1
    assert rtq.rt_workspace_reserve(-1, None) == INVALID


def test_noalloc_validation_and_scratch_limit():
    # every status below is decided before any CUDA call
    f = rtq.rt_qgemm_noalloc
    assert f(5, X, W, S, Y, 4, 16, 64, 0, None) == INVALID          # unknown format
    assert f(4, X, W, S, Y, 4, 16, 40, 0, None) == SHAPE            # q4 K granule
    assert f(8, X + 4, W, S, Y, 4, 16, 64, 0, None) == ALIGN        # X alignment
    assert f(4, X, W, S, X, 4, 16, 64, 0, None) == INVALID          # Y overlaps X
    assert f(4, X, W, S, Y, 4, 16, 64, 9, None) == INVALID          # unknown path
    assert f(4, X, W, S, Y, 4096, 16, 96, 2, None) == SHAPE         # forced TC needs K % 64
    # M * K * 2 bytes of scratch above the fixed array: rejected, nothing launched
    limit = rtq.NOALLOC_SCRATCH_BYTES
    assert rtq.plan(8, 4096, 512, 4096) == "tc_w_streamed" and 4096 * 4096 * 2 > limit
    assert f(8, 0x100000000, W, S, 0x300000000, 4096, 512, 4096, 0, None) == 8
    assert rtq.plan(4, 16383, 4096, 512) == "tc_x_resident" and 16383 * 512 * 2 < limit
    # the CTA-pair kernel needs no scratch, so its size is not limited
    assert rtq.plan(4, 65536, 4096, 512) == "tc_x_resident_pair" and 65536 * 512 * 2 > limit
    assert rtq.status_string(8) != "unknown status"


def test_block_driver_validation():
    blk = rtq._QBlockC(W, S, W, S, W, S, W, S, 0, 2048)
    assert rtq.rt_qblock_project(blk, 4, X, X, X, X, Y, Y, Y, Y, 0, None) == INVALID
    assert rtq.lib().rt_qblock_project(None, 4, X, X, X, X, Y, Y, Y, Y, 0, None) == INVALID


def test_block_grouped_launch_plan():
    # one grouped launch exactly where all four projections take the
    # weight-stationary kernel with a single activation tile
    assert rtq.block_fused(80, 512, 2048) == 1
    assert rtq.block_fused(17, 512, 2048) == 1 and rtq.block_fused(128, 512, 2048) == 1
    assert rtq.block_fused(16, 512, 2048) == 0            # AUTO takes SIMT for q4 at M <= 16
    assert rtq.block_fused(8, 512, 2048) == 0
    assert rtq.block_fused(8, 512, 2048, "tc") == 1
    assert rtq.block_fused(1, 512, 2048, "tc") == 1
    assert rtq.block_fused(1, 512, 2048, 3) == -1
    assert rtq.block_fused(129, 512, 2048) == 0           # the TMA-fed kernels
    assert rtq.block_fused(80, 512, 2048, "simt") == 0
    assert rtq.block_fused(0, 512, 2048) == 0
    assert rtq.block_fused(80, 512, 2000) == 0            # w2's K % 64 != 0: SIMT under AUTO
    assert rtq.block_fused(80, 512, 2000, "tc") == -1     # and rejected on forced TC
    assert rtq.block_fused(80, 0, 2048) == -1
    assert rtq.block_fused(80, 512, 2048, 9) == -1


def test_block_driver_rejects_overlapping_outputs():
    # distinct fake regions 16 MB apart: X_i at 0x1i000000, codes at 0x2i..,
    # scales at 0x3i.., Y_i at 0x4i..; every status is decided before any
    # CUDA call, and an error means nothing was enqueued
    Xs = [0x11000000, 0x12000000, 0x13000000, 0x14000000]
    Ws = [0x21000000, 0x22000000, 0x23000000, 0x24000000]
    Ss = [0x31000000, 0x32000000, 0x33000000, 0x34000000]
    Ys = [0x41000000, 0x42000000, 0x43000000, 0x44000000]
    blk = rtq._QBlockC(Ws[0], Ss[0], Ws[1], Ss[1], Ws[2], Ss[2], Ws[3], Ss[3], 512, 2048)
    f = rtq.rt_qblock_project

    def call(M, xs, ys, path=0):
        return f(blk, M, *xs, *ys, path, None)

    assert call(0, Xs, Ys) == RT_OK                                   # M == 0: no-op
    assert call(80, Xs, [Ys[0], Ys[1], Ys[0] + 4096, Ys[3]]) == INVALID  # Y_13 inside Y_qkvg
    assert call(80, Xs, [Ys[0], Xs[2], Ys[2], Ys[3]]) == INVALID      # Y_o is w13's input
    assert call(80, Xs, [Ys[0], Ys[1], Ys[2], Ws[0]]) == INVALID      # Y_2 on qkvg's codes
    assert call(80, Xs, [Ys[0], Ys[1], Ss[1], Ys[3]]) == INVALID      # Y_13 on wo's scales
    # the rule holds on the one-call-per-projection route too: at M = 4096,
    # Y_qkvg (32 MB) runs into Y_o
    assert rtq.block_fused(4096, 512, 2048) == 0
    assert call(4096, Xs, Ys) == INVALID
    assert call(80, Xs, Ys, path=9) == INVALID                        # unknown path


def test_binding_rejects_mismatched_shapes_before_any_launch():
    """The C layer sees pointers and sizes only, so the torch-level helpers
    check every tensor's shape against M, N and K first (host tensors with the
    right shapes get as far as the CUDA-tensor check)."""
    torch = pytest.importorskip("torch")
    M, N, K = 4, 16, 64
    X = torch.zeros((M, K))
    Wq4 = torch.zeros((N, K // 2), dtype=torch.uint8)
    sm = torch.zeros((N, K // 32, 2), dtype=torch.uint16)
    Wq8 = torch.zeros((N, K), dtype=torch.int8)
    s8 = torch.zeros((N,))
    with pytest.raises(ValueError, match="Wq"):
        rtq.qgemm_q4(X, Wq4[:, :16], sm)                 # codes of a K = 32 weight
    with pytest.raises(ValueError, match="scale_min"):
        rtq.qgemm_q4(X, Wq4, sm[:, :1])
    with pytest.raises(ValueError, match="Y"):
        rtq.qgemm_q4(X, Wq4, sm, Y=torch.zeros((M, N // 2)))
    with pytest.raises(ValueError, match="X"):
        rtq.qgemm_q4(X.view(-1), Wq4, sm)
    with pytest.raises(TypeError, match="CUDA"):
        rtq.qgemm_q4(X, Wq4, sm)                         # shapes fine, host memory
    with pytest.raises(ValueError, match="scale"):
        rtq.qgemm_q8(X, Wq8, s8[:8])
    with pytest.raises(ValueError, match="Wq"):
        rtq.qgemm_q8(X, Wq8[:, :32], s8)
    with pytest.raises(ValueError, match="fmt"):
        rtq.qgemm_noalloc(5, X, Wq8, s8, torch.zeros((M, N)))
    with pytest.raises(ValueError, match="scale_min"):
        rtq.dequant_q4_f32(Wq4, sm[:, :1])
    with pytest.raises(ValueError, match="scale"):
        rtq.dequant_q8_f32(Wq8, s8[:1])

    d, f = 64, 128
    blk = rtq.QBlock(torch.zeros((4 * d, d // 2), dtype=torch.uint8),
                     torch.zeros((4 * d, d // 32, 2), dtype=torch.uint16),
                     torch.zeros((d, d), dtype=torch.int8), torch.zeros((d,)),
                     torch.zeros((2 * f, d // 2), dtype=torch.uint8),
                     torch.zeros((2 * f, d // 32, 2), dtype=torch.uint16),
                     torch.zeros((d, f), dtype=torch.int8), torch.zeros((d,)), d_model=d, d_ff=f)
    Xs = [torch.zeros((M, d)), torch.zeros((M, d)), torch.zeros((M, d)), torch.zeros((M, f))]
    Ys = [torch.zeros((M, 4 * d)), torch.zeros((M, d)), torch.zeros((M, 2 * f)),
          torch.zeros((M, d))]
    with pytest.raises(ValueError, match="Y_13"):
        rtq.qblock_project(blk, *Xs, Ys[0], Ys[1], torch.zeros((M, f)), Ys[3])
    with pytest.raises(ValueError, match="X_w2"):
        rtq.qblock_project(blk, Xs[0], Xs[1], Xs[2], torch.zeros((M, d)), *Ys)
    with pytest.raises(TypeError, match="CUDA"):
        rtq.qblock_project(blk, *Xs, *Ys)                # shapes fine, host memory
    bad = rtq.QBlock(*(getattr(blk, n) for n in ("qkvg", "qkvg_sm", "wo", "wo_s", "w13",
                                                 "w13_sm")),
                     torch.zeros((d, d), dtype=torch.int8), blk.w2_s, d_model=d, d_ff=f)
    with pytest.raises(ValueError, match="w2"):
        bad.as_c()


def test_dequant_validation():
    assert rtq.rt_dequant_q4_f32(W, S, Y, 4, 40, None) == SHAPE
    assert rtq.rt_dequant_q4_f32(W + 1, S, Y, 4, 64, None) == ALIGN
    assert rtq.rt_dequant_q8_f32(None, S, Y, 4, 64, None) == INVALID
    assert rtq.rt_device_status(None, None) == INVALID


def test_debug_inject_rejects_bad_arguments():
    # checked before any CUDA call
    assert rtq.rt_debug_inject(2, 0) == INVALID
    assert rtq.rt_debug_inject(-1, 0) == INVALID
    assert rtq.rt_debug_inject(1, -5) == INVALID


# ---------------------------------------------------------------- quantizers
def test_quantizer_statuses():
    w = np.zeros((2, 40), dtype=np.float32)
    Wq = np.empty((2, 20), dtype=np.uint8)
    sm = np.empty((2, 2, 2), dtype=np.uint16)
    assert rtq.rt_quantize_q4_g32(w.ctypes.data, 2, 40, 21, Wq.ctypes.data, sm.ctypes.data) == SHAPE
    w = np.full((1, 32), np.nan, dtype=np.float32)
    assert rtq.rt_quantize_q4_g32(w.ctypes.data, 1, 32, 21, Wq.ctypes.data, sm.ctypes.data) == RANGE
    w = np.full((1, 32), 7e4, dtype=np.float32)
    assert rtq.rt_quantize_q4_g32(w.ctypes.data, 1, 32, 21, Wq.ctypes.data, sm.ctypes.data) == RANGE
    assert rtq.rt_quantize_q4_g32(w.ctypes.data, 1, 32, -1, Wq.ctypes.data, sm.ctypes.data) == INVALID
    assert rtq.rt_quantize_q8_row(None, 1, 32, None, None) == INVALID
    w = np.full((1, 16), np.inf, dtype=np.float32)
    q = np.empty((1, 16), dtype=np.int8)
    s = np.empty(1, dtype=np.float32)
    assert rtq.rt_quantize_q8_row(w.ctypes.data, 1, 16, q.ctypes.data, s.ctypes.data) == RANGE


@pytest.mark.parametrize("name,outliers", [("qkvg", False), ("w13", False), ("qkvg", True)])
def test_q4_quantizer_matches_oracle_bit_for_bit(name, outliers):
    W = wl.projection_weights(3, 0, name, outliers=outliers)
    if not outliers:
        W = W[:512]  # a slice keeps the single-threaded oracle fast
    Wq, sm = rtq.quantize_q4_g32(W)
    Wq_o, sm_o = oracle.quant_q4_g32(W)
    assert np.array_equal(Wq, Wq_o)
    assert np.array_equal(sm, sm_o)


def test_q4_quantizer_grid_sizes_and_degenerate_rows():
    W = wl.weights(48, 96, seed=31)
    W[5] = 0.25   # constant rows
    W[6] = 0.0
    W[7, :32] = -3.0
    for n_grid in (1, 2, 5, 21, 41):
        Wq, sm = rtq.quantize_q4_g32(W, n_grid=n_grid)
        Wq_o, sm_o = oracle.quant_q4_g32(W, n_grid=n_grid)
        assert np.array_equal(Wq, Wq_o) and np.array_equal(sm, sm_o), n_grid


@pytest.mark.parametrize("name,outliers", [("wo", False), ("w2", False), ("w2", True)])
def test_q8_quantizer_matches_oracle_bit_for_bit(name, outliers):
    W = wl.projection_weights(3, 0, name, outliers=outliers)
    W[1] = 0.0
    Wq, s = rtq.quantize_q8_row(W)
    Wq_o, s_o = oracle.quant_q8_row(W)
    assert np.array_equal(Wq, Wq_o)
    assert np.array_equal(s.view(np.uint32), s_o.view(np.uint32))


def test_empty_quantizer_inputs():
    Wq, sm = rtq.quantize_q4_g32(np.zeros((0, 64), dtype=np.float32))
    assert Wq.shape == (0, 32) and sm.shape == (0, 2, 2)
    q, s = rtq.quantize_q8_row(np.zeros((0, 16), dtype=np.float32))
    assert q.shape == (0, 16)


# ------------------------------------------------------------ projection lists
def _qproj_array(entries):
    arr = (rtq._QProjC * len(entries))()
    for i, e in enumerate(entries):
        arr[i] = rtq._QProjC(*e)
    return arr


def test_batch_validation_and_routes():
    # (fmt, reserved, X, Wq, scales, bias, Y, N, K) at fake, aligned, disjoint addresses
    GB = 1 << 30
    def entry(i, fmt=4, N=2048, K=512, X=None, Y=None):
        return (fmt, 0, X or (1 * GB + i * 16 * 2 ** 20), 2 * GB + i * 16 * 2 ** 20,
                3 * GB + i * 16 * 2 ** 20, None, Y or (4 * GB + i * 16 * 2 ** 20), N, K)
    plan, run = rtq.lib().rt_qgemm_batch_plan, rtq.lib().rt_qgemm_batch
    TC_LIST = 5
    ok = _qproj_array([entry(i) for i in range(12)])          # 12 x 16 tiles = 192 >= SMs
    assert plan(ok, 12, 80, 0) == TC_LIST
    assert plan(ok, 12, 80, 2) == TC_LIST
    assert plan(ok, 12, 80, 1) == 0                           # SIMT: one call per entry
    assert plan(ok, 12, 4, 0) == 0                            # AUTO takes SIMT for q4 at M <= 16
    assert plan(ok, 12, 200, 2) == 0                          # M > 128: per call
    assert plan(ok, 2, 80, 0) == 0                            # 32 tiles < SMs under AUTO
    assert plan(ok, 2, 80, 2) == TC_LIST                      # forced
    # shared activations are allowed
    shared = _qproj_array([entry(i, X=1 * GB) for i in range(3)])
    assert plan(shared, 3, 80, 2) == TC_LIST
    # q4 K % 128 != 0 runs per call; K % 64 != 0 needs SIMT under AUTO
    assert plan(_qproj_array([entry(0, K=192), entry(1)]), 2, 80, 2) == 0
    assert plan(_qproj_array([entry(0, K=96)]), 1, 80, 2) == -1
    # rejections, all before any CUDA call
    assert run(None, 1, 80, 0, None) == INVALID
    assert run(ok, -1, 80, 0, None) == INVALID
    assert run(ok, 12, -1, 0, None) == INVALID
    assert run(ok, 12, 80, 3, None) == INVALID                # no path 3
    assert run(_qproj_array([entry(0, fmt=5)]), 1, 80, 0, None) == INVALID
    bad = list(entry(0)); bad[1] = 1                           # reserved must be 0
    assert run(_qproj_array([tuple(bad)]), 1, 80, 0, None) == INVALID
    bad = list(entry(0)); bad[2] += 4                          # X misaligned
    assert run(_qproj_array([tuple(bad)]), 1, 80, 0, None) == ALIGN
    assert run(_qproj_array([entry(0, K=40)]), 1, 80, 0, None) == SHAPE
    # outputs may not overlap another entry's output or inputs
    assert run(_qproj_array([entry(0), entry(1, Y=4 * GB + 4096)]), 2, 80, 0, None) == INVALID
    assert run(_qproj_array([entry(0), entry(1, Y=2 * GB)]), 2, 80, 0, None) == INVALID
    assert run(_qproj_array([entry(0), entry(1, X=4 * GB + 64)]), 2, 80, 0, None) == INVALID
    # no-ops
    assert run(ok, 0, 80, 0, None) == RT_OK
    assert run(ok, 12, 0, 0, None) == RT_OK


def test_block_fmt_validation_and_routes():
    GB = 1 << 30
    def blk(fmts, reserved=0, d=512, f=2048):
        ws = [rtq._QWeightC(fm, reserved, (2 + i) * GB, (6 + i) * GB) for i, fm in enumerate(fmts)]
        return rtq._QBlockFmtC(*ws, d, f)
    fused = rtq.lib().rt_qblock_fused_fmt
    run = rtq.lib().rt_qblock_project_fmt
    import ctypes as C
    q8 = blk((8, 8, 8, 8))
    assert fused(C.byref(q8), 80, 0) == 1                  # one grouped launch
    assert fused(C.byref(q8), 2048, 0) == 0                # one call per projection
    assert fused(C.byref(q8), 1, 0) == 0                   # SIMT under AUTO (q8: M = 1)
    assert fused(C.byref(q8), 2, 0) == 1
    mixed = blk((4, 8, 4, 8))
    assert fused(C.byref(mixed), 80, 0) == rtq.block_fused(80, 512, 2048) == 1
    assert fused(C.byref(blk((8, 8, 5, 8))), 80, 0) == -1  # unknown format
    assert fused(C.byref(blk((8, 8, 8, 8), reserved=1)), 80, 0) == -1
    X = [10 * GB + i * GB // 4 for i in range(4)]
    Y = [20 * GB + i * GB // 4 for i in range(4)]
    assert run(C.byref(blk((8, 8, 9, 8))), 80, *X, *Y, 0, None) == INVALID
    assert run(C.byref(blk((8, 8, 8, 8), reserved=2)), 80, *X, *Y, 0, None) == INVALID
    assert run(None, 80, *X, *Y, 0, None) == INVALID
    Ybad = list(Y); Ybad[1] = Y[0] + 64                    # outputs overlap
    assert run(C.byref(q8), 80, *X, *Ybad, 0, None) == INVALID
    assert run(C.byref(q8), 0, *X, *Y, 0, None) == RT_OK   # M == 0: no-op


def test_block_route_bits():
    """rt_qblock_route_fmt / rt_qblock_route: which launches a block takes.
    Without a device the side-stream pre-pass bit is never set."""
    GB = 1 << 30
    import ctypes as C
    route = rtq.lib().rt_qblock_route_fmt

    def blk(fmts, d=512, f=2048, scale_off=0):
        ws = [rtq._QWeightC(fm, 0, (2 + i) * GB, (6 + i) * GB + scale_off) for i, fm in enumerate(fmts)]
        return rtq._QBlockFmtC(*ws, d, f)
    mixed, q8 = blk((4, 8, 4, 8)), blk((8, 8, 8, 8))
    G, XR = rtq.ROUTE_GROUPED_SMALL_M, rtq.ROUTE_X_RESIDENT_GROUP
    assert route(C.byref(mixed), 80, 0) == G                 # one grouped launch
    assert route(C.byref(q8), 4096, 0) == XR                 # qkvg, wo, w13 share a launch
    assert route(C.byref(mixed), 4096, 0) == XR
    assert route(C.byref(mixed), 129, 0) == XR
    assert route(C.byref(mixed), 16384, 0) == 0              # CTA-pair kernels, one call each
    assert route(C.byref(mixed), 4096, 1) == 0               # SIMT path: one call each
    assert route(C.byref(mixed), 4096, 2) == XR              # tensor cores forced
    # q4 scales only 4-byte aligned: qkvg and w13 leave the TMA kernels, wo alone stays
    assert route(C.byref(blk((4, 8, 4, 8), scale_off=4)), 4096, 0) == 0
    assert route(C.byref(blk((8, 8, 5, 8))), 4096, 0) == -1  # unknown format
    assert route(C.byref(mixed), -1, 0) == -1
    assert route(None, 80, 0) == -1
    # rt_qblock_route (mixed recipe) agrees with the per-format form
    mq = rtq._QBlockC(2 * GB, 6 * GB, 3 * GB, 7 * GB, 4 * GB, 8 * GB, 5 * GB, 9 * GB, 512, 2048)
    for M in (80, 129, 4096, 16384):
        assert rtq.lib().rt_qblock_route(C.byref(mq), M, 0) == route(C.byref(mixed), M, 0)


# --------------------------------------------------------------- FP8 E4M3
@pytest.mark.parametrize("outliers", [False, True])
def test_e4m3_quantizer_matches_oracle_bit_for_bit(outliers):
    W = wl.weights(256, 512, 4242)
    if outliers:
        W = wl.with_outliers(W, 4243)
    assert np.array_equal(rtq.quantize_e4m3(W), oracle.quant_e4m3(W))


def test_e4m3_quantizer_edges_match_oracle():
    finite = np.array([oracle.e4m3_to_double(b) for b in range(0x7F)])
    mids = (finite[:-1] + finite[1:]) / 2
    edge = np.array([464.0, 463.99997, 448.0, 2 ** -10, 2 ** -6, 2 ** -6 - 2 ** -12, 0.0, -0.0])
    W = np.concatenate([finite, -finite, mids, -mids, edge]).astype(np.float32)[None, :]
    assert np.array_equal(rtq.quantize_e4m3(W), oracle.quant_e4m3(W))
    for bad in (464.01, -1e6, np.nan, np.inf):
        with pytest.raises(rtq.RtqError) as e:
            rtq.quantize_e4m3(np.array([[0.5, bad]], dtype=np.float32))
        assert e.value.status == RANGE
    assert rtq.rt_quantize_e4m3(None, 4, None) == INVALID
    assert rtq.rt_quantize_e4m3(None, 0, None) == RT_OK


def test_e4m3_gemm_validation_and_plan():
    f = rtq.rt_gemm_e4m3
    assert f(None, W, Y, 4, 16, 64, 0, None) == INVALID           # null X with M > 0
    assert f(X, None, Y, 4, 16, 64, 0, None) == INVALID           # null weights
    assert f(X, W + 8, Y, 4, 16, 64, 0, None) == ALIGN            # W not 16-byte aligned
    assert f(X, W, X, 4, 16, 64, 0, None) == INVALID              # Y overlaps X
    assert f(X, W, Y, 4, 16, 24, 0, None) == SHAPE                # K % 16
    assert f(X, W, Y, 4, 16, 96, 2, None) == SHAPE                # forced TC needs K % 64
    assert f(None, W, None, 0, 16, 64, 0, None) == RT_OK          # M == 0
    assert rtq.plan(3, 80, 512, 2048) == "tc_w_stationary"
    assert rtq.plan(3, 4096, 512, 512) == "tc_x_resident"
    assert rtq.plan(3, 4096, 512, 2048) == "tc_w_streamed"
    assert rtq.plan(3, 1, 512, 2048) == "simt"
    assert rtq.plan(3, 4, 512, 2048) == "tc_w_stationary"
    assert rtq.auto_path(3, 80, 512, 48) == 1                     # K % 64 != 0 -> SIMT
    assert rtq.workspace_bytes(3, 4096, 512, 2048) == 4096 * 2048 * 2
    # a batch entry in e4m3 carries no scales
    arr = _qproj_array([(3, 0, X, W, 0, None, Y, 2048, 512)] * 1)
    assert rtq.lib().rt_qgemm_batch_plan(arr, 1, 80, 2) == 5


def test_bias_validation():
    f = rtq.lib().rt_qgemm
    GB = 1 << 30
    B = 5 * GB
    assert f(4, X, W, S, B + 2, Y, 4, 16, 64, 0, None) == ALIGN        # bias not 4-byte aligned
    assert f(4, X, W, S, Y + 64, Y, 4, 16, 64, 0, None) == INVALID     # bias overlaps Y
    assert f(9, X, W, S, B, Y, 4, 16, 64, 0, None) == INVALID          # unknown format
    assert f(3, X, W, None, B, Y, 4, 16, 24, 0, None) == SHAPE         # e4m3 K % 16
    assert f(4, None, W, S, None, None, 0, 16, 64, 0, None) == RT_OK   # M == 0
    # a list entry's output may not overlap another entry's bias
    arr = _qproj_array([(4, 0, X, W, S, B, Y, 16, 64), (4, 0, X, W, S, None, B, 16, 64)])
    assert rtq.lib().rt_qgemm_batch(arr, 2, 4, 0, None) == INVALID
