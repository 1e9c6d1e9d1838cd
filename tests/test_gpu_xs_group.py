"""Grouped launches of the activation-resident kernel on a GPU, through the
C ABI.

Above 128 activation rows, the K <= 512 projections of a block
(rt_qblock_project) or of a list (rt_qgemm_batch, per-entry route) run up to
four at a time in one launch of the activation-resident kernel, after one
pre-pass launch that rounds each one's activations into its own slice of the
workspace.  A launch whose problems share one format runs that format's
build; q4 mixed with q8 / e4m3 runs the mixed build (q4 scale words loaded
from global memory one item ahead).  Checked here:
  - every output against the oracle (max|dY| / max|Y| <= 4e-3 and the
    elementwise fp16 rounding bound);
  - the same bits as one rt_qgemm call per projection (the grouped kernel
    computes each tile exactly as the single-problem launch does);
  - problems of different K in one launch (128 to 512), ragged M and N,
    bias, e4m3 entries, lists longer than one launch holds, and entries the
    group leaves out (K = 2048, q4 scales only 4-byte aligned);
  - nothing written outside the outputs (NaN guard bands), bit-identical
    repeats.
Expected values come only from oracle/.
"""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

TC_TOL = 4e-3
U16 = 2.0 ** -11


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
    return float(np.max(np.abs(np.asarray(Y, np.float64) - Yref)) / max(np.max(np.abs(Yref)), 1e-300))


def within_bound(Y, X, What):
    """fp16 rounding of both operands plus fp32 accumulation, per output."""
    A = np.abs(X.astype(np.float64)) @ np.abs(What).T
    K = X.shape[1]
    slack = 2.0 ** -25 * (np.abs(What).sum(axis=1)[None, :] +
                          np.abs(X.astype(np.float64)).sum(axis=1)[:, None])
    bound = (2 * U16 + U16 * U16 + (K + 1) * 2.0 ** -23) * A + slack
    return not (np.abs(np.asarray(Y, np.float64) - X.astype(np.float64) @ What.T) > bound).any()


class Entry:
    """Host data of one projection and its oracle result (fmt 4, 8 or 3)."""

    def __init__(self, fmt, M, N, K, seed, bias=False):
        self.fmt, self.N, self.K = fmt, N, K
        self.X = wl.activations(M, K, seed)
        W = wl.with_outliers(wl.weights(N, K, seed + 1), seed + 2)
        if fmt == 4:
            self.q = oracle.quant_q4_g32(W)
            self.What = oracle.dequant_q4(*self.q)
        elif fmt == 8:
            self.q = oracle.quant_q8_row(W)
            self.What = oracle.dequant_q8(*self.q)
        else:
            self.q = (oracle.quant_e4m3(W), None)
            self.What = oracle.dequant_e4m3(self.q[0])
        self.b = (np.random.default_rng(seed + 3).standard_normal(N).astype(np.float32)
                  if bias else None)
        self.ref = self.X.astype(np.float64) @ self.What.T
        if self.b is not None:
            self.ref = self.ref + self.b.astype(np.float64)[None, :]


def device_list(rtq, entries, M, guard=64, scale_offset=None):
    """Device tensors; every Y is a 16-byte aligned view of one NaN-filled
    buffer with `guard` floats between outputs.  scale_offset: {index: k}
    places that q4 entry's scales k floats into a larger buffer (alignment
    tests)."""
    sizes = [M * e.N for e in entries]
    offs, off = [], guard
    for sz in sizes:
        offs.append(off)
        off = (off + sz + guard + 3) // 4 * 4
    flat = torch.full((off,), float("nan"), device="cuda")
    mask = torch.ones_like(flat, dtype=torch.bool)
    projs = []
    for i, (e, sz, o) in enumerate(zip(entries, sizes, offs)):
        sc = None
        if e.q[1] is not None:
            sc = dev(e.q[1])
            if scale_offset and i in scale_offset:
                k = 4 * scale_offset[i]                  # bytes past a 256-byte boundary
                nbytes = sc.numel() * sc.element_size()
                raw = torch.empty(nbytes + k, dtype=torch.uint8, device="cuda")
                raw[k:].copy_(sc.reshape(-1).view(torch.uint8))
                sc = raw[k:].view(sc.dtype).view(sc.shape)
        projs.append(rtq.Proj(e.fmt, dev(e.X), dev(e.q[0]), sc, flat[o:o + sz].view(M, e.N),
                              None if e.b is None else dev(e.b)))
        mask[o:o + sz] = False
    return projs, flat, mask


def single_call(rtq, e, p):
    """The same projection as one rt_qgemm call (same kernel plan)."""
    Y = torch.empty_like(p.Y)
    rtq.qgemm(e.fmt, p.X, p.Wq, p.scales, bias=p.bias, Y=Y)
    return Y


def check(rtq, entries, projs, flat, mask):
    torch.cuda.synchronize()
    assert bool(torch.isnan(flat[mask]).all()), "write outside an output"
    for i, (e, p) in enumerate(zip(entries, projs)):
        Y = p.Y.cpu().numpy()
        assert rel_err(Y, e.ref) <= TC_TOL, i
        if e.b is None:
            assert within_bound(Y, e.X, e.What), i
        assert torch.equal(p.Y, single_call(rtq, e, p)), f"entry {i}: grouped != single call"


# (M, [(fmt, N, K, bias), ...]) for rt_qgemm_batch above 128 rows
LISTS = [
    # mixed q4 / q8 / e4m3, ragged N, K 128..512 in one launch, 500 = 2 x 192 + 116
    (500, [(4, 130, 256, False), (8, 257, 512, True), (3, 200, 384, False), (4, 1000, 128, True)]),
    # six entries: a launch of four and one of two; one K = 2048 entry between them
    # (weight-streamed, outside the groups)
    (129, [(8, 384, 512, False), (4, 640, 512, False), (4, 128, 256, True), (3, 520, 128, False),
           (8, 300, 2048, False), (4, 768, 384, False), (8, 96, 256, True)]),
    # one format per launch: the q4 build (TMA-staged scales) and the q8 build
    (1000, [(4, 2048, 512, False), (4, 512, 256, True), (4, 1100, 384, False)]),
    (777, [(8, 512, 512, False), (8, 1536, 256, False), (8, 129, 128, True)]),
    (300, [(3, 1024, 512, False), (3, 256, 256, True)]),
]


@pytest.mark.parametrize("M,shapes", LISTS)
def test_batch_groups_match_oracle_and_single_calls(rtq_lib, M, shapes):
    entries = [Entry(f, M, n, k, seed=9100 + 17 * i + M, bias=b)
               for i, (f, n, k, b) in enumerate(shapes)]
    projs, flat, mask = device_list(rtq_lib, entries, M)
    assert rtq_lib.batch_plan(projs) == "per_call"
    rtq_lib.qgemm_batch(projs)
    check(rtq_lib, entries, projs, flat, mask)
    first = flat.clone()
    rtq_lib.qgemm_batch(projs)                      # repeat: the same bits
    torch.cuda.synchronize()
    assert torch.equal(torch.nan_to_num(first, nan=7.0), torch.nan_to_num(flat, nan=7.0))


def test_q4_scales_4_byte_aligned_leave_the_group(rtq_lib):
    """A q4 entry whose scales sit 4 bytes past a 16-byte boundary (allowed)
    cannot take a tensor map: it runs on the weight-stationary kernel, the
    rest of the list still as one launch; same results either way."""
    M = 400
    shapes = [(4, 512, 512, False), (8, 512, 512, False), (4, 256, 256, True)]
    entries = [Entry(f, M, n, k, seed=9300 + i, bias=b) for i, (f, n, k, b) in enumerate(shapes)]
    projs, flat, mask = device_list(rtq_lib, entries, M, scale_offset={0: 1})
    assert projs[0].scales.data_ptr() % 16 == 4
    rtq_lib.qgemm_batch(projs)
    check(rtq_lib, entries, projs, flat, mask)


def _sized_block(d_model, d_ff, M, seed):
    shapes = {"qkvg": (4, 4 * d_model, d_model), "wo": (8, d_model, d_model),
              "w13": (4, 2 * d_ff, d_model), "w2": (8, d_model, d_ff)}
    return {n: Entry(f, M, N, K, seed + 10 * i) for i, (n, (f, N, K)) in enumerate(shapes.items())}


# (M, d_model, d_ff): blocks above 128 rows through rt_qblock_project
BLOCKS = [
    (300, 256, 384),     # all four in one mixed launch (K 256 and 384); last block 108 rows
    (200, 128, 256),     # all four, K 128 and 256; 8 rows past the first block
    (1000, 512, 2048),   # qkvg, wo, w13 in one launch; w2 (K = 2048) weight-streamed
]


@pytest.mark.parametrize("M,d_model,d_ff", BLOCKS)
def test_block_driver_groups_the_x_resident_projections(rtq_lib, M, d_model, d_ff):
    names = ("qkvg", "wo", "w13", "w2")
    e = _sized_block(d_model, d_ff, M, seed=9500 + M)
    entries = [e[n] for n in names]
    projs, flat, mask = device_list(rtq_lib, entries, M)
    blk = rtq_lib.QBlock(projs[0].Wq, projs[0].scales, projs[1].Wq, projs[1].scales,
                         projs[2].Wq, projs[2].scales, projs[3].Wq, projs[3].scales,
                         d_model=d_model, d_ff=d_ff)
    assert rtq_lib.block_fused(M, d_model, d_ff, "auto") == 0
    rtq_lib.qblock_project(blk, *(p.X for p in projs), *(p.Y for p in projs))
    check(rtq_lib, entries, projs, flat, mask)


def test_default_block_takes_the_side_stream_pre_pass(rtq_lib):
    """RT-J's block at M = 4096 (the benchmark's configuration), mixed and
    all-int8 recipes: qkvg, wo and w13 share one launch, and w2's pre-pass
    runs on the second stream -- its lean blocks fit on the SMs beside the
    activation-resident CTAs (the check that would turn the overlap off if a
    kernel's register count grew past the room)."""
    M, d, f = 4096, 512, 2048
    both = rtq_lib.ROUTE_X_RESIDENT_GROUP | rtq_lib.ROUTE_SIDE_PREPASS
    e = _sized_block(d, f, 8, seed=9700)
    ten = {n: (dev(e[n].q[0]), dev(e[n].q[1])) for n in e}
    blk = rtq_lib.QBlock(*ten["qkvg"], *ten["wo"], *ten["w13"], *ten["w2"], d_model=d, d_ff=f)
    assert rtq_lib.block_route(blk, M) == both
    q8 = {n: oracle.quant_q8_row(wl.weights(N, K, 9800 + i))
          for i, (n, N, K) in enumerate((("qkvg", 4 * d, d), ("wo", d, d), ("w13", 2 * f, d),
                                         ("w2", d, f)))}
    blk8 = rtq_lib.QBlockFmt(*((8, dev(q8[n][0]), dev(q8[n][1])) for n in ("qkvg", "wo", "w13", "w2")),
                             d_model=d, d_ff=f)
    assert rtq_lib.block_route(blk8, M) == both
