"""rt_qgemm_batch on a GPU: every entry of a projection list against the
oracle, through the C ABI.

The list kernel (RT_KERNEL_TC_LIST) is checked on
  - RT-J block projection sets at M = 80 (mixed q4 / q8, the automatic route);
  - ragged shapes: M from 1 to 128 (every accumulator-ring and weight-ring
    depth the launch picks), N not a multiple of 128, q4 K from 128 to 1024,
    q8 K from 64 to 2048 (items that run chunk by chunk over 512-wide K);
  - entries sharing one activation buffer (the resident block is reused);
  - more entries than one launch holds (several launches);
  - no write outside any Y (NaN guard bands), bit-identical repeats and the
    same bits for the list in another order.
Expected values come only from oracle/; tolerances are the tensor-core gate
(max|dY| / max|Y| <= 4e-3) plus the elementwise fp16 rounding bound.
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
    """Host data of one list entry and its oracle result."""

    def __init__(self, fmt, M, N, K, seed, X=None, outliers=True):
        self.fmt, self.N, self.K = fmt, N, K
        self.X = wl.activations(M, K, seed) if X is None else X
        W = wl.weights(N, K, seed + 1)
        if outliers:
            W = wl.with_outliers(W, seed + 2)
        if fmt == 4:
            self.q = oracle.quant_q4_g32(W)
            self.What = oracle.dequant_q4(*self.q)
        else:
            self.q = oracle.quant_q8_row(W)
            self.What = oracle.dequant_q8(*self.q)
        self.ref = self.X.astype(np.float64) @ self.What.T


def device_list(rtq, entries, M, Xd=None, guard=64):
    """Device tensors of the entries; every Y is a 16-byte aligned view of one
    NaN-filled buffer with at least `guard` floats between outputs."""
    sizes = [M * e.N for e in entries]
    offs, off = [], guard
    for sz in sizes:
        offs.append(off)
        off = (off + sz + guard + 3) // 4 * 4
    flat = torch.full((off,), float("nan"), device="cuda")
    projs = []
    mask = torch.ones_like(flat, dtype=torch.bool)
    for i, (e, sz, o) in enumerate(zip(entries, sizes, offs)):
        X = Xd[i] if Xd is not None else dev(e.X)
        projs.append(rtq.Proj(e.fmt, X, dev(e.q[0]), dev(e.q[1]), flat[o:o + sz].view(M, e.N)))
        mask[o:o + sz] = False
    return projs, flat, mask


def check(entries, projs, flat, mask):
    assert bool(torch.isnan(flat[mask]).all()), "write outside an output"
    for i, (e, p) in enumerate(zip(entries, projs)):
        Y = p.Y.cpu().numpy()
        assert rel_err(Y, e.ref) <= TC_TOL, i
        assert within_bound(Y, e.X, e.What), i


def block_entries(M, n_blocks, seed):
    out = []
    for b in range(n_blocks):
        for j, name in enumerate(("qkvg", "wo", "w13", "w2")):
            spec = wl.BLOCK_PROJECTIONS[name]
            fmt = 4 if spec["fmt"] == "q4" else 8
            out.append(Entry(fmt, M, spec["N"], spec["K"], seed + 40 * b + 4 * j, outliers=False))
    return out


def test_block_sets_at_m80_take_the_list_kernel(rtq_lib):
    """Three RT-J blocks' projection sets at M = 80 (168 weight tiles): the
    automatic route is the list kernel; every output matches the oracle."""
    M = 80
    entries = block_entries(M, 3, seed=7000)
    projs, flat, mask = device_list(rtq_lib, entries, M)
    assert rtq_lib.batch_plan(projs) == "tc_list"
    rtq_lib.qgemm_batch(projs)
    torch.cuda.synchronize()
    check(entries, projs, flat, mask)
    first = flat.clone()
    rtq_lib.qgemm_batch(projs)                      # repeat: the same bits
    torch.cuda.synchronize()
    assert torch.equal(torch.nan_to_num(first, nan=7.0), torch.nan_to_num(flat, nan=7.0))
    # reversed list order: each tile is computed the same way by whichever CTA
    rtq_lib.qgemm_batch(list(reversed(projs)))
    torch.cuda.synchronize()
    assert torch.equal(torch.nan_to_num(first, nan=7.0), torch.nan_to_num(flat, nan=7.0))


# (M, [(fmt, N, K), ...]) with the list route forced (path "tc")
RAGGED = [
    (1, [(4, 130, 128), (8, 257, 64), (4, 512, 512), (8, 100, 2048)]),
    (16, [(4, 1, 256), (8, 384, 576), (4, 640, 1024), (8, 128, 512)]),
    (33, [(8, 300, 192), (4, 2048, 384), (8, 1000, 2048)]),
    (80, [(4, 2048, 512), (8, 512, 512), (4, 4096, 512), (8, 512, 2048), (4, 200, 640)]),
    (96, [(4, 384, 1024), (8, 700, 1088)]),
    (112, [(8, 520, 2048), (4, 129, 128)]),
    (128, [(4, 1024, 512), (8, 512, 2048), (4, 250, 896)]),
]


@pytest.mark.parametrize("M,shapes", RAGGED)
def test_ragged_lists_match_the_oracle(rtq_lib, M, shapes):
    entries = [Entry(f, M, n, k, seed=7100 + 13 * i + M) for i, (f, n, k) in enumerate(shapes)]
    projs, flat, mask = device_list(rtq_lib, entries, M)
    assert rtq_lib.batch_plan(projs, path="tc") == "tc_list"
    rtq_lib.qgemm_batch(projs, path="tc")
    torch.cuda.synchronize()
    check(entries, projs, flat, mask)


def test_entries_sharing_activations(rtq_lib):
    """Six q4 and q8 projections of K = 512 read one activation buffer, two
    q8 projections of K = 2048 another: one image each, kept resident."""
    M = 64
    X1 = wl.activations(M, 512, 7301)
    X2 = wl.activations(M, 2048, 7302)
    shapes = [(4, 2048, 512, X1), (8, 512, 512, X1), (4, 4096, 512, X1), (8, 512, 2048, X2),
              (4, 640, 512, X1), (8, 1536, 2048, X2), (4, 128, 512, X1), (8, 256, 512, X1)]
    entries = [Entry(f, M, n, k, 7310 + i, X=x) for i, (f, n, k, x) in enumerate(shapes)]
    Xd1, Xd2 = dev(X1), dev(X2)
    Xd = [Xd1 if e.K == 512 else Xd2 for e in entries]
    projs, flat, mask = device_list(rtq_lib, entries, M, Xd=Xd)
    rtq_lib.qgemm_batch(projs, path="tc")
    torch.cuda.synchronize()
    check(entries, projs, flat, mask)


def test_more_entries_than_one_launch(rtq_lib):
    """300 small projections (one launch holds 256): two list launches."""
    M = 24
    entries = [Entry(4 if i % 3 else 8, M, 128 + 64 * (i % 4), 128 * (1 + i % 4), 7400 + i,
                     outliers=False) for i in range(300)]
    projs, flat, mask = device_list(rtq_lib, entries, M)
    assert rtq_lib.batch_plan(projs) == "tc_list"
    rtq_lib.qgemm_batch(projs)
    torch.cuda.synchronize()
    check(entries, projs, flat, mask)


def test_routes_and_rejections(rtq_lib):
    M = 80
    entries = block_entries(M, 1, seed=7500)
    projs, flat, mask = device_list(rtq_lib, entries, M)
    # one block is 56 tiles, fewer than the SMs: one call per entry under AUTO
    assert rtq_lib.batch_plan(projs) == "per_call"
    assert rtq_lib.batch_plan(projs, path="tc") == "tc_list"
    assert rtq_lib.batch_plan(projs, path="simt") == "per_call"
    rtq_lib.qgemm_batch(projs)                       # the per-call route, same results
    torch.cuda.synchronize()
    check(entries, projs, flat, mask)
    # an output overlapping another entry's output is rejected before any launch
    bad = [projs[0], rtq_lib.Proj(projs[1].fmt, projs[1].X, projs[1].Wq, projs[1].scales,
                                  flat[64:64 + M * 512].view(M, 512))]   # entry 0's output
    with pytest.raises(rtq_lib.RtqError) as e:
        rtq_lib.qgemm_batch(bad, path="tc")
    assert e.value.status == rtq_lib.RT_ERR_INVALID_ARG
    rtq_lib.qgemm_batch([], M=M)                     # empty list: no-op
