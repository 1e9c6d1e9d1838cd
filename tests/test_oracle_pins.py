"""Pins for the CPU oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to a hand-worked example (tests/golden), a
closed form, an exact-arithmetic brute force on tiny inputs, an invariant, or
a library routine that computes the same special case (numpy's binary16
conversion).  A plausible slip in the oracle -- a swapped nibble, a dropped
min term, a wrong group index, a transposed operand, a double rounding in the
fp16 encoder, a wrong tie rule -- fails at least one of them.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl


def _hex_list(s):
    return [int(t, 16) for t in s.split()]


# ---------------------------------------------------------------------------
# binary16 encode / decode  (pinned to numpy's independent implementation)
# ---------------------------------------------------------------------------
def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got) & (got > 0), np.isinf(ref) & (ref > 0))


def test_f16_encode_matches_numpy_across_ranges():
    g = np.random.default_rng(123)
    xs = []
    for e in range(-30, 17):  # subnormals, normals, overflow
        xs.append(g.uniform(2.0 ** e, 2.0 ** (e + 1), size=200))
    xs = np.concatenate(xs)
    xs = np.concatenate([xs, -xs])
    # exact ties: halfway between adjacent binary16 values, in normal and subnormal range
    h = np.arange(1, 0x7BFF, 97, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    ties = (lo + hi) / 2
    special = np.array([0.0, -0.0, 65504.0, 65519.999, 65520.0, 70000.0, 2.0 ** -25,
                        1.5 * 2.0 ** -24, 3 * 2.0 ** -26, 2.0 ** -24, 2.0 ** -14,
                        (2.0 ** -14) * (1 - 2.0 ** -12), 0.1, 1.0 / 3.0])
    xs = np.concatenate([xs, ties, -ties, special, -special])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f16_from_double(float(x)) for x in xs], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(xs[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]


# ---------------------------------------------------------------------------
# packing and dequantization (E1, round trip, independent restatement)
# ---------------------------------------------------------------------------
def test_e1_pack_and_dequant(golden):
    fx = golden("e1_pack_dequant.txt")
    codes = np.array([int(t) for t in fx["codes"].split()], dtype=np.uint8)
    packed = oracle.pack_nibbles(codes)
    assert list(packed) == _hex_list(fx["bytes"])
    # one 32-wide group: the four worked codes then zeros
    row_codes = np.zeros(32, dtype=np.uint8)
    row_codes[:4] = codes
    Wq = oracle.pack_nibbles(row_codes).reshape(1, 16)
    sm = np.array([[[int(fx["scale16"], 16), int(fx["min16"], 16)]]], dtype=np.uint16)
    W = oracle.dequant_q4(Wq, sm)
    expect = [float(t) for t in fx["dequant"].split()]
    assert list(W[0, :4]) == expect
    assert np.all(W[0, 4:] == -1.0)  # code 0 -> min


def test_pack_unpack_round_trip():
    g = np.random.default_rng(7)
    codes = g.integers(0, 16, size=4096, dtype=np.uint8)
    packed = oracle.pack_nibbles(codes)
    assert packed.size == 2048
    assert np.array_equal(oracle.unpack_nibbles(packed), codes)
    # low nibble is the even index
    assert np.array_equal(packed & 0x0F, codes[0::2])
    assert np.array_equal(packed >> 4, codes[1::2])


def test_dequant_q4_group_indexing_against_numpy_view():
    """Every element of a multi-group, multi-row tensor equals nibble*scale+min
    with the group k//32 of its own row, as numpy reads the same bytes."""
    g = np.random.default_rng(11)
    N, K = 5, 96
    Wq = g.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sc = (g.uniform(0.001, 0.01, size=(N, K // 32))).astype(np.float16)
    mn = (g.uniform(-0.1, 0.0, size=(N, K // 32))).astype(np.float16)
    sm = np.stack([sc.view(np.uint16), mn.view(np.uint16)], axis=-1)
    got = oracle.dequant_q4(Wq, sm)
    nib = np.empty((N, K), dtype=np.int64)
    nib[:, 0::2] = Wq & 0x0F
    nib[:, 1::2] = Wq >> 4
    grp = np.arange(K) // 32
    ref = nib * sc.astype(np.float64)[:, grp] + mn.astype(np.float64)[:, grp]
    assert np.array_equal(got, ref)


def test_dequant_q8_exact():
    g = np.random.default_rng(12)
    q = g.integers(-127, 128, size=(4, 64), dtype=np.int8)
    s = g.uniform(1e-4, 1e-3, size=4).astype(np.float32)
    got = oracle.dequant_q8(q, s)
    for o in range(4):
        for k in range(64):
            assert Fraction(got[o, k]) == Fraction(int(q[o, k])) * Fraction(float(s[o]))


# ---------------------------------------------------------------------------
# q4 min-MSE clip search
# ---------------------------------------------------------------------------
def test_shrink_grid_endpoints():
    assert oracle.shrink_factor(0, 21) == 1.0
    assert oracle.shrink_factor(20, 21) == 0.8
    assert abs(oracle.shrink_factor(10, 21) - 0.9) < 1e-15
    assert oracle.shrink_factor(0, 1) == 1.0


def test_e2_clip_closed_form(golden):
    fx = golden("e2_clip_closed_form.txt")
    w = np.array([-1 + 0.5 * (i % 16) for i in range(32)], dtype=np.float32).reshape(1, 32)
    Wq, sm, js = oracle.quant_q4_g32(w, want_j=True)
    assert js[0, 0] == int(fx["jstar"])
    assert sm[0, 0, 0] == int(fx["scale16"], 16) and sm[0, 0, 1] == int(fx["min16"], 16)
    assert list(Wq[0]) == _hex_list(fx["bytes"])
    # every shrunk candidate clips something, so has positive error
    for j in range(1, 21):
        *_, err = oracle.q4_candidate(w[0], -1.0, 6.5, oracle.shrink_factor(j, 21))
        assert err > 0.0


def test_e5_degenerate_group(golden):
    fx = golden("e5_degenerate_group.txt")
    w = np.full((1, 32), np.float32(float(fx["value"])), dtype=np.float32)
    Wq, sm, js = oracle.quant_q4_g32(w, want_j=True)
    assert js[0, 0] == int(fx["jstar"])
    assert sm[0, 0, 0] == int(fx["scale16"], 16)
    assert sm[0, 0, 1] == int(fx["min16"], 16)
    assert oracle.f16_to_double(int(sm[0, 0, 1])) == float(fx["min_value"])
    assert np.all(Wq == 0)


def _numpy_grid_errors(w, n_grid):
    """Squared error of every grid point for one group, computed with numpy's own
    binary16 rounding (an implementation independent of the oracle's)."""
    w64 = w.astype(np.float64)
    lo, hi = w64.min(), w64.max()
    errs, params, codes = [], [], []
    for j in range(n_grid):
        s = 1.0 - (0.2 * j) / (n_grid - 1)
        sc = np.float64((s * hi - s * lo) / 15.0).astype(np.float16)
        mn = np.float64(s * lo).astype(np.float16)
        scd, mnd = float(sc), float(mn)
        if scd == 0.0:
            q = np.zeros(32)
        else:
            q = np.clip(np.rint((w64 - mnd) / scd), 0, 15)
        rec = q * scd + mnd
        errs.append(float(np.sum((w64 - rec) ** 2)))
        params.append((int(sc.view(np.uint16)), int(mn.view(np.uint16))))
        codes.append(q.astype(np.uint8))
    return np.array(errs), params, codes


@pytest.mark.parametrize("outliers", [False, True])
def test_clip_choice_is_bruteforce_argmin(outliers):
    N, K = 24, 256
    W = wl.weights(N, K, seed=4242)
    if outliers:
        W = wl.with_outliers(W, seed=4242, frac=0.2)
    Wq, sm, js = oracle.quant_q4_g32(W, n_grid=21, want_j=True)
    codes = oracle.unpack_nibbles(Wq.reshape(-1)).reshape(N, K)
    for o in range(N):
        for g in range(K // 32):
            errs, params, qs = _numpy_grid_errors(W[o, g * 32:(g + 1) * 32], 21)
            # the chosen point has the least error; ties keep the first
            j = int(js[o, g])
            assert errs[j] == errs.min()
            assert np.all(errs[:j] > errs[j])
            assert tuple(sm[o, g]) == params[j]
            assert np.array_equal(codes[o, g * 32:(g + 1) * 32], qs[j])
    if outliers:
        assert np.any(js > 0), "outlier groups should choose a clipped range"


def test_q4_reconstruction_error_bound():
    """With the unshrunk range every value lies within half a step of its
    reconstruction (plus the binary16 rounding of scale and min), so the
    chosen point's error is at most the s=1 error."""
    W = wl.weights(16, 128, seed=99)
    Wq, sm, js = oracle.quant_q4_g32(W, want_j=True)
    deq = oracle.dequant_q4(Wq, sm)
    for o in range(16):
        for g in range(4):
            w = W[o, g * 32:(g + 1) * 32]
            *_, err0 = oracle.q4_candidate(w, float(w.min()), float(w.max()), 1.0)
            err = float(np.sum((w.astype(np.float64) - deq[o, g * 32:(g + 1) * 32]) ** 2))
            assert err <= err0


# ---------------------------------------------------------------------------
# q8 per-row quantizer
# ---------------------------------------------------------------------------
def test_e3_q8_row(golden):
    fx = golden("e3_q8_row.txt")
    row = np.array([[float(t) for t in fx["row"].split()]], dtype=np.float32)
    q, s = oracle.quant_q8_row(row)
    assert float(s[0]) == float(fx["scale"])
    assert list(q[0]) == [int(t) for t in fx["codes"].split()]


def test_q8_invariants():
    W = wl.with_outliers(wl.weights(64, 512, seed=5), seed=5)
    W[3] = 0.0  # zero row
    q, s = oracle.quant_q8_row(W)
    assert s[3] == 0 and np.all(q[3] == 0)
    amax = np.abs(W).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(127.0)).astype(np.float32))
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    deq = q.astype(np.float64) * s.astype(np.float64)[:, None]
    assert np.all(np.abs(W - deq) <= s.astype(np.float64)[:, None] / 2 * (1 + 1e-6))
    nz = np.nonzero(amax > 0)[0]
    arg = np.abs(W[nz]).argmax(axis=1)
    assert np.all(np.abs(q[nz, arg]) == 127)


# ---------------------------------------------------------------------------
# GEMM: exact brute force on tiny inputs, closed forms, orientation
# ---------------------------------------------------------------------------
def _exact_q4_weights(Wq, sm):
    N, K2 = Wq.shape
    K = 2 * K2
    out = [[None] * K for _ in range(N)]
    for o in range(N):
        for k in range(K):
            b = int(Wq[o, k // 2])
            nib = (b & 15) if k % 2 == 0 else (b >> 4)
            sc = Fraction(float(np.uint16(sm[o, k // 32, 0]).view(np.float16)))
            mn = Fraction(float(np.uint16(sm[o, k // 32, 1]).view(np.float16)))
            out[o][k] = nib * sc + mn
    return out


def test_gemm_q4_tiny_exact_bruteforce():
    g = np.random.default_rng(3)
    M, N, K = 3, 5, 64
    X = g.standard_normal((M, K)).astype(np.float32)
    W = wl.weights(N, K, seed=17)
    Wq, sm = oracle.quant_q4_g32(W)
    Y = oracle.gemm_q4(X, Wq, sm)
    assert Y.shape == (M, N)
    What = _exact_q4_weights(Wq, sm)
    for m in range(M):
        for o in range(N):
            exact = sum(Fraction(float(X[m, k])) * What[o][k] for k in range(K))
            assert abs(float(exact) - Y[m, o]) <= 1e-14 * max(1.0, abs(float(exact)))


def test_gemm_q8_tiny_exact_bruteforce():
    g = np.random.default_rng(4)
    M, N, K = 4, 3, 48
    X = g.standard_normal((M, K)).astype(np.float32)
    q = g.integers(-127, 128, size=(N, K), dtype=np.int8)
    s = g.uniform(1e-4, 1e-3, size=N).astype(np.float32)
    Y = oracle.gemm_q8(X, q, s)
    for m in range(M):
        for o in range(N):
            exact = sum(Fraction(float(X[m, k])) * int(q[o, k]) * Fraction(float(s[o]))
                        for k in range(K))
            assert abs(float(exact) - Y[m, o]) <= 1e-14 * max(1.0, abs(float(exact)))


def test_gemm_identity_input_gives_transposed_weights():
    """X = I_K turns the projection into W_hat^T exactly (E4)."""
    N, K = 40, 64
    W = wl.weights(N, K, seed=21)
    Wq, sm = oracle.quant_q4_g32(W)
    Y = oracle.gemm_q4(np.eye(K, dtype=np.float32), Wq, sm)
    assert np.array_equal(Y, oracle.dequant_q4(Wq, sm).T)
    q, s = oracle.quant_q8_row(W)
    Y8 = oracle.gemm_q8(np.eye(K, dtype=np.float32), q, s)
    assert np.array_equal(Y8, oracle.dequant_q8(q, s).T)


def test_gemm_ones_input_closed_form():
    """X = 1 gives, per output, sum over groups of scale*sum(codes) + 32*min."""
    N, K = 6, 128
    W = wl.weights(N, K, seed=22)
    Wq, sm = oracle.quant_q4_g32(W)
    Y = oracle.gemm_q4(np.ones((2, K), dtype=np.float32), Wq, sm)
    for o in range(N):
        tot = Fraction(0)
        for g in range(K // 32):
            byts = Wq[o, g * 16:(g + 1) * 16].astype(int)
            csum = int(np.sum(byts & 15) + np.sum(byts >> 4))
            sc = Fraction(float(np.uint16(sm[o, g, 0]).view(np.float16)))
            mn = Fraction(float(np.uint16(sm[o, g, 1]).view(np.float16)))
            tot += sc * csum + 32 * mn
        assert Y[0, o] == Y[1, o]
        assert abs(Y[0, o] - float(tot)) <= 1e-15 * abs(float(tot)) + 1e-300


def test_gemm_q8_identity_weights_reproduce_input():
    K = 32
    q = (127 * np.eye(K)).astype(np.int8)
    s = np.full(K, np.float32(1.0) / np.float32(127.0), dtype=np.float32)
    X = np.random.default_rng(5).standard_normal((3, K)).astype(np.float32)
    Y = oracle.gemm_q8(X, q, s)
    assert np.allclose(Y, X, rtol=1e-7, atol=0)


def test_gemm_row_subset_matches_full():
    X = wl.activations(9, 64, seed=1)
    W = wl.weights(7, 64, seed=2)
    Wq, sm = oracle.quant_q4_g32(W)
    full = oracle.gemm_q4(X, Wq, sm)
    rows = np.array([0, 4, 8])
    assert np.array_equal(oracle.gemm_q4(X, Wq, sm, rows=rows), full[rows])


def test_quantizer_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.quant_q4_g32(np.full((1, 32), np.inf, dtype=np.float32))
    with pytest.raises(ValueError):
        oracle.quant_q4_g32(np.full((1, 32), 1e5, dtype=np.float32))


# ---------------------------------------------------------------- FP8 E4M3
torch = pytest.importorskip("torch")


def test_e6_e4m3_hand_worked(golden):
    g = golden("e6_e4m3.txt")
    codes = [int(c, 16) for c in g["codes"].split()]
    values = [float(v) for v in g["values"].split()]
    assert [oracle.e4m3_to_double(c) for c in codes] == values
    ins = [float(v) for v in g["encode_in"].split()]
    outs = [int(c, 16) for c in g["encode_out"].split()]
    assert [oracle.e4m3_from_double(x) for x in ins] == outs


def test_e4m3_decode_all_codes_match_torch():
    """Every one of the 256 codes against PyTorch's own float8_e4m3fn decoding."""
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_to_double(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.isnan(got).sum() == 2          # 0x7F and 0xFF


def test_e4m3_encode_matches_torch_rounding():
    """The nearest-value search against PyTorch's float -> float8_e4m3fn cast on
    every finite value, every midpoint (ties), random values across the
    binades and the subnormals, and the edge up to 464."""
    finite = np.array([oracle.e4m3_to_double(b) for b in range(0x7F)])
    mids = (finite[:-1] + finite[1:]) / 2
    g = np.random.default_rng(11)
    rnd = np.concatenate([g.uniform(-448, 448, 2000), g.normal(0, 0.02, 2000),
                          g.uniform(-2 ** -6, 2 ** -6, 1000), np.linspace(440, 464, 97)])
    xs = np.concatenate([finite, -finite, mids, -mids, rnd]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_from_double(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_out_of_range_is_rejected():
    for x in (464.0001, -500.0, 1e30, float("nan"), float("inf")):
        assert oracle.e4m3_from_double(x) is None
    with pytest.raises(ValueError):
        oracle.quant_e4m3(np.array([[0.1, 600.0]], dtype=np.float32))


def test_gemm_e4m3_identity_and_bruteforce():
    W = wl.weights(24, 32, 5)
    Wq = oracle.quant_e4m3(W)
    What = oracle.dequant_e4m3(Wq)
    # X = I gives the dequantized weights transposed, exactly
    assert np.array_equal(oracle.gemm_e4m3(np.eye(32, dtype=np.float32), Wq), What.T)
    # a tiny product against exact rational arithmetic
    X = wl.activations(3, 32, 6)
    Y = oracle.gemm_e4m3(X, Wq)
    for m in range(3):
        for o in range(0, 24, 5):
            exact = sum(Fraction(float(X[m, k])) * Fraction(What[o, k]) for k in range(32))
            assert abs(Fraction(Y[m, o]) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 80)
