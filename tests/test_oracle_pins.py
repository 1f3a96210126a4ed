"""Pins for the CPU oracle: each check ties it to something other than itself.

* Hadamard: scipy's Sylvester construction, H H^T = b I, the explicit (-1)^popcount(i&j) matrix,
  and the involution H(Hx) = b x -- exact on small integers.
* Transform: a float64 reference built from scipy's Hadamard matrix, within the fp32 rounding bound,
  and absorption invariance X diag(1/s) H (W diag(s) H / b)^T = X W^T to 1e-5.
* MXFP4: the hand-derived OCP MX v1.0 cases in tests/golden/ocp_mxfp4_cases.txt, a brute-force
  nearest-grid search (a second, independent restatement written here), the defining property of
  the shared exponent (block maximum lands in E2M1's top binade), and exact round trips of on-grid
  values for every code and every reachable scale.
* GEMM: an exact rational sum (fractions) on tiny shapes.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ocp_mxfp4_cases.txt")
GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _golden(kind):
    out = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == kind:
                out.append(parts[1:])
    return out


# ---------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_matrix_is_sylvester(b):
    cols = [oracle.fwht_f32(np.eye(b, dtype=np.float32)[j]) for j in range(b)]
    H = np.stack(cols, axis=1).astype(np.float64)  # column j = H e_j
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(b).astype(np.float64))
    np.testing.assert_array_equal(H @ H.T, b * np.eye(b))
    explicit = np.array([[(-1) ** bin(i & j).count("1") for j in range(b)] for i in range(b)], np.float64)
    np.testing.assert_array_equal(H, explicit)


@pytest.mark.parametrize("b", [16, 32, 64, 128])
def test_fwht_exact_on_small_integers_and_involution(b):
    rng = np.random.default_rng(b)
    explicit = np.array([[(-1) ** bin(i & j).count("1") for j in range(b)] for i in range(b)], np.float64)
    for _ in range(20):
        x = rng.integers(-1000, 1000, size=b).astype(np.float32)
        y = oracle.fwht_f32(x)
        np.testing.assert_array_equal(y.astype(np.float64), explicit @ x.astype(np.float64))
        np.testing.assert_array_equal(oracle.fwht_f32(y).astype(np.float64), b * x.astype(np.float64))


def _blockdiag_h(K, b):
    H = scipy.linalg.hadamard(b).astype(np.float64)
    return scipy.linalg.block_diag(*([H] * (K // b)))


@pytest.mark.parametrize("b", [1, 16, 32, 64, 128])
@pytest.mark.parametrize("absorb", [False, True])
def test_transform_matches_float64_reference(b, absorb):
    g = torch.Generator().manual_seed(7 + b)
    K, rows = 256, 8
    x = (torch.randn(rows, K, generator=g) * 3).to(torch.bfloat16)
    m = torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69).to(torch.float32)
    y = oracle.transform_rows(x, m, b, absorb)
    xd = x.to(torch.float64).numpy()
    md = m.to(torch.float64).numpy()
    Hb = _blockdiag_h(K, b) if b > 1 else np.eye(K)
    ref = (xd * md) @ Hb
    if absorb and b > 1:
        ref = ref / b
    absterm = np.abs(xd * md) @ np.abs(Hb)
    if absorb and b > 1:
        absterm = absterm / b
    bound = (math.log2(b) + 2) * 2.0 ** -24 * absterm + 1e-30
    assert np.all(np.abs(y.astype(np.float64) - ref) <= bound)


@pytest.mark.parametrize("b", [16, 32, 64, 128])
def test_absorption_invariance(b):
    """X diag(1/s) H_b (W diag(s) H_b / b)^T equals X W^T to 1e-5 relative (unquantized)."""
    g = torch.Generator().manual_seed(100 + b)
    M, K, N = 12, 512, 24
    X = torch.randn(M, K, generator=g).to(torch.bfloat16)
    X[:, :4] *= 50
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    s = torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69).to(torch.float32)
    inv_s = np.float32(1.0) / s.numpy()
    xa = oracle.transform_rows(X, inv_s, b, absorb=False).astype(np.float64)
    wa = oracle.transform_rows(W, s, b, absorb=True).astype(np.float64)
    got = xa @ wa.T
    ref = X.to(torch.float64).numpy() @ W.to(torch.float64).numpy().T
    scale = np.abs(X.to(torch.float64).numpy()) @ np.abs(W.to(torch.float64).numpy()).T
    assert np.max(np.abs(got - ref) / scale) < 1e-5
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-5


def test_absorption_breaks_without_inverse_factor():
    """The pin has teeth: dropping the 1/b factor (a plausible mistake) fails it by far."""
    g = torch.Generator().manual_seed(5)
    X = torch.randn(4, 64, generator=g).to(torch.bfloat16)
    W = torch.randn(8, 64, generator=g).to(torch.bfloat16)
    xa = oracle.transform_rows(X, None, 32, absorb=False).astype(np.float64)
    wa_wrong = oracle.transform_rows(W, None, 32, absorb=False).astype(np.float64)
    ref = X.double().numpy() @ W.double().numpy().T
    assert np.linalg.norm(xa @ wa_wrong.T - ref) / np.linalg.norm(ref) > 1.0


# ---------------------------------------------------------------- E2M1 / E8M0
def brute_force_code(t: float) -> int:
    """Nearest E2M1 magnitude by exhaustive search in exact rationals; a tie goes to the code with
    an even mantissa bit (code bit 0); |t| > 6 clamps to 6; the sign bit follows the input's sign."""
    sign = 8 if math.copysign(1.0, t) < 0 else 0
    a = Fraction(abs(t)) if math.isfinite(t) else Fraction(10 ** 40)
    best = None
    for code, v in enumerate(GRID):
        d = abs(a - Fraction(v))
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return sign | best[1]


def test_e2m1_golden_cases():
    cases = _golden("code")
    assert len(cases) >= 20
    for val, code, *_ in cases:
        t = float(np.float32(float(val)))
        assert oracle.e2m1_code(t) == int(code, 16), (val, code)
        assert brute_force_code(t) == int(code, 16), (val, code)


def test_e2m1_matches_brute_force_on_ties_and_random():
    pts = []
    for i in range(len(GRID) - 1):  # every midpoint and its fp32 neighbours
        mid = np.float32((GRID[i] + GRID[i + 1]) / 2)
        pts += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(10))]
    pts += [np.float32(v) for v in GRID] + [np.float32(6.0001), np.float32(1e-45), np.float32(3e38)]
    rng = np.random.default_rng(0)
    pts += list(rng.uniform(0, 8, 4000).astype(np.float32))
    pts += list((rng.standard_normal(2000) * 3).astype(np.float32))
    for p in pts:
        for t in (float(p), -float(p)):
            assert oracle.e2m1_code(t) == brute_force_code(t), t


def test_e8m0_golden_cases():
    for amax, E, *_ in _golden("exp"):
        assert oracle.e8m0_exponent(float(np.float32(float(amax)))) == int(E), amax


def test_e8m0_puts_block_max_in_top_binade():
    """Defining property of the shared exponent: amax / 2^(E-127) lies in [4, 8) whenever E is not
    clamped, i.e. the largest element uses E2M1's top exponent (emax_elem = 2)."""
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        np.exp2(rng.uniform(-120, 125, 3000)),
        np.exp2(np.arange(-124, 126)),                      # exact powers of two
        np.nextafter(np.exp2(np.arange(-120, 126)).astype(np.float32), np.float32(0)),  # just below them
    ]).astype(np.float32)
    for a in vals:
        E = oracle.e8m0_exponent(float(a))
        r = Fraction(float(a)) / Fraction(2) ** (E - 127)
        assert 4 <= r < 8, (a, E)


def test_mxfp4_pack_golden():
    for v0, v1, E, byte in _golden("pack"):
        E = int(E)
        y = np.zeros(32, np.float32)
        y[0], y[1] = float(v0), float(v1)
        y[31] = 4.0 * 2.0 ** (E - 127)
        codes, sf = oracle.mxfp4_quantize(y)
        assert int(sf[0, 0]) == E
        assert int(codes[0, 0]) == int(byte, 16), (v0, v1, hex(codes[0, 0]))


def test_mxfp4_round_trip_every_code_every_scale():
    """Values already on the MXFP4 grid come back bit-exactly, for all 16 codes and every E8M0
    value reachable from finite fp32 data (0..252)."""
    codes16 = np.arange(16, dtype=np.uint8)
    vals = np.array([oracle.e2m1_value(int(c)) for c in codes16])
    assert list(vals[:8]) == GRID and list(-vals[8:]) == GRID
    for E in range(0, 253):
        y = np.zeros(32, np.float64)
        y[:16] = vals
        y[16:] = vals[::-1]
        y = (y * 2.0 ** (E - 127)).astype(np.float32)
        assert np.all(np.isfinite(y))
        codes, sf = oracle.mxfp4_quantize(y)
        assert int(sf[0, 0]) == E
        expect = np.concatenate([codes16, codes16[::-1]])
        got = np.empty(32, np.uint8)
        got[0::2] = codes[0] & 15
        got[1::2] = codes[0] >> 4
        np.testing.assert_array_equal(got, expect)
        back = oracle.dequant(codes, sf)[0]
        np.testing.assert_array_equal(back, y.astype(np.float64))


def test_mxfp4_quantize_matches_brute_force_rows():
    rng = np.random.default_rng(3)
    y = (rng.standard_normal((16, 128)) * np.exp2(rng.integers(-20, 20, (16, 1)))).astype(np.float32)
    y[3] = 0
    y[4, :32] = 1e-40
    codes, sf = oracle.mxfp4_quantize(y)
    for r in range(16):
        for g in range(4):
            blk = y[r, 32 * g:32 * g + 32]
            amax = float(np.max(np.abs(blk)))
            if amax == 0:
                E = 0
            else:
                p = math.floor(math.log2(Fraction(amax))) if amax >= 2.0 ** -149 else -149
                # exact floor(log2) by search (log2 of a Fraction is float; correct it exactly)
                while Fraction(2) ** p > Fraction(amax):
                    p -= 1
                while Fraction(2) ** (p + 1) <= Fraction(amax):
                    p += 1
                E = min(max(p - 2 + 127, 0), 254)
            assert sf[r, g] == E
            for i in range(32):
                t = float(Fraction(float(blk[i])) / Fraction(2) ** (E - 127))
                c = (codes[r, (32 * g + i) // 2] >> (4 * (i & 1))) & 15
                assert c == brute_force_code(t), (r, g, i)


# ---------------------------------------------------------------- GEMM
def test_linear_exact_rational_sum():
    rng = np.random.default_rng(11)
    for M, N, K in [(1, 1, 32), (3, 5, 64), (7, 4, 64)]:
        Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
        Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
        Asf = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
        Wsf = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
        Y, T = oracle.linear(Aq, Asf, Wq, Wsf)

        def val(q, sf, r, k):
            c = (q[r, k // 2] >> (4 * (k & 1))) & 15
            mag = Fraction(GRID[c & 7])
            return (-mag if c & 8 else mag) * Fraction(2) ** (int(sf[r, k // 32]) - 127)

        for m in range(M):
            for n in range(N):
                terms = [val(Aq, Asf, m, k) * val(Wq, Wsf, n, k) for k in range(K)]
                exact = sum(terms, Fraction(0))
                tabs = sum((abs(t) for t in terms), Fraction(0))
                assert abs(Fraction(Y[m, n]) - exact) <= Fraction(1, 10 ** 12) * tabs
                assert abs(Fraction(T[m, n]) - tabs) <= Fraction(1, 10 ** 12) * tabs


def test_linear_row_subset_and_grouped_reduce_to_dense():
    rng = np.random.default_rng(12)
    M, N, K, E = 20, 6, 128, 3
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    Asf = rng.integers(110, 140, (M, K // 32), dtype=np.uint8)
    Wq = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    Wsf = rng.integers(110, 140, (E, N, K // 32), dtype=np.uint8)
    off = np.array([0, 7, 7, 20], np.int32)  # expert 1 is empty
    Yg, Tg = oracle.grouped_linear(Aq, Asf, off, Wq, Wsf)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        Yd, Td = oracle.linear(Aq[lo:hi], Asf[lo:hi], Wq[e], Wsf[e])
        np.testing.assert_array_equal(Yg[lo:hi], Yd)
        np.testing.assert_array_equal(Tg[lo:hi], Td)
    rows = [19, 0, 8]
    Ys, _ = oracle.grouped_linear(Aq, Asf, off, Wq, Wsf, rows=rows)
    np.testing.assert_array_equal(Ys, Yg[sorted(rows)])
    Yd, _ = oracle.linear(Aq, Asf, Wq[2], Wsf[2], rows=[3, 9])
    Yf, _ = oracle.linear(Aq, Asf, Wq[2], Wsf[2])
    np.testing.assert_array_equal(Yd, Yf[[3, 9]])


def test_linear_matmul_equals_the_ordered_sum():
    """The library-matmul form of the GEMM oracle equals the exact rational sum on tiny shapes and
    the ordered C loop elsewhere, to float64 rounding (K * 2^-52 of T), with extreme scales, row
    subsets, W chunking across the chunk size and the grouped form with empty experts."""
    rng = np.random.default_rng(13)
    M, N, K = 3, 5, 64
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Asf = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
    Wsf = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
    Y, T = oracle.linear_matmul(Aq, Asf, Wq, Wsf)

    def val(q, sf, r, k):
        c = (q[r, k // 2] >> (4 * (k & 1))) & 15
        mag = Fraction(GRID[c & 7])
        return (-mag if c & 8 else mag) * Fraction(2) ** (int(sf[r, k // 32]) - 127)

    for m in range(M):
        for n in range(N):
            terms = [val(Aq, Asf, m, k) * val(Wq, Wsf, n, k) for k in range(K)]
            tabs = sum((abs(t) for t in terms), Fraction(0))
            assert abs(Fraction(Y[m, n]) - sum(terms, Fraction(0))) <= Fraction(1, 10 ** 12) * tabs
            assert abs(Fraction(T[m, n]) - tabs) <= Fraction(1, 10 ** 12) * tabs
    M, N, K = 37, 300, 1024
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Asf = rng.integers(1, 254, (M, K // 32), dtype=np.uint8)
    Wsf = rng.integers(60, 190, (N, K // 32), dtype=np.uint8)
    rows = [36, 0, 17]
    Yl, Tl = oracle.linear(Aq, Asf, Wq, Wsf, rows=rows)
    Ym, Tm = oracle.linear_matmul(Aq, Asf, Wq, Wsf, rows=rows, n_chunk=128)
    assert np.all(np.abs(Ym - Yl) <= K * 2.0 ** -52 * Tl)
    assert np.all(np.abs(Tm - Tl) <= K * 2.0 ** -52 * Tl)
    E = 4
    off = np.array([0, 9, 9, 30, 37], np.int32)        # expert 1 is empty
    Wqe = rng.integers(0, 256, (E, 64, K // 2), dtype=np.uint8)
    Wsfe = rng.integers(110, 140, (E, 64, K // 32), dtype=np.uint8)
    Yg, Tg = oracle.grouped_linear(Aq, Asf, off, Wqe, Wsfe)
    Ygm, Tgm = oracle.grouped_linear_matmul(Aq, Asf, off, Wqe, Wsfe)
    assert np.all(np.abs(Ygm - Yg) <= K * 2.0 ** -52 * Tg)
    assert np.all(np.abs(Tgm - Tg) <= K * 2.0 ** -52 * Tg)
    Ys, _ = oracle.grouped_linear_matmul(Aq, Asf, off, Wqe, Wsfe, rows=[30, 2, 29, 9])
    sub = [2, 9, 29, 30]
    assert np.all(np.abs(Ys - Yg[sub]) <= K * 2.0 ** -52 * Tg[sub])


# ---------------------------------------------------------------- composed pipeline
def test_prep_and_act_quant_compose_to_transform_then_quantize():
    g = torch.Generator().manual_seed(21)
    M, K, N, b = 5, 256, 7, 32
    X = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    s = torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69).to(torch.float32)
    Wq, Wsf, inv_s = oracle.prep_weights(W, s, b)
    np.testing.assert_array_equal(inv_s, np.float32(1.0) / s.numpy())
    c2, s2 = oracle.mxfp4_quantize(oracle.transform_rows(W, s, b, absorb=True))
    np.testing.assert_array_equal(Wq, c2)
    np.testing.assert_array_equal(Wsf, s2)
    Xq, Xsf = oracle.act_quant(X, inv_s, b)
    c3, s3 = oracle.mxfp4_quantize(oracle.transform_rows(X, inv_s, b, absorb=False))
    np.testing.assert_array_equal(Xq, c3)
    np.testing.assert_array_equal(Xsf, s3)
    # grouped act-quant reduces to the dense one per expert
    inv2 = np.stack([inv_s, inv_s[::-1].copy()])
    off = [0, 2, 5]
    Gq, Gsf = oracle.act_quant(X, inv2, b, offsets=off)
    for e in range(2):
        q, sf = oracle.act_quant(X[off[e]:off[e + 1]], inv2[e], b)
        np.testing.assert_array_equal(Gq[off[e]:off[e + 1]], q)
        np.testing.assert_array_equal(Gsf[off[e]:off[e + 1]], sf)


def test_quantized_layer_approximates_unquantized_product():
    """End-to-end sanity: the W4A4 product stays close to X W^T (MXFP4 noise only). A random,
    uncalibrated s spreads channel magnitudes 16x and costs accuracy; that is expected."""
    g = torch.Generator().manual_seed(22)
    M, K, N, b = 16, 512, 32, 32
    X = torch.randn(M, K, generator=g).to(torch.bfloat16)
    X[:, [3, 100]] *= 50
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    s = torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69).to(torch.float32)
    ref = X.double().numpy() @ W.double().numpy().T
    for scale, bound in ((None, 0.25), (s, 0.6)):
        Wq, Wsf, inv_s = oracle.prep_weights(W, scale, b)
        Xq, Xsf = oracle.act_quant(X, inv_s, b)
        Y, _ = oracle.linear(Xq, Xsf, Wq, Wsf)
        rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
        assert rel < bound, rel


# ---------------------------------------------------------------- MoE combine
def test_bf16_rne_matches_torch_cast():
    """The oracle's fp32 -> bf16 rounding equals torch's round-to-nearest-even cast, including exact
    ties (odd and even kept bit), subnormals, signed zeros and values near the top of the range."""
    g = torch.Generator().manual_seed(31)
    v = torch.randn(4000, generator=g) * torch.exp(torch.randn(4000, generator=g) * 20)
    ties = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130 * 1.5,
                         1e-40, -0.0, 0.0, 3.0e38, -3.0e38, 2.0 ** -126 * (1 + 2.0 ** -8)])
    v = torch.cat([v, ties]).to(torch.float32)
    v = v[torch.isfinite(v)]
    ref = v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.bf16_rne(v.numpy()), ref)


def test_moe_combine_definition():
    """Properties that fix the combine: with one choice of weight 1 it copies rows exactly; dropped
    choices (pos outside Y) equal omitting them; the fp32 result is within the rounding bound of the
    exact float64 weighted sum (2 * topk roundings of 2^-24 each, relative to sum |w y|)."""
    g = torch.Generator().manual_seed(32)
    y_rows, N, T, topk = 40, 24, 9, 6
    Y = torch.randn(y_rows, N, generator=g).to(torch.bfloat16)
    pos = torch.randint(0, y_rows, (T, topk), generator=g).to(torch.int32).numpy()
    w = torch.rand(T, topk, generator=g).numpy().astype(np.float32)
    one = oracle.moe_combine(Y, pos[:, :1], np.ones((T, 1), np.float32))
    np.testing.assert_array_equal(one, Y.float().numpy()[pos[:, 0]])
    out = oracle.moe_combine(Y, pos, w)
    yd = Y.double().numpy()
    exact = np.einsum("tj,tjn->tn", w.astype(np.float64), yd[pos])
    tabs = np.einsum("tj,tjn->tn", np.abs(w.astype(np.float64)), np.abs(yd[pos]))
    assert np.all(np.abs(out - exact) <= 2 * topk * 2.0 ** -24 * tabs)
    dropped = pos.copy()
    dropped[:, 2] = -1
    dropped[0, 4] = y_rows          # past the end: also skipped
    got = oracle.moe_combine(Y, dropped, w)
    keep = [0, 1, 3, 4, 5]           # rows 1.. lose choice 2
    np.testing.assert_array_equal(got[1:], oracle.moe_combine(Y, pos[1:, keep], w[1:, keep]))
    keep0 = [0, 1, 3, 5]             # row 0 loses choices 2 and 4
    np.testing.assert_array_equal(got[:1], oracle.moe_combine(Y, pos[:1, keep0], w[:1, keep0]))


# ---------------------------------------------------------------- fused SwiGLU
def test_exp_f32_against_the_exponential():
    """The fixed fp32 exp is within 4 ulp of exp over its range, exact at 0, and clamps outside it."""
    import math

    xs = np.concatenate([np.linspace(-100, 88, 40001), np.float32([-0.0, 1e-30, -1e-30, 0.34657359, -0.34657359,
                                                                   1.0, -1.0, 87.99, -99.99])]).astype(np.float32)
    for x in xs:
        e = oracle.exp_f32(float(x))
        ref = math.exp(float(x))
        if ref >= 2.0 ** -126:
            assert abs(e - ref) <= 4 * float(np.spacing(np.float32(ref))), (x, e, ref)
        else:   # subnormal results: within 4 units of the smallest subnormal step
            assert abs(e - ref) <= 4 * 2.0 ** -149, (x, e, ref)
    assert oracle.exp_f32(0.0) == 1.0
    assert oracle.exp_f32(-1000.0) == oracle.exp_f32(-100.0)
    assert oracle.exp_f32(1000.0) == oracle.exp_f32(88.0)


def test_swiglu_f32_definition():
    import math

    rng = np.random.default_rng(41)
    for g, u in zip(rng.normal(0, 4, 3000).astype(np.float32), rng.normal(0, 2, 3000).astype(np.float32)):
        ref = float(g) * float(u) / (1.0 + math.exp(-float(g)))
        got = oracle.swiglu_f32(float(g), float(u))
        assert abs(got - ref) <= 8 * float(np.spacing(np.float32(abs(ref)))) + 1e-38, (g, u, got, ref)
    assert oracle.swiglu_f32(0.0, 5.0) == 0.0
    assert oracle.swiglu_f32(200.0, 3.0) == 600.0          # exp(-200) clamps to exp(-100): silu(g) = g
    tiny = oracle.swiglu_f32(-200.0, 3.0)                   # exp(200) clamps to exp(88): -200 / (1 + e^88) * 3
    assert -1e-33 < tiny < 0.0


def test_swiglu_act_quant_composes_swiglu_transform_and_mxfp4():
    """swiglu_act_quant equals: the elementwise fixed SwiGLU, the fp32 multiply by 1/s, the fixed-order
    butterflies per block, then MXFP4 (each step its own pinned oracle function)."""
    rng = np.random.default_rng(42)
    M, I = 5, 256
    G = rng.normal(0, 3, (M, I)).astype(np.float32)
    U = rng.normal(0, 1, (M, I)).astype(np.float32)
    inv = np.exp(rng.uniform(-2.0, 0.7, I)).astype(np.float32)
    for b in (1, 16, 32, 64):
        H = np.array([[oracle.swiglu_f32(float(G[m, i]), float(U[m, i])) for i in range(I)] for m in range(M)],
                     np.float32)
        V = (H * inv).astype(np.float32)
        if b > 1:
            V = np.stack([np.concatenate([oracle.fwht_f32(V[m, k:k + b]) for k in range(0, I, b)]) for m in range(M)])
        c_ref, s_ref = oracle.mxfp4_quantize(V)
        c, s = oracle.swiglu_act_quant(G, U, inv, b)
        np.testing.assert_array_equal(c, c_ref)
        np.testing.assert_array_equal(s, s_ref)


# ---------------------------------------------------------------- Flip-Refinement
def _flip_case(seed, N=6, K=256, b=32, M=512):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    s = torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69).to(torch.float32)
    X = torch.randn(M, K, generator=g)
    X[:, :4] *= 20.0                                          # correlated, uneven channels
    X = (X + 0.5 * X.roll(1, dims=1)).to(torch.bfloat16)
    Wq, Wsf, inv = oracle.prep_weights(W, s, b)
    Xt = oracle.transform_rows(X, inv, b, absorb=False).astype(np.float64)
    H = (Xt.T @ Xt / M).astype(np.float32)
    w = oracle.transform_rows(W, s, b, absorb=True).astype(np.float64)
    return W, s, b, Wq, Wsf, H, w


def _exact_loss(q, sf, w, H):
    e = oracle.dequant(q, sf) - w
    return np.einsum("nk,kj,nj->n", e, H.astype(np.float64), e)


def test_flip_refine_separable_hessian_moves_nothing():
    """With a diagonal positive H the loss separates per code, and the prepared (nearest) codes are
    already optimal: no move lowers it."""
    W, s, b, Wq, Wsf, H, w = _flip_case(51)
    for D in (np.eye(H.shape[0], dtype=np.float32), np.diag(np.diag(H)).astype(np.float32)):
        q, flips = oracle.flip_refine(W, s, b, D, 2, Wq, Wsf)
        np.testing.assert_array_equal(q, Wq)
        assert np.all(flips == 0)


def test_flip_refine_loss_never_increases_and_converges_to_a_local_minimum():
    W, s, b, Wq, Wsf, H, w = _flip_case(52)
    prev = _exact_loss(Wq, Wsf, w, H)
    q = Wq
    total = 0
    for sweep in range(12):
        q, flips = oracle.flip_refine(W, s, b, H, 1, q, Wsf)
        cur = _exact_loss(q, Wsf, w, H)
        assert np.all(cur <= prev * (1 + 1e-12) + 1e-300), (sweep, cur, prev)
        total += int(flips.sum())
        prev = cur
        if flips.sum() == 0:
            break
    assert flips.sum() == 0, "did not converge"
    assert total > 0 and np.all(prev < _exact_loss(Wq, Wsf, w, H))
    # brute force: no single neighbouring move lowers the exact loss of any row
    N, K = w.shape
    grid = oracle.dequant(q, Wsf)
    Hd = H.astype(np.float64)
    E = Wsf.astype(np.int64) - 127
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    signed = np.concatenate([-vals[:0:-1], vals])               # index t + 7 for t in [-7, 7]
    for n in range(N):
        e = grid[n] - w[n]
        base = e @ Hd @ e
        for k in range(K):
            scale = 2.0 ** E[n, k // 32]
            t = int(np.argmin(np.abs(signed * scale - grid[n, k])))
            for tc in (t - 1, t + 1):
                if 0 <= tc < 15:
                    e2 = e.copy()
                    e2[k] += signed[tc] * scale - grid[n, k]
                    assert e2 @ Hd @ e2 >= base * (1 - 1e-12), (n, k)


# ---------------------------------------------------------------- weight-only (W4A16)
def test_act_transform_bf16_composes_transform_and_rounding():
    g = torch.Generator().manual_seed(61)
    X = (torch.randn(7, 512, generator=g) * 10).to(torch.bfloat16)
    inv = (1.0 / torch.exp(torch.rand(512, generator=g) * 2.77 - 0.69)).to(torch.float32).numpy()
    for b in (1, 16, 32, 64, 128):
        ref = torch.from_numpy(oracle.transform_rows(X, inv, b, absorb=False)).to(torch.bfloat16)
        got = oracle.act_transform_bf16(X, inv, b)
        np.testing.assert_array_equal(got, ref.view(torch.int16).numpy().view(np.uint16))


def test_w4a16_linear_exact_on_tiny_inputs():
    """b = 1 and no s: the activations are X itself (already bf16), so Y is the exact rational sum of
    X times the dequantized codes."""
    rng = np.random.default_rng(62)
    M, N, K = 3, 4, 64
    X = torch.from_numpy(rng.normal(0, 1, (M, K)).astype(np.float32)).to(torch.bfloat16)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Wsf = rng.integers(110, 140, (N, K // 32), dtype=np.uint8)
    Y, T = oracle.w4a16_linear(X, None, 1, Wq, Wsf)
    xv = [[Fraction(float(v)) for v in row] for row in X.float().numpy()]
    for m in range(M):
        for n in range(N):
            terms = []
            for k in range(K):
                c = (Wq[n, k // 2] >> (4 * (k & 1))) & 15
                w = (-1 if c & 8 else 1) * Fraction(GRID[c & 7]) * Fraction(2) ** (int(Wsf[n, k // 32]) - 127)
                terms.append(xv[m][k] * w)
            tabs = sum((abs(t) for t in terms), Fraction(0))
            assert abs(Fraction(Y[m, n]) - sum(terms, Fraction(0))) <= Fraction(1, 10 ** 12) * tabs
            assert abs(Fraction(T[m, n]) - tabs) <= Fraction(1, 10 ** 12) * tabs


def test_w4a16_beats_w4a4_on_outlier_channels():
    """With outlier channels, keeping the (transformed) activations in bf16 loses less than MXFP4
    activations: the weight-only layer is closer to X W^T than the W4A4 layer."""
    g = torch.Generator().manual_seed(63)
    M, K, N, b = 16, 1024, 64, 32
    X = torch.randn(M, K, generator=g)
    X[:, [5, 300, 777]] *= 40
    X = X.to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    s = torch.exp(torch.rand(K, generator=g) * 2.77 - 0.69).to(torch.float32)
    ref = X.double().numpy() @ W.double().numpy().T
    Wq, Wsf, inv = oracle.prep_weights(W, s, b)
    Yw, _ = oracle.w4a16_linear(X, inv, b, Wq, Wsf)
    Xq, Xsf = oracle.act_quant(X, inv, b)
    Ya, _ = oracle.linear(Xq, Xsf, Wq, Wsf)
    err_w = np.linalg.norm(Yw - ref) / np.linalg.norm(ref)
    err_a = np.linalg.norm(Ya - ref) / np.linalg.norm(ref)
    assert err_w < err_a, (err_w, err_a)
