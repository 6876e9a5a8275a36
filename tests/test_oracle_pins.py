"""Pins for the CPU oracle: each check ties an oracle function to something
other than itself (an independent Philox implementation, closed forms,
hand-derived worked examples, brute-force enumeration with exact rationals,
numpy), so that a dropped term, a wrong sign or index or a transposed operand
fails at least one of them. CPU only."""
import json
import math
import subprocess
import sys
from fractions import Fraction
from pathlib import Path

import numpy as np
import pytest

import oracle
from quantized_lora_merge_b200 import workloads as wl

GOLDEN = Path(__file__).resolve().parent / "golden"


# ---------------------------------------------------------------------------
# a1: Philox4x32-10 against Triton's independent implementation
# ---------------------------------------------------------------------------
def test_philox_matches_independent_implementation():
    rng = np.random.default_rng(12345)
    cases = [[0, 0, 0, 0, 0, 0], [2**32 - 1] * 6, [1, 0, 0, 0, 1, 0], [0, 1, 0, 0, 0, 0],
             [0, 0, 7, 0, 1, 0], [123, 0, 5, 0, 1, 0]]
    cases += rng.integers(0, 2**32, size=(26, 6), dtype=np.uint64).tolist()
    script = Path(__file__).resolve().parent / "philox_triton_reference.py"
    res = subprocess.run([sys.executable, str(script), json.dumps(cases)], check=True,
                         capture_output=True, text=True, timeout=600)
    expected = json.loads(res.stdout.strip().splitlines()[-1])
    for case, exp in zip(cases, expected):
        got = oracle.philox4x32_10(case[:4], case[4:]).tolist()
        assert got == exp, f"Philox mismatch for counter/key {case}"


def test_aux_word_counter_layout():
    """Element e of stream (seed, sid) is word e%4 of the block whose counter
    is (e//4 low, e//4 high, sid, 0) under key (seed low, seed high); checked
    through the independently pinned block function, including a block index
    above 2^32 and a seed above 2^32."""
    for seed, sid, e in [(1, 0, 0), (1, 0, 7), (1, 3, 1023), (2**40 + 5, 9, 2**34 + 6),
                         (1, 2**32 - 1, 5)]:
        block = e >> 2
        words = oracle.philox4x32_10([block & 0xFFFFFFFF, block >> 32, sid, 0],
                                     [seed & 0xFFFFFFFF, seed >> 32])
        assert oracle.aux_word(seed, sid, e) == int(words[e & 3])


def test_philox_output_is_uniform():
    """Chi-square of 2^16 words over 256 top-byte bins, and bit balance."""
    words = np.concatenate([oracle.philox4x32_10([b, 0, 1, 0], [7, 0]) for b in range(1 << 14)])
    words = words.astype(np.uint64)
    counts = np.bincount((words >> 24).astype(np.int64), minlength=256)
    expected = words.size / 256
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    assert chi2 < 256 + 6 * math.sqrt(2 * 256)
    bits = np.unpackbits(words.astype(np.uint32).view(np.uint8))
    assert abs(bits.mean() - 0.5) < 4 * 0.5 / math.sqrt(bits.size)


# ---------------------------------------------------------------------------
# a1: the Laplace sampler
# ---------------------------------------------------------------------------
def test_laplace_closed_forms():
    g = json.loads((GOLDEN / "laplace_closed_form.json").read_text())
    for case in g["cases"]:
        expected = eval(case["R_expr"], {"ln": math.log, "log": math.log, "log1p": math.log1p})
        got = float(oracle.laplace_from_word(case["x"])[0])
        assert got == pytest.approx(expected, rel=1e-15, abs=1e-300), case


def test_laplace_inverse_cdf_round_trip():
    """F(R(x)) = u(x) with F the textbook Laplace(0,1) CDF."""
    rng = np.random.default_rng(5)
    xs = rng.integers(0, 2**32, size=4000, dtype=np.uint64).astype(np.uint32)
    R = oracle.laplace_from_word(xs)
    u = (2.0 * (xs >> 9).astype(np.float64) + 1.0) * 2.0**-24
    F = np.where(R < 0, 0.5 * np.exp(R), 1.0 - 0.5 * np.exp(-R))
    assert np.max(np.abs(F - u)) < 1e-15


def test_laplace_symmetry_exact():
    """Complementing the 23 uniform bits maps u to 1-u, hence R to -R exactly."""
    rng = np.random.default_rng(6)
    xs = rng.integers(0, 2**32, size=2000, dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(oracle.laplace_from_word(xs ^ np.uint32(0xFFFFFE00)),
                          -oracle.laplace_from_word(xs))


def test_laplace_moments():
    """Laplace(0,1): mean 0, variance 2, excess kurtosis 3, P(|R|>t)=e^-t."""
    R = oracle.aux_R(1024, 1024, seed=1, stream_id=0).ravel()
    N = R.size
    assert abs(R.mean()) < 4 * math.sqrt(2.0 / N)
    var = R.var()
    assert abs(var - 2.0) < 4 * math.sqrt(20.0 / N)
    kurt = np.mean(R**4) / var**2 - 3.0
    assert abs(kurt - 3.0) < 0.1
    for t in (0.5, 1.0, 2.0, 4.0):
        p = math.exp(-t)
        assert abs(np.mean(np.abs(R) > t) - p) < 5 * math.sqrt(p * (1 - p) / N)
    assert np.max(np.abs(R)) <= 23 * math.log(2) + 1e-12


# ---------------------------------------------------------------------------
# a2: sigma and VMC
# ---------------------------------------------------------------------------
def test_population_std_closed_form_ramp():
    for N in (1, 2, 10, 1001):
        x = np.arange(N, dtype=np.float64) * 3.0 + 7.0
        assert oracle.population_std(x) == pytest.approx(3.0 * math.sqrt((N * N - 1) / 12.0),
                                                         rel=1e-14, abs=1e-14)


def test_std_f32_and_sigma_r_against_numpy():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((37, 53)) * 0.02 + 0.5).astype(np.float32)
    assert oracle.std_f32(W) == pytest.approx(float(np.std(W.astype(np.float64))), rel=1e-12)
    R = oracle.aux_R(37, 53, 1, 4)
    assert oracle.sigma_r(37, 53, 1, 4) == pytest.approx(float(np.std(R)), rel=1e-12)


def test_vmc_scale_laws():
    sw, sr = 0.02, 1.41
    assert oracle.vmc_scale(sw, sr, 0.0) == 1.0
    # alpha = 1 matches sigma exactly: std(c R) = sigma_W
    R = oracle.aux_R(64, 64, 1, 0)
    c1 = oracle.vmc_scale(sw, float(np.std(R)), 1.0)
    assert np.std(c1 * R) == pytest.approx(sw, rel=1e-13)
    # exponent law: c(2a) = c(a)^2, and c < 1 grows toward 1 as alpha shrinks
    assert oracle.vmc_scale(sw, sr, 3.0) == pytest.approx(oracle.vmc_scale(sw, sr, 1.5) ** 2,
                                                          rel=1e-14)
    assert oracle.vmc_scale(sw, sr, 0.5) > oracle.vmc_scale(sw, sr, 1.5)


# ---------------------------------------------------------------------------
# a3 / a6: the affine quantizer
# ---------------------------------------------------------------------------
def test_affine_quantizer_worked_examples():
    g = json.loads((GOLDEN / "affine_quantizer_worked.json").read_text())
    for case in g["cases"]:
        q = oracle.affine_quantize_row(case["x"], case["bits"])
        assert q["scale"] == pytest.approx(case["scale"], rel=1e-15), case
        assert q["zero"] == case["zero"], case
        assert q["codes"].tolist() == case["codes"], case


def _brute_force_code(x: Fraction, scale: Fraction, zero: int, qmax: int) -> int:
    best, best_err = None, None
    for q in range(qmax + 1):
        err = abs(x - scale * (q - zero))
        if best is None or err < best_err or (err == best_err and (q - zero) % 2 == 0):
            best, best_err = q, err
    return best


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_affine_quantizer_brute_force(bits):
    """Every code is the exact argmin over all 2^b codes of |x - s(q - z)|,
    ties to the even (q - z); zero is exactly representable; the extremes of a
    row that spans both signs land on codes 0 and 2^b - 1 (the grid is tight);
    every value inside the range is reproduced within s/2."""
    rng = np.random.default_rng(bits)
    qmax = 2**bits - 1
    for trial in range(60):
        n = int(rng.integers(1, 17))
        x = rng.standard_normal(n) * 10 ** rng.uniform(-3, 1)
        if trial % 7 == 0:
            x = np.abs(x)
        if trial % 11 == 0:
            x = -np.abs(x)
        q = oracle.affine_quantize_row(x, bits)
        scale, zero = Fraction(q["scale"]), q["zero"]
        assert 0 <= zero <= qmax
        for xi, ci in zip(x, q["codes"]):
            assert ci == _brute_force_code(Fraction(float(xi)), scale, zero, qmax)
            assert abs(Fraction(float(xi)) - scale * (ci - zero)) <= scale / 2 * (1 + 1e-12)
        if x.min() < 0 < x.max():
            assert q["codes"][int(np.argmin(x))] == 0
            assert q["codes"][int(np.argmax(x))] == qmax


# ---------------------------------------------------------------------------
# a1-a3: layer preparation (AQS + VMC)
# ---------------------------------------------------------------------------
def _small_layer(d, n, r, w_bits, sid, variant="mul", out_bits=8):
    spec = wl.LayerSpec("t", d, n, r, w_bits, variant, out_bits, stream_id=sid)
    return spec, wl.host_W(spec), wl.host_A(spec), wl.host_B(spec)


@pytest.mark.parametrize("w_bits", [4, 8])
def test_gen_aux_composition(w_bits):
    """sigma_W, sigma_R against numpy; R* = c R; each row is the pinned affine
    quantizer of W - R*; and the AQS reconstruction s(W_round - z) + R*
    reproduces W within s/2 (a wrong sign on R* would miss by ~2|R*|)."""
    spec, W, _, _ = _small_layer(24, 40, 4, w_bits, sid=3)
    g = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, w_bits, want_r_star=True)
    R = oracle.aux_R(24, 40, spec.seed, spec.stream_id)
    assert g["sigma_w"] == pytest.approx(float(np.std(W.astype(np.float64))), rel=1e-12)
    assert g["sigma_r"] == pytest.approx(float(np.std(R)), rel=1e-12)
    assert g["c"] == pytest.approx((g["sigma_w"] / g["sigma_r"]) ** spec.alpha, rel=1e-14)
    np.testing.assert_allclose(g["r_star"], g["c"] * R, rtol=1e-15, atol=0)
    for i in range(24):
        q = oracle.affine_quantize_row(W[i].astype(np.float64) - g["r_star"][i], w_bits)
        assert g["codes"][i].tolist() == q["codes"].tolist()
        assert g["s"][i] == q["scale"] and g["z"][i] == q["zero"]
    recon = g["s"][:, None] * (g["codes"] - g["z"][:, None]) + g["r_star"]
    assert np.all(np.abs(recon - W) <= g["s"][:, None] / 2 * (1 + 1e-9))


def test_gen_aux_row_subset_matches_full():
    spec, W, _, _ = _small_layer(20, 16, 4, 8, sid=1)
    full = oracle.gen_aux(W, 1, 1, 1.5, 8)
    part = oracle.gen_aux(W, 1, 1, 1.5, 8, row_begin=7, row_count=5)
    assert np.array_equal(full["codes"][7:12], part["codes"])
    assert np.array_equal(full["s"][7:12], part["s"])


# ---------------------------------------------------------------------------
# a4-a5: the MLA adaptation term
# ---------------------------------------------------------------------------
def _prepared(d, n, r, w_bits, sid):
    spec, W, A, B = _small_layer(d, n, r, w_bits, sid)
    g = oracle.gen_aux(W, spec.seed, sid, spec.alpha, w_bits, want_r_star=True)
    return spec, W, A, B, g


@pytest.mark.parametrize("w_bits,d,n,r", [(8, 16, 16, 4), (4, 12, 20, 3), (8, 9, 33, 16)])
def test_mla_identity(w_bits, d, n, r):
    """[s + (R* + AB)/D] * D = Q[W - R*] + R* + AB on D != 0 (AQS and MLA give
    the same pre-quantization weight), with AB from numpy and R* from the
    pinned sampler; U = s where D = 0."""
    spec, W, A, B, g = _prepared(d, n, r, w_bits, sid=2)
    s32 = g["s"].astype(np.float32)
    U, D = oracle.mla_rows(g["codes"], s32, g["z"], A, B, spec.seed, 2, g["sigma_w"],
                           g["sigma_r"], spec.alpha)
    AB = A.astype(np.float64) @ B.astype(np.float64)
    rhs = s32.astype(np.float64)[:, None] * D + g["r_star"] + AB
    nz = D != 0
    scale = np.abs(s32.astype(np.float64)[:, None] * D) + np.abs(g["r_star"]) + np.abs(AB)
    assert np.all(np.abs(U * D - rhs)[nz] <= 1e-13 * scale[nz])
    assert np.array_equal(U[~nz], np.broadcast_to(s32.astype(np.float64)[:, None], U.shape)[~nz])
    assert np.array_equal(D, g["codes"].astype(np.int64) - g["z"][:, None])


def test_mla_exact_rational_on_4x4():
    """The same identity term by term in exact rationals on a 4x4 layer: the
    oracle's fp64 U differs from the exact quotient by at most one rounding."""
    spec, W, A, B, g = _prepared(4, 4, 2, 8, sid=5)
    s32 = g["s"].astype(np.float32)
    U, D = oracle.mla_rows(g["codes"], s32, g["z"], A, B, spec.seed, 5, g["sigma_w"],
                           g["sigma_r"], spec.alpha)
    for i in range(4):
        for j in range(4):
            if D[i, j] == 0:
                continue
            ab = sum(Fraction(float(A[i, k])) * Fraction(float(B[k, j])) for k in range(2))
            exact = (Fraction(float(s32[i])) + (Fraction(float(g["r_star"][i, j])) + ab)
                     / int(D[i, j]))
            assert abs(Fraction(float(U[i, j])) - exact) <= abs(exact) * Fraction(1, 2**50)


# ---------------------------------------------------------------------------
# a6: IntLoRA_MUL
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w_bits,u_bits", [(8, 8), (4, 4)])
def test_merge_mul_composition(w_bits, u_bits):
    """U_round, s_bar, z_bar are the pinned affine quantizer applied to the
    pinned U row; P = (U_round - z_bar) * D in integer arithmetic."""
    spec, W, A, B, g = _prepared(10, 24, 4, w_bits, sid=7)
    s32 = g["s"].astype(np.float32)
    m = oracle.merge_mul(g["codes"], s32, g["z"], A, B, spec.seed, 7, g["sigma_w"], g["sigma_r"],
                         spec.alpha, u_bits)
    U, D = oracle.mla_rows(g["codes"], s32, g["z"], A, B, spec.seed, 7, g["sigma_w"],
                           g["sigma_r"], spec.alpha)
    for i in range(10):
        q = oracle.affine_quantize_row(U[i], u_bits)
        assert m["u_round"][i].tolist() == q["codes"].tolist()
        assert m["sbar"][i] == q["scale"] and m["zbar"][i] == q["zero"]
        want = [(int(a) - q["zero"]) * int(b) for a, b in zip(q["codes"], D[i])]
        assert m["P"][i].tolist() == want
    lim = (2**w_bits - 1) * (2**u_bits - 1)
    assert np.abs(m["P"]).max() <= lim


def test_merge_mul_ab_zero_special_case():
    """AB zero-initialised: W'_pre = Q[W - R*] + R*, and after MUL quantization
    |s_bar P - (Q[W-R*] + R*)| <= s_bar |D| / 2 on D != 0, P = 0 on D = 0."""
    spec, W, A, B, g = _prepared(12, 32, 4, 8, sid=11)
    s32 = g["s"].astype(np.float32).astype(np.float64)
    A0 = np.zeros_like(A)
    m = oracle.merge_mul(g["codes"], s32.astype(np.float32), g["z"], A0, B, spec.seed, 11,
                         g["sigma_w"], g["sigma_r"], spec.alpha, 8)
    D = g["codes"].astype(np.int64) - g["z"][:, None]
    target = s32[:, None] * D + g["r_star"]
    err = np.abs(m["sbar"][:, None] * m["P"] - target)
    nz = D != 0
    assert np.all(err[nz] <= (m["sbar"][:, None] * np.abs(D) / 2 * (1 + 1e-9))[nz])
    assert np.all(m["P"][~nz] == 0)


def test_merge_mul_bit_width_limit():
    """W' -> W + AB as the bit widths grow. At a fixed base width the MUL
    output converges to the MLA weight Q[W-R*] + R* + AB like 2^-b_U; growing
    the base width as well (with b_U = b_W + 12) drives it to W + AB."""
    spec, W, A, B = _small_layer(16, 48, 4, 8, sid=13)
    AB = A.astype(np.float64) @ B.astype(np.float64)
    errs_u = []
    g8 = oracle.gen_aux(W, spec.seed, 13, spec.alpha, 8, want_r_star=True)
    s8 = g8["s"].astype(np.float32)
    D8 = g8["codes"].astype(np.int64) - g8["z"][:, None]
    mla = s8.astype(np.float64)[:, None] * D8 + g8["r_star"] + AB
    for ub in (8, 12, 16, 20):
        m = oracle.merge_mul(g8["codes"], s8, g8["z"], A, B, spec.seed, 13, g8["sigma_w"],
                             g8["sigma_r"], spec.alpha, ub)
        nz = D8 != 0
        errs_u.append(np.linalg.norm((m["sbar"][:, None] * m["P"] - mla)[nz])
                      / np.linalg.norm(mla[nz]))
    for a, b in zip(errs_u, errs_u[1:]):
        assert b < a / 8          # 4 more bits: at least 8x smaller
    errs_w = []
    for wb in (4, 8, 12, 16):
        g = oracle.gen_aux(W, spec.seed, 13, spec.alpha, wb, want_r_star=True)
        s = g["s"].astype(np.float32)
        m = oracle.merge_mul(g["codes"], s, g["z"], A, B, spec.seed, 13, g["sigma_w"],
                             g["sigma_r"], spec.alpha, wb + 12)
        D = g["codes"].astype(np.int64) - g["z"][:, None]
        nz = D != 0
        target = W.astype(np.float64) + AB
        errs_w.append(np.linalg.norm((m["sbar"][:, None] * m["P"] - target)[nz])
                      / np.linalg.norm(target[nz]))
    for a, b in zip(errs_w, errs_w[1:]):
        assert b < a / 8
    assert errs_w[-1] < 1e-4


# ---------------------------------------------------------------------------
# a7: IntLoRA_SHIFT
# ---------------------------------------------------------------------------
def test_shift_quantizer_worked_examples():
    g = json.loads((GOLDEN / "shift_quantizer_worked.json").read_text())
    for case in g["cases"]:
        q = oracle.shift_quantize_row(case["U"], case["D"], case["bits"])
        assert q["sbar"] == case["sbar"], case
        assert q["shift"].tolist() == case["shift"], case
        assert q["M"].tolist() == case["M"], case


def _brute_force_shift(v: Fraction, kmax: int) -> int:
    """Nearest integer to -log2|v| by exact comparisons of v^2 with the
    half-integer powers 2^-(2k+1), clamped to [0, kmax]."""
    if v == 0:
        return kmax
    v2 = v * v
    k = 0
    while k < kmax and v2 <= Fraction(1, 2 ** (2 * k + 1)):
        k += 1
    return k


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_shift_quantizer_brute_force(bits):
    rng = np.random.default_rng(40 + bits)
    kmax = 2**bits - 1
    for _ in range(60):
        n = int(rng.integers(1, 17))
        U = rng.standard_normal(n) * np.exp(rng.uniform(-6, 0, n))
        D = rng.integers(-15, 16, n)
        if n > 2:
            U[0] = 0.0
        q = oracle.shift_quantize_row(U, D, bits)
        sbar = Fraction(float(np.max(np.abs(U)))) if np.any(U != 0) else Fraction(1)
        assert Fraction(q["sbar"]) == sbar
        for u, dv, k, m in zip(U, D, q["shift"], q["M"]):
            v = Fraction(float(u)) / sbar
            assert k == _brute_force_shift(v, kmax)
            sign = (v > 0) - (v < 0)
            assert m == sign * (int(dv) >> int(k))   # Python >> is a floor shift


def test_merge_shift_composition():
    spec, W, A, B, g = _prepared(10, 24, 8, 4, sid=17)
    s32 = g["s"].astype(np.float32)
    m = oracle.merge_shift(g["codes"], s32, g["z"], A, B, spec.seed, 17, g["sigma_w"],
                           g["sigma_r"], spec.alpha, 4)
    U, D = oracle.mla_rows(g["codes"], s32, g["z"], A, B, spec.seed, 17, g["sigma_w"],
                           g["sigma_r"], spec.alpha)
    for i in range(10):
        q = oracle.shift_quantize_row(U[i], D[i], 4)
        assert m["sbar"][i] == q["sbar"]
        assert m["shift"][i].tolist() == q["shift"].tolist()
        assert m["M"][i].tolist() == q["M"].tolist()
    assert np.abs(m["M"]).max() <= 15


# ---------------------------------------------------------------------------
# a8: STE backward
# ---------------------------------------------------------------------------
def test_ste_backward_against_numpy():
    spec = wl.LayerSpec("t", 19, 45, 6, 8, "mul", 8, stream_id=21)
    Gb = wl.host_G_bits(spec)
    Ab = wl.to_bf16_bits(wl.host_A(spec))
    Bb = wl.to_bf16_bits(wl.host_B(spec))
    G, A, B = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb))
    dA, dB = oracle.ste_backward(G, A, B)
    np.testing.assert_allclose(dA, G @ B.T, rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(dB, A.T @ G, rtol=1e-12, atol=1e-18)
    rows, cols = np.array([0, 5, 18]), np.array([0, 44, 7])
    sA, sB = oracle.ste_sampled(Gb, Ab, Bb, rows, cols)
    np.testing.assert_allclose(sA, dA[rows], rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(sB, dB[:, cols], rtol=1e-12, atol=1e-18)


# ---------------------------------------------------------------------------
# Integer inference GEMM on the merged weights (Y = X W'^T)
# ---------------------------------------------------------------------------
def test_int_planes_bounds():
    assert [oracle.int_planes(v) for v in (0, 127, 128, 16383, 16384, 2**21 - 1, 2**21)] == \
        [1, 1, 2, 2, 3, 3, 0]
    # merged-weight bounds: |P| <= (2^b_W - 1)(2^b_U - 1) (MUL), |M| <= 2^b_W - 1 (SHIFT)
    assert oracle.int_planes(15 * 15) == 2 and oracle.int_planes(255 * 255) == 3
    assert oracle.int_planes(15) == 1 and oracle.int_planes(255) == 2


@pytest.mark.parametrize("planes,lo,hi", [(1, -128, 127), (2, -16384, 16383)])
def test_int_digits_exhaustive(planes, lo, hi):
    """Every w in range: the digits rebuild w in base 128, lower digits lie in
    [0, 127] and the top digit in [-128, 127] (which makes them unique)."""
    w = np.arange(lo, hi + 1, dtype=np.int64).reshape(1, -1)
    dig, bad = oracle.int_digits(w, planes)
    assert bad == 0
    dig = dig[0].astype(np.int64)                     # [planes][n]
    rebuilt = sum(dig[k] * 128**k for k in range(planes))
    assert np.array_equal(rebuilt, w[0])
    for k in range(planes - 1):
        assert dig[k].min() >= 0 and dig[k].max() <= 127


def test_int_digits_three_planes_and_overflow():
    rng = np.random.default_rng(5)
    w = np.concatenate([rng.integers(-2**21, 2**21, 4000), [-2**21, 2**21 - 1, 0, -1, 127, -128]])
    dig, bad = oracle.int_digits(w.reshape(2, -1), 3)
    assert bad == 0
    d = dig.astype(np.int64)
    assert np.array_equal(d[:, 0] + 128 * d[:, 1] + 16384 * d[:, 2], w.reshape(2, -1))
    for planes, out in ((1, [128, -129, 5]), (2, [16384, -16385, 3])):
        _, bad = oracle.int_digits(np.array([out], np.int64), planes)
        assert bad == 2


def test_int_gemm_brute_force_tiny():
    rng = np.random.default_rng(8)
    X = rng.integers(-128, 128, (3, 5)).astype(np.int8)
    W = rng.integers(-300, 300, (4, 5))
    xs, ws = rng.uniform(0.01, 1, 3), rng.uniform(0.01, 1, 4)
    Y = oracle.int_gemm_rows(X, xs, W, ws)
    for t in range(3):
        for i in range(4):
            acc = sum(int(X[t, j]) * int(W[i, j]) for j in range(5))
            assert Y[t, i] == acc * xs[t] * ws[i]
    np.testing.assert_array_equal(oracle.int_gemm_rows(X, xs, W, ws, rows=[2, 0]), Y[[2, 0]])


def test_int_gemm_is_the_dequantized_matmul_of_merged_weights():
    """Y equals numpy's fp64 matmul of the dequantized activations with the
    merged weight W' = s_bar P of an oracle MUL merge, and equals the sum of
    the digit-plane products scaled by 128^k."""
    spec, W, A, B, g = _prepared(12, 40, 4, 4, sid=3)
    s32 = g["s"].astype(np.float32)
    m = oracle.merge_mul(g["codes"], s32, g["z"], A, B, spec.seed, 3, g["sigma_w"], g["sigma_r"],
                         spec.alpha, 4)
    P, sbar = m["P"], m["sbar"]
    rng = np.random.default_rng(4)
    X = rng.integers(-127, 128, (7, 40)).astype(np.int8)
    xs = rng.uniform(1e-3, 1e-2, 7)
    Y = oracle.int_gemm_rows(X, xs, P, sbar)
    Wm = sbar[:, None] * P
    np.testing.assert_allclose(Y, (xs[:, None] * X) @ Wm.T, rtol=1e-12, atol=1e-300)
    planes = oracle.int_planes(int(np.abs(P).max()))
    dig, bad = oracle.int_digits(P, planes)
    assert bad == 0
    acc = sum(128**k * (X.astype(np.int64) @ dig[:, k, :].astype(np.int64).T) for k in range(planes))
    np.testing.assert_allclose(Y, acc * xs[:, None] * sbar[None, :], rtol=1e-15, atol=0)


def test_row_views_equal_whole_layer_functions():
    """quantize_rows / merge_mul_rows (rows given alone, c given) reproduce the
    pinned whole-layer functions on a slice of rows, flat index included."""
    spec, W, A, B, g = _prepared(21, 36, 4, 4, sid=13)
    rows = slice(7, 15)
    q = oracle.quantize_rows(W[rows], spec.seed, 13, g["c"], 4, 7)
    for k in ("codes", "s", "z", "pre", "zpre"):
        np.testing.assert_array_equal(q[k], g[k][rows])
    s32 = g["s"].astype(np.float32)
    m = oracle.merge_mul(g["codes"], s32, g["z"], A, B, spec.seed, 13, g["sigma_w"], g["sigma_r"],
                         spec.alpha, 4)
    mr = oracle.merge_mul_rows(g["codes"][rows], s32[rows], g["z"][rows], A[rows], B, spec.seed,
                               13, g["c"], 4, 7)
    for k in ("u_round", "sbar", "zbar", "P", "pre", "zpre"):
        np.testing.assert_array_equal(mr[k], m[k][rows])


def test_results_do_not_depend_on_the_thread_count():
    """One host thread and all of them give the same bits: the statistics add
    row sums in row order and every parallel loop writes its own outputs (the
    benchmark's single-core figure relies on this)."""
    spec, W, A, B, g = _prepared(37, 52, 8, 8, sid=17)
    s32 = g["s"].astype(np.float32)
    many = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        assert oracle.num_threads() == 1
        g1 = oracle.gen_aux(W, spec.seed, 17, spec.alpha, 8)
        m1 = oracle.merge_mul(g1["codes"], g1["s"].astype(np.float32), g1["z"], A, B, spec.seed, 17,
                              g1["sigma_w"], g1["sigma_r"], spec.alpha, 8)
    finally:
        oracle.set_num_threads(many)
    assert oracle.num_threads() == many
    m = oracle.merge_mul(g["codes"], s32, g["z"], A, B, spec.seed, 17, g["sigma_w"], g["sigma_r"],
                         spec.alpha, 8)
    assert g1["sigma_w"] == g["sigma_w"] and g1["sigma_r"] == g["sigma_r"]
    for k in ("codes", "s", "z"):
        np.testing.assert_array_equal(g1[k], g[k])
    for k in ("u_round", "sbar", "zbar", "P"):
        np.testing.assert_array_equal(m1[k], m[k])


# ---------------------------------------------------------------------------
# auxiliary laws of the ablation: Gaussian, Cauchy, Student-t (2 dof)
# ---------------------------------------------------------------------------
def _law_sample(dist):
    return oracle.aux_R(1024, 1024, 1, 3, dist=dist).ravel()


def _frac_close(frac, p, n, z=4.5):
    return abs(frac - p) <= z * math.sqrt(p * (1 - p) / n)


def test_gaussian_law_moments_and_tails():
    x = _law_sample(oracle.GAUSSIAN)
    n = x.size
    assert abs(x.mean()) < 4.5 / math.sqrt(n)
    assert abs(x.var() - 1.0) < 4.5 * math.sqrt(2.0 / n)
    k = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert abs(k - 3.0) < 4.5 * math.sqrt(24.0 / n)
    for t in (0.5, 1.0, 1.96, 3.0):      # P(|Z| > t) = erfc(t / sqrt 2)
        assert _frac_close(np.mean(np.abs(x) > t), math.erfc(t / math.sqrt(2.0)), n)
    # Box-Muller pairs: words 2p and 2p+1 share the radius, so the pair's
    # squared norm is -2 ln u of word 2p, independent of the angle word
    pairs = x.reshape(-1, 2)
    r2 = (pairs ** 2).sum(axis=1)
    assert abs(np.mean(r2) - 2.0) < 4.5 * 2.0 / math.sqrt(r2.size)   # chi-square(2): mean 2, sd 2
    assert _frac_close(np.mean(r2 > 2.0), math.exp(-1.0), r2.size)   # P(chi2_2 > t) = e^(-t/2)


def test_cauchy_law_cdf_and_symmetry():
    x = _law_sample(oracle.CAUCHY)
    n = x.size
    for t in (-10.0, -1.0, -0.25, 0.0, 0.5, 1.0, 3.0, 50.0):   # F(t) = 1/2 + atan(t) / pi
        assert _frac_close(np.mean(x <= t), 0.5 + math.atan(t) / math.pi, n)
    assert _frac_close(np.mean(np.abs(x) < 1.0), 0.5, n)         # quartiles at -1, +1


def test_student_t2_law_cdf():
    x = _law_sample(oracle.STUDENT_T2)
    n = x.size
    for t in (-5.0, -2.0, -0.5, 0.0, 1.0, 3.0, 20.0):   # F(t) = 1/2 + t / (2 sqrt(2 + t^2))
        assert _frac_close(np.mean(x <= t), 0.5 + t / (2.0 * math.sqrt(2.0 + t * t)), n)


def test_laws_share_the_laplace_stream_and_layout():
    """Law 0 is the pinned Laplace sampler; every law reads element e from
    block e / 4 (a different element of the same block changes the value)."""
    np.testing.assert_array_equal(oracle.aux_R(3, 8, 1, 5, dist=oracle.LAPLACE),
                                  oracle.aux_R(3, 8, 1, 5))
    for dist in (oracle.GAUSSIAN, oracle.CAUCHY, oracle.STUDENT_T2):
        a = oracle.aux_R(3, 8, 1, 5, dist=dist)
        assert np.all(np.isfinite(a))
        assert [oracle.aux_value(1, 5, e, dist) for e in range(24)] == a.ravel().tolist()


@pytest.mark.parametrize("dist", [1, 2, 3])
def test_gen_aux_and_merge_compose_under_other_laws(dist):
    """sigma_R is the population std of the law's R; the base quantization and
    the MUL merge use c = (sigma_W / sigma_R)^alpha and R of that law."""
    spec, W, A, B = _small_layer(10, 24, 4, 4, 19)
    g = oracle.gen_aux(W, spec.seed, 19, spec.alpha, 4, want_r_star=True, dist=dist)
    R = oracle.aux_R(10, 24, spec.seed, 19, dist=dist)
    assert abs(g["sigma_r"] - np.std(R)) <= 1e-12 * np.std(R)
    assert abs(g["sigma_r"] - oracle.sigma_r(10, 24, spec.seed, 19, dist=dist)) <= 1e-12 * g["sigma_r"]
    c = oracle.vmc_scale(np.std(W.astype(np.float64)), np.std(R), spec.alpha)
    np.testing.assert_allclose(g["r_star"], c * R, rtol=1e-12)
    for i in range(10):
        q = oracle.affine_quantize_row(W[i].astype(np.float64) - g["r_star"][i], 4)
        assert g["codes"][i].tolist() == q["codes"].tolist()
    s32 = g["s"].astype(np.float32)
    U, D = oracle.mla_rows(g["codes"], s32, g["z"], A, B, spec.seed, 19, g["sigma_w"], g["sigma_r"],
                           spec.alpha, dist=dist)
    AB = A.astype(np.float64) @ B.astype(np.float64)
    nz = D != 0
    np.testing.assert_allclose((U * D)[nz], (s32.astype(np.float64)[:, None] * D + g["r_star"] + AB)[nz],
                               rtol=1e-11, atol=1e-14)


def test_ste_masked_pins():
    """The masked STE is the plain one on G (.) [W_round != z]: all-kept
    equals the plain STE, all-masked gives zero, and a random mask equals
    numpy's matmul of the masked gradient; the sampled form agrees."""
    spec = wl.LayerSpec("t", 11, 24, 4, 4, "mul", 4, stream_id=23)
    Gb = wl.host_G_bits(spec)
    Ab = wl.to_bf16_bits(wl.host_A(spec))
    Bb = wl.to_bf16_bits(wl.host_B(spec))
    G, A, B = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb))
    rng = np.random.default_rng(31)
    codes = rng.integers(0, 16, (11, 24))
    z = rng.integers(0, 16, 11)
    never = np.broadcast_to((z[:, None] + 1) % 16, (11, 24))        # never equal to z
    for a, b in zip(oracle.ste_backward_masked(G, A, B, never, z), oracle.ste_backward(G, A, B)):
        np.testing.assert_array_equal(a, b)
    dA0, dB0 = oracle.ste_backward_masked(G, A, B, np.repeat(z[:, None], 24, axis=1), z)
    assert not dA0.any() and not dB0.any()
    M = (codes != z[:, None]).astype(np.float64)
    dA, dB = oracle.ste_backward_masked(G, A, B, codes, z)
    np.testing.assert_allclose(dA, (G * M) @ B.T, rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(dB, A.T @ (G * M), rtol=1e-12, atol=1e-18)
    rows, cols = np.array([0, 4, 10]), np.array([1, 23])
    sA, sB = oracle.ste_sampled_masked(Gb, Ab, Bb, codes, z, rows, cols)
    np.testing.assert_allclose(sA, dA[rows], rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(sB, dB[:, cols], rtol=1e-12, atol=1e-18)


# ---------------------------------------------------------------------------
# training forward: fake-quantized bf16 merged weight and the layer GEMM
# ---------------------------------------------------------------------------
def _bf16_nearest_even(x32):
    """bf16 pattern of an fp32 value by exact comparison with its two bf16
    neighbours (ties to the even pattern)."""
    bits = int(np.float32(x32).view(np.uint32))
    lo = bits >> 16
    hi = lo + 1
    val = Fraction(float(np.float32(x32)))
    f = lambda p: Fraction(float(np.array([p << 16], np.uint32).view(np.float32)[0]))
    dl, dh = abs(val - f(lo)), abs(f(hi) - val)
    if dl < dh or (dl == dh and lo % 2 == 0):
        return lo
    return hi


def test_fakequant_bf16_rounding_brute_force():
    rng = np.random.default_rng(17)
    Q = rng.integers(-65025, 65026, (6, 40))
    sbar = rng.uniform(1e-5, 1e-2, 6).astype(np.float32)
    Q[0, :3] = [0, 1, -1]
    got = oracle.fakequant_bf16(Q, sbar)
    for i in range(6):
        for j in range(40):
            prod = np.float32(sbar[i]) * np.float32(Q[i, j])      # one fp32 rounding
            assert got[i, j] == _bf16_nearest_even(prod)
    # exact ties: 1 + 2^-8 (+ 2^-7) sit halfway between bf16 neighbours
    ties = oracle.fakequant_bf16(np.array([[257, 259]]), np.array([2.0**-8], np.float32))
    assert ties.tolist() == [[0x3F80, 0x3F82]]


def test_linear_rows_brute_force_and_numpy():
    rng = np.random.default_rng(18)
    X = wl.to_bf16_bits(rng.standard_normal((3, 16)).astype(np.float32))
    W = wl.to_bf16_bits(rng.standard_normal((5, 16)).astype(np.float32))
    Y = oracle.linear_rows(X, W)
    xf, wf = wl.bf16_bits_to_f32(X).astype(np.float64), wl.bf16_bits_to_f32(W).astype(np.float64)
    for t in range(3):
        for i in range(5):
            assert abs(Y[t, i] - sum(float(xf[t, j]) * float(wf[i, j]) for j in range(16))) < 1e-12
    np.testing.assert_allclose(Y, xf @ wf.T, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(oracle.linear_rows(X, W, rows=[2]), Y[[2]])


def test_train_backward_brute_force_and_reassociation():
    """G = dY^T X, dX = dY W', dA = G B^T, dB = A^T G: brute force on a tiny
    case, and the low-rank reassociation dA = dY^T (X B^T), dB = (dY A)^T X
    that a fused backward would use holds to rounding."""
    rng = np.random.default_rng(44)
    T, d, n, r = 3, 4, 5, 2
    bits = lambda *shape: wl.to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    Xb, dYb, Wb, Ab, Bb = bits(T, n), bits(T, d), bits(d, n), bits(d, r), bits(r, n)
    o = oracle.train_backward(Xb, dYb, Wb, Ab, Bb)
    X, dY, W, A, B = (wl.bf16_bits_to_f32(b).astype(np.float64) for b in (Xb, dYb, Wb, Ab, Bb))
    for i in range(d):
        for j in range(n):
            assert abs(o["G"][i, j] - sum(dY[t, i] * X[t, j] for t in range(T))) < 1e-12
    for t in range(T):
        for j in range(n):
            assert abs(o["dX"][t, j] - sum(dY[t, i] * W[i, j] for i in range(d))) < 1e-12
    np.testing.assert_allclose(o["dA"], dY.T @ (X @ B.T), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(o["dB"], (dY @ A).T @ X, rtol=1e-12, atol=1e-14)
