"""Pins for the CPU oracle: things other than the oracle itself fix its output.

  * the hand-worked 4x16 example (tests/golden/hand_4x16.json), re-derived here
    with exact rational arithmetic;
  * the definition of correct rounding, checked on the exact mean;
  * brute force with exact rationals on tiny shapes;
  * closed forms and invariants (code range, |q| <= 127, zero fractions of
    Gaussian / Laplace weights, scale invariance, identity weights);
  * planted mistakes: plausible bugs put into the oracle must fail a pin.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from bit_ternary_b200 import workloads as WL

F32_MAX = Fraction(np.finfo(np.float32).max.item())


# --------------------------------------------------------------------------
# helpers written from definitions (independent of the oracle's own code)
# --------------------------------------------------------------------------
def exact(v) -> Fraction:
    return Fraction(float(v))


def f32_neighbours(r: np.float32):
    lo = np.nextafter(r, np.float32(-np.inf), dtype=np.float32)
    hi = np.nextafter(r, np.float32(np.inf), dtype=np.float32)
    return lo, hi


def is_correctly_rounded(r: np.float32, true: Fraction) -> bool:
    """r is an fp32 nearest to `true`; on a tie its significand is even."""
    d = abs(exact(r) - true)
    for nb in f32_neighbours(np.float32(r)):
        if not np.isfinite(nb):
            continue
        dn = abs(exact(nb) - true)
        if dn < d:
            return False
        if dn == d and (int(np.float32(r).view(np.uint32)) & 1):
            return False
    return True


def rn_f32(true: Fraction) -> np.float32:
    """Nearest fp32 by search over candidates around float(true).

    float(Fraction) is the nearest double; the nearest fp32 is one of the few
    fp32 values next to np.float32 of that double. Pick by exact distance,
    ties to even significand.
    """
    c = np.float32(float(true))
    cands = {c, *f32_neighbours(c)}
    best = None
    for v in cands:
        if not np.isfinite(v):
            continue
        key = (abs(exact(v) - true), int(np.float32(v).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return np.float32(best[1])


def exact_mean_abs(W: np.ndarray) -> Fraction:
    total = Fraction(0)
    # sum via integer numerators over a common power-of-two denominator
    acc = 0
    for v in np.abs(W.astype(np.float64)).ravel():
        num, den = float(v).as_integer_ratio()
        acc += num * ((1 << 149) // den)
    total = Fraction(acc, 1 << 149)
    return total / W.size


def load_golden(golden_dir):
    with open(os.path.join(golden_dir, "hand_4x16.json")) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# the hand-worked example
# --------------------------------------------------------------------------
def test_golden_hand_example_oracle(golden_dir):
    g = load_golden(golden_dir)
    W = np.array(g["W"], np.float32)
    x = np.array(g["x"], np.float32)
    mean = O.absmean_exact(W)
    assert mean == np.float32(g["mean"])
    codes, mean_c = O.weight_quant(W)
    assert np.array_equal(codes, np.array(g["codes"], np.int8))
    assert (codes == 0).mean() == g["zero_fraction"]
    packed, D = O.pack_weights(W)
    assert [hex(int(v)) for v in packed[:, 0]] == g["packed_hex"]
    assert D.shape == (4, 1) and np.all(D == np.float32(g["mean"]))
    q, s_x = O.act_quant(x)
    assert np.array_equal(q, np.array(g["q"], np.int8))
    assert np.array_equal(s_x, np.array(g["s_x"], np.float32))
    y, parts = O.bitlinear_forward(x, packed, D, 16, return_parts=True)
    assert np.array_equal(parts["acc"], np.array(g["acc"]))
    got = [[hex(int(v)) for v in row] for row in y.view(np.uint32)]
    assert got == g["y_hex"]


def test_golden_hand_example_exact_rationals(golden_dir):
    """Re-derive the fixture from the formulas with Fractions only."""
    g = load_golden(golden_dir)
    W = [[Fraction(v) for v in row] for row in g["W"]]
    x = [[Fraction(v) for v in row] for row in g["x"]]
    mean = sum(abs(v) for row in W for v in row) / 64
    assert mean == Fraction(1, 4)
    s = 1 / mean  # exactly 4

    def rint_half_even(v: Fraction) -> int:
        f = math.floor(v)
        r = v - f
        if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2 == 1):
            return f + 1
        return f

    codes = [[max(-1, min(1, rint_half_even(v * s))) for v in row] for row in W]
    assert codes == g["codes"]
    words = [sum((c + 1) << (2 * k) for k, c in enumerate(row)) for row in codes]
    assert [hex(w) for w in words] == g["packed_hex"]
    # ActQuant: s_x = 127 / max|x| (exact for these tokens), q = rint(x*s_x)
    q = []
    for row in x:
        sx = Fraction(127) / max(abs(v) for v in row)
        q.append([max(-128, min(127, rint_half_even(v * sx))) for v in row])
    assert q == g["q"]
    acc = [[sum(a * b for a, b in zip(qr, cr)) for cr in codes] for qr in q]
    assert acc == g["acc"]
    sxs = [Fraction(v) for v in g["s_x"]]
    for m in range(2):
        for n in range(4):
            t = rn_f32(Fraction(acc[m][n]) / sxs[m])
            y = rn_f32(exact(t) * mean)
            assert hex(int(np.float32(y).view(np.uint32))) == g["y_hex"][m][n]


# --------------------------------------------------------------------------
# exact mean, correct rounding
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_absmean_is_correctly_rounded(seed):
    rng = np.random.default_rng(seed)
    n = [7, 64, 1000, 4096, 20000, 3][seed]
    kind = seed % 3
    if kind == 0:
        W = rng.standard_normal(n).astype(np.float32) * np.float32(0.02)
    elif kind == 1:  # wide dynamic range, including subnormals and zeros
        W = (rng.standard_normal(n) * 2.0 ** rng.integers(-140, 60, n)).astype(np.float32)
        W[::5] = 0.0
    else:
        W = rng.laplace(0, 0.02, n).astype(np.float32)
    got = O.absmean_exact(W)
    assert is_correctly_rounded(got, exact_mean_abs(W))


def test_absmean_large_vs_bigint():
    """10^6 elements: the oracle mean equals the big-int reference exactly."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal(1_000_000) * 0.02).astype(np.float32)
    ref = rn_f32(exact_mean_abs(W))
    assert O.absmean_exact(W) == ref


def test_round_fraction_matches_single_rounding_of_doubles():
    """For a value that is exactly a double, fp32 conversion of that double is a
    single correctly rounded step (numpy), so both must agree bit for bit."""
    rng = np.random.default_rng(5)
    vals = np.abs(rng.standard_normal(3000) * 2.0 ** rng.integers(-149, 120, 3000))
    # include exact ties: fp32 midpoints
    mids = []
    for v in rng.standard_normal(200).astype(np.float32):
        v = np.abs(v)
        nx = np.nextafter(v, np.float32(np.inf))
        mids.append((float(v) + float(nx)) / 2.0)
    for d in list(vals) + mids:
        assert O.round_fraction_to_f32(Fraction(float(d))) == np.float32(d)


def test_absmean_rejects_nonfinite():
    W = np.ones((2, 16), np.float32)
    W[1, 3] = np.inf
    with pytest.raises(FloatingPointError):
        O.absmean_exact(W)


# --------------------------------------------------------------------------
# brute force with exact rationals on tiny shapes
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(8))
def test_bruteforce_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(1, 5))
    K = 16 * int(rng.integers(1, 3))
    M = int(rng.integers(1, 4))
    # multiples of 2^-8 keep every product exact
    W = (rng.integers(-40, 41, (N, K)) / 256.0).astype(np.float32)
    x = (rng.integers(-300, 301, (M, K)) / 256.0).astype(np.float32)
    if seed == 0:
        x[0] = 0.0  # all-zero token: floor path
    packed, D = O.pack_weights(W)
    y, parts = O.bitlinear_forward(x, packed, D, K, return_parts=True)

    # exact mean and its rounding
    mean = Fraction(int(np.abs(W * 256).sum().round()), 256 * W.size)
    mean_f = max(rn_f32(mean), O.FLOOR)
    assert D[0, 0] == mean_f
    s = rn_f32(1 / exact(mean_f))
    codes = np.array([[max(-1, min(1, round_half_even(rn_f32(exact(w) * exact(s)))))
                       for w in row] for row in W], np.int8)
    assert np.array_equal(parts["codes"], codes)
    for m in range(M):
        amax = max(abs(exact(v)) for v in x[m])
        mx = max(rn_f32(amax), O.FLOOR)
        sx = rn_f32(Fraction(127) / exact(mx))
        assert parts["s_x"][m] == sx
        qrow = [max(-128, min(127, round_half_even(rn_f32(exact(v) * exact(sx))))) for v in x[m]]
        assert list(parts["q"][m]) == qrow
        for n in range(N):
            acc = sum(int(a) * int(b) for a, b in zip(qrow, codes[n]))
            assert parts["acc"][m, n] == acc
            t = rn_f32(Fraction(acc) / exact(sx))
            yv = rn_f32(exact(t) * exact(mean_f))
            assert y[m, n].view(np.uint32) == np.float32(yv).view(np.uint32)


def round_half_even(v) -> int:
    v = Fraction(float(v)) if not isinstance(v, Fraction) else v
    f = math.floor(v)
    r = v - f
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2 == 1):
        return f + 1
    return f


# --------------------------------------------------------------------------
# invariants and closed forms on workload-shaped inputs
# --------------------------------------------------------------------------
def test_zero_fraction_gaussian_and_laplace():
    """Closed forms: P(|z| < 0.5*E|z|) for the two weight laws.

    Gaussian: E|z| = sigma*sqrt(2/pi), so P = erf(0.5*sqrt(2/pi)/sqrt(2)) ~ 0.3101.
    Laplace(b): E|z| = b, P(|z| < b/2) = 1 - exp(-1/2) ~ 0.3935.
    """
    Wn = WL.weight(2560, 2560, "normal", 1000)
    Wl = WL.weight(2560, 2560, "laplace", 1003)
    cn, _ = O.weight_quant(Wn)
    cl, _ = O.weight_quant(Wl)
    pn = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    pl = 1 - math.exp(-0.5)
    assert abs((cn == 0).mean() - pn) < 0.002
    assert abs((cl == 0).mean() - pl) < 0.002
    assert set(np.unique(cn)) <= {-1, 0, 1}
    # packed fields never hold 3
    packed = O.pack_codes(cn)
    f = (packed.astype(np.int64)[..., None] >> (2 * np.arange(16))) & 3
    assert not np.any(f == 3)


def test_pack_roundtrip_and_layout():
    rng = np.random.default_rng(3)
    codes = rng.integers(-1, 2, (5, 48)).astype(np.int8)
    p = O.pack_codes(codes)
    assert p.shape == (5, 3) and p.dtype == np.uint32
    assert np.array_equal(O.unpack_codes(p, 48), codes)
    # column k of row n lives in word k//16, bits 2*(k%16)
    for n in range(5):
        for k in range(48):
            fld = (int(p[n, k // 16]) >> (2 * (k % 16))) & 3
            assert fld == codes[n, k] + 1


def test_actquant_invariants():
    x = WL.activations(64, 6912, "student_t", 1001, meta={"df": 3.0})
    q, s_x = O.act_quant(x)
    assert q.min() >= -127 and q.max() <= 127  # -128 unreachable
    for m in range(x.shape[0]):
        k = int(np.argmax(np.abs(x[m])))
        assert abs(int(q[m, k])) == 127
        assert np.sign(q[m, k]) == np.sign(x[m, k])


def test_scale_invariance_powers_of_two():
    W = WL.weight(64, 256, "normal", 7)
    x = WL.activations(4, 256, "normal", 7)
    c0, m0 = O.weight_quant(W)
    q0, s0 = O.act_quant(x)
    for j in (-7, -1, 3, 9):
        c1, m1 = O.weight_quant(W * np.float32(2.0 ** j))
        assert np.array_equal(c0, c1) and m1 == m0 * np.float32(2.0 ** j)
        q1, s1 = O.act_quant(x * np.float32(2.0 ** j))
        assert np.array_equal(q0, q1)


def test_constant_magnitude_weights():
    a = np.float32(0.0371)
    rng = np.random.default_rng(1)
    W = (np.where(rng.random((8, 64)) < 0.5, -1, 1) * a).astype(np.float32)
    codes, mean_c = O.weight_quant(W)
    assert mean_c == a
    assert np.array_equal(codes, np.sign(W).astype(np.int8))


def test_identity_weights_give_dequantised_x():
    """W = a*I: codes = I, so y = dequant(x) * D (a textbook reduction)."""
    K = 32
    W = (np.eye(K) * 0.5).astype(np.float32)
    x = WL.activations(3, K, "normal", 2)
    packed, D = O.pack_weights(W)
    assert np.array_equal(O.unpack_codes(packed, K), np.eye(K, dtype=np.int8))
    y, parts = O.bitlinear_forward(x, packed, D, K, return_parts=True)
    q, s_x = parts["q"], parts["s_x"]
    expect = ((q.astype(np.float32) / s_x[:, None]).astype(np.float32) * D[0, 0]).astype(np.float32)
    assert np.array_equal(y, expect)
    assert D[0, 0] == np.float32(0.5 / K)


def test_onehot_token():
    """x = v*e_k: q = sign(v)*127 at k, so acc[n] = sign(v)*127*code[n,k]."""
    W = WL.weight(16, 64, "normal", 9)
    packed, D = O.pack_weights(W)
    codes = O.unpack_codes(packed, 64)
    x = np.zeros((1, 64), np.float32)
    x[0, 5] = np.float32(-3.25)
    _, parts = O.bitlinear_forward(x, packed, D, 64, return_parts=True)
    assert np.array_equal(parts["acc"][0], -127 * codes[:, 5].astype(np.int64))


def test_acc_bound_and_fake_quant_agreement():
    """|acc| <= 127 * nnz(row); y equals the literal fake-quant F.linear up to
    fp32 rounding (BitVLA page §2's 'exactly' claim)."""
    W = WL.weight(96, 1152, "normal", 1002)
    x = WL.activations(8, 1152, "outlier_channels", 1002, meta={"frac": 0.01, "scale": 20.0})
    packed, D = O.pack_weights(W)
    y, parts = O.bitlinear_forward(x, packed, D, 1152, return_parts=True)
    nnz = (parts["codes"] != 0).sum(axis=1)
    assert np.all(np.abs(parts["acc"]) <= 127 * nnz[None, :])
    ref = O.fake_quant_linear(x, W)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 1e-6


def test_shape_errors():
    with pytest.raises(ValueError):
        O.pack_codes(np.zeros((2, 20), np.int8))
    with pytest.raises(ValueError):
        O.absmean_exact(np.zeros((0, 16), np.float32))


# --------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# --------------------------------------------------------------------------
PLANTS = {
    "round_half_away_from_zero": lambda mp: mp.setattr(
        O.bitlinear_oracle.np, "rint",
        lambda a: np.sign(a) * np.floor(np.abs(a) + 0.5)),
    "msb_first_pack": lambda mp: mp.setattr(
        O.bitlinear_oracle, "pack_codes",
        lambda c: np.sum(((c.astype(np.int64) + 1).reshape(c.shape[0], -1, 16))
                         << (30 - 2 * np.arange(16)), axis=2).astype(np.uint32)),
    "mean_not_abs": lambda mp: mp.setattr(
        O.bitlinear_oracle, "absmean_exact",
        lambda W: np.float32(np.mean(W, dtype=np.float64))),
    "reciprocal_scale_order": lambda mp: mp.setattr(
        O.bitlinear_oracle, "rescale",
        lambda acc, s_x, D: ((acc.astype(np.float32) * (np.float32(1) / s_x)[:, None]).astype(np.float32)
                             * D.reshape(1, -1)).astype(np.float32)),
    "codes_read_as_k_by_n": lambda mp: mp.setattr(
        O.bitlinear_oracle, "int_matmul",
        lambda q, c: q.astype(np.int64) @ c.astype(np.int64).reshape(q.shape[1], -1)),
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_planted_mistake_is_caught(plant, monkeypatch, golden_dir):
    PLANTS[plant](monkeypatch)
    with pytest.raises(AssertionError):
        test_golden_hand_example_oracle(golden_dir)


# ------------------------------------------------------------- bf16 inputs
BF16_KNOWN = {  # bit pattern -> value (bf16 = sign, 8 exponent bits, 7 fraction bits)
    0x3F80: 1.0, 0xC000: -2.0, 0x3E80: 0.25, 0x4049: 3.140625, 0x0001: 2.0 ** -133,
    0x0080: 2.0 ** -126, 0x7F7F: (2.0 - 2.0 ** -7) * 2.0 ** 127, 0x8000: -0.0,
    0x7F80: float("inf"), 0xFF80: float("-inf"),
}


def test_bf16_widening_known_values():
    bits = np.array(sorted(BF16_KNOWN), dtype=np.uint16)
    got = O.bf16_to_f32(bits)
    want = np.array([BF16_KNOWN[int(b)] for b in bits], dtype=np.float64)
    assert got.dtype == np.float32
    assert np.array_equal(got.astype(np.float64), want)
    assert np.signbit(got[bits.tolist().index(0x8000)])


def test_bf16_widening_matches_library_on_every_pattern():
    torch = pytest.importorskip("torch")
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_to_f32(bits)
    lib = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), lib[~nan].view(np.uint32))


def test_bf16_round_trip_of_fp32_with_empty_low_half():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(1000).astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    assert np.array_equal(O.bf16_to_f32((v.view(np.uint32) >> 16).astype(np.uint16)), v)


def test_bf16_widening_planted_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(O, "bf16_to_f32", lambda b: np.asarray(b, np.uint16).view(np.float16).astype(np.float32))
    with pytest.raises(AssertionError):
        test_bf16_widening_known_values()


# ------------------------------------------------------- RMSNorm + ActQuant
def _rms_ref64(x, g, eps):
    """fp64 RMSNorm from torch's own routine (a library reference)."""
    torch = pytest.importorskip("torch")
    xt = torch.from_numpy(x.astype(np.float64))
    gt = torch.from_numpy(g.astype(np.float64))
    return torch.nn.functional.rms_norm(xt, (x.shape[1],), gt, float(eps)).numpy()


def test_rmsnorm_matches_library_fp64_within_rounding():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal((6, 1024)), 20 * rng.standard_t(3, (2, 1024))]).astype(np.float32)
    x[1] *= np.float32(1e-3)
    g = rng.uniform(0.5, 2.0, 1024).astype(np.float32)
    n = O.rmsnorm(x, g)
    ref = _rms_ref64(x, g, O.RMS_EPS)
    ulp = np.spacing(np.abs(n).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(n.astype(np.float64) - ref) <= 4 * ulp)


def test_mean_square_exact_brute_force_rational():
    from fractions import Fraction
    rng = np.random.default_rng(12)
    for K in (16, 48, 96):
        for scale in (1.0, 1e-20, 1e18, 1e-42):
            row = (rng.standard_normal(K) * scale).astype(np.float32)
            want = O.round_fraction_to_f32(sum(Fraction(float(v)) ** 2 for v in row) / K)
            assert O.mean_square_exact(row) == want


def test_mean_square_exact_tie_rounds_to_even():
    a = np.float32(1 + 2.0 ** -12)  # a^2 = 1 + 2^-11 + 2^-24: halfway between two fp32 neighbours
    assert O.mean_square_exact(np.full(32, a, np.float32)) == np.float32(1 + 2.0 ** -11)
    # b^2 = 1 + 4098.5*2^-23 + 2^-34 + 2^-46: a hair above a midpoint, so it rounds up to 4099
    b = np.float32(1 + 2.0 ** -12 + 2.0 ** -23)
    assert O.mean_square_exact(np.full(16, b, np.float32)) == np.float32(1 + 4099 * 2.0 ** -23)
    c = np.float32(1 + 3 * 2.0 ** -12)  # c^2 = 1 + 12292.5*2^-23 exactly: a tie, to the even 12292
    assert O.mean_square_exact(np.full(16, c, np.float32)) == np.float32(1 + 12292 * 2.0 ** -23)


def _sqrt_rn_f32(v: Fraction) -> np.float32:
    """Nearest fp32 to sqrt(v), decided by exact squares of the midpoints
    between neighbouring fp32 values (sqrt of an fp32 is never a midpoint)."""
    c = np.float32(math.sqrt(float(v)))
    cands = sorted({np.nextafter(np.nextafter(c, np.float32(0)), np.float32(0)), np.nextafter(c, np.float32(0)), c,
                    np.nextafter(c, np.float32(np.inf)),
                    np.nextafter(np.nextafter(c, np.float32(np.inf)), np.float32(np.inf))})
    for i in range(1, len(cands) - 1):
        lo = (exact(cands[i - 1]) + exact(cands[i])) / 2
        hi = (exact(cands[i]) + exact(cands[i + 1])) / 2
        if lo * lo <= v < hi * hi:
            return np.float32(cands[i])
    raise AssertionError("no candidate brackets sqrt(v)")


def test_rmsnorm_hand_row_exact_rationals():
    """Reading 11's rounding order, re-derived step by step with rationals on
    a hand row: x = the primes 2..19 with alternating signs, so sum x^2 = 1027
    and ms = 1027/8 = 128.375 exactly; eps = 1e-6 is below half an ulp of
    128.375 (2^-16), so RN(ms + eps) = ms. Then RN(sqrt), RN(1/.), RN(x*r),
    RN(.*g). The row is chosen so that the reading is pinned to the bit: one
    rounding of 1/sqrt(v) instead of two gives another r, and scaling by
    RN(r*g) instead of x*r first changes two of the eight outputs."""
    x = np.array([2, -3, 5, -7, 11, -13, 17, -19], np.float32)
    g = np.array([0.125, 1.0, 0.75, 1.125, 1.25, 1.125, 0.25, 1.625], np.float32)
    eps = O.RMS_EPS
    ms_exact = sum(Fraction(int(v)) ** 2 for v in x) / 8
    assert ms_exact == Fraction(1027, 8)
    ms = rn_f32(ms_exact)
    assert exact(ms) == ms_exact
    v = rn_f32(exact(ms) + exact(eps))
    assert v == ms  # eps is below half an ulp of 128.375
    sq = _sqrt_rn_f32(exact(v))
    r = rn_f32(1 / exact(sq))
    n = [rn_f32(exact(rn_f32(exact(a) * exact(r))) * exact(b)) for a, b in zip(x, g)]
    got = O.rmsnorm(x[None, :], g, eps)[0]
    assert [int(t) for t in got.view(np.uint32)] == [int(np.float32(t).view(np.uint32)) for t in n]
    # the pin discriminates: the alternatives give other bits
    # one rounding of 1/sqrt(v): the fp32 c with 1/hi^2 < v <= 1/lo^2 for the
    # midpoints lo < c < hi around it
    c0 = np.float32(1.0 / math.sqrt(float(exact(v))))
    cands = sorted({np.nextafter(c0, np.float32(0)), c0, np.nextafter(c0, np.float32(1))})
    r_once = [cands[i] for i in range(1, len(cands) - 1)
              if 1 / ((exact(cands[i]) + exact(cands[i + 1])) / 2) ** 2 < exact(v)
              <= 1 / ((exact(cands[i - 1]) + exact(cands[i])) / 2) ** 2]
    assert [hex(int(np.float32(t).view(np.uint32))) for t in r_once] == ["0x3db4c137"]
    alt = [rn_f32(exact(a) * exact(rn_f32(exact(r) * exact(b)))) for a, b in zip(x, g)]
    assert sum(np.float32(p) != np.float32(q) for p, q in zip(alt, n)) == 2
    assert hex(int(np.float32(r).view(np.uint32))) == "0x3db4c138"


def test_rmsnorm_act_quant_constant_row_and_g_scaling():
    x = np.full((2, 64), 3.0, np.float32)
    g = np.ones(64, np.float32)
    q, s = O.rmsnorm_act_quant(x, g)
    assert np.all(q == 127)
    q2, s2 = O.rmsnorm_act_quant(x, 2 * g)  # n doubles exactly: same codes, half the scale
    assert np.array_equal(q, q2) and np.array_equal(s2, s / np.float32(2))


RMS_PLANTS = {
    "mean_over_k_minus_1": lambda row: O.round_fraction_to_f32(
        sum(__import__("fractions").Fraction(float(v)) ** 2 for v in row) / (row.size - 1)),
    "no_square": lambda row: O.round_fraction_to_f32(
        sum(abs(__import__("fractions").Fraction(float(v))) for v in row) / row.size),
}


@pytest.mark.parametrize("plant", sorted(RMS_PLANTS))
def test_rmsnorm_planted_mistake_is_caught(plant, monkeypatch):
    monkeypatch.setattr(O.bitlinear_oracle, "mean_square_exact", RMS_PLANTS[plant])
    with pytest.raises(AssertionError):
        test_rmsnorm_matches_library_fp64_within_rounding()
