"""Pins for the per-256-block scale oracle (oracle/block_oracle.py).

"Core AI model zoo - BitVLA", §2 "Generalizing the ternary kernel", names
BitCPM's per-256-block scale as the alternative to BitNet's per-row D [N, 1].
The reading pinned here: blocks of 256 consecutive columns inside a row (a
shorter last block when K % 256 != 0), each quantised with the per-tensor
absmean formula of §1, D [N, ceil(K/256)], and the product as the fp32 sum, in
ascending block order, of t_b = RN(RN(acc_b / s_x) * D[n, b]).

What fixes the oracle's output here, other than the oracle itself:
  * two hand-worked rows whose values are derived in the comments below (a
    block mean that is an exact fp32 tie, a tail block, the 1e-5 floor, and a
    sum whose value depends on the order of the block terms);
  * brute force with exact rationals on tiny shapes (every step re-derived from
    the definitions with Fractions);
  * the reduction to the per-tensor forward when a row has one block;
  * scale invariance of a single block under powers of two;
  * planted mistakes that must fail one of these pins.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from oracle import block_oracle as BO


# ------------------------------------------------ helpers from definitions
def exact(v) -> Fraction:
    return Fraction(float(v))


def rn_f32(true: Fraction) -> np.float32:
    """Nearest fp32 to a rational, ties to even significand (search around
    float(true) and pick by exact distance)."""
    c = np.float32(float(true))
    cands = {c, np.nextafter(c, np.float32(-np.inf)), np.nextafter(c, np.float32(np.inf))}
    best = None
    for v in cands:
        if not np.isfinite(v):
            continue
        key = (abs(exact(v) - true), int(np.float32(v).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, np.float32(v))
    return best[1]


def rint_half_even(v: Fraction) -> int:
    f = math.floor(v)
    r = v - f
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2 == 1):
        return f + 1
    return f


def bits(v) -> int:
    return int(np.float32(v).view(np.uint32))


def rational_block_forward(W: np.ndarray, x: np.ndarray):
    """Every step of the reading with Fractions: codes, D, q, s_x, y."""
    N, K = W.shape
    nb = -(-K // 256)
    floor = exact(np.float32(1e-5))
    codes = [[0] * K for _ in range(N)]
    D = [[None] * nb for _ in range(N)]
    for n in range(N):
        for b in range(nb):
            k0, k1 = 256 * b, min(256 * b + 256, K)
            mean = rn_f32(sum(abs(exact(W[n, k])) for k in range(k0, k1)) / (k1 - k0))
            mean_c = max(exact(mean), floor)
            s = exact(rn_f32(1 / mean_c))
            D[n][b] = np.float32(float(mean_c))
            for k in range(k0, k1):
                codes[n][k] = max(-1, min(1, rint_half_even(exact(rn_f32(exact(W[n, k]) * s)))))
    M = x.shape[0]
    y = np.zeros((M, N), np.float32)
    for m in range(M):
        amax = max(max(abs(exact(v)) for v in x[m]), floor)
        s_x = exact(rn_f32(Fraction(127) / amax))
        q = [max(-128, min(127, rint_half_even(exact(rn_f32(exact(v) * s_x))))) for v in x[m]]
        for n in range(N):
            acc_y = None
            for b in range(nb):
                k0, k1 = 256 * b, min(256 * b + 256, K)
                acc = sum(q[k] * codes[n][k] for k in range(k0, k1))
                t = rn_f32(exact(rn_f32(Fraction(acc) / s_x)) * exact(D[n][b]))
                acc_y = t if acc_y is None else rn_f32(exact(acc_y) + exact(t))
            y[m, n] = acc_y
    return np.array(codes, np.int8), np.array(D, np.float32), y


# ------------------------------------------------------- hand-worked rows
def hand_tie_example():
    """N=2, K=272 (blocks of 256 and 16 columns), M=2.

    Row 0, block 0: the cycle 0.5, -0.25, 0, 1 (64 times): sum|w| = 112,
      mean = 0.4375 (exact), s = RN(16/7); 0.5*s = 1.14 -> 1, -0.25*s = -0.57
      -> -1, 0 -> 0, 1*s = 2.29 -> 2 -> clamp 1.
    Row 0, block 1: 0.125, -0.375 (8 times): mean = 0.25, s = 4; 0.125*4 = 0.5
      rounds half to even -> 0; -0.375*4 = -1.5 -> -2 -> clamp -1.
    Row 1, block 0: +1, -1 alternating, except column 255 = -(1 + 2^-16):
      sum|w| = 256 + 2^-16, mean = 1 + 2^-24, the midpoint of 1 and 1 + 2^-23,
      so it rounds to the even significand: 1.0. s = 1, codes +1/-1.
    Row 1, block 1: sixteen values 2^-20: mean 2^-20 < 1e-5, so D = RN(1e-5);
      2^-20 * RN(1/RN(1e-5)) = 0.095 -> code 0.
    x: token 0 = ((37*k) mod 255) - 127 (integers, max 127, so s_x = 1, q = x);
      token 1 = 0.3 * ((k mod 17) - 8) in fp32.
    """
    K = 272
    W = np.zeros((2, K), np.float32)
    W[0, :256] = np.tile(np.array([0.5, -0.25, 0.0, 1.0], np.float32), 64)
    W[0, 256:] = np.tile(np.array([0.125, -0.375], np.float32), 8)
    W[1, :256] = np.where(np.arange(256) % 2 == 0, 1.0, -1.0).astype(np.float32)
    W[1, 255] = -(1.0 + 2.0 ** -16)
    W[1, 256:] = np.float32(2.0 ** -20)
    k = np.arange(K)
    x = np.zeros((2, K), np.float32)
    x[0] = ((37 * k) % 255 - 127).astype(np.float32)
    x[1] = ((k % 17) - 8).astype(np.float32) * np.float32(0.3)
    return W, x


def hand_order_example():
    """N=1, K=528 (blocks of 256, 256 and 16 columns), M=1: a sum whose value
    depends on the order of the block terms.

    W: block 0 all 16 (mean 16, s = 1/16, codes +1); blocks 1 and 2 all 2^-10
    (mean 2^-10 > 1e-5, codes +1). x: columns 0..7 = 127, column 8 = 8,
    column 256 = 1, column 512 = 1, the rest 0; max|x| = 127, so s_x = 1 and
    q = x. acc = (1024, 1, 1), terms t = (1024*16, 2^-10, 2^-10) =
    (2^14, 2^-10, 2^-10). In block order: 2^14 + 2^-10 is the midpoint of 2^14
    and 2^14 + 2^-9 (the ulp of 2^14 is 2^-9), which rounds to the even 2^14;
    adding 2^-10 again gives 2^14. Summed in reverse order, or summed exactly
    and rounded once, it would be 2^14 + 2^-9.
    """
    K = 528
    W = np.full((1, K), np.float32(2.0 ** -10))
    W[0, :256] = 16.0
    x = np.zeros((1, K), np.float32)
    x[0, :8] = 127.0
    x[0, 8] = 8.0
    x[0, 256] = 1.0
    x[0, 512] = 1.0
    return W, x


def test_hand_tie_example():
    W, x = hand_tie_example()
    codes, D = O.weight_quant_blocks(W)
    assert D.shape == (2, 2)
    assert D[0, 0] == np.float32(0.4375) and D[0, 1] == np.float32(0.25)
    assert D[1, 0] == np.float32(1.0), "the mean 1 + 2^-24 is a tie and rounds to even"
    assert D[1, 1] == np.float32(1e-5)
    assert np.array_equal(codes[0, :256], np.tile(np.array([1, -1, 0, 1], np.int8), 64))
    assert np.array_equal(codes[0, 256:], np.tile(np.array([0, -1], np.int8), 8))
    assert np.array_equal(codes[1, :256], np.where(np.arange(256) % 2 == 0, 1, -1).astype(np.int8))
    assert not codes[1, 256:].any()
    packed, D2 = O.pack_weights_blocks(W)
    assert np.array_equal(D2, D)
    y, parts = O.bitlinear_forward_blocks(x, packed, D, 272, return_parts=True)
    assert parts["s_x"][0] == np.float32(1.0)
    assert np.array_equal(parts["q"][0], x[0].astype(np.int8))
    # Row 1 has codes +1/-1 alternating on block 0 and 0 on block 1, with q = x
    # for token 0: acc_0 = sum of x[even] - sum of x[odd] over columns 0..255.
    xk = x[0, :256].astype(np.int64)
    assert parts["acc_blocks"][0][0, 1] == xk[0::2].sum() - xk[1::2].sum()
    assert parts["acc_blocks"][1][0, 1] == 0
    c_want, D_want, y_want = rational_block_forward(W, x)
    assert np.array_equal(c_want, codes) and np.array_equal(D_want, D)
    assert [bits(v) for v in y.ravel()] == [bits(v) for v in y_want.ravel()]


def test_hand_order_example():
    W, x = hand_order_example()
    packed, D = O.pack_weights_blocks(W)
    assert np.array_equal(D, np.array([[16.0, 2.0 ** -10, 2.0 ** -10]], np.float32))
    y, parts = O.bitlinear_forward_blocks(x, packed, D, 528, return_parts=True)
    assert [int(a[0, 0]) for a in parts["acc_blocks"]] == [1024, 1, 1]
    assert [float(t[0, 0]) for t in parts["terms"]] == [2.0 ** 14, 2.0 ** -10, 2.0 ** -10]
    assert bits(y[0, 0]) == bits(np.float32(2.0 ** 14)) == 0x46800000
    assert np.float32(2.0 ** 14) + np.float32(2.0 ** -9) != np.float32(2.0 ** 14)  # the other order differs


# ------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed,N,K,M", [(0, 3, 528, 2), (1, 2, 272, 3), (2, 4, 48, 2), (3, 2, 784, 1)])
def test_bruteforce_rational(seed, N, K, M):
    rng = np.random.default_rng(seed)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    W[0, :16] *= np.float32(64.0)  # one block with a different scale
    x = rng.standard_t(3, (M, K)).astype(np.float32)
    codes, D = O.weight_quant_blocks(W)
    packed, _ = O.pack_weights_blocks(W)
    y = O.bitlinear_forward_blocks(x, packed, D, K)
    c_want, D_want, y_want = rational_block_forward(W, x)
    assert np.array_equal(codes, c_want)
    assert np.array_equal(D.view(np.uint32), D_want.view(np.uint32))
    assert np.array_equal(y.view(np.uint32), y_want.view(np.uint32))


# ----------------------------------------------------- reductions, invariants
@pytest.mark.parametrize("N,K", [(1, 256), (5, 16), (3, 144)])
def test_one_block_equals_per_tensor_forward(N, K):
    """With K <= 256 each row is one block; for N == 1 that block is the whole
    tensor, so codes and D equal the per-tensor pack, and for any N the forward
    equals the per-tensor forward with D[n] = D[n, 0]."""
    rng = np.random.default_rng(K + N)
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = rng.normal(0, 1, (3, K)).astype(np.float32)
    packed, D = O.pack_weights_blocks(W)
    assert D.shape == (N, 1)
    if N == 1:
        p1, D1 = O.pack_weights(W)
        assert np.array_equal(p1, packed) and np.array_equal(D1, D)
    y = O.bitlinear_forward_blocks(x, packed, D, K)
    y1 = O.bitlinear_forward(x, packed, D[:, 0], K)
    assert np.array_equal(y.view(np.uint32), y1.view(np.uint32))


def test_blocks_are_row_local():
    """Changing one block's weights changes only that block's codes and D."""
    rng = np.random.default_rng(7)
    W = rng.normal(0, 0.02, (3, 784)).astype(np.float32)
    c0, D0 = O.weight_quant_blocks(W)
    W2 = W.copy()
    W2[1, 256:512] *= np.float32(3.0)
    W2[1, 300] = np.float32(0.5)
    c1, D1 = O.weight_quant_blocks(W2)
    changed = D1 != D0
    assert changed[1, 1] and changed.sum() == 1
    mask = np.ones_like(c0, bool)
    mask[1, 256:512] = False
    assert np.array_equal(c0[mask], c1[mask])


@pytest.mark.parametrize("j", [-6, -1, 3, 9])
def test_block_scale_invariance(j):
    rng = np.random.default_rng(11)
    W = rng.normal(0, 0.02, (2, 528)).astype(np.float32)
    c0, D0 = O.weight_quant_blocks(W)
    W2 = W.copy()
    W2[0, 256:512] *= np.float32(2.0 ** j)
    c1, D1 = O.weight_quant_blocks(W2)
    assert np.array_equal(c0, c1)
    assert D1[0, 1] == D0[0, 1] * np.float32(2.0 ** j)
    D1[0, 1] = D0[0, 1]
    assert np.array_equal(D0, D1)


def test_block_zero_fraction_gaussian():
    """A block of Gaussian weights gives the closed-form zero fraction of the
    per-tensor case, erf(sqrt(2/pi)/2/sqrt(2)) = 0.3101, up to sampling."""
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (256, 2560)).astype(np.float32)
    codes, D = O.weight_quant_blocks(W)
    want = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    assert abs((codes == 0).mean() - want) < 0.005
    assert set(np.unique(codes).tolist()) <= {-1, 0, 1}
    assert np.all(D > 0)


def test_forward_within_rounding_of_exact_product():
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, (8, 1152)).astype(np.float32)
    x = rng.normal(0, 1, (3, 1152)).astype(np.float32)
    packed, D = O.pack_weights_blocks(W)
    y, parts = O.bitlinear_forward_blocks(x, packed, D, 1152, return_parts=True)
    nb = D.shape[1]
    for m in range(3):
        for n in range(8):
            ex = sum(Fraction(int(parts["acc_blocks"][b][m, n])) * exact(D[n, b]) for b in range(nb)) \
                / exact(parts["s_x"][m])
            scale = sum(abs(exact(parts["terms"][b][m, n])) for b in range(nb))
            assert abs(exact(y[m, n]) - ex) <= scale * Fraction(3 * nb, 2 ** 24)


def test_shape_errors():
    with pytest.raises(ValueError):
        O.num_blocks(24)
    packed, D = O.pack_weights_blocks(np.ones((2, 272), np.float32))
    with pytest.raises(ValueError):
        O.bitlinear_forward_blocks(np.ones((1, 272), np.float32), packed, D[:, :1], 272)


# ----------------------------------------------------------- planted mistakes
def _flattened_blocks(W):
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    flat = W.reshape(-1)
    codes = np.empty(flat.size, np.int8)
    means = np.empty(flat.size, np.float32)
    for k0 in range(0, flat.size, 256):
        c, m = O.weight_quant(flat[k0:k0 + 256].reshape(1, -1))
        codes[k0:k0 + 256] = c[0]
        means[k0:k0 + 256] = m
    nb = -(-K // 256)
    D = np.stack([means.reshape(N, K)[:, min(256 * b, K - 1)] for b in range(nb)], axis=1)
    return codes.reshape(N, K), D


def _per_row_mean(W):
    W = np.ascontiguousarray(W, np.float32)
    nb = -(-W.shape[1] // 256)
    rows = [O.weight_quant(W[n:n + 1]) for n in range(W.shape[0])]
    return (np.concatenate([c for c, _ in rows]),
            np.array([[m] * nb for _, m in rows], np.float32))


def _forward_summed(order):
    def fwd(x, packed, D, K, return_parts=False):
        codes = O.unpack_codes(packed, K)
        q, s_x = O.act_quant(x)
        terms = [O.rescale(O.int_matmul(q[:, k0:k1], codes[:, k0:k1]), s_x, D[:, b])
                 for b, (k0, k1) in enumerate(BO.block_bounds(K))]
        if order == "exact":
            y = np.sum(np.stack(terms).astype(np.float64), axis=0).astype(np.float32)
        else:
            y = terms[-1].copy()
            for t in reversed(terms[:-1]):
                y = (y + t).astype(np.float32)
        if return_parts:
            return y, {"q": q, "s_x": s_x, "terms": terms,
                       "acc_blocks": [O.int_matmul(q[:, k0:k1], codes[:, k0:k1]) for k0, k1 in BO.block_bounds(K)]}
        return y
    return fwd


def _forward_d_first(x, packed, D, K, return_parts=False):
    codes = O.unpack_codes(packed, K)
    q, s_x = O.act_quant(x)
    y, accs, terms = None, [], []
    for b, (k0, k1) in enumerate(BO.block_bounds(K)):
        accs.append(O.int_matmul(q[:, k0:k1], codes[:, k0:k1]))
        a = accs[-1].astype(np.float32)
        terms.append(((a * D[:, b][None, :]).astype(np.float32) / s_x[:, None]).astype(np.float32))
        y = terms[-1] if y is None else (y + terms[-1]).astype(np.float32)
    if return_parts:
        return y, {"q": q, "s_x": s_x, "terms": terms, "acc_blocks": accs}
    return y


BLOCK_PLANTS = {
    "blocks_over_flattened_tensor": ("weight_quant_blocks", _flattened_blocks),
    "one_mean_per_row": ("weight_quant_blocks", _per_row_mean),
    "terms_summed_in_reverse": ("bitlinear_forward_blocks", _forward_summed("reverse")),
    "terms_summed_exactly_rounded_once": ("bitlinear_forward_blocks", _forward_summed("exact")),
    "scale_by_D_before_s_x": ("bitlinear_forward_blocks", _forward_d_first),
}


@pytest.mark.parametrize("plant", sorted(BLOCK_PLANTS))
def test_planted_mistake_is_caught(plant, monkeypatch):
    name, fn = BLOCK_PLANTS[plant]
    monkeypatch.setattr(BO, name, fn)
    monkeypatch.setattr(O, name, fn)
    failed = False
    for pin in (test_hand_tie_example, test_hand_order_example):
        try:
            pin()
        except (AssertionError, ValueError, TypeError, KeyError):
            failed = True
    if not failed:
        try:
            test_bruteforce_rational(0, 3, 528, 2)
        except AssertionError:
            failed = True
    assert failed, f"planted mistake {plant} passed every pin"
