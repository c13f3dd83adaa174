"""Plain, slow CPU oracle for the BitNet b1.58 BitLinear (W1.58-A8).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this module. The product
path (bit_ternary_b200) never imports it, and it imports nothing from there.

What it computes, and where the pages define it:

  WeightQuant  "Core AI model zoo - BitVLA", §1 "What the checkpoint actually
               is": per-tensor absmean, s = 1/mean(|W|),
               codes = round(W*s).clamp(-1, 1). The same formula appears in
               "BitNet-Embeddings I2_S guide" §3.3, "I2_S Ternary Packing".
  Encoding     BitVLA page §2, "Generalizing the ternary kernel": codes are
               stored as code+1 (-1->0, 0->1, +1->2), 16 codes per 32-bit
               lane chunk, and the scale D is one fp32 per output row, [N, 1].
  ActQuant     BitVLA page §1: per-token int8 absmax,
               round(x*127/max|x|).clamp(-128, 127), dequantised by
               /(127/max|x|). I2_S guide §2 ("8-bit activations, absmax,
               per-token").
  Product      BitVLA page §2: the wrapper quantises x and then the kernel
               equals F.linear(ActQuant(x), WeightQuant(W)). Here that is an
               exact integer contraction acc = q . code, then the two scales.

Readings where the pages are silent (the plainest reading in each case):
  * mean(|W|) is the exact real mean, correctly rounded to fp32.
  * A floor of 1e-5 guards mean(|W|) and max|x| (an all-zero tensor or token).
  * s = RN(1/mean); the code is rint(RN(W*s)) (the W*s spelling of §1).
  * s_x = RN(127/max|x|); q = rint(RN(x*s_x)).
  * round() is round-half-to-even (torch.round).
  * Bit order: code+1 for column k sits in bits [2*(k%16), 2*(k%16)+2) of word
    k/16 (LSB first); the row stride is exactly K/16 words.
  * y[m,n] = RN( RN(float(acc[m,n]) / s_x[m]) * D[n] ).
  * Per-projection RMSNorm before ActQuant ("BitNet-Embeddings I2_S guide"
    §3.1; rms_norm_eps = 1e-6): ms = mean(x^2) over the row is the exact real
    mean, correctly rounded to fp32 once; r = RN(1/RN(sqrt(RN(ms + eps))));
    n = RN(RN(x*r)*g); then ActQuant of n.
  * bf16 inputs (the BitVLA checkpoint is a bf16 latent master, §1; the codes
    are built from it, §2) are widened to fp32 exactly (a bf16 is the upper
    half of an fp32) and then follow the fp32 definition above.

Every step is fp32 with IEEE round-to-nearest-even (numpy float32 arithmetic);
integer steps are exact (Python ints / int64).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

FLOOR = np.float32(1e-5)
QMAX = 127

__all__ = [
    "FLOOR",
    "absmean_exact",
    "weight_quant",
    "pack_codes",
    "unpack_codes",
    "pack_weights",
    "act_quant",
    "int_matmul",
    "rescale",
    "bitlinear_forward",
    "bitlinear_forward_rows",
    "fake_quant_linear",
    "round_fraction_to_f32",
    "bf16_to_f32",
    "pack_weights_bf16",
    "act_quant_bf16",
    "bitlinear_forward_bf16",
    "RMS_EPS",
    "mean_square_exact",
    "rmsnorm",
    "rmsnorm_act_quant",
    "bitlinear_forward_rmsnorm",
]


# --------------------------------------------------------------------------
# Exact mean of |W|, correctly rounded to fp32
# --------------------------------------------------------------------------
def round_fraction_to_f32(value: Fraction) -> np.float32:
    """Round a non-negative rational to the nearest fp32, ties to even.

    Plain definition of IEEE round-to-nearest-even: find the binade, scale the
    value so the significand has 24 integer bits, take the integer part and
    round with the exact remainder. Subnormal results use the fixed 2^-149
    quantum. Values beyond FLT_MAX are not expected (a mean of finite fp32
    values never exceeds FLT_MAX) and raise.
    """
    if value < 0:
        raise ValueError("negative value")
    if value == 0:
        return np.float32(0.0)
    num, den = value.numerator, value.denominator
    # e = floor(log2(value)), from bit lengths, then fixed up exactly.
    e = num.bit_length() - den.bit_length()
    if Fraction(2) ** e > value:
        e -= 1
    if Fraction(2) ** (e + 1) <= value:
        e += 1
    # Quantum (weight of the last significand bit): 2^(e-23), never below 2^-149.
    q_exp = max(e - 23, -149)
    scaled = value / (Fraction(2) ** q_exp)
    sig, rem = divmod(scaled.numerator, scaled.denominator)
    twice = 2 * rem
    if twice > scaled.denominator or (twice == scaled.denominator and sig % 2 == 1):
        sig += 1
    result = Fraction(sig) * (Fraction(2) ** q_exp)
    if result > Fraction(np.finfo(np.float32).max.item()):
        raise OverflowError("mean exceeds FLT_MAX")
    # sig < 2^25 and the exponent is in range, so float64 and fp32 hold it exactly.
    out = np.float32(float(result))
    assert Fraction(float(out)) == result
    return out


def absmean_exact(W: np.ndarray) -> np.float32:
    """mean(|W|) over the whole tensor: exact sum, correctly rounded division.

    Each |w| is m * 2^(max(e,1) - 150), with e the biased exponent and m the
    24-bit significand (implicit bit included for e > 0). Summing m per
    exponent is exact integer work, independent of order; the total is then an
    exact rational divided by the element count and rounded once.
    """
    a = np.ascontiguousarray(W, dtype=np.float32).reshape(-1)
    n = a.size
    if n == 0:
        raise ValueError("empty weight")
    bits = a.view(np.uint32) & np.uint32(0x7FFFFFFF)
    exps = (bits >> np.uint32(23)).astype(np.int64)
    if np.any(exps == 255):
        raise FloatingPointError("non-finite weight")
    mant = (bits & np.uint32(0x7FFFFF)).astype(np.int64)
    mant = np.where(exps > 0, mant | (1 << 23), mant)
    # Per-exponent integer sums. bincount accumulates in float64, so split the
    # 24-bit significand into two 12-bit halves: each half-sum stays far below
    # 2^53 and is therefore exact.
    hi = np.bincount(exps, weights=(mant >> 12).astype(np.float64), minlength=256)
    lo = np.bincount(exps, weights=(mant & 0xFFF).astype(np.float64), minlength=256)
    assert n < (1 << 40)
    total = 0  # in units of 2^-149
    for e in range(255):
        s = (int(hi[e]) << 12) + int(lo[e])
        if s:
            total += s << (max(e, 1) - 1)
    return round_fraction_to_f32(Fraction(total, n) / (Fraction(2) ** 149))


# --------------------------------------------------------------------------
# WeightQuant and the packed format
# --------------------------------------------------------------------------
def weight_quant(W: np.ndarray):
    """Ternary codes int8 [N, K] and the (floored) per-tensor scale mean.

    BitVLA page §1: s = 1/mean(|W|), codes = round(W*s).clamp(-1, 1); the
    dequantised weight is codes/s, i.e. codes * mean.
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    mean = absmean_exact(W)
    mean_c = np.float32(max(mean, FLOOR))
    s = np.float32(np.float32(1.0) / mean_c)
    t = (W * s).astype(np.float32)  # one fp32 multiply per element
    codes = np.clip(np.rint(t), -1, 1).astype(np.int8)
    return codes, mean_c


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """int8 codes [N, K] in {-1,0,1} -> uint32 [N, K/16] holding code+1.

    BitVLA page §2: 16 codes per 32-bit lane chunk, stored as code+1; K must be
    a multiple of 16. Column k goes to bits 2*(k%16) of word k//16.
    """
    N, K = codes.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    u = (codes.astype(np.int64) + 1).reshape(N, K // 16, 16)
    if u.min(initial=1) < 0 or u.max(initial=1) > 2:
        raise ValueError("codes outside {-1,0,1}")
    shifts = (2 * np.arange(16, dtype=np.int64))
    words = np.sum(u << shifts, axis=2)  # fields do not overlap: sum == OR
    return words.astype(np.uint32)


def unpack_codes(packed: np.ndarray, K: int) -> np.ndarray:
    """Inverse of pack_codes. Raises if a field holds the unused value 3."""
    N = packed.shape[0]
    w = packed.astype(np.int64).reshape(N, K // 16, 1)
    fields = (w >> (2 * np.arange(16, dtype=np.int64))) & 3
    if np.any(fields == 3):
        raise ValueError("packed field holds 3")
    return (fields - 1).reshape(N, K).astype(np.int8)


def pack_weights(W: np.ndarray):
    """fp32 W [N, K] -> (packed uint32 [N, K/16], D fp32 [N, 1])."""
    codes, mean_c = weight_quant(W)
    N = W.shape[0]
    D = np.full((N, 1), mean_c, dtype=np.float32)
    return pack_codes(codes), D


# --------------------------------------------------------------------------
# ActQuant
# --------------------------------------------------------------------------
def act_quant(x: np.ndarray):
    """Per-token int8 absmax: q int8 [M, K], s_x fp32 [M] (= 127/max|x|).

    BitVLA page §1: round(x*127/max|x|).clamp(-128, 127); the dequantised
    activation is q / (127/max|x|), so s_x is kept as 127/max|x|.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    mx = np.maximum(amax, FLOOR).astype(np.float32)
    s_x = (np.float32(QMAX) / mx).astype(np.float32)
    t = (x * s_x[:, None]).astype(np.float32)
    q = np.clip(np.rint(t), -128, 127).astype(np.int8)
    return q, s_x


# --------------------------------------------------------------------------
# Contraction and rescale
# --------------------------------------------------------------------------
def int_matmul(q: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[m, k] * codes[n, k], exact (int64), checked to fit int32."""
    acc = q.astype(np.int64) @ codes.astype(np.int64).T
    if acc.size and np.abs(acc).max() >= 2**31:
        raise OverflowError("accumulator exceeds int32")
    return acc


def rescale(acc: np.ndarray, s_x: np.ndarray, D: np.ndarray) -> np.ndarray:
    """y = RN(RN(float(acc) / s_x[m]) * D[n]).

    BitVLA page §1 dequantises activations by /(127/max|x|) and weights by /s
    (= * mean); page §2 stores that weight factor per row as D [N, 1].
    float(acc) is exact because |acc| < 2^24 for every supported shape.
    """
    if acc.size and np.abs(acc).max() >= 2**24:
        raise OverflowError("accumulator not exactly representable in fp32")
    a = acc.astype(np.float32)
    t = (a / s_x.astype(np.float32)[:, None]).astype(np.float32)
    return (t * D.reshape(1, -1).astype(np.float32)).astype(np.float32)


def bitlinear_forward(x: np.ndarray, packed: np.ndarray, D: np.ndarray, K: int,
                      return_parts: bool = False):
    """y = F.linear(ActQuant(x), WeightQuant(W)) from the packed weights.

    BitVLA page §2: the wrapper applies ActQuant and the kernel contracts the
    int8 activations with the ternary codes and applies the per-row scale.
    """
    codes = unpack_codes(packed, K)
    q, s_x = act_quant(x)
    acc = int_matmul(q, codes)
    y = rescale(acc, s_x, D)
    if return_parts:
        return y, {"q": q, "s_x": s_x, "acc": acc, "codes": codes}
    return y


def bitlinear_forward_rows(x: np.ndarray, packed: np.ndarray, D: np.ndarray, K: int,
                           rows: np.ndarray, return_parts: bool = False):
    """The forward for a subset of token rows only (ActQuant is per token)."""
    xs = np.ascontiguousarray(x[np.asarray(rows)], dtype=np.float32)
    return bitlinear_forward(xs, packed, D, K, return_parts=return_parts)


def fake_quant_linear(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Literal F.linear(ActQuant(x), WeightQuant(W)) with dequantised operands.

    The float reading of BitVLA page §2's "equals F.linear(ActQuant(x),
    WeightQuant(W)) exactly", evaluated in fp64. It differs from
    bitlinear_forward only by summation order and the final fp32 roundings.
    """
    codes, mean_c = weight_quant(W)
    s = np.float32(np.float32(1.0) / mean_c)
    q, s_x = act_quant(x)
    xq = q.astype(np.float64) / s_x.astype(np.float64)[:, None]
    wq = codes.astype(np.float64) / np.float64(s)
    return xq @ wq.T


# --------------------------------------------------------------------------
# bf16 inputs
# --------------------------------------------------------------------------
def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 values given as their 16-bit patterns (uint16) -> fp32, exactly.

    BitVLA page §1: the checkpoint is a bf16 latent master, quantised on the
    fly; §2 builds the codes from it. A bf16 is the upper 16 bits of the fp32
    with the same value, so the widening is a shift of the bit pattern.
    """
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def pack_weights_bf16(W_bits: np.ndarray):
    """WeightQuant + pack of a bf16 master weight [N, K] (uint16 bit patterns)."""
    return pack_weights(bf16_to_f32(W_bits))


def act_quant_bf16(x_bits: np.ndarray):
    """ActQuant of bf16 activations [M, K] (uint16 bit patterns)."""
    return act_quant(bf16_to_f32(x_bits))


def bitlinear_forward_bf16(x_bits: np.ndarray, packed: np.ndarray, D: np.ndarray, K: int,
                           return_parts: bool = False):
    """The forward from bf16 activations (uint16 bit patterns) [M, K]."""
    return bitlinear_forward(bf16_to_f32(x_bits), packed, D, K, return_parts=return_parts)


# --------------------------------------------------------------------------
# Per-projection RMSNorm + ActQuant
# --------------------------------------------------------------------------
RMS_EPS = np.float32(1e-6)


def mean_square_exact(row: np.ndarray) -> np.float32:
    """mean(x^2) over one row: exact sum of squares, correctly rounded division.

    x = m * 2^(ee-150) (ee = max(biased exponent, 1), m the 24-bit
    significand), so x^2 = m^2 * 2^(2*(ee-1)) units of 2^-298: integer sums,
    then one rounding of the exact rational to fp32.
    """
    a = np.ascontiguousarray(row, dtype=np.float32).reshape(-1)
    bits = a.view(np.uint32) & np.uint32(0x7FFFFFFF)
    exps = (bits >> np.uint32(23)).astype(np.int64)
    if np.any(exps == 255):
        raise FloatingPointError("non-finite activation")
    mant = (bits & np.uint32(0x7FFFFF)).astype(np.int64)
    mant = np.where(exps > 0, mant | (1 << 23), mant)
    total = 0  # in units of 2^-298
    for m, e in zip(mant.tolist(), exps.tolist()):
        if m:
            total += (m * m) << (2 * (max(e, 1) - 1))
    return round_fraction_to_f32(Fraction(total, a.size) / (Fraction(2) ** 298))


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: np.float32 = RMS_EPS) -> np.ndarray:
    """n = RMSNorm(x, g) per row, in fp32 (I2_S guide §3.1: each projection
    normalises its input with its own norm.weight g before activation_quant).

    ms = mean(x^2) exact, rounded once; r = RN(1 / RN(sqrt(RN(ms + eps))));
    n[k] = RN(RN(x[k] * r) * g[k]).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32).reshape(1, -1)
    out = np.empty_like(x)
    for i in range(x.shape[0]):
        ms = mean_square_exact(x[i])
        v = np.float32(ms + np.float32(eps))
        r = np.float32(np.float32(1.0) / np.sqrt(v))
        out[i] = ((x[i] * r).astype(np.float32) * g[0]).astype(np.float32)
    return out


def rmsnorm_act_quant(x: np.ndarray, g: np.ndarray, eps: np.float32 = RMS_EPS):
    """ActQuant(RMSNorm(x, g)): q int8 [M, K], s_x fp32 [M]."""
    return act_quant(rmsnorm(x, g, eps))


def bitlinear_forward_rmsnorm(x: np.ndarray, g: np.ndarray, packed: np.ndarray, D: np.ndarray, K: int,
                              eps: np.float32 = RMS_EPS, return_parts: bool = False):
    """y = F.linear(ActQuant(RMSNorm(x, g)), WeightQuant(W)) (I2_S guide §3.1 chain)."""
    return bitlinear_forward(rmsnorm(x, g, eps), packed, D, K, return_parts=return_parts)
