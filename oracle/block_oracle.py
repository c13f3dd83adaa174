"""Plain, slow CPU oracle for the per-256-block scale variant of the BitLinear.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this module. The product
path (bit_ternary_b200) never imports it, and it imports nothing from there.

"Core AI model zoo - BitVLA", §2 "Generalizing the ternary kernel", names two
ways to scale the ternary codes: BitNet's per-tensor absmean, stored per row as
D [N, 1] (the main oracle, bitlinear_oracle.py), and BitCPM's per-256-block
scale, which the page names as the contrast without defining it. The plainest
reading, taken here:

  * A block is 256 consecutive columns of one row: block b of row n holds
    columns [256*b, min(256*b + 256, K)). The last block of a row holds
    K - 256*(nb - 1) columns (a multiple of 16, since K % 16 == 0), where
    nb = ceil(K / 256). No block spans two rows.
  * Each block is quantised with the page's per-tensor formula (BitVLA §1)
    applied to the block alone: mean = mean(|W|) over the block (exact,
    rounded once to fp32), mean_c = max(mean, 1e-5), s = RN(1/mean_c),
    code = clamp(rint(RN(W*s)), -1, 1). The codes are stored exactly as in the
    per-tensor format (code+1, 16 per 32-bit word, LSB first); a word never
    straddles two blocks because 256 is a multiple of 16.
  * D is fp32 [N, nb], D[n, b] = mean_c of block (n, b).
  * ActQuant is unchanged (per token, over the whole row of x).
  * Product: per block, acc_b[m, n] = sum over the block's columns of
    q[m, k]*code[n, k] (exact integer), and the block's dequantised term is the
    per-tensor rescale applied with the block's scale,
    t_b = RN(RN(float(acc_b) / s_x[m]) * D[n, b]). The terms are added in fp32
    in ascending block order: y = t_0, then y = RN(y + t_b) for b = 1..nb-1
    (the order in which a matvec walks K). With one block (K <= 256) this is
    exactly the per-tensor forward with D[n] = D[n, 0].

Every step is fp32 with IEEE round-to-nearest-even (numpy float32 arithmetic);
integer steps are exact.
"""
from __future__ import annotations

import numpy as np

from . import bitlinear_oracle as _core

BLOCK = 256

__all__ = [
    "BLOCK",
    "num_blocks",
    "block_bounds",
    "weight_quant_blocks",
    "pack_weights_blocks",
    "bitlinear_forward_blocks",
]


def num_blocks(K: int) -> int:
    """nb = ceil(K / 256) scale blocks per row."""
    if K <= 0 or K % 16:
        raise ValueError("K must be a positive multiple of 16")
    return (K + BLOCK - 1) // BLOCK


def block_bounds(K: int):
    """[(k0, k1)] column ranges of the blocks of a row, in ascending order."""
    return [(b * BLOCK, min(b * BLOCK + BLOCK, K)) for b in range(num_blocks(K))]


def weight_quant_blocks(W: np.ndarray):
    """Ternary codes int8 [N, K] and per-block scales D fp32 [N, nb].

    Each block (n, b) is quantised on its own with the per-tensor absmean
    formula of BitVLA §1 (exact mean of |W| over the block, floor 1e-5,
    s = RN(1/mean_c), code = clamp(rint(RN(W*s)), -1, 1)).
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    bounds = block_bounds(K)
    codes = np.empty((N, K), dtype=np.int8)
    D = np.empty((N, len(bounds)), dtype=np.float32)
    for n in range(N):
        for b, (k0, k1) in enumerate(bounds):
            c, mean_c = _core.weight_quant(W[n:n + 1, k0:k1])
            codes[n, k0:k1] = c[0]
            D[n, b] = mean_c
    return codes, D


def pack_weights_blocks(W: np.ndarray):
    """fp32 W [N, K] -> (packed uint32 [N, K/16], D fp32 [N, nb])."""
    codes, D = weight_quant_blocks(W)
    return _core.pack_codes(codes), D


def bitlinear_forward_blocks(x: np.ndarray, packed: np.ndarray, D: np.ndarray, K: int,
                             return_parts: bool = False):
    """y [M, N] from per-block scaled ternary weights.

    acc_b = q[:, block] . code[:, block]^T (exact); t_b = RN(RN(acc_b/s_x)*D[:, b]);
    y = t_0 + t_1 + ... + t_{nb-1}, each addition an fp32 rounding, left to right.
    """
    codes = _core.unpack_codes(packed, K)
    D = np.ascontiguousarray(D, dtype=np.float32)
    bounds = block_bounds(K)
    if D.shape != (codes.shape[0], len(bounds)):
        raise ValueError(f"D must be [N, {len(bounds)}]")
    q, s_x = _core.act_quant(x)
    accs, terms = [], []
    y = None
    for b, (k0, k1) in enumerate(bounds):
        acc = _core.int_matmul(q[:, k0:k1], codes[:, k0:k1])
        t = _core.rescale(acc, s_x, D[:, b])
        accs.append(acc)
        terms.append(t)
        y = t.copy() if y is None else (y + t).astype(np.float32)
    if return_parts:
        return y, {"q": q, "s_x": s_x, "acc_blocks": accs, "terms": terms, "codes": codes}
    return y
