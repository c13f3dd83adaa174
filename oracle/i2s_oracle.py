"""Plain CPU oracle for I2_S import/export of packed BitLinear weights.

TEST INFRASTRUCTURE, like the rest of this package: only tests/,
__graft_entry__.smoke() and bench.py's cpu_baseline / reference legs may
import it; the product path never does.

What the format is ("BitNet-Embeddings I2_S guide", section "I2_S Ternary
Packing"):
  * codes come from the per-tensor absmean quantiser, scale = 1/mean(|w|),
    q = round(w * scale).clamp(-1, 1);
  * each code is stored as 2 bits, -1 -> 0, 0 -> 1, +1 -> 2 (code + 1);
  * every 128 values form one block of 32 bytes, and each byte holds four
    values as (c0 << 6) | (c1 << 4) | (c2 << 2) | c3;
  * the fp32 scale is appended after the packed data.

Readings where the page is silent (the plainest reading in each case):
  * The blocks run over the whole tensor, flattened row-major ([N, K], K
    contiguous), so a block may span two rows when K % 128 != 0.
  * A tail shorter than 128 values is padded to a whole block with the code 0
    (stored 1); import ignores the padding.
  * Which four values of a block share a byte is not stated. Two readings are
    provided: "consecutive" (byte j holds values 4j, 4j+1, 4j+2, 4j+3 as
    c0..c3) and "quarters" (byte j holds values j, j+32, j+64, j+96 as c0..c3,
    so one 32-byte block splits into four 32-value runs by the shift alone).
  * The appended scale is the quantiser's own `scale` = 1/mean(|w|), stored
    little-endian right after the last block. With the BitLinear pack's
    D = mean_c (one value for every row), export writes RN(1/D) — which is
    exactly the quantiser's s = RN(1/mean_c) — and import sets every D[n] to
    RN(1/scale).
  * A field holding 3 (no code), a scale that is not finite and positive, or
    a reciprocal of it that is not finite, make an I2_S buffer invalid.
"""
from __future__ import annotations

import numpy as np

from .bitlinear_oracle import pack_codes, unpack_codes, weight_quant

I2S_BLOCK = 128      # values per block
I2S_BLOCK_BYTES = 32  # bytes per block
I2S_LAYOUTS = ("consecutive", "quarters")

__all__ = [
    "I2S_BLOCK",
    "I2S_BLOCK_BYTES",
    "I2S_LAYOUTS",
    "i2s_nbytes",
    "i2s_encode_codes",
    "i2s_decode_codes",
    "i2s_export",
    "i2s_import",
    "i2s_from_weight",
]


def i2s_nbytes(N: int, K: int) -> int:
    """Bytes of an I2_S tensor of N*K values: whole blocks plus the fp32 scale."""
    nblocks = -(-(N * K) // I2S_BLOCK)
    return nblocks * I2S_BLOCK_BYTES + 4


def _block_groups(stored: np.ndarray, layout: str) -> np.ndarray:
    """[nblocks, 128] stored 2-bit values -> [nblocks, 32, 4]: the four values
    (c0, c1, c2, c3) that share byte j of each block."""
    nb = stored.shape[0]
    if layout == "consecutive":
        return stored.reshape(nb, 32, 4)
    if layout == "quarters":
        return stored.reshape(nb, 4, 32).transpose(0, 2, 1)
    raise ValueError(f"unknown I2_S layout {layout!r}")


def i2s_encode_codes(codes: np.ndarray, layout: str = "consecutive") -> np.ndarray:
    """Ternary codes (any shape, values in {-1, 0, 1}, row-major order) ->
    the packed blocks, uint8 [nblocks * 32] (no scale)."""
    flat = np.asarray(codes).reshape(-1).astype(np.int64)
    if flat.size and (flat.min() < -1 or flat.max() > 1):
        raise ValueError("codes must be -1, 0 or +1")
    nblocks = -(-flat.size // I2S_BLOCK)
    stored = np.ones(nblocks * I2S_BLOCK, dtype=np.int64)  # padding: code 0 -> 1
    stored[: flat.size] = flat + 1
    g = _block_groups(stored.reshape(nblocks, I2S_BLOCK), layout)
    byte = (g[..., 0] << 6) | (g[..., 1] << 4) | (g[..., 2] << 2) | g[..., 3]
    return byte.reshape(-1).astype(np.uint8)


def i2s_decode_codes(blocks: np.ndarray, count: int, layout: str = "consecutive") -> np.ndarray:
    """Packed blocks (uint8) -> the first `count` codes, int8 in {-1, 0, 1}.
    Raises ValueError if one of those values holds the field 3."""
    b = np.asarray(blocks, dtype=np.uint8).astype(np.int64)
    nblocks = b.size // I2S_BLOCK_BYTES
    if nblocks * I2S_BLOCK < count:
        raise ValueError("buffer too short")
    b = b[: nblocks * I2S_BLOCK_BYTES].reshape(nblocks, 32)
    g = np.stack([(b >> 6) & 3, (b >> 4) & 3, (b >> 2) & 3, b & 3], axis=-1)  # [nb, 32, 4]
    if layout == "consecutive":
        stored = g.reshape(nblocks, I2S_BLOCK)
    elif layout == "quarters":
        stored = g.transpose(0, 2, 1).reshape(nblocks, I2S_BLOCK)
    else:
        raise ValueError(f"unknown I2_S layout {layout!r}")
    stored = stored.reshape(-1)[:count]
    if np.any(stored == 3):
        raise ValueError("an I2_S field holds 3, which is no code")
    return (stored - 1).astype(np.int8)


def i2s_export(packed: np.ndarray, D: np.ndarray, K: int, layout: str = "consecutive") -> np.ndarray:
    """BitLinear packed weights [N, K/16] + D [N, 1] -> one I2_S buffer
    (uint8: blocks, then the fp32 scale RN(1/D)). Every row must share D."""
    Dv = np.asarray(D, dtype=np.float32).reshape(-1)
    if Dv.size == 0:
        raise ValueError("no rows")
    if not np.all(Dv == Dv[0]):
        raise ValueError("I2_S holds one scale per tensor; the rows of D differ")
    if not (np.isfinite(Dv[0]) and Dv[0] > 0):
        raise ValueError("D must be finite and positive")
    codes = unpack_codes(np.asarray(packed), K)
    with np.errstate(over="ignore"):
        scale = np.float32(np.float32(1.0) / Dv[0])
    if not np.isfinite(scale):
        raise ValueError("the reciprocal of D is not finite, so no I2_S scale holds it")
    return np.concatenate([i2s_encode_codes(codes, layout), np.array([scale], "<f4").view(np.uint8)])


def i2s_import(buf: np.ndarray, N: int, K: int, layout: str = "consecutive"):
    """One I2_S buffer of an [N, K] tensor -> (packed uint32 [N, K/16],
    D fp32 [N, 1] = RN(1/scale))."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    if buf.size != i2s_nbytes(N, K):
        raise ValueError("buffer size does not match N*K")
    scale = buf[-4:].copy().view("<f4")[0]
    if not (np.isfinite(scale) and scale > 0):
        raise ValueError("the I2_S scale must be finite and positive")
    with np.errstate(over="ignore"):
        d = np.float32(np.float32(1.0) / np.float32(scale))
    if not np.isfinite(d):
        raise ValueError("the reciprocal of the I2_S scale is not finite")
    codes = i2s_decode_codes(buf[:-4], N * K, layout).reshape(N, K)
    return pack_codes(codes), np.full((N, 1), d, dtype=np.float32)


def i2s_from_weight(W: np.ndarray, layout: str = "consecutive") -> np.ndarray:
    """The I2_S page's own recipe applied to a weight: absmean codes, blocks,
    then the quantiser's scale s = RN(1/mean_c)."""
    codes, mean_c = weight_quant(np.asarray(W, dtype=np.float32))
    s = np.float32(np.float32(1.0) / mean_c)
    return np.concatenate([i2s_encode_codes(codes, layout), np.array([s], "<f4").view(np.uint8)])
