"""Pins for the I2_S oracle ("BitNet-Embeddings I2_S guide", section "I2_S
Ternary Packing"): a hand-worked block, closed forms for uniform blocks, an
independent bit-string construction of the byte formula, brute force over
every position in a block, the tail padding, the round trip through the
BitLinear pack, invalid buffers, and planted mistakes that the pins catch."""
import json
import os

import numpy as np
import pytest

import oracle as O
from oracle import i2s_oracle


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "i2s_block.json")) as f:
        return json.load(f)


def _hex(xs):
    return np.array([int(v, 16) for v in xs], dtype=np.uint8)


@pytest.mark.parametrize("layout", O.I2S_LAYOUTS)
def test_golden_hand_block(golden_dir, layout):
    g = _golden(golden_dir)
    got = O.i2s_encode_codes(np.array(g["codes"], np.int8), layout)
    assert np.array_equal(got, _hex(g["bytes_" + layout]))
    back = O.i2s_decode_codes(got, 128, layout)
    assert np.array_equal(back, np.array(g["codes"], np.int8))


def test_golden_scale_bytes(golden_dir):
    g = _golden(golden_dir)["scale_mean_quarter"]
    W = np.where(np.arange(128) % 3 == 0, -0.25, 0.25).astype(np.float32).reshape(1, 128)
    buf = O.i2s_from_weight(W)
    assert buf.size == 32 + 4
    assert np.array_equal(buf[-4:], _hex(g["scale_bytes_le"]))
    codes = O.i2s_decode_codes(buf[:-4], 128)
    assert np.array_equal(codes, np.sign(W.reshape(-1)).astype(np.int8))


@pytest.mark.parametrize("layout", O.I2S_LAYOUTS)
@pytest.mark.parametrize("code,byte", [(-1, 0x00), (0, 0x55), (1, 0xAA)])
def test_uniform_blocks(layout, code, byte):
    got = O.i2s_encode_codes(np.full(256, code, np.int8), layout)
    assert got.size == 64 and np.all(got == byte)


def _bitstring_encode(codes, layout):
    """Independent construction: for each block, write the stored values as
    2-bit binary strings in the order c0, c1, c2, c3 of byte 0, then byte 1,
    ..., and cut the string into bytes (MSB first)."""
    flat = [int(c) + 1 for c in np.asarray(codes).reshape(-1)]
    flat += [1] * ((-len(flat)) % 128)
    out = []
    for b0 in range(0, len(flat), 128):
        blk = flat[b0:b0 + 128]
        if layout == "consecutive":
            order = [4 * j + i for j in range(32) for i in range(4)]
        else:
            order = [j + 32 * i for j in range(32) for i in range(4)]
        bits = "".join(format(blk[v], "02b") for v in order)
        out += [int(bits[8 * t:8 * t + 8], 2) for t in range(32)]
    return np.array(out, dtype=np.uint8)


@pytest.mark.parametrize("layout", O.I2S_LAYOUTS)
def test_every_position_in_a_block(layout):
    for i in range(128):
        for c in (-1, 1):
            codes = np.zeros(128, np.int8)
            codes[i] = c
            got = O.i2s_encode_codes(codes, layout)
            assert np.array_equal(got, _bitstring_encode(codes, layout)), (i, c)
            j, f = (i // 4, i % 4) if layout == "consecutive" else (i % 32, i // 32)
            want = np.full(32, 0x55, np.uint8)
            want[j] = (0x55 & ~(3 << (6 - 2 * f))) | ((c + 1) << (6 - 2 * f))
            assert np.array_equal(got, want), (i, c)


@pytest.mark.parametrize("layout", O.I2S_LAYOUTS)
@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (5, 1152), (7, 4304), (2, 128)])
def test_random_codes_against_bitstring(layout, N, K):
    rng = np.random.default_rng(N * 7919 + K)
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    got = O.i2s_encode_codes(codes, layout)
    assert got.size == O.i2s_nbytes(N, K) - 4
    assert np.array_equal(got, _bitstring_encode(codes, layout))
    assert np.array_equal(O.i2s_decode_codes(got, N * K, layout), codes.reshape(-1))


def test_tail_block_is_padded_with_zero_codes():
    codes = np.full((3, 48), -1, np.int8)  # 144 values: one full block + 16
    for layout in O.I2S_LAYOUTS:
        got = O.i2s_encode_codes(codes, layout)
        assert got.size == 64
        assert np.all(got[:32] == 0x00)
        tail = got[32:]
        if layout == "consecutive":
            assert np.all(tail[:4] == 0x00) and np.all(tail[4:] == 0x55)
        else:
            assert np.all(tail[:16] == 0x15) and np.all(tail[16:] == 0x55)


def test_sizes():
    assert O.i2s_nbytes(1, 16) == 36
    assert O.i2s_nbytes(2560, 2560) == 2560 * 2560 // 4 + 4
    assert O.i2s_nbytes(3, 48) == 68
    assert O.i2s_nbytes(0, 16) == 4


@pytest.mark.parametrize("layout", O.I2S_LAYOUTS)
@pytest.mark.parametrize("N,K,dist", [(3, 48, "normal"), (64, 1152, "laplace"), (17, 4304, "normal")])
def test_round_trip_through_the_bitlinear_pack(layout, N, K, dist):
    rng = np.random.default_rng(K + N)
    W = (rng.standard_normal((N, K)) if dist == "normal" else rng.laplace(size=(N, K))).astype(np.float32) * 0.02
    packed, D = O.pack_weights(W)
    buf = O.i2s_export(packed, D, K, layout)
    # export of the pack equals the page's own recipe applied to W
    assert np.array_equal(buf, O.i2s_from_weight(W, layout))
    p2, D2 = O.i2s_import(buf, N, K, layout)
    assert np.array_equal(p2, packed)
    s = np.float32(np.float32(1) / D[0, 0])
    assert np.array_equal(D2, np.full((N, 1), np.float32(np.float32(1) / s), np.float32))


def test_exact_scale_round_trips_exactly():
    W = np.full((2, 64), 0.5, np.float32)
    packed, D = O.pack_weights(W)
    p2, D2 = O.i2s_import(O.i2s_export(packed, D, 64), 2, 64)
    assert np.array_equal(D2, D) and np.array_equal(p2, packed)


def test_import_rejects_invalid_buffers():
    N, K = 3, 48
    packed, D = O.pack_weights(np.ones((N, K), np.float32))
    good = O.i2s_export(packed, D, K)
    bad = good.copy()
    bad[0] |= 0xC0  # value 0 holds 3
    with pytest.raises(ValueError, match="3"):
        O.i2s_import(bad, N, K)
    pad = good.copy()
    pad[40] = 0xFF  # padding only (values 144..): ignored
    O.i2s_import(pad, N, K)
    for scale in (0.0, -1.0, np.nan, np.inf, 1e-45):
        b = good.copy()
        b[-4:] = np.array([scale], "<f4").view(np.uint8)
        with pytest.raises(ValueError):
            O.i2s_import(b, N, K)
    with pytest.raises(ValueError):
        O.i2s_import(good[:-1], N, K)


def test_export_rejects_per_row_scales():
    packed, D = O.pack_weights(np.ones((2, 16), np.float32))
    D2 = D.copy()
    D2[1, 0] = 2.0
    with pytest.raises(ValueError, match="differ"):
        O.i2s_export(packed, D2, 16)
    for d in (0.0, -1.0, np.nan, np.inf, 1e-45):  # no finite positive scale 1/d
        with pytest.raises(ValueError):
            O.i2s_export(packed, np.full((2, 1), d, np.float32), 16)


# planted mistakes: each must fail the hand-worked block
PLANTS = {
    "fields_lsb_first": lambda mp: mp.setattr(
        i2s_oracle, "_block_groups",
        lambda stored, layout: stored.reshape(stored.shape[0], 32, 4)[..., ::-1]
        if layout == "consecutive" else stored.reshape(stored.shape[0], 4, 32).transpose(0, 2, 1)[..., ::-1]),
    "layouts_swapped": lambda mp: mp.setattr(
        i2s_oracle, "_block_groups",
        lambda stored, layout: stored.reshape(stored.shape[0], 4, 32).transpose(0, 2, 1)
        if layout == "consecutive" else stored.reshape(stored.shape[0], 32, 4)),
    "quarters_not_transposed": lambda mp: mp.setattr(
        i2s_oracle, "_block_groups",
        lambda stored, layout: stored.reshape(stored.shape[0], 4, 32).reshape(stored.shape[0], 32, 4)),
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_planted_mistake_is_caught(plant, monkeypatch, golden_dir):
    PLANTS[plant](monkeypatch)
    with pytest.raises(AssertionError):
        for layout in O.I2S_LAYOUTS:
            test_golden_hand_block(golden_dir, layout)


def test_planted_twos_complement_codes_are_caught(monkeypatch, golden_dir):
    """Codes stored as 2-bit two's complement (-1 -> 3, 0 -> 0, +1 -> 1)
    instead of code + 1."""
    def twos_complement(codes, layout="consecutive"):
        flat = np.asarray(codes).reshape(-1).astype(np.int64)
        nb = -(-flat.size // 128)
        stored = np.zeros(nb * 128, np.int64)
        stored[:flat.size] = flat & 3
        g = i2s_oracle._block_groups(stored.reshape(nb, 128), layout)
        return ((g[..., 0] << 6) | (g[..., 1] << 4) | (g[..., 2] << 2) | g[..., 3]).reshape(-1).astype(np.uint8)

    monkeypatch.setattr(O, "i2s_encode_codes", twos_complement)
    with pytest.raises(AssertionError):
        test_golden_hand_block(golden_dir, "consecutive")


def test_round_trip_property_random_shapes():
    """Random shapes (K % 16 == 0, any N, tails of every length mod 128) and
    random codes: decode(encode(c)) == c in both groupings, and the encoded
    bytes agree with the bit-string construction."""
    rng = np.random.default_rng(20261202)
    for _ in range(60):
        N = int(rng.integers(1, 9))
        K = 16 * int(rng.integers(1, 40))
        codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        for layout in O.I2S_LAYOUTS:
            blocks = O.i2s_encode_codes(codes, layout)
            assert blocks.size == 32 * (-(-(N * K) // 128))
            assert np.array_equal(O.i2s_decode_codes(blocks, N * K, layout), codes.reshape(-1))
            assert np.array_equal(blocks, _bitstring_encode(codes, layout))
