"""GPU parity of the per-256-block scale variant against its CPU oracle.

"Core AI model zoo - BitVLA", section 2, names BitCPM's per-256-block scale
as the alternative to the per-row D [N, 1]; the reading (blocks of 256
consecutive columns inside a row, per-block absmean, D [N, ceil(K/256)], the
block terms added in fp32 in ascending order) is the one oracle/block_oracle.py
states and tests/test_block_oracle.py pins. Packed codes and D are compared bit
for bit, and so is y (the kernel takes the same fp32 roundings in the same
order), which is stricter than the 1e-6 relative bar.

Blocks are row-local, so full-size weights are checked on a sample of rows:
the oracle quantises only those rows and contracts only with them.
"""
import numpy as np
import pytest

import oracle as O
from bit_ternary_b200 import workloads as WL

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL_TOL = 1e-6


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_ternary_b200 import build, bitlinear, _lib

    build.build_library()
    assert _lib.lib().bitlinear_device_check() == 0, "device is not sm_100"
    return bitlinear


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def assert_y_bitexact(y_gpu, y_ref):
    y_gpu = np.asarray(y_gpu, np.float32)
    assert y_gpu.shape == y_ref.shape
    den = np.maximum(np.abs(y_ref), np.float32(np.finfo(np.float32).tiny))
    rel = np.abs(y_gpu.astype(np.float64) - y_ref.astype(np.float64)) / den
    assert rel.max(initial=0.0) <= REL_TOL
    assert np.array_equal(y_gpu.view(np.uint32), y_ref.view(np.uint32))


def test_hand_examples_gpu(B):
    from test_block_oracle import hand_order_example, hand_tie_example

    for W, x in (hand_tie_example(), hand_order_example()):
        K = W.shape[1]
        packed, D = B.pack_weights_blocks(dev(W))
        p_ref, D_ref = O.pack_weights_blocks(W)
        assert np.array_equal(u32(packed), p_ref)
        assert np.array_equal(D.cpu().numpy().view(np.uint32), D_ref.view(np.uint32))
        y = B.forward_blocks(dev(x), packed, D).cpu().numpy()
        assert_y_bitexact(y, O.bitlinear_forward_blocks(x, p_ref, D_ref, K))
    # the order-dependent row of hand_order_example: 2^14 exactly
    assert y.view(np.uint32)[0, 0] == 0x46800000


PACK_SHAPES = [(1, 16), (3, 272), (17, 528), (33, 1152), (64, 4304), (129, 6912), (2, 131072)]


@pytest.mark.parametrize("N,K", PACK_SHAPES)
@pytest.mark.parametrize("dist", ["normal", "laplace"])
def test_pack_blocks_bitexact(B, N, K, dist):
    W = WL.weight(N, K, dist, N + K)
    packed, D = B.pack_weights_blocks(dev(W))
    p_ref, D_ref = O.pack_weights_blocks(W)
    assert D.shape == (N, O.num_blocks(K))
    assert np.array_equal(u32(packed), p_ref)
    assert np.array_equal(D.cpu().numpy().view(np.uint32), D_ref.view(np.uint32))


def _hard_blocks():
    """Blocks whose mean an fp64 sum cannot round by itself: exact fp32 ties,
    values a hair either side of a tie, exponents far apart (the fp64 sum is
    inexact), subnormals, values near FLT_MAX, and an all-zero block."""
    rows = []
    one = np.ones(256, np.float32)
    for delta in (0.0, 2.0 ** -23, -(2.0 ** -23), 2.0 ** -22):
        r = one.copy()
        r[255] = np.float32(1.0 + 2.0 ** -16 + delta)  # mean 1 + 2^-24 (+ delta/256)
        rows.append(r)
    r = one.copy()
    r[7] = np.float32(3.0 + 2.0 ** -16)  # mean 1 + 2^-7 + 2^-24: a tie in another binade
    rows.append(r)
    # 128 x 2^100 + 2^83 puts the mean on the midpoint of 2^99 and 2^99 + 2^76;
    # 127 values of 2^-100, far below any fp64 sum's resolution, decide it
    # upwards. Without them it is a tie and rounds to the even 2^99.
    for tiny in (2.0 ** -100, 0.0):
        r = np.full(256, np.float32(tiny))
        r[:128] = np.float32(2.0 ** 100)
        r[128] = np.float32(2.0 ** 83)
        rows.append(r)
    rows.append(np.full(256, np.float32(1e-45)))  # the smallest subnormal
    r = np.zeros(256, np.float32)
    r[:3] = np.float32(np.finfo(np.float32).tiny)
    r[3] = np.float32(2.0 ** -149)
    rows.append(r)
    rows.append(np.full(256, np.finfo(np.float32).max))
    r = np.full(256, np.float32(0.375))
    r[200] = np.float32(0.375 + 2.0 ** -10)  # mean 0.375 + 2^-18: exactly representable
    rows.append(r)
    rows.append(np.zeros(256, np.float32))
    W = np.stack(rows).astype(np.float32)
    W[:, 1::3] *= -1  # signs do not enter the mean
    return W


def test_pack_blocks_exact_mean_paths(B):
    W = _hard_blocks()
    W = np.concatenate([W, W[:, :128]], axis=1)  # a second, 128-column block per row
    packed, D = B.pack_weights_blocks(dev(W))
    p_ref, D_ref = O.pack_weights_blocks(W)
    assert np.array_equal(D.cpu().numpy().view(np.uint32), D_ref.view(np.uint32))
    assert np.array_equal(u32(packed), p_ref)
    assert D_ref[0, 0] == np.float32(1.0)  # the tie rounded to even


def test_pack_blocks_nonfinite_rejected(B):
    from bit_ternary_b200._lib import BitLinearError

    W = WL.weight(4, 528, "normal", 3)
    W[2, 300] = np.inf
    with pytest.raises(BitLinearError, match="NONFINITE"):
        B.pack_weights_blocks(dev(W))
    W[2, 300] = np.nan
    with pytest.raises(BitLinearError, match="NONFINITE"):
        B.pack_weights_blocks(dev(W))


FWD_CASES = [
    (1, 1, 16), (1, 33, 272), (3, 257, 528), (16, 100, 1152), (1, 300, 4304), (5, 64, 6912),
    (17, 65, 528), (40, 33, 2560), (1, 7, 131072), (2, 3, 4096 + 16),
    # K % 256 == 0 (one lane per block): few blocks per row, rows across chunk edges
    (1, 1, 256), (3, 5, 256), (2, 70, 512), (1, 33, 1024), (4, 1000, 768), (16, 45, 2048),
    # one token, K % 256 == 0, at most 32 blocks per row (activation codes held in registers)
    (1, 1000, 2560), (1, 77, 6912), (1, 129, 8192), (1, 5, 768), (1, 4097, 512),
    (1, 300, 2048), (1, 1025, 3072),
    # M >= 128: one tensor-core GEMM per block, the epilogue adding each term to y
    (128, 300, 528), (200, 256, 2560), (300, 1000, 1152), (256, 4304, 4304), (129, 33, 6912), (385, 130, 272),
]


@pytest.mark.parametrize("M,N,K", FWD_CASES)
def test_forward_blocks_bitexact(B, M, N, K):
    seed = M * 1000 + N + K
    W = WL.weight(N, K, "laplace", seed)
    W[0, : min(K, 256)] *= np.float32(40.0)  # one block with its own scale
    x = WL.activations(M, K, "student_t", seed, meta={"df": 3.0})
    packed, D = B.pack_weights_blocks(dev(W))
    p_ref, D_ref = O.pack_weights_blocks(W)
    assert np.array_equal(u32(packed), p_ref)
    y = B.forward_blocks(dev(x), packed, D).cpu().numpy()
    assert_y_bitexact(y, O.bitlinear_forward_blocks(x, p_ref, D_ref, K))
    # and again into a poisoned output buffer: every entry is written
    out = torch.full((M, N), float("nan"), device="cuda")
    B.forward_blocks(dev(x), packed, D, out=out)
    assert_y_bitexact(out.cpu().numpy(), O.bitlinear_forward_blocks(x, p_ref, D_ref, K))


def test_forward_blocks_zero_sizes_and_validation(B):
    from bit_ternary_b200._lib import BitLinearError

    W = WL.weight(8, 272, "normal", 5)
    packed, D = B.pack_weights_blocks(dev(W))
    y = B.forward_blocks(torch.zeros((0, 272), device="cuda"), packed, D)
    assert y.shape == (0, 8)
    with pytest.raises(ValueError):
        B.forward_blocks(torch.zeros((1, 272), device="cuda"), packed, D[:, :1].contiguous())
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(BitLinearError, match="WORKSPACE"):
        B.forward_blocks(torch.zeros((1, 272), device="cuda"), packed, D, ws=small)
    # the tensor-core route needs the per-block row sums too: the plain forward workspace is short
    short = torch.empty(B.workspace_size(200, 8, 272), dtype=torch.uint8, device="cuda")
    with pytest.raises(BitLinearError, match="WORKSPACE"):
        B.forward_blocks(torch.zeros((200, 272), device="cuda"), packed, D, ws=short)


def _rows(n, k=64):
    return np.unique(np.concatenate([np.arange(0, n, max(1, n // k)), [n - 1]]))


@pytest.mark.parametrize("key,li,M", [("decode_layer_set", 0, 1), ("decode_layer_set", 2, 1),
                                      ("decode_layer_set", 3, 1), ("siglip_m256", 0, 256),
                                      ("siglip_m256", 1, 256), ("prefill_sweep", 1, 512)])
def test_forward_blocks_workload_shapes_sampled(B, key, li, M):
    """Full-size weights of the workload layers; the oracle packs and contracts
    a sample of weight rows (blocks are row-local), for a sample of tokens."""
    wl = WL.WORKLOADS[key]
    layer = wl.layers[li]
    W = WL.weight(layer.N, layer.K, wl.w_dist, wl.seed, layer=li)
    x = WL.activations(M, layer.K, wl.x_dist, wl.seed, layer=li, meta=wl.meta)
    packed, D = B.pack_weights_blocks(dev(W))
    y = B.forward_blocks(dev(x), packed, D).cpu().numpy()
    rows = _rows(layer.N)
    toks = _rows(M, 16)
    p_ref, D_ref = O.pack_weights_blocks(W[rows])
    assert np.array_equal(u32(packed)[rows], p_ref)
    assert np.array_equal(D.cpu().numpy()[rows].view(np.uint32), D_ref.view(np.uint32))
    y_ref = O.bitlinear_forward_blocks(x[toks], p_ref, D_ref, layer.K)
    assert_y_bitexact(y[np.ix_(toks, rows)], y_ref)


# -------------------------------------------------------------- bf16 inputs
def _bf16(a):
    """fp32 array -> (bf16 bit patterns uint16, the same values as fp32), by truncation."""
    bits = (np.ascontiguousarray(a, np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return bits, O.bf16_to_f32(bits)


@pytest.mark.parametrize("M,N,K", [(1, 300, 2560), (1, 77, 528), (5, 64, 6912), (130, 257, 1152), (1, 129, 8192)])
def test_blocks_bf16_inputs_bitexact(B, M, N, K):
    """bf16 master weights and bf16 activations, widened exactly: the same as
    the fp32 path on the widened values (pack, and each forward route)."""
    Wb, Wf = _bf16(WL.weight(N, K, "laplace", M + N + K))
    xb, xf = _bf16(WL.activations(M, K, "student_t", M + K, meta={"df": 3.0}))
    packed, D = B.pack_weights_blocks(torch.from_numpy(Wb.view(np.int16)).cuda().view(torch.bfloat16))
    p_ref, D_ref = O.pack_weights_blocks(Wf)
    assert np.array_equal(u32(packed), p_ref)
    assert np.array_equal(D.cpu().numpy().view(np.uint32), D_ref.view(np.uint32))
    y = B.forward_blocks(torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16), packed, D).cpu().numpy()
    assert_y_bitexact(y, O.bitlinear_forward_blocks(xf, p_ref, D_ref, K))
