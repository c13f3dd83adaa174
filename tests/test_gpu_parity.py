"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar (numerics of the BitVLA page, sections 1-2, with the readings in the
oracle's header): packed codes, D, int8 activation codes, s_x, row sums and
int32 accumulators are bit-exact; fp32 outputs are within 1e-6 relative of the
oracle (the kernels use the same two correctly rounded steps, so they are
expected to match bit for bit, and that is asserted too where noted).
"""
import json
import os

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


def assert_y_close(y_gpu, y_ref, bitexact=True):
    y_gpu = np.asarray(y_gpu, np.float32)
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu))
    den = np.maximum(np.abs(y_ref), np.float32(np.finfo(np.float32).tiny))
    rel = np.abs(y_gpu.astype(np.float64) - y_ref.astype(np.float64)) / den
    assert rel.max(initial=0.0) <= REL_TOL
    if bitexact:
        assert np.array_equal(y_gpu.view(np.uint32), y_ref.view(np.uint32))


# ------------------------------------------------------------ golden example
def test_golden_hand_example_gpu(B, golden_dir):
    with open(os.path.join(golden_dir, "hand_4x16.json")) as f:
        g = json.load(f)
    W = np.array(g["W"], np.float32)
    x = np.array(g["x"], np.float32)
    packed, D = B.pack_weights(dev(W))
    assert [hex(int(v) & 0xFFFFFFFF) for v in packed.cpu().numpy()[:, 0]] == g["packed_hex"]
    assert np.all(D.cpu().numpy() == np.float32(g["mean"]))
    q, s_x, rs = B.quant_act(dev(x))
    assert np.array_equal(q.cpu().numpy(), np.array(g["q"], np.int8))
    assert np.array_equal(s_x.cpu().numpy(), np.array(g["s_x"], np.float32))
    acc = B.forward_acc(dev(x), packed).cpu().numpy()
    assert np.array_equal(acc, np.array(g["acc"]))
    y = B.forward(dev(x), packed, D).cpu().numpy()
    assert [[hex(int(v)) for v in row] for row in y.view(np.uint32)] == g["y_hex"]


# ------------------------------------------------------------------- pack
PACK_SHAPES = [(1, 16), (3, 48), (17, 496), (31, 528), (33, 1152), (64, 4304), (257, 6912), (2560, 2560)]


@pytest.mark.parametrize("N,K", PACK_SHAPES)
@pytest.mark.parametrize("dist", ["normal", "laplace"])
def test_pack_bitexact(B, N, K, dist):
    W = WL.weight(N, K, dist, 7000 + N + K)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.array_equal(D.cpu().numpy(), D_ref)


def test_pack_full_gate_up_shape(B):
    """Largest weight of the decode layer set (13824 x 2560 = 35.4M weights)."""
    W = WL.weight(13824, 2560, "normal", 1001, layer=2)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.array_equal(D.cpu().numpy(), D_ref)


def test_pack_special_values(B):
    W = WL.weight(8, 64, "normal", 3)
    W[0, :5] = [0.0, -0.0, 1e-45, -1e-42, 3.4e38]  # zeros, subnormals, huge
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.array_equal(D.cpu().numpy(), D_ref)


def test_pack_exact_path_on_mean_ties(B):
    """Tensors whose exact mean of |W| lies on, or a hair off, the midpoint of
    two fp32 values (and one where values 200 binades apart decide it): the
    fp64 pass cannot round these, so the exact integer path must."""
    one = np.ones(256, np.float32)
    cases = []
    for delta in (0.0, 2.0 ** -23, -(2.0 ** -23)):
        r = one.copy()
        r[255] = np.float32(1.0 + 2.0 ** -16 + delta)  # mean 1 + 2^-24 (+ delta / 256)
        cases.append(r.reshape(16, 16))
    for tiny in (2.0 ** -100, 0.0):
        r = np.full(256, np.float32(tiny))
        r[:128] = np.float32(2.0 ** 100)
        r[128] = np.float32(2.0 ** 83)  # mean on the midpoint of 2^99 and 2^99 + 2^76, decided by the tiny values
        cases.append(r.reshape(8, 32))
    for W in cases:
        W = W.copy()
        W[:, 1::3] *= -1
        packed, D = B.pack_weights(dev(W))
        p_ref, D_ref = O.pack_weights(W)
        assert np.array_equal(D.cpu().numpy().view(np.uint32), D_ref.view(np.uint32))
        assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert O.absmean_exact(cases[0]) == np.float32(1.0)


def test_pack_async_back_to_back_sticky_status(B):
    """Asynchronous packs sharing one zero-filled workspace: a non-finite
    weight in the middle is reported once by pack_status, and the packs
    before and after it are still bit-exact."""
    Ws = [WL.weight(64, 528, "normal", 11), WL.weight(33, 1152, "laplace", 12), WL.weight(200, 2560, "normal", 13)]
    Ws[1][5, 17] = np.inf
    ws = B.pack_workspace("cuda")
    outs = [B.pack_weights(dev(W), ws=ws, sync=False) for W in Ws]
    assert B.pack_status(ws) == 5  # BL_ERR_NONFINITE
    assert B.pack_status(ws) == 0  # read and cleared
    for i in (0, 2):
        p_ref, D_ref = O.pack_weights(Ws[i])
        assert np.array_equal(outs[i][0].cpu().numpy().view(np.uint32), p_ref)
        assert np.array_equal(outs[i][1].cpu().numpy(), D_ref)
    out = B.pack_weights(dev(Ws[2]), ws=ws, sync=False)
    assert B.pack_status(ws) == 0
    assert np.array_equal(out[0].cpu().numpy(), outs[2][0].cpu().numpy())


def test_pack_all_zero_uses_floor(B):
    W = np.zeros((4, 32), np.float32)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.all(D.cpu().numpy() == np.float32(1e-5))


def test_pack_nonfinite_rejected(B):
    from bit_ternary_b200._lib import BitLinearError

    W = np.ones((4, 32), np.float32)
    W[2, 7] = np.nan
    with pytest.raises(BitLinearError, match="NONFINITE"):
        B.pack_weights(dev(W))


# --------------------------------------------------------------- ActQuant
@pytest.mark.parametrize("M,K", [(1, 16), (3, 2560), (17, 1152), (64, 6912), (5, 4304)])
def test_quant_act_bitexact(B, M, K):
    x = WL.activations(M, K, "student_t", 77 + K, meta={"df": 3.0})
    if M > 1:
        x[-1] = 0.0  # all-zero token: floor path
    q, s_x, rs = B.quant_act(dev(x))
    q_ref, s_ref = O.act_quant(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)
    assert np.array_equal(rs.cpu().numpy(), q_ref.astype(np.int64).sum(axis=1))


# ---------------------------------------------------------------- forward
def run_case(B, M, N, K, wdist="normal", xdist="normal", seed=0):
    W = WL.weight(N, K, wdist, seed)
    x = WL.activations(M, K, xdist, seed, meta={"df": 3.0, "frac": 0.02, "scale": 20.0})
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    y_ref, parts = O.bitlinear_forward(x, p_ref, D_ref, K, return_parts=True)
    xd = dev(x)
    acc = B.forward_acc(xd, packed).cpu().numpy()
    assert np.array_equal(acc, parts["acc"])
    y = B.forward(xd, packed, D).cpu().numpy()
    assert_y_close(y, y_ref)


GEMV_CASES = [
    (1, 1, 16), (1, 17, 48), (1, 31, 496), (1, 33, 528), (2, 64, 1152), (1, 2560, 2560),
    (4, 100, 4304), (8, 4304, 1152), (9, 257, 6912), (16, 300, 2560), (1, 3840, 2560), (13, 65, 80),
]


@pytest.mark.parametrize("M,N,K", GEMV_CASES)
def test_forward_gemv(B, M, N, K):
    run_case(B, M, N, K, xdist="student_t", seed=M * 1000 + N + K)


@pytest.mark.parametrize("M,N,K", [(1, 2560, 2560), (3, 300, 528), (16, 257, 6912), (1, 33, 48), (200, 129, 1152)])
def test_forward_per_row_scale(B, M, N, K):
    """D is a per-row [N,1] scale: distinct values per row must land on their
    own rows (decode and tensor-core paths)."""
    rng = np.random.default_rng(N * 7 + K)
    W = WL.weight(N, K, "normal", 31)
    x = WL.activations(M, K, "student_t", 32, meta={"df": 3.0})
    packed, _ = B.pack_weights(dev(W))
    p_ref, _ = O.pack_weights(W)
    D_rows = rng.uniform(1e-3, 2.0, size=(N, 1)).astype(np.float32)
    y = B.forward(dev(x), packed, dev(D_rows)).cpu().numpy()
    assert_y_close(y, O.bitlinear_forward(x, p_ref, D_rows, K))


@pytest.mark.parametrize("M", [1, 3, 100])
def test_quant_ties_round_to_even(B, M):
    """Products x*s_x that land exactly on .5 round to even (rint), in the
    decode kernel's own quantiser (M <= 16) and in the ActQuant kernel (M > 16).
    amax = 127 gives s_x = 1, so the codes are rint(x)."""
    K = 64
    halves = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5, 3.5, 4.5], np.float32)
    x = np.zeros((M, K), np.float32)
    for m in range(M):
        row = np.resize(np.roll(halves, m), K)
        row[10 + (7 * m) % (K - 10)] = 127.0 if m % 2 == 0 else -127.0
        x[m] = row
    W = WL.weight(48, K, "normal", 77)
    packed, _ = B.pack_weights(dev(W))
    p_ref, _ = O.pack_weights(W)
    q_ref, s_ref = O.act_quant(x)
    assert np.all(s_ref == 1.0)
    assert q_ref[0, 0] == 0 and q_ref[0, 1] == 2 and q_ref[0, 2] == 2 and q_ref[0, 6] == 126
    _, parts = O.bitlinear_forward(x, p_ref, np.ones((48, 1), np.float32), K, return_parts=True)
    acc = B.forward_acc(dev(x), packed).cpu().numpy()
    assert np.array_equal(acc, parts["acc"])


def test_gemv_streamed_rounds(B):
    """A decode layer too large for one shot of shared memory per CTA
    (~38 MB of packed weights): the kernel streams double-buffered rounds.
    Codes are drawn directly (uniform over {-1,0,1}), D per row; sampled
    rows are checked against the oracle on those rows' weights."""
    M, N, K = 1, 9477, 16384
    rng = np.random.default_rng(99)
    packed = np.empty((N, K // 16), dtype=np.uint32)
    for r0 in range(0, N, 512):
        r1 = min(N, r0 + 512)
        packed[r0:r1] = O.pack_codes(rng.integers(-1, 2, size=(r1 - r0, K), dtype=np.int8))
    D_rows = rng.uniform(1e-3, 2.0, size=(N, 1)).astype(np.float32)
    x = WL.activations(M, K, "student_t", 98, meta={"df": 3.0})
    y = B.forward(dev(x), dev(packed.view(np.int32)), dev(D_rows)).cpu().numpy()
    rows = np.array(sorted(set(range(0, N, 5)) | set(range(N - 40, N))))
    y_ref = O.bitlinear_forward(x, packed[rows], D_rows[rows], K)
    assert_y_close(y[:, rows], y_ref)


GEMM_CASES = [
    (17, 16, 16), (17, 128, 128), (100, 129, 256), (256, 4304, 1152), (256, 1152, 4304),
    (300, 700, 2560), (129, 33, 6912), (512, 384, 528), (1000, 257, 48), (640, 640, 640),
]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_forward_gemm(B, M, N, K):
    run_case(B, M, N, K, wdist="laplace", xdist="outlier_channels", seed=M + N * 7 + K)


def test_gemm_rescale_extreme_token_scales(B):
    """The tensor-core epilogue divides by s_x through a reciprocal with two
    FMA corrections. Tokens whose max|x| spans 1e-30 .. 3e38 (s_x from ~1e32
    down to ~4e-37, quotients from 0 to beyond the fp32 range, where the
    IEEE division takes over) must still match the oracle bit for bit,
    infinities included."""
    M, N, K = 160, 96, 512
    W = WL.weight(N, K, "normal", 77)
    x = WL.activations(M, K, "normal", 78)
    with np.errstate(over="ignore"):
        scales = (10.0 ** np.linspace(-31, 38, M)).astype(np.float32)
        x = (x * scales[:, None]).astype(np.float32)
    x[~np.isfinite(x)] = np.float32(3e38)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    y = B.forward(dev(x), packed, D).cpu().numpy()
    with np.errstate(over="ignore"):
        y_ref = O.bitlinear_forward(x, p_ref, D_ref, K)
    assert np.array_equal(y.view(np.uint32), y_ref.view(np.uint32))
    assert np.isinf(y_ref).any() and np.isfinite(y_ref).any()


def test_gemm_edge_zero_tokens_and_rows(B):
    """All-zero token (floor path) and rows whose weights ternarise to 0."""
    M, N, K = 40, 200, 512
    W = WL.weight(N, K, "normal", 5)
    W[3] = 1e-9  # ternarises to all zeros
    x = WL.activations(M, K, "normal", 5)
    x[7] = 0.0
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    y_ref = O.bitlinear_forward(x, p_ref, D_ref, K)
    y = B.forward(dev(x), packed, D).cpu().numpy()
    assert_y_close(y, y_ref)
    assert np.all(y[7] == 0.0)


def test_output_written_exactly(B):
    """Every element of y is written, nothing past it (poisoned guard), and the
    values match the oracle."""
    # (37, 131): plain-store epilogue (N % 4 != 0); (37, 132) and (300, 260):
    # TMA bulk-store epilogue, which must clip the M and N tails.
    for (M, N, K) in [(1, 33, 64), (37, 131, 272), (37, 132, 272), (300, 260, 528)]:
        W = WL.weight(N, K, "normal", 1)
        x = WL.activations(M, K, "normal", 1)
        packed, D = B.pack_weights(dev(W))
        buf = torch.full((M * N + 4096,), float("nan"), device="cuda")
        y = buf[: M * N].view(M, N)
        B.forward(dev(x), packed, D, out=y)
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
        assert torch.isnan(buf[M * N:]).all()
        p_ref, D_ref = O.pack_weights(W)
        assert_y_close(y.cpu().numpy(), O.bitlinear_forward(x, p_ref, D_ref, K))


def test_D_row_layout_enforced(B):
    W = WL.weight(8, 32, "normal", 2)
    packed, D = B.pack_weights(dev(W))
    with pytest.raises(ValueError, match=r"\[N, 1\]"):
        B.forward(dev(np.ones((1, 32), np.float32)), packed, D.reshape(1, -1))


def test_forward_host_matches_device(B):
    M, N, K = 3, 500, 1024
    W = WL.weight(N, K, "normal", 9)
    x = WL.activations(M, K, "normal", 9)
    packed, D = B.pack_weights(dev(W))
    y_dev = B.forward(dev(x), packed, D).cpu().numpy()
    xh = torch.from_numpy(x).pin_memory()
    y_host = B.forward_host(xh, packed, D).numpy()
    assert np.array_equal(y_dev.view(np.uint32), y_host.view(np.uint32))
    # and the tensor-core path
    M = 300
    x = WL.activations(M, K, "normal", 10)
    y_dev = B.forward(dev(x), packed, D).cpu().numpy()
    y_host = B.forward_host(torch.from_numpy(x).pin_memory(), packed, D).numpy()
    assert np.array_equal(y_dev.view(np.uint32), y_host.view(np.uint32))


def test_forward_host_async_shared_workspace(B):
    """Several asynchronous host calls on one stream share a workspace; after
    one synchronise every y_host holds its own result (decode and GEMM paths)."""
    shapes = [(1, 3840, 2560), (1, 2560, 2560), (5, 700, 1152), (40, 300, 512)]
    calls, refs = [], []
    for i, (M, N, K) in enumerate(shapes):
        W = WL.weight(N, K, "normal", 900 + i)
        x = WL.activations(M, K, "student_t", 910 + i, meta={"df": 3.0})
        packed, D = B.pack_weights(dev(W))
        calls.append((torch.from_numpy(x).pin_memory(), packed, D,
                      torch.empty((M, N), dtype=torch.float32).pin_memory()))
        refs.append(_oracle_y(W, x))
    L = __import__("bit_ternary_b200._lib", fromlist=["lib"]).lib()
    ws_bytes = max(L.bitlinear_host_workspace_size(M, N, K) for (M, N, K) in shapes)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    for xh, packed, D, yh in calls:
        B.forward_host(xh, packed, D, y_host=yh, ws=ws, sync=False)
    torch.cuda.current_stream().synchronize()
    for (_, _, _, yh), ref in zip(calls, refs):
        assert_y_close(yh.numpy(), ref)
    with pytest.raises(ValueError):
        B.forward_host(torch.zeros(1, 16), calls[0][1][:, :1].contiguous(), calls[0][2], sync=False)


@pytest.mark.parametrize("M,N,K", [(1, 300, 2560), (16, 257, 6912), (5, 33, 4304), (37, 257, 528),
                                   (300, 700, 1152)])
def test_forward_q_from_quant_act(B, M, N, K):
    """forward_q on quant_act's natural-order codes equals the oracle's
    contraction and rescale of the same codes; arbitrary codes (-128 included)
    and scales too."""
    W = WL.weight(N, K, "normal", 60 + K)
    x = WL.activations(M, K, "student_t", 61 + M, meta={"df": 3.0})
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    q, s_x, _ = B.quant_act(dev(x))
    y = B.forward_q(q, s_x, packed, D).cpu().numpy()
    assert_y_close(y, O.bitlinear_forward(x, p_ref, D_ref, K))
    rng = np.random.default_rng(M + N + K)
    q2 = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    s2 = rng.uniform(0.5, 300.0, size=M).astype(np.float32)
    codes = O.unpack_codes(p_ref, K)
    y_ref = O.rescale(O.int_matmul(q2, codes), s2, D_ref)
    y2 = B.forward_q(dev(q2), dev(s2), packed, D).cpu().numpy()
    assert_y_close(y2, y_ref)


def test_workspace_error_word_clear_after_gemm(B):
    M, N, K = 200, 256, 512
    W = WL.weight(N, K, "normal", 4)
    x = WL.activations(M, K, "normal", 4)
    packed, D = B.pack_weights(dev(W))
    ws = torch.full((B.workspace_size(M, N, K),), 0x5A, dtype=torch.uint8, device="cuda")
    B.forward(dev(x), packed, D, ws=ws)
    assert B.workspace_error(ws) == 0


def test_misaligned_and_small_workspace_rejected(B):
    from bit_ternary_b200._lib import BitLinearError

    M, N, K = 2, 64, 64
    W = WL.weight(N, K, "normal", 4)
    packed, D = B.pack_weights(dev(W))
    x = torch.zeros(M * K + 1, device="cuda")[1:].view(M, K)  # 4-byte offset
    with pytest.raises(BitLinearError, match="ALIGN"):
        B.forward(x, packed, D)
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(BitLinearError, match="WORKSPACE"):
        B.forward(torch.zeros(M, K, device="cuda"), packed, D, ws=small)


# ------------------------------------------------ workload shapes (full size)
def _layer_case(B, key, li, M, rows=None):
    wl = WL.WORKLOADS[key]
    layer = wl.layers[li]
    W = WL.weight(layer.N, layer.K, wl.w_dist, wl.seed, layer=li)
    x = WL.activations(M, layer.K, wl.x_dist, wl.seed, layer=li, meta=wl.meta)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    y = B.forward(dev(x), packed, D).cpu().numpy()
    if rows is None:
        y_ref = O.bitlinear_forward(x, p_ref, D_ref, layer.K)
        assert_y_close(y, y_ref)
    else:
        y_ref = O.bitlinear_forward_rows(x, p_ref, D_ref, layer.K, rows)
        assert_y_close(y[rows], y_ref)


@pytest.mark.parametrize("li", range(4))
def test_decode_layer_set_full(B, li):
    _layer_case(B, "decode_layer_set", li, 1)


def test_decode_2560_full(B):
    _layer_case(B, "decode_2560", 0, 1)


@pytest.mark.parametrize("li", range(2))
def test_siglip_full(B, li):
    _layer_case(B, "siglip_m256", li, 256)


def _sample_rows(M, extra=()):
    rows = set(range(0, M, 64)) | {0, M - 1} | set(int(r) for r in extra)
    return np.array(sorted(rows))


@pytest.mark.parametrize("li", range(3))
@pytest.mark.parametrize("M", [512, 2048, 4096])
def test_prefill_sweep_sampled(B, li, M):
    _layer_case(B, "prefill_sweep", li, M, rows=_sample_rows(M))


@pytest.mark.parametrize("kind", ["acc", "n_tail"])
def test_gemm_wide_tiles_output_paths(B, kind):
    """Launches large enough for the 192-token tiles, through the two output
    paths the prefill sweep does not reach: the exact int32 accumulators
    (bitlinear_forward_acc), and y rows that do not start on a 16-byte
    boundary (N % 4 != 0: plain stores instead of TMA stores). Sampled token
    rows, every output column."""
    M, K = 4096, 2560
    N = 13824 if kind == "acc" else 3843
    W = WL.weight(N, K, "laplace", 71)
    x = WL.activations(M, K, "normal", 72)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    rows = _sample_rows(M, extra=(4095 - 64, 191, 192))  # either side of a 192-token tile edge
    if kind == "acc":
        acc = B.forward_acc(dev(x), packed).cpu().numpy()
        q, _ = O.act_quant(x[rows])
        acc_ref = O.int_matmul(q, O.unpack_codes(p_ref, K))
        assert np.array_equal(acc[rows].astype(np.int64), acc_ref)
    else:
        y = B.forward(dev(x), packed, D).cpu().numpy()
        y_ref = O.bitlinear_forward_rows(x, p_ref, D_ref, K, rows)
        assert_y_close(y[rows], y_ref)


@pytest.mark.parametrize("li", range(6))
def test_embed_batch_sampled(B, li):
    M = 32768
    seed = WL.WORKLOADS["embed_batch"].seed
    _layer_case(B, "embed_batch", li, M, rows=_sample_rows(M, WL.outlier_rows(M, seed)))


def test_bounded_wait_reports_device_error(B):
    """A barrier wait that can never complete gives up within its limit and the
    host sees BL_ERR_DEVICE; the context stays usable afterwards."""
    import time

    from bit_ternary_b200 import _lib

    L = _lib.lib()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    assert L.bitlinear_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 20_000_000, stream) == 0
    assert L.bitlinear_workspace_error(ws.data_ptr(), ws.numel(), stream) == 6  # BL_ERR_DEVICE
    assert time.perf_counter() - t0 < 5.0
    assert int(ws[:4].view(torch.int32).item()) == 0  # cleared by the read
    assert L.bitlinear_workspace_error(ws.data_ptr(), ws.numel(), stream) == 0
    run_case(B, 2, 40, 64, seed=3)  # the context still works


# ------------------------------------------------------------ batched calls
def _oracle_y(W, x):
    p_ref, D_ref = O.pack_weights(W)
    return O.bitlinear_forward(x, p_ref, D_ref, W.shape[1])


@pytest.mark.parametrize("flags", [0, 1])
def test_forward_batch_grouped_matches_oracle(B, flags):
    """Decode-sized calls of different shapes fused into grouped launches, with
    a tensor-core call in the middle and a group split by the 8-call limit."""
    shapes = [(1, 3840, 2560), (1, 2560, 2560), (2, 100, 528), (1, 13824 // 8, 2560), (3, 257, 6912),
              (40, 300, 512),  # tensor-core path in the middle
              (1, 33, 48), (16, 64, 1152), (1, 17, 16), (1, 500, 1024), (1, 64, 64), (5, 31, 4304),
              (1, 48, 256), (2, 129, 2560)]
    calls, refs = [], []
    for i, (M, N, K) in enumerate(shapes):
        W = WL.weight(N, K, "normal", 500 + i)
        x = WL.activations(M, K, "student_t", 600 + i, meta={"df": 3.0})
        packed, D = B.pack_weights(dev(W))
        calls.append((dev(x), packed, D, None))
        refs.append(_oracle_y(W, x))
    outs = B.forward_batch(calls, flags=flags)
    torch.cuda.synchronize()
    for y, ref in zip(outs, refs):
        assert_y_close(y.cpu().numpy(), ref)


def test_forward_batch_chain_with_early_weights(B):
    """A dependent chain (each call's x is the previous call's y) with the
    early-weights flag: activations must still be read only after the
    previous kernel finished."""
    K = 2560
    Ws = [WL.weight(K, K, "normal", 700 + i) for i in range(4)]
    packs = [B.pack_weights(dev(W)) for W in Ws]
    x0 = WL.activations(1, K, "normal", 7)
    xd = dev(x0)
    for (packed, D) in packs:
        (xd,) = B.forward_batch([(xd, packed, D, None)], flags=1)
    torch.cuda.synchronize()
    ref = x0
    for W in Ws:
        ref = _oracle_y(W, ref)
    assert_y_close(xd.cpu().numpy(), ref)


def test_forward_batch_rejects_before_launch(B):
    from bit_ternary_b200._lib import BitLinearError

    W = WL.weight(64, 64, "normal", 1)
    packed, D = B.pack_weights(dev(W))
    good = (dev(np.ones((1, 64), np.float32)), packed, D, None)
    bad_y = torch.zeros(1 * 64 + 1, device="cuda")[1:].view(1, 64)
    with pytest.raises(BitLinearError, match="ALIGN"):
        B.forward_batch([good, (good[0], packed, D, bad_y)])


@pytest.mark.parametrize("flags", [2, 3])
def test_forward_batch_one_launch_per_call(B, flags):
    """Every call in its own launch (with and without early weights): the same
    bits as the grouped launches, and the oracle's."""
    shapes = [(1, 2560, 2560), (2, 100, 528), (1, 33, 48), (40, 300, 512), (16, 64, 1152), (3, 257, 6912)]
    calls, refs = [], []
    for i, (M, N, K) in enumerate(shapes):
        W = WL.weight(N, K, "normal", 800 + i)
        x = WL.activations(M, K, "normal", 900 + i)
        packed, D = B.pack_weights(dev(W))
        calls.append((dev(x), packed, D, None))
        refs.append(_oracle_y(W, x))
    outs = B.forward_batch(calls, flags=flags)
    grouped = B.forward_batch(calls, flags=0)
    torch.cuda.synchronize()
    for y, g, ref in zip(outs, grouped, refs):
        assert_y_close(y.cpu().numpy(), ref)
        assert torch.equal(y, g)


def _pinned(a):
    t = torch.empty(a.shape, dtype=torch.float32, pin_memory=True)
    t.copy_(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)))
    return t


@pytest.mark.parametrize("flags", [0, 3])
def test_forward_batch_host(B, flags):
    """Host activations and outputs: views of one pinned buffer (merged
    copies), a call with its own buffers, blocks whose bytes are not a
    multiple of 16, an empty call, and a tensor-core call."""
    shapes = [(1, 2560, 2560), (3, 33, 48), (0, 64, 64), (2, 129, 528), (40, 300, 512), (1, 17, 16)]
    Ws = [WL.weight(N, K, "normal", 1000 + i) for i, (M, N, K) in enumerate(shapes)]
    xs = [WL.activations(M, K, "student_t", 1100 + i, meta={"df": 3.0}) for i, (M, N, K) in enumerate(shapes)]
    packs = [B.pack_weights(dev(W)) for W in Ws]
    x_all = torch.empty(sum(M * K for M, N, K in shapes), dtype=torch.float32, pin_memory=True)
    y_all = torch.full((sum(M * N for M, N, K in shapes),), float("nan"), dtype=torch.float32, pin_memory=True)
    calls, xo, yo = [], 0, 0
    for i, (M, N, K) in enumerate(shapes):
        xv = x_all[xo:xo + M * K].view(M, K)
        yv = y_all[yo:yo + M * N].view(M, N)
        xo += M * K
        yo += M * N
        if i == 3:  # its own buffers: breaks both runs
            xv = _pinned(np.zeros((M, K), np.float32))
            yv = torch.empty((M, N), dtype=torch.float32, pin_memory=True)
        xv.copy_(torch.from_numpy(xs[i]))
        calls.append((xv, packs[i][0], packs[i][1], yv))
    outs = B.forward_batch_host(calls, flags=flags)
    torch.cuda.synchronize()
    for i, (y, W, x) in enumerate(zip(outs, Ws, xs)):
        assert y.data_ptr() == calls[i][3].data_ptr()
        assert_y_close(y.numpy(), _oracle_y(W, x))
    # every slot of the shared output buffer that a call owns was written
    yo = 0
    for i, (M, N, K) in enumerate(shapes):
        if i != 3:
            assert not torch.isnan(y_all[yo:yo + M * N]).any()
        yo += M * N


def test_forward_batch_host_chain_reuses_workspace(B):
    """Repeated batched host calls on one stream and one workspace, each
    feeding its output back as the next input."""
    K = 1024
    W = WL.weight(K, K, "normal", 1200)
    packed, D = B.pack_weights(dev(W))
    x0 = WL.activations(2, K, "normal", 1201)
    xh = _pinned(x0)
    yh = torch.empty((2, K), dtype=torch.float32, pin_memory=True)
    ws = None
    ref = x0
    for _ in range(3):
        if ws is None:
            ws = torch.empty(B.batch_host_workspace_size([(2, K, K)]), dtype=torch.uint8, device="cuda")
        B.forward_batch_host([(xh, packed, D, yh)], flags=1, ws=ws)
        torch.cuda.synchronize()
        ref = _oracle_y(W, ref)
        assert_y_close(yh.numpy(), ref)
        xh.copy_(yh)


# ------------------------------------------------------------ bf16 inputs
def _bf16(a):
    """fp32 numpy array -> (bf16 CUDA tensor, its uint16 bit patterns)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.cuda(), bits


@pytest.mark.parametrize("N,K,dist", [(3, 48, "normal"), (257, 6912, "laplace"), (2560, 2560, "normal"),
                                      (33, 1152, "laplace")])
def test_pack_bf16_bitexact(B, N, K, dist):
    Wt, bits = _bf16(WL.weight(N, K, dist, 40 + K))
    packed, D = B.pack_weights(Wt)
    p_ref, D_ref = O.pack_weights_bf16(bits)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.array_equal(D.cpu().numpy(), D_ref)


def test_pack_bf16_special_values(B):
    bits = np.array([[0x0001, 0x8001, 0x0000, 0x8000, 0x3F80, 0xBF80, 0x0080, 0x7F7F] * 2], dtype=np.uint16)
    Wt = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    packed, D = B.pack_weights(Wt)
    p_ref, D_ref = O.pack_weights_bf16(bits)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.array_equal(D.cpu().numpy(), D_ref)


@pytest.mark.parametrize("M,K", [(1, 2560), (3, 528), (64, 6912), (17, 16400)])
def test_quant_act_bf16_bitexact(B, M, K):
    xt, bits = _bf16(WL.activations(M, K, "student_t", 50 + K, meta={"df": 3.0}))
    q, s_x, rs = B.quant_act(xt)
    q_ref, s_ref = O.act_quant_bf16(bits)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)
    assert np.array_equal(rs.cpu().numpy(), q_ref.astype(np.int64).sum(axis=1))


@pytest.mark.parametrize("M,N,K", [(1, 3840, 2560), (1, 2560, 6912), (5, 257, 528), (16, 300, 2560),
                                   (40, 700, 1152), (300, 129, 6912)])
def test_forward_bf16(B, M, N, K):
    """bf16 master weight and bf16 activations, decode (M <= 16) and tensor-core paths."""
    Wt, wbits = _bf16(WL.weight(N, K, "normal", 70 + N))
    xt, xbits = _bf16(WL.activations(M, K, "student_t", 71 + M, meta={"df": 3.0}))
    packed, D = B.pack_weights(Wt)
    p_ref, D_ref = O.pack_weights_bf16(wbits)
    y = B.forward(xt, packed, D).cpu().numpy()
    assert_y_close(y, O.bitlinear_forward_bf16(xbits, p_ref, D_ref, K))


# --------------------------------------------------- RMSNorm + ActQuant
@pytest.mark.parametrize("K", [1024, 2560])
def test_rmsnorm_quant_act_many_tokens_per_cta(B, K):
    """Enough tokens that every persistent CTA of the RMSNorm quantiser walks
    many of them (the next row's loads in flight while the current one is
    quantised): sampled tokens, including both ends, bit for bit."""
    M = 20000
    x = WL.activations(M, K, "outlier_tokens", 90 + K, meta={"frac": 0.02, "scale": 20.0})
    g = np.random.default_rng(91 + K).uniform(0.5, 2.0, K).astype(np.float32)
    q, s_x, rs = B.rmsnorm_quant_act(dev(x), dev(g))
    rows = _sample_rows(M, extra=(1, 147, 148, 149, 1775, 1776, 1777, M - 2))
    q_ref, s_ref = O.rmsnorm_act_quant(x[rows], g)
    assert np.array_equal(q.cpu().numpy()[rows], q_ref)
    assert np.array_equal(s_x.cpu().numpy()[rows], s_ref)
    assert np.array_equal(rs.cpu().numpy()[rows], q_ref.astype(np.int64).sum(axis=1))


@pytest.mark.parametrize("M,K,xdist", [(1, 2560, "student_t"), (5, 1024, "outlier_tokens"), (64, 3072, "normal"),
                                       (300, 640, "student_t"), (17, 16384, "normal")])
def test_rmsnorm_quant_act_bitexact(B, M, K, xdist):
    x = WL.activations(M, K, xdist, 80 + K, meta={"df": 3.0, "frac": 0.02, "scale": 20.0})
    x[0, :5] = 0.0
    g = np.random.default_rng(K).uniform(0.5, 2.0, K).astype(np.float32)
    q, s_x, rs = B.rmsnorm_quant_act(dev(x), dev(g))
    q_ref, s_ref = O.rmsnorm_act_quant(x, g)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)
    assert np.array_equal(rs.cpu().numpy(), q_ref.astype(np.int64).sum(axis=1))


def test_rmsnorm_exact_path_on_rounding_ties_and_zero_row(B):
    """Rows whose mean square is an exact fp32 rounding tie (or a hair above
    one) leave the fp64 interval ambiguous, so the kernel takes the exact
    integer path; an all-zero row gives ms = 0; a tiny row gives a subnormal ms."""
    B2 = B
    K = 64
    rows = [np.full(K, 1 + 2.0 ** -12, np.float32), np.full(K, 1 + 3 * 2.0 ** -12, np.float32),
            np.full(K, 1 + 2.0 ** -12 + 2.0 ** -23, np.float32), np.zeros(K, np.float32),
            np.full(K, 3.0 * 2.0 ** -70, np.float32)]
    x = np.stack(rows)
    g = np.linspace(0.5, 1.5, K).astype(np.float32)
    q, s_x, _ = B2.rmsnorm_quant_act(dev(x), dev(g))
    q_ref, s_ref = O.rmsnorm_act_quant(x, g)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)


@pytest.mark.parametrize("M,N,K", [(1, 3840, 2560), (1, 2560, 6912), (8, 300, 4304), (37, 700, 1024),
                                   (300, 1024, 3072), (16, 129, 528), (9, 64, 16384)])
def test_forward_rmsnorm(B, M, N, K):
    W = WL.weight(N, K, "normal", 90 + N)
    x = WL.activations(M, K, "outlier_tokens", 91 + M, meta={"df": 3.0, "frac": 0.02, "scale": 20.0})
    g = np.random.default_rng(N).uniform(0.5, 2.0, K).astype(np.float32)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    y = B.forward_rmsnorm(dev(x), dev(g), packed, D).cpu().numpy()
    assert_y_close(y, O.bitlinear_forward_rmsnorm(x, g, p_ref, D_ref, K))


def test_forward_rmsnorm_decode_exact_path(B):
    """The decode kernel's own RMSNorm: rows whose mean square sits on (or a
    hair from) an fp32 rounding tie take the exact integer path, a zero row
    gives ms = 0, a tiny row a subnormal ms; outputs equal the oracle's."""
    K, N = 64, 40
    rows = [np.full(K, 1 + 2.0 ** -12, np.float32), np.full(K, 1 + 3 * 2.0 ** -12, np.float32),
            np.full(K, 1 + 2.0 ** -12 + 2.0 ** -23, np.float32), np.zeros(K, np.float32),
            np.full(K, 3.0 * 2.0 ** -70, np.float32)]
    x = np.stack(rows)
    x[:, ::3] *= -1.0
    g = np.linspace(0.5, 1.5, K).astype(np.float32)
    W = WL.weight(N, K, "normal", 95)
    packed, D = B.pack_weights(dev(W))
    p_ref, D_ref = O.pack_weights(W)
    y = B.forward_rmsnorm(dev(x), dev(g), packed, D).cpu().numpy()
    assert_y_close(y, O.bitlinear_forward_rmsnorm(x, g, p_ref, D_ref, K))


@pytest.mark.parametrize("M,K", [(1, 2560), (16, 6912), (3, 528), (300, 1152)])
def test_forward_prepared_shares_one_quantisation(B, M, K):
    """prepare_act once, then forward_prepared with three weights (decode
    kernel for M <= 16, tensor-core kernel above): each equals the oracle."""
    x = WL.activations(M, K, "student_t", 110 + M, meta={"df": 3.0})
    ws = torch.zeros(B.workspace_size(M, 1, K), dtype=torch.uint8, device="cuda")
    B.prepare_act(dev(x), ws)
    for i, N in enumerate([300, 17, 2560]):
        W = WL.weight(N, K, "laplace", 120 + i)
        packed, D = B.pack_weights(dev(W))
        p_ref, D_ref = O.pack_weights(W)
        y = B.forward_prepared(M, K, packed, D, ws).cpu().numpy()
        assert_y_close(y, O.bitlinear_forward(x, p_ref, D_ref, K))
    assert B.workspace_error(ws) == 0


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (1, 1, 4304), (2, 15, 64), (7, 4305, 1152), (16, 16, 16),
                                   (1, 65536, 256), (3, 97, 16384)])
def test_decode_ring_shapes(B, M, N, K):
    """Decode kernel edge shapes: single words, one-row problems with a row
    that is not 16-byte aligned, N tails, many small tiles per CTA (a ring of
    many tiles that wraps), and tiles of 64 KB (K = 16384)."""
    run_case(B, M, N, K, xdist="student_t", seed=3 * M + N + K)


# ------------------------------------------------------------ I2_S import/export
I2S_SHAPES = [(1, 16), (3, 48), (5, 1152), (17, 4304), (2560, 2560), (7, 6912)]


@pytest.mark.parametrize("layout", ["consecutive", "quarters"])
@pytest.mark.parametrize("N,K", I2S_SHAPES)
def test_i2s_export_bitexact(B, layout, N, K):
    W = WL.weight(N, K, "normal", 1300 + K + N)
    p_ref, D_ref = O.pack_weights(W)
    buf = B.i2s_export(dev(p_ref.view(np.int32)), dev(D_ref), layout)
    assert np.array_equal(buf.cpu().numpy(), O.i2s_export(p_ref, D_ref, K, layout))


@pytest.mark.parametrize("layout", ["consecutive", "quarters"])
@pytest.mark.parametrize("N,K", I2S_SHAPES)
def test_i2s_import_bitexact_arbitrary_codes(B, layout, N, K):
    """Random valid fields (not only what a pack produces) and random bytes in
    the tail padding, with a scale that is not a power of two."""
    rng = np.random.default_rng(N * 131 + K)
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    blocks = O.i2s_encode_codes(codes, layout)
    pad = blocks.size * 4 - N * K  # padding values at the end of the last block
    if pad:
        # overwrite the padding fields of the last block with random 2-bit values, 3 included
        got = O.i2s_decode_codes(blocks, N * K, layout)
        assert np.array_equal(got, codes.reshape(-1))
        last = blocks[-32:].copy()
        junk = rng.integers(0, 256, size=32).astype(np.uint8)
        order = np.arange(128).reshape(32, 4) if layout == "consecutive" else np.arange(128).reshape(4, 32).T
        for byte in range(32):
            for f in range(4):
                v = order[byte, f]  # value index within the block
                if (blocks.size - 32) * 4 + v >= N * K:
                    sh = 6 - 2 * f
                    last[byte] = (int(last[byte]) & (0xFF ^ (3 << sh))) | (int(junk[byte]) & (3 << sh))
        blocks = np.concatenate([blocks[:-32], last])
    scale = np.float32(7.3)
    buf = np.concatenate([blocks, np.array([scale], "<f4").view(np.uint8)])
    packed, D = B.i2s_import(dev(buf), N, K, layout)
    p_ref, D_ref = O.i2s_import(buf, N, K, layout)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    assert np.array_equal(D.cpu().numpy(), D_ref)


@pytest.mark.parametrize("layout", ["consecutive", "quarters"])
def test_i2s_round_trip_and_forward(B, layout):
    """pack -> export -> import gives the same codes; the forward from the
    imported weights equals the oracle's forward with the imported D."""
    N, K, M = 300, 1152, 5
    W = WL.weight(N, K, "laplace", 1400)
    x = WL.activations(M, K, "normal", 1401)
    packed, D = B.pack_weights(dev(W))
    buf = B.i2s_export(packed, D, layout)
    assert np.array_equal(buf.cpu().numpy(), O.i2s_from_weight(W, layout))
    p2, D2 = B.i2s_import(buf, N, K, layout)
    assert torch.equal(p2, packed)
    p_ref, D_ref = O.i2s_import(buf.cpu().numpy(), N, K, layout)
    assert np.array_equal(D2.cpu().numpy(), D_ref)
    y = B.forward(dev(x), p2, D2)
    torch.cuda.synchronize()
    assert_y_close(y.cpu().numpy(), O.bitlinear_forward(x, p_ref, D_ref, K))


def test_i2s_rejects_invalid_buffers(B):
    from bit_ternary_b200._lib import BitLinearError

    N, K = 3, 48
    W = WL.weight(N, K, "normal", 1500)
    p_ref, D_ref = O.pack_weights(W)
    good = O.i2s_export(p_ref, D_ref, K)
    for layout in ("consecutive", "quarters"):
        bad = good.copy()
        bad[5] |= 0x0C  # a data value holds 3
        with pytest.raises(BitLinearError, match="FORMAT"):
            B.i2s_import(dev(bad), N, K, layout)
    for scale in (0.0, -2.0, np.nan, np.inf, 1e-45):
        b = good.copy()
        b[-4:] = np.array([scale], "<f4").view(np.uint8)
        with pytest.raises(BitLinearError, match="FORMAT"):
            B.i2s_import(dev(b), N, K)
    D_rows = D_ref.copy()
    D_rows[2, 0] *= 2
    with pytest.raises(BitLinearError, match="FORMAT"):
        B.i2s_export(dev(p_ref.view(np.int32)), dev(D_rows))
    p3 = p_ref.copy()
    p3[1, 2] |= np.uint32(3 << 10)  # a packed field holds 3
    with pytest.raises(BitLinearError, match="FORMAT"):
        B.i2s_export(dev(p3.view(np.int32)), dev(D_ref))
    # the context still works, and a good buffer still imports
    packed, D = B.i2s_import(dev(good), N, K)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)


def test_i2s_async_conversions_share_one_status_word(B):
    """Several asynchronous conversions with one status check; a bad buffer
    among them sets the word, the read clears it."""
    ws = B.i2s_workspace("cuda")
    outs = []
    for i, (N, K) in enumerate([(3, 48), (64, 1152), (5, 4304)]):
        W = WL.weight(N, K, "normal", 1600 + i)
        p_ref, D_ref = O.pack_weights(W)
        for layout in ("consecutive", "quarters"):
            buf = B.i2s_export(dev(p_ref.view(np.int32)), dev(D_ref), layout, ws=ws, sync=False)
            outs.append((B.i2s_import(buf, N, K, layout, ws=ws, sync=False), buf, p_ref, D_ref, K, layout))
    assert B.i2s_status(ws) == 0
    for (packed, D), buf, p_ref, D_ref, K, layout in outs:
        assert np.array_equal(buf.cpu().numpy(), O.i2s_export(p_ref, D_ref, K, layout))
        assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)
    bad = outs[0][1].clone()
    bad[0] = 0xFF
    B.i2s_import(bad, 3, 48, ws=ws, sync=False)
    B.i2s_import(outs[0][1], 3, 48, ws=ws, sync=False)
    assert B.i2s_status(ws) == 9
    assert B.i2s_status(ws) == 0


@pytest.mark.parametrize("M", [1, 3])
def test_decode_stacked_weights_stream(B, M):
    """The decode kernel over 16 stacked copies of the gate_up weight (221184
    rows, the streaming measurement's shape): every block of 13824 rows equals
    the oracle's output for one copy, bit for bit."""
    W = WL.weight(13824, 2560, "normal", 1700)
    x = WL.activations(M, 2560, "normal", 1701)
    p_ref, D_ref = O.pack_weights(W)
    ref = O.bitlinear_forward(x, p_ref, D_ref, 2560)
    packed = dev(p_ref.view(np.int32)).repeat(16, 1).contiguous()
    D = dev(D_ref).repeat(16, 1).contiguous()
    y = B.forward(dev(x), packed, D)
    torch.cuda.synchronize()
    assert_y_close(y.cpu().numpy(), np.tile(ref, (1, 16)))
