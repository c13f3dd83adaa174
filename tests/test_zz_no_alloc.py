"""bitlinear_forward_noalloc: the forward for callers that cannot allocate.

A plugin inside a framework that owns all device memory, or a C caller with no
device allocator, cannot pass bitlinear_forward a workspace. This entry point
runs the same forward on a fixed scratch array inside the library. These tests
call it through the C ABI and check that it gives the same output as
bitlinear_forward with a caller workspace. They check two calls in a row,
because the scratch is shared and keeps the previous call's contents. They
also check that work larger than the scratch is refused.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL_TOL = 1e-6  # the tolerance the parity tests use for fp32 outputs
BL_ERR_WORKSPACE = 4


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_ternary_b200 import _lib, bitlinear, build, workloads

    build.build_library()
    return _lib.lib(), bitlinear, workloads


def _case(B, WL, M, N, K, seed):
    W = torch.from_numpy(WL.weight(N, K, "laplace", seed)).cuda()
    x = torch.from_numpy(WL.activations(M, K, "outlier_channels", seed,
                                        meta={"frac": 0.01, "scale": 20.0})).cuda()
    packed, D = B.pack_weights(W)
    return x, packed, D


def _noalloc(L, x, packed, D, M, N, K):
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = L.bitlinear_forward_noalloc(x.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr(),
                                     stream)
    assert st == 0, f"bitlinear_forward_noalloc returned {st}"
    torch.cuda.synchronize()
    return y


def _assert_close(y, y_ref):
    a = y.cpu().numpy()
    b = y_ref.cpu().numpy()
    assert np.all(np.isfinite(a))
    den = np.maximum(np.abs(b), np.finfo(np.float32).tiny)
    assert (np.abs(a.astype(np.float64) - b) / den).max() <= REL_TOL


def test_noalloc_matches_forward_on_two_calls_in_a_row(env):
    L, B, WL = env
    # Two different tensor-core-path shapes back to back: the second call finds
    # the first call's data still in the shared scratch.
    for (M, N, K, seed) in [(300, 700, 2560, 11), (96, 1152, 4304, 12)]:
        x, packed, D = _case(B, WL, M, N, K, seed)
        y_ref = B.forward(x, packed, D)  # existing entry point, caller workspace
        y = _noalloc(L, x, packed, D, M, N, K)
        _assert_close(y, y_ref)


def test_noalloc_decode_shape(env):
    L, B, WL = env
    M, N, K = 1, 2560, 2560
    x, packed, D = _case(B, WL, M, N, K, 13)
    _assert_close(_noalloc(L, x, packed, D, M, N, K), B.forward(x, packed, D))


def test_noalloc_rejects_work_larger_than_scratch(env):
    L, _, _ = env
    limit = 16 * 1024 * 1024
    M, K = 8192, 4096  # M*K = 32 MiB of quantised activations > 16 MiB
    assert L.bitlinear_workspace_size(M, 64, K) > limit
    # Refused before any GPU access, so the pointers are never read.
    st = L.bitlinear_forward_noalloc(0x10000, M, 64, K, 0x10000, 0x10000, 0x10000, None)
    assert st == BL_ERR_WORKSPACE
