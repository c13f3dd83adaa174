"""bitlinear_forward_noalloc: the forward for callers that cannot allocate.

A plugin inside a framework that owns all device memory, or a C caller with no
device allocator, cannot pass bitlinear_forward a workspace. This entry point
runs the same forward on a fixed scratch array inside the library. These tests
call it through the C ABI and check its output bit for bit against the CPU
oracle and against bitlinear_forward with a caller workspace. They check two
calls in a row, because the scratch is shared and keeps the previous call's
contents. They also check that work larger than the scratch is refused, and
that a device-side failure recorded in the scratch reaches the caller through
bitlinear_noalloc_error.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest

import oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

BL_ERR_WORKSPACE = 4
BL_ERR_DEVICE = 6


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_ternary_b200 import _lib, bitlinear, build, workloads

    build.build_library()
    return _lib.lib(), bitlinear, workloads


def _case(B, WL, M, N, K, seed):
    W = WL.weight(N, K, "laplace", seed)
    x = WL.activations(M, K, "outlier_channels", seed, meta={"frac": 0.01, "scale": 20.0})
    packed, D = B.pack_weights(torch.from_numpy(W).cuda())
    p_ref, D_ref = O.pack_weights(W)
    return x, packed, D, O.bitlinear_forward(x, p_ref, D_ref, K)


def _noalloc(L, x, packed, D, M, N, K):
    xd = torch.from_numpy(x).cuda()
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = L.bitlinear_forward_noalloc(xd.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr(),
                                     stream)
    assert st == 0, f"bitlinear_forward_noalloc returned {st}"
    torch.cuda.synchronize()
    return y


def _assert_bits(y, y_ref):
    a = np.asarray(y, np.float32)
    assert a.shape == y_ref.shape
    assert np.array_equal(a.view(np.uint32), y_ref.view(np.uint32))


def test_noalloc_matches_oracle_on_two_calls_in_a_row(env):
    L, B, WL = env
    # Tensor-core shapes, then decode shapes, back to back: each call finds
    # the previous call's data still in the shared scratch.
    for (M, N, K, seed) in [(300, 700, 2560, 11), (96, 1152, 4304, 12), (1, 2560, 2560, 13), (16, 300, 6912, 14)]:
        x, packed, D, y_ref = _case(B, WL, M, N, K, seed)
        y = _noalloc(L, x, packed, D, M, N, K).cpu().numpy()
        _assert_bits(y, y_ref)
        # the existing entry point with a caller workspace gives the same bits
        _assert_bits(B.forward(torch.from_numpy(x).cuda(), packed, D).cpu().numpy(), y)
    assert L.bitlinear_noalloc_error(torch.cuda.current_stream().cuda_stream) == 0


def test_noalloc_error_reports_a_recorded_device_failure(env):
    """A bounded wait that runs out in the scratch's own error word (the
    self-test: a barrier nothing completes, no fault or hang) is reported by
    bitlinear_noalloc_error once, then cleared; later calls still work."""
    L, B, WL = env
    stream = torch.cuda.current_stream().cuda_stream
    assert L.bitlinear_noalloc_selftest_wait_timeout(20_000_000, stream) == 0
    assert L.bitlinear_noalloc_error(stream) == BL_ERR_DEVICE
    assert L.bitlinear_noalloc_error(stream) == 0
    M, N, K = 2, 40, 64
    x, packed, D, y_ref = _case(B, WL, M, N, K, 15)
    _assert_bits(_noalloc(L, x, packed, D, M, N, K).cpu().numpy(), y_ref)
    assert L.bitlinear_noalloc_error(stream) == 0


def test_noalloc_rejects_work_larger_than_scratch(env):
    L, _, _ = env
    limit = 16 * 1024 * 1024
    M, K = 8192, 4096  # M*K = 32 MiB of quantised activations > 16 MiB
    assert L.bitlinear_workspace_size(M, 64, K) > limit
    # Refused before any GPU access, so the pointers are never read.
    st = L.bitlinear_forward_noalloc(0x10000, M, 64, K, 0x10000, 0x10000, 0x10000, None)
    assert st == BL_ERR_WORKSPACE
