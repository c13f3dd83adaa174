"""PyTorch-facing API of the B200 BitLinear: pack_weights, quant_act, forward.

PyTorch supplies device memory and streams; the arithmetic is in
libbitlinear (C ABI, include/bitlinear.h). Shapes follow torch.nn.Linear:
W [N, K] (out_features x in_features), x [M, K], y [M, N]. The per-row scale D
is a [N, 1] tensor, as the ternary kernel of "Core AI model zoo - BitVLA"
section 2 requires ([1, N] is rejected: that layout made the Metal kernel of
the page read out of bounds).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _lib

__all__ = [
    "pack_weights",
    "pack_status",
    "pack_workspace",
    "quant_act",
    "forward",
    "forward_acc",
    "forward_host",
    "forward_batch",
    "prepare_act",
    "forward_prepared",
    "forward_q",
    "rmsnorm_quant_act",
    "forward_rmsnorm",
    "block_scales",
    "pack_weights_blocks",
    "forward_blocks",
    "blocks_workspace_size",
    "workspace_size",
    "workspace_error",
    "BitLinear",
]


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need_cuda(t: torch.Tensor, name: str, dtype: torch.dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_D(D: torch.Tensor, N: int) -> None:
    if tuple(D.shape) != (N, 1):
        raise ValueError(f"D must have shape [N, 1] = [{N}, 1], got {list(D.shape)}")
    _need_cuda(D, "D", torch.float32)


def _alloc_ws(nbytes: int, device: torch.device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks.
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.lib().bitlinear_workspace_size(M, N, K))


def _float_input(t: torch.Tensor, name: str) -> str:
    """'' for fp32, '_bf16' for bf16 (passed to the library as its bit patterns)."""
    if t.dtype == torch.bfloat16:
        _need_cuda(t, name, torch.bfloat16)
        return "_bf16"
    _need_cuda(t, name, torch.float32)
    return ""


def pack_weights(W: torch.Tensor, ws: Optional[torch.Tensor] = None,
                 sync: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """WeightQuant + pack: fp32 or bf16 W [N, K] -> (packed int32 [N, K/16], D fp32 [N, 1]).

    sync=False (fp32 W only) enqueues the pack without waiting; a non-finite
    weight is then recorded in ws (zero-filled before the first call) and
    reported by pack_status(ws)."""
    sfx = _float_input(W, "W")
    if not sync and sfx:
        raise ValueError("the asynchronous pack takes fp32 W")
    if not sync and ws is None:
        raise ValueError("the asynchronous pack needs a caller workspace (zero-filled before the first call)")
    if not sync:
        sfx = "_async"
    N, K = W.shape
    packed = torch.empty((N, K // 16), dtype=torch.int32, device=W.device)
    D = torch.empty((N, 1), dtype=torch.float32, device=W.device)
    L = _lib.lib()
    if ws is None:
        ws = _alloc_ws(L.bitlinear_pack_workspace_size(N, K), W.device)
    _lib.call("bitlinear_pack_weights" + sfx, W.data_ptr(), N, K, packed.data_ptr(), D.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(W.device))
    return packed, D


def pack_status(ws: torch.Tensor) -> int:
    """Synchronises the stream, reads and clears the status word of a pack workspace:
    BL_OK (0) or BL_ERR_NONFINITE (5)."""
    return int(_lib.lib().bitlinear_pack_status(ws.data_ptr(), ws.numel(), _stream_handle(ws.device)))


def pack_workspace(device) -> torch.Tensor:
    """A zero-filled pack workspace, as the asynchronous pack wants it."""
    return torch.zeros(int(_lib.lib().bitlinear_pack_workspace_size(1, 16)), dtype=torch.uint8, device=device)


def quant_act(x: torch.Tensor):
    """ActQuant: fp32 or bf16 x [M, K] -> (q int8 [M, K], s_x fp32 [M], rowsum int32 [M])."""
    sfx = _float_input(x, "x")
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty((M,), dtype=torch.float32, device=x.device)
    rs = torch.empty((M,), dtype=torch.int32, device=x.device)
    _lib.call("bitlinear_quant_act" + sfx, x.data_ptr(), M, K, q.data_ptr(), s_x.data_ptr(), rs.data_ptr(),
              _stream_handle(x.device))
    return q, s_x, rs


def _fwd_args(x, packed, K, allow_bf16=False):
    if not (allow_bf16 and x.dtype == torch.bfloat16):
        _need_cuda(x, "x", torch.float32)
    else:
        _need_cuda(x, "x", torch.bfloat16)
    _need_cuda(packed, "packed", torch.int32)
    if x.dim() != 2 or packed.dim() != 2:
        raise ValueError("x must be [M, K] and packed [N, K/16]")
    M, Kx = x.shape
    if Kx != K or packed.shape[1] * 16 != K:
        raise ValueError(f"K mismatch: x has {Kx}, packed has {packed.shape[1] * 16}")
    return M, packed.shape[0]


def forward(x: torch.Tensor, packed: torch.Tensor, D: torch.Tensor,
            out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = F.linear(ActQuant(x), WeightQuant(W)) from packed weights; x fp32 or bf16, y fp32."""
    K = x.shape[-1]
    M, N = _fwd_args(x, packed, K, allow_bf16=True)
    fn = "bitlinear_forward_bf16" if x.dtype == torch.bfloat16 else "bitlinear_forward"
    _check_D(D, N)
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x.device)
    _need_cuda(y, "out", torch.float32)
    need = workspace_size(M, N, K)
    if ws is None:
        ws = _alloc_ws(need, x.device)
    _lib.call(fn, x.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(x.device))
    return y


def forward_acc(x: torch.Tensor, packed: torch.Tensor, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Exact int32 accumulators acc[m, n] = sum_k q[m, k] * code[n, k]."""
    K = x.shape[-1]
    M, N = _fwd_args(x, packed, K)
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    if ws is None:
        ws = _alloc_ws(workspace_size(M, N, K), x.device)
    _lib.call("bitlinear_forward_acc", x.data_ptr(), M, N, K, packed.data_ptr(), acc.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(x.device))
    return acc


def prepare_act(x: torch.Tensor, ws: torch.Tensor) -> torch.Tensor:
    """Quantise x [M, K] once into `ws` for several forward_prepared calls."""
    _need_cuda(x, "x", torch.float32)
    M, K = x.shape
    _lib.call("bitlinear_prepare_act", x.data_ptr(), M, K, ws.data_ptr(), ws.numel(), _stream_handle(x.device))
    return ws


def forward_prepared(M: int, K: int, packed: torch.Tensor, D: torch.Tensor, ws: torch.Tensor,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Contraction + rescale from a workspace filled by prepare_act (tensor-core path)."""
    _need_cuda(packed, "packed", torch.int32)
    N = packed.shape[0]
    if packed.shape[1] * 16 != K:
        raise ValueError("K mismatch with packed")
    _check_D(D, N)
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=packed.device)
    _need_cuda(y, "out", torch.float32)
    _lib.call("bitlinear_forward_prepared", M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(packed.device))
    return y


def forward_q(q: torch.Tensor, s_x: torch.Tensor, packed: torch.Tensor, D: torch.Tensor,
              out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y from pre-quantised activations: q int8 [M,K] (natural order) and s_x fp32 [M]
    as quant_act returns them."""
    _need_cuda(q, "q", torch.int8)
    _need_cuda(s_x, "s_x", torch.float32)
    if q.dim() != 2 or not q.is_contiguous() or not s_x.is_contiguous():
        raise ValueError("q must be a contiguous [M, K] tensor and s_x contiguous")
    M, K = q.shape
    if s_x.numel() != M:
        raise ValueError("s_x must hold one scale per token")
    _need_cuda(packed, "packed", torch.int32)
    N = packed.shape[0]
    if packed.shape[1] * 16 != K:
        raise ValueError("K mismatch with packed")
    _check_D(D, N)
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=q.device)
    _need_cuda(y, "out", torch.float32)
    if ws is None:
        ws = _alloc_ws(_lib.lib().bitlinear_workspace_size(M, N, K), q.device)
    _lib.call("bitlinear_forward_q", q.data_ptr(), s_x.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(),
              y.data_ptr(), ws.data_ptr(), ws.numel(), _stream_handle(q.device))
    return y


def rmsnorm_quant_act(x: torch.Tensor, g: torch.Tensor, eps: float = 1e-6):
    """ActQuant(RMSNorm(x, g)): fp32 x [M, K], norm weight g [K] -> (q int8 [M, K], s_x [M], rowsum [M])."""
    _need_cuda(x, "x", torch.float32)
    _need_cuda(g, "g", torch.float32)
    M, K = x.shape
    if g.numel() != K:
        raise ValueError("g must hold K weights")
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty((M,), dtype=torch.float32, device=x.device)
    rs = torch.empty((M,), dtype=torch.int32, device=x.device)
    _lib.call("bitlinear_rmsnorm_quant_act", x.data_ptr(), g.data_ptr(), float(eps), M, K, q.data_ptr(),
              s_x.data_ptr(), rs.data_ptr(), _stream_handle(x.device))
    return q, s_x, rs


def forward_rmsnorm(x: torch.Tensor, g: torch.Tensor, packed: torch.Tensor, D: torch.Tensor, eps: float = 1e-6,
                    out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = F.linear(ActQuant(RMSNorm(x, g)), WeightQuant(W)) from packed weights."""
    K = x.shape[-1]
    M, N = _fwd_args(x, packed, K)
    _need_cuda(g, "g", torch.float32)
    if g.numel() != K:
        raise ValueError("g must hold K weights")
    _check_D(D, N)
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x.device)
    _need_cuda(y, "out", torch.float32)
    if ws is None:
        ws = _alloc_ws(workspace_size(M, N, K), x.device)
    _lib.call("bitlinear_forward_rmsnorm", x.data_ptr(), g.data_ptr(), float(eps), M, N, K, packed.data_ptr(),
              D.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(), _stream_handle(x.device))
    return y


def block_scales(K: int) -> int:
    """nb = ceil(K / 256): scale blocks per row of the per-256-block variant."""
    nb = int(_lib.lib().bitlinear_block_scales(K))
    if nb <= 0:
        raise ValueError(f"invalid K = {K}")
    return nb


def blocks_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.lib().bitlinear_blocks_workspace_size(M, N, K))


def pack_weights_blocks(W: torch.Tensor, ws: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-256-block WeightQuant + pack: fp32 or bf16 W [N, K] -> (packed int32 [N, K/16], D fp32 [N, nb])."""
    sfx = _float_input(W, "W")
    N, K = W.shape
    nb = block_scales(K)
    packed = torch.empty((N, K // 16), dtype=torch.int32, device=W.device)
    D = torch.empty((N, nb), dtype=torch.float32, device=W.device)
    L = _lib.lib()
    if ws is None:
        ws = _alloc_ws(L.bitlinear_pack_workspace_size(N, K), W.device)
    _lib.call("bitlinear_pack_weights_blocks" + sfx, W.data_ptr(), N, K, packed.data_ptr(), D.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(W.device))
    return packed, D


def forward_blocks(x: torch.Tensor, packed: torch.Tensor, D: torch.Tensor,
                   out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y [M, N] from per-256-block scaled weights (D fp32 [N, ceil(K/256)]); x fp32 or bf16, y fp32."""
    K = x.shape[-1]
    M, N = _fwd_args(x, packed, K, allow_bf16=True)
    fn = "bitlinear_forward_blocks_bf16" if x.dtype == torch.bfloat16 else "bitlinear_forward_blocks"
    nb = block_scales(K)
    if tuple(D.shape) != (N, nb):
        raise ValueError(f"D must have shape [N, nb] = [{N}, {nb}], got {list(D.shape)}")
    _need_cuda(D, "D", torch.float32)
    y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x.device)
    _need_cuda(y, "out", torch.float32)
    if ws is None:
        ws = _alloc_ws(blocks_workspace_size(M, N, K), x.device)
    _lib.call(fn, x.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(x.device))
    return y


def forward_batch(calls, flags: int = 0, ws: Optional[torch.Tensor] = None):
    """Run independent BitLinears [(x, packed, D, out), ...] in one C call.

    Decode-sized calls (M <= 16) are fused into grouped launches; `flags` may
    hold BL_FLAG_STREAM_WEIGHTS_EARLY (weights are static, so the decode
    kernels may stream them while the previous work on the stream finishes)
    and BL_FLAG_ONE_LAUNCH_PER_CALL (every call in its own launch, in order,
    for calls that stand for dependent layers). Returns the list of outputs.
    """
    n = len(calls)
    arr = (_lib.LinearCall * max(n, 1))()
    outs = []
    device = None
    for i, (x, packed, D, out) in enumerate(calls):
        K = x.shape[-1]
        M, N = _fwd_args(x, packed, K)
        _check_D(D, N)
        y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x.device)
        _need_cuda(y, "out", torch.float32)
        arr[i] = _lib.LinearCall(x.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr())
        outs.append(y)
        device = x.device
    if n == 0:
        return outs
    L = _lib.lib()
    if ws is None:
        ws = _alloc_ws(L.bitlinear_batch_workspace_size(arr, n), device)
    _lib.call("bitlinear_forward_batch", arr, n, flags, ws.data_ptr(), ws.numel(), _stream_handle(device))
    return outs


def forward_batch_host(calls, flags: int = 0, ws: Optional[torch.Tensor] = None):
    """forward_batch with host activations and outputs: calls are
    [(x_host, packed, D, y_host), ...] with x_host / y_host pinned CPU fp32
    tensors (y_host None: allocated pinned) and packed / D on the device.
    Enqueued on the current stream; the outputs are valid once it has been
    synchronised. Calls whose host blocks follow one another in memory (views
    of one pinned buffer) move in one copy each way. Returns the outputs."""
    n = len(calls)
    arr = (_lib.LinearCall * max(n, 1))()
    outs = []
    device = None
    for i, (x, packed, D, y) in enumerate(calls):
        if x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous() or x.dim() != 2:
            raise ValueError("x_host must be a contiguous 2-D fp32 CPU tensor")
        M, K = x.shape
        _need_cuda(packed, "packed", torch.int32)
        N = packed.shape[0]
        _check_D(D, N)
        if y is None:
            y = torch.empty((M, N), dtype=torch.float32, pin_memory=True)
        if y.is_cuda or y.dtype != torch.float32 or not y.is_contiguous() or tuple(y.shape) != (M, N):
            raise ValueError("y_host must be a contiguous fp32 CPU tensor of shape (M, N)")
        if M and N and not (x.is_pinned() and y.is_pinned()):
            raise ValueError("the batched host call needs pinned x_host and y_host")
        arr[i] = _lib.LinearCall(x.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(), y.data_ptr())
        outs.append(y)
        device = packed.device
    if n == 0:
        return outs
    L = _lib.lib()
    if ws is None:
        ws = _alloc_ws(L.bitlinear_batch_host_workspace_size(arr, n), device)
    _lib.call("bitlinear_forward_batch_host", arr, n, flags, ws.data_ptr(), ws.numel(), _stream_handle(device))
    return outs


def batch_host_workspace_size(calls) -> int:
    """Workspace bytes for forward_batch_host over [(M, N, K), ...]."""
    n = len(calls)
    arr = (_lib.LinearCall * max(n, 1))()
    for i, (M, N, K) in enumerate(calls):
        arr[i] = _lib.LinearCall(0, M, N, K, 0, 0, 0)
    return int(_lib.lib().bitlinear_batch_host_workspace_size(arr, n))


def forward_host(x_host: torch.Tensor, packed: torch.Tensor, D: torch.Tensor,
                 y_host: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 sync: bool = True) -> torch.Tensor:
    """End-to-end call with host x / y. sync=True: synchronous (pinned memory
    recommended). sync=False: enqueued on the current stream; x_host and y_host
    must be pinned, and y_host is valid after the stream is synchronised."""
    if x_host.is_cuda or x_host.dtype != torch.float32 or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous fp32 CPU tensor")
    M, K = x_host.shape
    _need_cuda(packed, "packed", torch.int32)
    N = packed.shape[0]
    _check_D(D, N)
    if y_host is None:
        y_host = torch.empty((M, N), dtype=torch.float32, pin_memory=True)
    if not sync and not (x_host.is_pinned() and y_host.is_pinned()):
        raise ValueError("the asynchronous host call needs pinned x_host and y_host")
    L = _lib.lib()
    if ws is None:
        ws = _alloc_ws(L.bitlinear_host_workspace_size(M, N, K), packed.device)
    fn = "bitlinear_forward_host" if sync else "bitlinear_forward_host_async"
    _lib.call(fn, x_host.data_ptr(), M, N, K, packed.data_ptr(), D.data_ptr(),
              y_host.data_ptr(), ws.data_ptr(), ws.numel(), _stream_handle(packed.device))
    return y_host


_I2S_LAYOUTS = {"consecutive": _lib.BL_I2S_CONSECUTIVE, "quarters": _lib.BL_I2S_QUARTERS}


def i2s_bytes(N: int, K: int) -> int:
    """Size of the I2_S buffer of an [N, K] tensor (blocks plus the fp32 scale)."""
    return int(_lib.lib().bitlinear_i2s_bytes(N, K))


def i2s_workspace(device) -> torch.Tensor:
    """A zeroed workspace (status word) for the I2_S conversions."""
    return torch.zeros(max(256, int(_lib.lib().bitlinear_i2s_workspace_size())), dtype=torch.uint8, device=device)


def i2s_export(packed: torch.Tensor, D: torch.Tensor, layout: str = "consecutive",
               out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
               sync: bool = True) -> torch.Tensor:
    """BitLinear packed weights + D -> one I2_S buffer (uint8 CUDA tensor).
    sync=True: raises BitLinearError (BL_ERR_FORMAT) on a field holding 3 or
    rows of D that differ. sync=False: enqueued on the current stream; errors
    collect in ws (zeroed by i2s_workspace) until i2s_status(ws)."""
    _need_cuda(packed, "packed", torch.int32)
    N, K = packed.shape[0], packed.shape[1] * 16
    _check_D(D, N)
    nbytes = i2s_bytes(N, K)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=packed.device)
    _need_cuda(out, "out", torch.uint8)
    if out.numel() != nbytes:
        raise ValueError(f"out must hold {nbytes} bytes")
    if ws is None:
        if not sync:
            raise ValueError("the asynchronous conversion needs a workspace from i2s_workspace()")
        ws = i2s_workspace(packed.device)
    fn = "bitlinear_i2s_export" if sync else "bitlinear_i2s_export_async"
    _lib.call(fn, packed.data_ptr(), D.data_ptr(), N, K, _I2S_LAYOUTS[layout], out.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(packed.device))
    return out


def i2s_import(buf: torch.Tensor, N: int, K: int, layout: str = "consecutive",
               out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None, ws: Optional[torch.Tensor] = None,
               sync: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """One I2_S buffer (uint8 CUDA tensor) of an [N, K] tensor -> (packed
    int32 [N, K/16], D fp32 [N, 1]). sync=True: raises BitLinearError
    (BL_ERR_FORMAT) on a field holding 3 or a scale that is not finite and
    positive. sync=False: as for i2s_export."""
    _need_cuda(buf, "buf", torch.uint8)
    if buf.numel() != i2s_bytes(N, K):
        raise ValueError(f"buf must hold {i2s_bytes(N, K)} bytes")
    if out is None:
        packed = torch.empty((N, K // 16), dtype=torch.int32, device=buf.device)
        D = torch.empty((N, 1), dtype=torch.float32, device=buf.device)
    else:
        packed, D = out
        _need_cuda(packed, "packed", torch.int32)
        _check_D(D, N)
        if tuple(packed.shape) != (N, K // 16):
            raise ValueError("packed must be [N, K/16]")
    if ws is None:
        if not sync:
            raise ValueError("the asynchronous conversion needs a workspace from i2s_workspace()")
        ws = i2s_workspace(buf.device)
    fn = "bitlinear_i2s_import" if sync else "bitlinear_i2s_import_async"
    _lib.call(fn, buf.data_ptr(), N, K, _I2S_LAYOUTS[layout], packed.data_ptr(), D.data_ptr(),
              ws.data_ptr(), ws.numel(), _stream_handle(buf.device))
    return packed, D


def i2s_status(ws: torch.Tensor) -> int:
    """Synchronise and read/clear the status word of asynchronous I2_S
    conversions: 0 (BL_OK) or 9 (BL_ERR_FORMAT)."""
    return int(_lib.lib().bitlinear_i2s_status(ws.data_ptr(), ws.numel(), _stream_handle(ws.device)))


def workspace_error(ws: torch.Tensor) -> int:
    """Synchronise and read/clear the device error word of a forward workspace."""
    return int(_lib.lib().bitlinear_workspace_error(ws.data_ptr(), ws.numel(), _stream_handle(ws.device)))


class BitLinear:
    """A packed BitNet b1.58 linear layer: holds packed codes and D [N, 1]."""

    def __init__(self, packed: torch.Tensor, D: torch.Tensor):
        _need_cuda(packed, "packed", torch.int32)
        _check_D(D, packed.shape[0])
        self.packed = packed
        self.D = D
        self.out_features = packed.shape[0]
        self.in_features = packed.shape[1] * 16
        self._ws = None

    @classmethod
    def from_float(cls, W: torch.Tensor) -> "BitLinear":
        packed, D = pack_weights(W.contiguous().float())
        return cls(packed, D)

    def workspace(self, M: int) -> torch.Tensor:
        need = workspace_size(M, self.out_features, self.in_features)
        if self._ws is None or self._ws.numel() < need:
            self._ws = _alloc_ws(need, self.packed.device)
        return self._ws

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features).contiguous().float()
        y = forward(x2, self.packed, self.D, ws=self.workspace(x2.shape[0]))
        return y.reshape(*lead, self.out_features)
