"""Python binding of libbitlinear.so (BitNet b1.58 BitLinear forward, B200).

Argument marshalling only: every function allocates its outputs (and a
workspace, unless one is passed) with torch on the tensors' device and calls
the C entry point of the same name on the current CUDA stream.  All the
arithmetic runs in the library's CUDA kernels; there is no fallback.  If the
shared library is missing, loading it raises with the build command.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

_c_i64 = ctypes.c_int64
_c_p = ctypes.c_void_p
_c_sz = ctypes.c_size_t

_SIGS = {
    "bitlinear_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bitlinear_version": (ctypes.c_int, []),
    "bitlinear_packed_bytes": (_c_sz, [_c_i64, _c_i64]),
    "bitlinear_pack_workspace_bytes": (_c_sz, [_c_i64, _c_i64]),
    "bitlinear_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64]),
    "bitlinear_host_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64]),
    "bitlinear_pack_weights": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "bitlinear_quant_act": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p]),
    "bitlinear_dequant_weights": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p]),
    "bitlinear_forward_host_async": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p,
                                                    ctypes.c_uint, _c_p, ctypes.c_size_t, _c_p]),
    "bitlinear_forward_debug_ex": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p,
                                                  _c_p, _c_p, _c_p, ctypes.c_int, ctypes.c_uint, _c_p,
                                                  ctypes.c_size_t, _c_p]),
    "bitlinear_forward_grouped": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p, ctypes.c_int, _c_p, _c_p, _c_p,
                                                 ctypes.c_uint, _c_p, ctypes.c_size_t, _c_p]),
    "bitlinear_forward": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_sz,
                                         _c_p]),
    "bitlinear_forward_ex": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, ctypes.c_uint,
                                            _c_p, _c_sz, _c_p]),
    "bitlinear_forward_q8": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p,
                                            _c_p, _c_sz, _c_p]),
    "bitlinear_forward_debug": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p,
                                               _c_p, _c_p, _c_p, ctypes.c_int, _c_p, _c_sz, _c_p]),
    "bitlinear_forward_host": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p,
                                              _c_sz, _c_p]),
    "bitlinear_check_status": (ctypes.c_int, [_c_p, _c_sz, _c_p]),
    "bitlinear_forward_noalloc": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p]),
    "bitlinear_noalloc_check_status": (ctypes.c_int, [_c_p]),
    "bitlinear_test_force_timeout": (ctypes.c_int, [ctypes.c_int]),
    "bitlinear_absmean_bins": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p]),
    "bitlinear_pack_weights_from_bins": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_p, _c_p, _c_p,
                                                        _c_sz, _c_p]),
    "bitlinear_act_absmax": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p]),
    "bitlinear_forward_partial": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_p, ctypes.c_uint,
                                                 _c_p, _c_sz, _c_p]),
    "bitlinear_epilogue_sum": (ctypes.c_int, [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p,
                                              ctypes.c_uint, _c_p]),
    "bitlinear_measure_i8_peak": (ctypes.c_int, [ctypes.c_int, _c_p, _c_p, _c_sz, _c_p]),
}

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded shared library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -m bitlinear_fwd_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def status_string(status: int) -> str:
    return lib().bitlinear_status_string(int(status)).decode()


def _check(st: int, where: str) -> None:
    if st != 0:
        raise BitLinearError(st, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return t.contiguous()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, device=None, min_numel: int = 0) -> None:
    """Host-side check of one tensor argument: dtype, exact shape, device and
    contiguity, so that a wrong argument raises here instead of making a
    kernel read or write out of bounds."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.numel() < min_numel:
        raise ValueError(f"{name} needs at least {min_numel} elements, got {t.numel()}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_forward(x: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor, bias, out, ws,
                   n_scales: int = 1, x_on_host: bool = False) -> tuple:
    """The arguments shared by the forward entry points, checked on the host
    before anything is enqueued: dtypes (TypeError), then shapes and layout
    (BitLinearError BITLINEAR_ERR_SHAPE for K, ValueError otherwise), then
    devices (ValueError).  Returns (M, N, K)."""
    lib()                                        # a missing library is reported first
    if x.dim() != 2:
        raise ValueError(f"x must be 2-D [M, K], got {tuple(x.shape)}")
    M, K = x.shape
    if K % 64 != 0 or K <= 0:
        raise BitLinearError(-2, f"K = {K} must be a positive multiple of 64")
    if packed.dim() != 2:
        raise ValueError(f"packed must be 2-D [N, K/4], got {tuple(packed.shape)}")
    N = packed.shape[0]
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(w_scale, "w_scale", torch.float32, None, min_numel=n_scales)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if out is not None:
        _need(out, "y_host" if x_on_host else "out", torch.bfloat16, (M, N))
    if ws is not None:
        _need(ws, "ws", torch.uint8)
    dev = packed.device
    if dev.type != "cuda":
        raise ValueError(f"packed must be on a CUDA device, got {dev}")
    if x_on_host:
        if x.device.type != "cpu":
            raise ValueError("x_host must be a host (CPU) tensor")
        if out is not None and out.device.type != "cpu":
            raise ValueError("y_host must be a host (CPU) tensor")
    else:
        for t, name in ((x, "x"), (out, "out")):
            if t is not None and t.device != dev:
                raise ValueError(f"{name} is on {t.device}, packed on {dev}")
    for t, name in ((w_scale, "w_scale"), (bias, "bias"), (ws, "ws")):
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, packed on {dev}")
    return M, N, K


def packed_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_packed_bytes(N, K))


def workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_workspace_bytes(M, N, K))


def host_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_host_workspace_bytes(M, N, K))


def pack_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_pack_workspace_bytes(N, K))


def workspace(M: int, N: int, K: int, device, host: bool = False) -> torch.Tensor:
    n = host_workspace_bytes(M, N, K) if host else workspace_bytes(M, N, K)
    if n == 0:
        raise BitLinearError(-2, "workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def bitlinear_pack_weights(w: torch.Tensor, ws: Optional[torch.Tensor] = None):
    """_weight_quant + 2-bit packing.  w: float32 [N, K] on the GPU.
    Returns (packed uint8 [N, K/4], w_scale float32 [1], w_mean float32 [1])."""
    w = w.contiguous()
    if w.dtype != torch.float32 or w.dim() != 2:
        raise TypeError("w must be a float32 [N, K] tensor")
    if w.device.type != "cuda":
        raise ValueError("w must be on a CUDA device")
    N, K = w.shape
    if ws is not None:
        _need(ws, "ws", torch.uint8, None, w.device, min_numel=pack_workspace_bytes(N, K))
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=w.device)
    w_scale = torch.empty(1, dtype=torch.float32, device=w.device)
    w_mean = torch.empty(1, dtype=torch.float32, device=w.device)
    if ws is None:
        ws = torch.empty(pack_workspace_bytes(N, K), dtype=torch.uint8, device=w.device)
    _check(lib().bitlinear_pack_weights(_ptr(w), N, K, _ptr(packed), _ptr(w_scale), _ptr(w_mean), _ptr(ws),
                                        ws.numel(), _stream(w.device)), "bitlinear_pack_weights")
    return packed, w_scale, w_mean


def bitlinear_quant_act(x: torch.Tensor):
    """activation_norm_quant.  x: bf16 [M, K].  Returns (xq int8, s_x f32, rowsum i32)."""
    x = _bits(x)
    if x.dim() != 2 or x.device.type != "cuda":
        raise ValueError("x must be a 2-D CUDA tensor [M, K]")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    rs = torch.empty(M, dtype=torch.int32, device=x.device)
    _check(lib().bitlinear_quant_act(_ptr(x), M, K, _ptr(xq), _ptr(s_x), _ptr(rs), _stream(x.device)),
           "bitlinear_quant_act")
    return xq, s_x, rs


def bitlinear_dequant_weights(packed: torch.Tensor, w_scale: torch.Tensor) -> torch.Tensor:
    """bf16 export of packed weights: w [N, K] bf16 = u / s_w (zeros +0)."""
    lib()
    if packed.dim() != 2:
        raise ValueError("packed must be 2-D [N, K/4]")
    if packed.device.type != "cuda":
        raise ValueError("packed must be on a CUDA device")
    N, K = packed.shape[0], packed.shape[1] * 4
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(w_scale, "w_scale", torch.float32, None, packed.device, min_numel=1)
    out = torch.empty((N, K), dtype=torch.bfloat16, device=packed.device)
    _check(lib().bitlinear_dequant_weights(_ptr(packed), N, K, _ptr(w_scale), _ptr(out), _stream(packed.device)),
           "bitlinear_dequant_weights")
    return out


WEIGHTS_RESIDENT = 1
BF16_FAITHFUL = 2


def bitlinear_forward(x: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor,
                      bias: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """BitLinear.forward: y bf16 [M, N] from x bf16 [M, K] and packed weights.
    flags=WEIGHTS_RESIDENT calls bitlinear_forward_ex (see the C header)."""
    x = _bits(x)
    M, N, K = _check_forward(x, packed, w_scale, bias, out, ws)
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = workspace(M, N, K, x.device)
    b = None if bias is None else _bits(bias)
    if flags:
        st = lib().bitlinear_forward_ex(_ptr(x), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b), _ptr(y), flags,
                                        _ptr(ws), ws.numel(), _stream(x.device))
        _check(st, "bitlinear_forward_ex")
    else:
        _check(lib().bitlinear_forward(_ptr(x), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b), _ptr(y),
                                       _ptr(ws), ws.numel(), _stream(x.device)), "bitlinear_forward")
    return y


MAX_GROUPS = 8


def bitlinear_forward_grouped(x: torch.Tensor, packed: torch.Tensor, group_rows, w_scales: torch.Tensor,
                              bias: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                              out: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """Layers sharing the input x (q/k/v, gate/up): packed [N, K/4] stacked row-wise,
    group_rows their row counts, w_scales [G] f32.  Returns y bf16 [M, N], layer g in
    its own column block."""
    x = _bits(x)
    M, N, K = _check_forward(x, packed, w_scales, bias, out, ws, n_scales=len(group_rows))
    if sum(int(r) for r in group_rows) != N:
        raise ValueError(f"group_rows sum to {sum(int(r) for r in group_rows)}, packed has {N} rows")
    rows = (ctypes.c_int64 * len(group_rows))(*[int(r) for r in group_rows])
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = workspace(M, N, K, x.device)
    _check(lib().bitlinear_forward_grouped(_ptr(x), M, K, _ptr(packed), rows, len(group_rows), _ptr(w_scales),
                                           _ptr(bias), _ptr(y), flags, _ptr(ws), ws.numel(), _stream(x.device)),
           "bitlinear_forward_grouped")
    return y


def bitlinear_forward_q8(xq: torch.Tensor, s_x: torch.Tensor, rowsum: torch.Tensor, packed: torch.Tensor,
                         w_scale: torch.Tensor, bias: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Contraction + epilogue on activations from bitlinear_quant_act."""
    if xq.dim() != 2:
        raise ValueError("xq must be 2-D [M, K]")
    M, K = xq.shape
    _need(xq, "xq", torch.int8, (M, K))
    _need(s_x, "s_x", torch.float32, (M,))
    _need(rowsum, "rowsum", torch.int32, (M,))
    N = packed.shape[0]
    _check_forward(xq, packed, w_scale, bias, out, ws)
    for t, name in ((s_x, "s_x"), (rowsum, "rowsum")):
        if t.device != packed.device:
            raise ValueError(f"{name} is on {t.device}, packed on {packed.device}")
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    if ws is None:
        ws = torch.zeros(256, dtype=torch.uint8, device=xq.device)
    b = None if bias is None else _bits(bias)
    _check(lib().bitlinear_forward_q8(_ptr(xq), _ptr(s_x), _ptr(rowsum), M, K, _ptr(packed), N, _ptr(w_scale),
                                      _ptr(b), _ptr(y), _ptr(ws), ws.numel(), _stream(xq.device)),
           "bitlinear_forward_q8")
    return y


def bitlinear_forward_debug(x: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor,
                            bias: Optional[torch.Tensor] = None, engine: int = 0,
                            ws: Optional[torch.Tensor] = None, flags: int = 0) -> dict:
    """Forward with intermediates: y, xq, s_x, acc (int32), y32 (float32).
    flags=BF16_FAITHFUL calls bitlinear_forward_debug_ex."""
    x = _bits(x)
    M, N, K = _check_forward(x, packed, w_scale, bias, None, ws)
    dev = x.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    s_x = torch.empty(M, dtype=torch.float32, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev)
    y32 = torch.empty((M, N), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(M, N, K, dev)
    b = None if bias is None else _bits(bias)
    if flags:
        _check(lib().bitlinear_forward_debug_ex(_ptr(x), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b), _ptr(y),
                                                _ptr(xq), _ptr(s_x), _ptr(acc), _ptr(y32), engine, flags, _ptr(ws),
                                                ws.numel(), _stream(dev)), "bitlinear_forward_debug_ex")
    else:
        _check(lib().bitlinear_forward_debug(_ptr(x), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b), _ptr(y),
                                             _ptr(xq), _ptr(s_x), _ptr(acc), _ptr(y32), engine, _ptr(ws),
                                             ws.numel(), _stream(dev)), "bitlinear_forward_debug")
    return {"y": y, "xq": xq, "s_x": s_x, "acc": acc, "y32": y32, "ws": ws}


def bitlinear_forward_host(x_host: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor,
                           bias: Optional[torch.Tensor] = None, y_host: Optional[torch.Tensor] = None,
                           ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Forward from host activations to a host output (synchronous)."""
    x_host = _bits(x_host)
    M, N, K = _check_forward(x_host, packed, w_scale, bias, y_host, ws, x_on_host=True)
    dev = packed.device
    if y_host is None:
        y_host = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
    if ws is None:
        ws = workspace(M, N, K, dev, host=True)
    b = None if bias is None else _bits(bias)
    _check(lib().bitlinear_forward_host(_ptr(x_host), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b),
                                        _ptr(y_host), _ptr(ws), ws.numel(), _stream(dev)),
           "bitlinear_forward_host")
    return y_host


def bitlinear_forward_host_async(x_host: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor,
                                 bias: Optional[torch.Tensor] = None, y_host: Optional[torch.Tensor] = None,
                                 ws: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """Stream-ordered host-to-host forward: enqueues the copies and kernels and
    returns; y_host is valid once the current stream is synchronised."""
    x_host = _bits(x_host)
    M, N, K = _check_forward(x_host, packed, w_scale, bias, y_host, ws, x_on_host=True)
    dev = packed.device
    if y_host is None:
        y_host = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
    if ws is None:
        ws = workspace(M, N, K, dev, host=True)
    b = None if bias is None else _bits(bias)
    _check(lib().bitlinear_forward_host_async(_ptr(x_host), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b),
                                              _ptr(y_host), flags, _ptr(ws), ws.numel(), _stream(dev)),
           "bitlinear_forward_host_async")
    return y_host


def bitlinear_forward_noalloc(x: torch.Tensor, packed: torch.Tensor, w_scale: torch.Tensor,
                              bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bitlinear_forward with the library's fixed device scratch instead of a
    workspace (for callers that cannot allocate; see the C header)."""
    x = _bits(x)
    M, N, K = _check_forward(x, packed, w_scale, bias, out, None)
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    b = None if bias is None else _bits(bias)
    _check(lib().bitlinear_forward_noalloc(_ptr(x), M, K, _ptr(packed), N, _ptr(w_scale), _ptr(b), _ptr(y),
                                           _stream(x.device)), "bitlinear_forward_noalloc")
    return y


def bitlinear_check_status(ws: torch.Tensor) -> int:
    """Status of the most recent call that used workspace ws (synchronises)."""
    return int(lib().bitlinear_check_status(_ptr(ws), ws.numel(), _stream(ws.device)))


def bitlinear_noalloc_check_status(device=None) -> int:
    """Status of the noalloc calls on the current device since the last
    reset (synchronises the current stream)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(lib().bitlinear_noalloc_check_status(_stream(dev)))


def bitlinear_test_force_timeout(on: bool) -> bool:
    """Test hook: while on, every forward's kernels take one wait that runs out
    (1 ms) and report BITLINEAR_ERR_TIMEOUT.  Returns the previous setting."""
    return bool(lib().bitlinear_test_force_timeout(1 if on else 0))


# ---- tensor-parallel K-split pieces (see the C header) ----------------------

ABSMEAN_BINS = 320
MAX_PARTS = 8


def bitlinear_absmean_bins(w: torch.Tensor) -> torch.Tensor:
    """Exact exponent bins of sum |w| over this shard: uint64 [320] as int64
    (two's complement); the bins of several shards add."""
    lib()
    if w.dim() != 2:
        raise ValueError("w must be 2-D [N, K]")
    _need(w, "w", torch.float32)
    if w.device.type != "cuda":
        raise ValueError("w must be on a CUDA device")
    N, K = w.shape
    bins = torch.empty(ABSMEAN_BINS, dtype=torch.int64, device=w.device)
    _check(lib().bitlinear_absmean_bins(_ptr(w), N, K, _ptr(bins), _stream(w.device)), "bitlinear_absmean_bins")
    return bins


def bitlinear_pack_weights_from_bins(w: torch.Tensor, bins: torch.Tensor, n_total: int,
                                     ws: Optional[torch.Tensor] = None):
    """Pack one shard with s_w from the summed bins of all shards.
    Returns (packed, w_scale, w_mean) as bitlinear_pack_weights does."""
    lib()
    if w.dim() != 2:
        raise ValueError("w must be 2-D [N, K]")
    _need(w, "w", torch.float32)
    _need(bins, "bins", torch.int64, (ABSMEAN_BINS,), w.device)
    if w.device.type != "cuda":
        raise ValueError("w must be on a CUDA device")
    N, K = w.shape
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=w.device)
    w_scale = torch.empty(1, dtype=torch.float32, device=w.device)
    w_mean = torch.empty(1, dtype=torch.float32, device=w.device)
    if ws is None:
        ws = torch.empty(pack_workspace_bytes(N, K), dtype=torch.uint8, device=w.device)
    _check(lib().bitlinear_pack_weights_from_bins(_ptr(w), N, K, _ptr(bins), int(n_total), _ptr(packed),
                                                  _ptr(w_scale), _ptr(w_mean), _ptr(ws), ws.numel(),
                                                  _stream(w.device)), "bitlinear_pack_weights_from_bins")
    return packed, w_scale, w_mean


def bitlinear_act_absmax(x: torch.Tensor) -> torch.Tensor:
    """Each token's absmax over this K-shard of x, float32 [M]."""
    x = _bits(x)
    if x.dim() != 2 or x.device.type != "cuda":
        raise ValueError("x must be a 2-D CUDA tensor [M, K]")
    M, K = x.shape
    out = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().bitlinear_act_absmax(_ptr(x), M, K, _ptr(out), _stream(x.device)), "bitlinear_act_absmax")
    return out


def bitlinear_forward_partial(x: torch.Tensor, absmax: torch.Tensor, packed: torch.Tensor,
                              ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                              flags: int = 0) -> torch.Tensor:
    """int32 [M, N] partial sums of one K-shard, quantised with the whole
    row's absmax."""
    x = _bits(x)
    M, N, K = _check_forward(x, packed, absmax, None, None, ws)
    _need(absmax, "absmax", torch.float32, (M,), packed.device)
    acc = out if out is not None else torch.empty((M, N), dtype=torch.int32, device=x.device)
    _need(acc, "out", torch.int32, (M, N), packed.device)
    if ws is None:
        ws = workspace(M, N, K, x.device)
    _check(lib().bitlinear_forward_partial(_ptr(x), M, K, _ptr(absmax), _ptr(packed), N, _ptr(acc), flags,
                                           _ptr(ws), ws.numel(), _stream(x.device)), "bitlinear_forward_partial")
    return acc


def bitlinear_epilogue_sum(partials, absmax: torch.Tensor, w_scale: torch.Tensor,
                           bias: Optional[torch.Tensor] = None, flags: int = 0, acc_out: Optional[torch.Tensor] = None,
                           out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y bf16 [M, N] from int32 partial sums (a tensor or a list of them, all
    [M, N]), the tokens' absmax over the whole K, s_w and the bias."""
    lib()
    parts = [partials] if isinstance(partials, torch.Tensor) else list(partials)
    if not 1 <= len(parts) <= MAX_PARTS:
        raise ValueError(f"1 .. {MAX_PARTS} partial sums")
    M, N = parts[0].shape
    dev = parts[0].device
    for p in parts:
        _need(p, "partial", torch.int32, (M, N))
    _need(absmax, "absmax", torch.float32, (M,), dev)
    _need(w_scale, "w_scale", torch.float32, None, dev, min_numel=1)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,), dev)
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _need(y, "out", torch.bfloat16, (M, N), dev)
    if acc_out is not None:
        _need(acc_out, "acc_out", torch.int32, (M, N), dev)
    arr = (ctypes.c_void_p * len(parts))(*[p.data_ptr() for p in parts])
    _check(lib().bitlinear_epilogue_sum(arr, len(parts), M, N, _ptr(absmax), _ptr(w_scale), _ptr(bias), _ptr(y),
                                        _ptr(acc_out), flags, _stream(dev)), "bitlinear_epilogue_sum")
    return y


def measure_i8_peak(iters: int = 20000, reps: int = 3, device=None) -> dict:
    """The dense int8 tensor-core rate, timed with CUDA events on the current
    stream (best of ``reps`` launches after one warm-up): int8 TOPS and
    MAC/clock/SM at the given SM clock is left to the caller."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    grid = ctypes.c_int(0)
    call = lambda: _check(lib().bitlinear_measure_i8_peak(iters, ctypes.byref(grid), _ptr(ws), ws.numel(),
                                                          _stream(dev)), "bitlinear_measure_i8_peak")
    call()
    torch.cuda.synchronize(dev)
    best = None
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    if bitlinear_check_status(ws) != 0:
        raise BitLinearError(-6, "bitlinear_measure_i8_peak")
    ops = 2.0 * 128 * 256 * 32 * 4 * iters * grid.value
    return {"tops": ops / (best * 1e-3) / 1e12, "ms": best, "iters": iters, "grid": grid.value,
            "macs_per_sm": ops / 2 / grid.value}
