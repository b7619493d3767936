"""ctypes front end of the C++ CPU oracle (``bitlinear_oracle.cpp``).

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests, the
smoke entry point and the benchmark's CPU baseline legs may use it.  It
does not call the numpy oracle; the two restate the same pages
independently, and the tests hold each to the same pins.

The functions have the numpy oracle's names, arguments and return values,
so a test can run against either.  ``build()`` compiles the library with
g++ into this folder; the first call of any function builds it if it is
missing or older than its source.
"""

from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "bitlinear_oracle.cpp")
LIBRARY = os.path.join(HERE, "liboracle_cpp.so")

# IEEE float arithmetic as written: no contraction into FMAs, no fast-math
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
            "-Wall", "-Wextra"]

ERRORS = {-1: "bad argument", -2: "invalid 2-bit code 3", -3: "non-finite weight",
          -4: "size beyond the oracle's exact arithmetic"}

_lib = None


def build(force: bool = False) -> str:
    """Compile the library if it is missing, stale, or ``force``; return its path."""
    if force or not os.path.exists(LIBRARY) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE):
        tmp = f"{LIBRARY}.{os.getpid()}.tmp"
        subprocess.run(["g++", *CXXFLAGS, SOURCE, "-o", tmp], check=True)
        os.replace(tmp, LIBRARY)
    return LIBRARY


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "oracle_bf16_to_f32": [_P, _I64, _P],
    "oracle_f32_to_bf16": [_P, _I64, _P],
    "oracle_act_quant": [_P, _I64, _I64, ctypes.c_int, _P, _P, _P],
    "oracle_absmean": [_P, _I64, _P],
    "oracle_ternarise": [_P, _I64, ctypes.c_float, _P],
    "oracle_pack": [_P, _I64, _I64, _P],
    "oracle_unpack": [_P, _I64, _I64, _P],
    "oracle_contract": [_P, _P, _I64, _I64, _I64, _P],
    "oracle_epilogue": [_P, _I64, _I64, _P, ctypes.c_float, _P, ctypes.c_int, _P, _P],
    "oracle_pack_weights": [_P, _I64, _I64, _P, _P, _P],
    "oracle_forward": [_P, _I64, _I64, _P, _I64, ctypes.c_int, _P, _P, _P, ctypes.c_int,
                       _P, _P, _P, _P, _P, _P],
    "oracle_dequant": [_P, _I64, _I64, ctypes.c_float, _P],
}


def _load(path: str) -> ctypes.CDLL:
    handle = ctypes.CDLL(path)
    for name, args in _SIGS.items():
        fn = getattr(handle, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    handle.oracle_weight_scale.argtypes = [ctypes.c_float]
    handle.oracle_weight_scale.restype = ctypes.c_float
    return handle


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _load(build())
    return _lib


@contextlib.contextmanager
def planted(mistake: int, workdir: str):
    """Inside the block, every function runs a copy of the oracle built with
    one planted mistake (``ORACLE_PLANT``: 1 floor for round in the
    activation quantisation, 2 multiply for divide in the epilogue, 3 i and j
    swapped in the packing).  Only for tests of the pins themselves."""
    global _lib
    path = os.path.join(workdir, f"liboracle_cpp_plant{int(mistake)}.so")
    subprocess.run(["g++", *CXXFLAGS, f"-DORACLE_PLANT={int(mistake)}", SOURCE, "-o", path], check=True)
    saved = lib()
    _lib = _load(path)
    try:
        yield
    finally:
        _lib = saved


def _call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise ValueError(f"{name}: {ERRORS.get(st, st)}")


def _arr(a, dtype) -> np.ndarray:
    return np.asarray(a, dtype=dtype, order="C")


def _ptr(a):
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------------------
# bfloat16 storage
# ---------------------------------------------------------------------------

def bf16_to_f32(bits) -> np.ndarray:
    b = _arr(bits, np.uint16)
    out = np.empty(b.shape, np.float32)
    _call("oracle_bf16_to_f32", _ptr(b), b.size, _ptr(out))
    return out


def f32_to_bf16_rne(x) -> np.ndarray:
    v = _arr(x, np.float32)
    out = np.empty(v.shape, np.uint16)
    _call("oracle_f32_to_bf16", _ptr(v), v.size, _ptr(out))
    return out


# ---------------------------------------------------------------------------
# the steps
# ---------------------------------------------------------------------------

def _act_quant(x_bits, bf16_mode: int):
    x = _arr(x_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s_x = np.empty(M, np.float32)
    r = np.empty(M, np.int32)
    _call("oracle_act_quant", _ptr(x), M, K, bf16_mode, _ptr(q), _ptr(s_x), _ptr(r))
    return q, s_x, r


def act_quant(x_bits):
    """(q int8 [M,K], s_x float32 [M], rowsum int32 [M])."""
    return _act_quant(x_bits, 0)


def act_quant_bf16(x_bits):
    return _act_quant(x_bits, 1)


def absmean(w) -> np.float32:
    a = _arr(w, np.float32)
    out = np.zeros(1, np.float32)
    _call("oracle_absmean", _ptr(a), a.size, _ptr(out))
    return out[0]


def weight_scale(mean) -> np.float32:
    return np.float32(lib().oracle_weight_scale(float(np.float32(mean))))


def ternarise(w, s_w) -> np.ndarray:
    a = _arr(w, np.float32)
    u = np.empty(a.shape, np.int8)
    _call("oracle_ternarise", _ptr(a), a.size, float(np.float32(s_w)), _ptr(u))
    return u


def pack(u) -> np.ndarray:
    a = _arr(u, np.int8)
    N, K = a.shape
    out = np.empty((N, K // 4), np.uint8)
    _call("oracle_pack", _ptr(a), N, K, _ptr(out))
    return out


def unpack(packed, K: int | None = None) -> np.ndarray:
    p = _arr(packed, np.uint8)
    N, KB = p.shape
    K = KB * 4 if K is None else K
    if K != KB * 4:
        raise ValueError("K must be four times the packed row length")
    u = np.empty((N, K), np.int8)
    _call("oracle_unpack", _ptr(p), N, K, _ptr(u))
    return u


def contract(q, u) -> np.ndarray:
    qa, ua = _arr(q, np.int8), _arr(u, np.int8)
    M, K = qa.shape
    N = ua.shape[0]
    acc = np.empty((M, N), np.int32)
    _call("oracle_contract", _ptr(qa), _ptr(ua), M, N, K, _ptr(acc))
    return acc


def _epilogue(acc, s_x, s_w, bias_bits, bf16_mode: int):
    a = _arr(acc, np.int32)
    M, N = a.shape
    sx = _arr(s_x, np.float32)
    b = None if bias_bits is None else _arr(bias_bits, np.uint16)
    y32 = np.empty((M, N), np.float32)
    y = np.empty((M, N), np.uint16)
    _call("oracle_epilogue", _ptr(a), M, N, _ptr(sx), float(np.float32(s_w)), _ptr(b), bf16_mode,
          _ptr(y32), _ptr(y))
    return y32, y


def epilogue(acc, s_x, s_w, bias_bits=None):
    """(y32 float32 [M,N], y bf16 bits [M,N])."""
    return _epilogue(acc, s_x, s_w, bias_bits, 0)


def epilogue_bf16(acc, s_x, s_w, bias_bits=None):
    return _epilogue(acc, s_x, s_w, bias_bits, 1)


def pack_weights(w):
    """(packed uint8 [N, K/4], s_w float32, mean float32)."""
    a = _arr(w, np.float32)
    N, K = a.shape
    packed = np.empty((N, K // 4), np.uint8)
    s = np.zeros(2, np.float32)
    _call("oracle_pack_weights", _ptr(a), N, K, _ptr(packed), _ptr(s[0:1]), _ptr(s[1:2]))
    return packed, s[0], s[1]


def _forward(x_bits, packed, group_rows, s_ws, bias_bits, K, bf16_mode: int):
    x = _arr(x_bits, np.uint16)
    p = _arr(packed, np.uint8)
    M, Kx = x.shape
    N, KB = p.shape
    K = KB * 4 if K is None else K
    if K != Kx or K != KB * 4:
        raise ValueError("x and packed disagree on K")
    rows = _arr(group_rows, np.int64)
    sw = _arr([np.float32(s) for s in s_ws], np.float32)
    if rows.size != sw.size:
        raise ValueError("one scale per group")
    b = None if bias_bits is None else _arr(bias_bits, np.uint16)
    q = np.empty((M, K), np.int8)
    s_x = np.empty(M, np.float32)
    r = np.empty(M, np.int32)
    acc = np.empty((M, N), np.int32)
    y32 = np.empty((M, N), np.float32)
    y = np.empty((M, N), np.uint16)
    _call("oracle_forward", _ptr(x), M, K, _ptr(p), N, rows.size, _ptr(rows), _ptr(sw), _ptr(b), bf16_mode,
          _ptr(q), _ptr(s_x), _ptr(r), _ptr(acc), _ptr(y32), _ptr(y))
    return {"q": q, "s_x": s_x, "rowsum": r, "acc": acc, "y32": y32, "y": y}


def forward(x_bits, packed, s_w, bias_bits=None, K: int | None = None):
    """BitLinear.forward on packed weights; a dict with q, s_x, rowsum, acc, y32, y."""
    return _forward(x_bits, packed, [np.shape(packed)[0]], [s_w], bias_bits, K, 0)


def forward_grouped(x_bits, packed, group_rows, s_ws, bias_bits=None, K: int | None = None):
    return _forward(x_bits, packed, group_rows, s_ws, bias_bits, K, 0)


def forward_bf16(x_bits, packed, s_w, bias_bits=None, K: int | None = None):
    return _forward(x_bits, packed, [np.shape(packed)[0]], [s_w], bias_bits, K, 1)


def dequant(packed, s_w, K: int | None = None) -> np.ndarray:
    """bf16 bits [N, K] of u / s_w."""
    p = _arr(packed, np.uint8)
    N, KB = p.shape
    K = KB * 4 if K is None else K
    if K != KB * 4:
        raise ValueError("K must be four times the packed row length")
    out = np.empty((N, K), np.uint16)
    _call("oracle_dequant", _ptr(p), N, K, float(np.float32(s_w)), _ptr(out))
    return out
