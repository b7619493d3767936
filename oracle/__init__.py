"""CPU oracle of the BitNet b1.58 BitLinear forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
cpu-baseline / reference legs of ``bench.py`` may import or call this module.
The product path (``bitlinear_fwd_b200``) never does, and shares no code with
it: the only common dependency is the seeded input generator ``synth``.

Plain numpy, one step per function, in the order and notation of the source
pages.  Sources (cited by short name below):

* [FE-univ]  Falcon-LLM team, "Falcon-Edge: a series of powerful, universal
  and fine-tunable 1.58bit language models" (blog; Arabic translation at
  n77n.net, Korean at molayo1419.me), section "Falcon-Edge, a series of
  universal models": the listings ``activation_norm_quant``,
  ``class BitLinear`` (``post_quant_process`` and ``forward``) and
  ``_weight_quant`` with the state-dict loop.
* [GN-BitNet] "BitNet: inference framework for 1-bit LLMs" (GeekNews,
  news.hada.io), Hacker News comments section: the weights are stored in
  2 bits (four codes).
* [Era-1bit] "The Era of 1-bit LLMs" (aitrends.kr summary), TL;DR: every
  weight is ternary {-1, 0, 1}.

Readings where the pages leave a step open (each is also listed in the
design notes):

* ``round()`` is round-half-to-even (PyTorch's rule); ``np.rint`` does that.
* Scales and the products x*scale, w*scale are float32 (bf16 input widens
  exactly); the clamp constant is the float32 literal 1e-5f.
* ``w.abs().mean()`` is the mean of the exact sum, rounded once to float32
  (any summation order gives a result within a few ulp of it; this one is
  unique).
* ``F.linear`` on the integer-valued operands is the exact integer sum
  ``acc = sum_k q*u`` (int32 suffices: |acc| <= 127*K).
* The epilogue is one float32 product d = s_x*s_w, one float32 division
  acc/d, then an optional float32 bias add, then one round-to-nearest-even
  to bfloat16.
* The 2-bit packing (the pages name ``unpack_weights`` but do not define
  it) stores code u+1 in {0,1,2}; row n of the packed matrix is K/16
  little-endian uint32 words; word g holds k = 16g + 4i + j in bits
  8j + 2i .. 8j + 2i + 1 (byte j, bit pair i).  Code 3 is invalid.
* bf16-faithful mode (``*_bf16`` functions): the listings run on a bf16
  module.  Every tensor op rounds its result to bf16; PyTorch computes
  elementwise bf16 ops in float32 and rounds once to bf16.  PyTorch evaluates
  ``127.0 / t`` as ``t.reciprocal() * 127.0`` (two roundings); the
  float32 mode reads that formula as one division instead.  The weight scale
  is the module's bf16 copy of s_w.  ``F.linear`` accumulates the exact
  integer products and rounds the sum once to bf16.  ``clamp_(min=1e-5)``
  bounds by bf16(1e-5).
* The bf16 export of the state-dict loop (``param_value / param_scale``)
  divides in float32 (the dtype of W) and rounds once to bfloat16 (RNE).
  It starts from the packed codes, so a zero is +0: ``round()`` can give
  -0.0 for small negative weights, and two bits do not keep that sign.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
things other than itself: a hand-worked example, exact rational arithmetic,
brute force over small domains, integer matmul, closed forms and invariants.
"""

from __future__ import annotations

import math

import numpy as np

F32 = np.float32
CLAMP_MIN = np.float32(1e-5)      # the listings' clamp_(min=1e-5), as float32
QMAX = 127.0                      # activation_norm_quant's 127.0


# ---------------------------------------------------------------------------
# bfloat16 <-> float32 (storage conversions, not part of the method)
# ---------------------------------------------------------------------------

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32; exact."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bfloat16, ties to even (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Step 1: activation quantisation  ([FE-univ] activation_norm_quant)
# ---------------------------------------------------------------------------

def act_quant(x_bits: np.ndarray):
    """Per-token absmax quantisation of bf16 activations to int8.

    For each row m: a = max_k |x[m,k]|; s_x = 127 / max(a, 1e-5);
    q = clamp(round(x * s_x), -128, 127).  Also returns the row sums of q
    (an integer by-product that the oracle does not need, but the CUDA path
    reports, so it is checked too).
    Returns (q int8 [M,K], s_x float32 [M], rowsum int32 [M]).
    """
    x = bf16_to_f32(x_bits)
    M, K = x.shape
    if M == 0:
        return np.zeros((0, K), np.int8), np.zeros(0, np.float32), np.zeros(0, np.int32)
    a = np.abs(x).max(axis=1)
    s_x = F32(QMAX) / np.maximum(a, CLAMP_MIN)
    t = x * s_x[:, None]
    q = np.clip(np.rint(t), -128, 127).astype(np.int8)
    rowsum = q.astype(np.int64).sum(axis=1).astype(np.int32)
    return q, s_x.astype(np.float32), rowsum


# ---------------------------------------------------------------------------
# Step 2a: weight absmean scale  ([FE-univ] _weight_quant, first line)
# ---------------------------------------------------------------------------

def exact_abs_sum(w: np.ndarray):
    """Exact sum of |w| over the whole tensor as an integer S with
    sum |w| = S * 2**-149, plus the element count.

    A finite float32 |w| is m * 2**(max(e,1) - 150) with e its biased
    exponent and m its 24-bit significand (hidden bit set when e > 0), i.e.
    (m << (max(e,1) - 1)) units of 2**-149.  Significands are first summed
    per exponent: each per-exponent sum is an integer below 2**24 * n, held
    exactly in float64 while n < 2**29.
    """
    bits = np.ascontiguousarray(w, dtype=np.float32).view(np.uint32).ravel() & np.uint32(0x7FFFFFFF)
    n = bits.size
    if n >= (1 << 29):
        raise ValueError("tensor too large for the exact per-exponent float64 sums")
    e = (bits >> np.uint32(23)).astype(np.int64)
    if n and int(e.max()) == 255:
        raise ValueError("non-finite weight")
    m = (bits & np.uint32(0x7FFFFF)) | np.where(e > 0, np.uint32(0x800000), np.uint32(0))
    per_exp = np.bincount(e, weights=m.astype(np.float64), minlength=256)
    S = 0
    for ex in range(256):
        v = int(per_exp[ex])
        if v:
            S += v << (max(ex, 1) - 1)
    return S, n


def round_to_f32(num: int, den: int) -> np.float32:
    """float32 nearest to num/den (num >= 0, den > 0), ties to even; the
    result's last place is never below 2**-149 (gradual underflow)."""
    if num == 0:
        return F32(0.0)
    e = num.bit_length() - den.bit_length() - 24
    # move e until 2**23 <= num / (den * 2**e) < 2**24
    while True:
        n_s = num << max(-e, 0)
        d_s = den << max(e, 0)
        if n_s < (d_s << 23):
            e -= 1
        elif n_s >= (d_s << 24):
            e += 1
        else:
            break
    e = max(e, -149)
    n_s = num << max(-e, 0)
    d_s = den << max(e, 0)
    q, r = divmod(n_s, d_s)
    if 2 * r > d_s or (2 * r == d_s and (q & 1)):
        q += 1
    return F32(math.ldexp(q, e))


def absmean(w: np.ndarray) -> np.float32:
    """mean(|w|) over the whole tensor, exactly rounded to float32."""
    S, n = exact_abs_sum(w)
    if n == 0:
        raise ValueError("empty weight")
    return round_to_f32(S, n << 149)


def weight_scale(mean: np.float32) -> np.float32:
    """s_w = 1 / max(mean, 1e-5) in float32 ([FE-univ] _weight_quant)."""
    return F32(F32(1.0) / np.maximum(F32(mean), CLAMP_MIN))


# ---------------------------------------------------------------------------
# Step 2b: ternarisation  ([FE-univ] _weight_quant, second line)
# ---------------------------------------------------------------------------

def ternarise(w: np.ndarray, s_w: np.float32) -> np.ndarray:
    """u = clamp(round(w * s_w), -1, 1) as int8 ([Era-1bit]: u in {-1,0,1})."""
    t = np.asarray(w, dtype=np.float32) * F32(s_w)
    return np.clip(np.rint(t), -1, 1).astype(np.int8)


# ---------------------------------------------------------------------------
# Step 2c: 2-bit packing  ([GN-BitNet] 2 bits per weight; layout: module doc)
# ---------------------------------------------------------------------------

def pack(u: np.ndarray) -> np.ndarray:
    """Pack ternary u [N,K] (K % 16 == 0) into uint8 [N, K/4]."""
    N, K = u.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    if np.any((u < -1) | (u > 1)):
        raise ValueError("not ternary")
    code = (u.astype(np.int64) + 1).astype(np.uint64)  # u + 1 in {0, 1, 2}
    c = code.reshape(N, K // 16, 4, 4)                 # [n, g, i, j], k = 16g + 4i + j
    i = np.arange(4, dtype=np.uint64)[:, None]
    j = np.arange(4, dtype=np.uint64)[None, :]
    shift = np.uint64(8) * j + np.uint64(2) * i        # bit position of (i, j)
    words = (c << shift).sum(axis=(2, 3), dtype=np.uint64).astype("<u4")
    return np.ascontiguousarray(words).view(np.uint8).reshape(N, K // 4)


def unpack(packed: np.ndarray, K: int | None = None) -> np.ndarray:
    """Inverse of ``pack``: uint8 [N, K/4] -> ternary int8 [N, K].
    Raises ValueError on the unused code 3."""
    N, KB = packed.shape
    K = KB * 4 if K is None else K
    words = np.ascontiguousarray(packed).view("<u4").astype(np.uint64)  # [N, K/16]
    i = np.arange(4, dtype=np.uint64)[:, None]
    j = np.arange(4, dtype=np.uint64)[None, :]
    shift = np.uint64(8) * j + np.uint64(2) * i
    c = (words[:, :, None, None] >> shift) & np.uint64(3)
    if np.any(c == 3):
        raise ValueError("invalid 2-bit code 3")
    return (c.astype(np.int64) - 1).astype(np.int8).reshape(N, K)


# ---------------------------------------------------------------------------
# Step 3: the contraction  ([FE-univ] BitLinear.forward, F.linear)
# ---------------------------------------------------------------------------

def contract(q: np.ndarray, u: np.ndarray, block: int = 2048) -> np.ndarray:
    """acc[m,n] = sum_k q[m,k] * u[n,k], exact, as int32.

    Uses a float64 matrix product as the library step: every product and
    every partial sum is an integer of magnitude <= 127*K < 2**53, so the
    result is exact in any summation order.  Row blocks of u bound memory.
    """
    M, K = q.shape
    N = u.shape[0]
    if 127 * K >= (1 << 31):
        raise ValueError("K too large for int32 accumulation")
    qf = q.astype(np.float64)
    acc = np.empty((M, N), dtype=np.int32)
    for n0 in range(0, N, block):
        uf = u[n0:n0 + block].astype(np.float64)
        acc[:, n0:n0 + block] = (qf @ uf.T).astype(np.int64).astype(np.int32)
    return acc


# ---------------------------------------------------------------------------
# Step 4: epilogue  ([FE-univ] BitLinear.post_quant_process and bias add)
# ---------------------------------------------------------------------------

def epilogue(acc: np.ndarray, s_x: np.ndarray, s_w: np.float32, bias_bits=None):
    """y = acc / (s_x * s_w) (+ bias), float32, then bfloat16 (RNE).

    Returns (y32 float32 [M,N], y bf16 bits uint16 [M,N]).  |acc| < 2**24 so
    its float32 conversion is exact.
    """
    d = np.asarray(s_x, np.float32) * F32(s_w)
    y32 = acc.astype(np.float32) / d[:, None]
    if bias_bits is not None:
        y32 = y32 + bf16_to_f32(bias_bits)[None, :]
    y32 = y32.astype(np.float32)
    return y32, f32_to_bf16_rne(y32)


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def pack_weights(w: np.ndarray):
    """[FE-univ] _weight_quant followed by packing: (packed, s_w, mean)."""
    w = np.asarray(w, dtype=np.float32)
    mean = absmean(w)
    s_w = weight_scale(mean)
    return pack(ternarise(w, s_w)), s_w, mean


def forward(x_bits: np.ndarray, packed: np.ndarray, s_w: np.float32, bias_bits=None, K: int | None = None):
    """[FE-univ] BitLinear.forward on packed weights.

    Returns a dict with every intermediate: q, s_x, rowsum, acc, y32, y.
    """
    q, s_x, rowsum = act_quant(x_bits)
    u = unpack(packed, K)
    acc = contract(q, u)
    y32, y = epilogue(acc, s_x, s_w, bias_bits)
    return {"q": q, "s_x": s_x, "rowsum": rowsum, "acc": acc, "y32": y32, "y": y}


def forward_grouped(x_bits: np.ndarray, packed: np.ndarray, group_rows, s_ws, bias_bits=None,
                    K: int | None = None):
    """Several BitLinear layers that read the same input (q/k/v, gate/up):
    [FE-univ] BitLinear.forward applied to each group of rows of the stacked
    packed matrix with that group's scale; the outputs side by side in one
    [M, sum(rows)] array.  Returns the same dict as ``forward``."""
    q, s_x, rowsum = act_quant(x_bits)
    u = unpack(packed, K)
    acc = contract(q, u)
    y32 = np.empty(acc.shape, np.float32)
    y = np.empty(acc.shape, np.uint16)
    off = 0
    for rows, s_w in zip(group_rows, s_ws):
        b = None if bias_bits is None else bias_bits[off:off + rows]
        y32[:, off:off + rows], y[:, off:off + rows] = epilogue(acc[:, off:off + rows], s_x, s_w, b)
        off += rows
    assert off == acc.shape[1]
    return {"q": q, "s_x": s_x, "rowsum": rowsum, "acc": acc, "y32": y32, "y": y}


# ---------------------------------------------------------------------------
# bf16-faithful mode: the listings' dtype semantics on a bf16 module
# ---------------------------------------------------------------------------

def _bf16(v) -> np.ndarray:
    """Round float32 values to bf16 (RNE) and widen back to float32."""
    return bf16_to_f32(f32_to_bf16_rne(np.asarray(v, np.float32)))


def act_quant_bf16(x_bits: np.ndarray):
    """[FE-univ] activation_norm_quant on bf16 tensors, evaluated as PyTorch
    does: ``127.0 / t`` is ``t.reciprocal() * 127.0``, so scale =
    bf16(bf16(1 / max(a, bf16(1e-5))) * 127), then q = clamp(round(bf16(x *
    scale)), -128, 127).
    Returns (q int8 [M,K], s_x float32 [M] holding bf16 values, rowsum int32)."""
    x = bf16_to_f32(x_bits)
    M, K = x.shape
    if M == 0:
        return np.zeros((0, K), np.int8), np.zeros(0, np.float32), np.zeros(0, np.int32)
    a = np.abs(x).max(axis=1)
    s_x = _bf16(_bf16(F32(1.0) / np.maximum(a, _bf16(CLAMP_MIN))) * F32(QMAX))
    t = _bf16(x * s_x[:, None])                 # bf16 * bf16 is exact in float32, then one rounding
    q = np.clip(np.rint(t), -128, 127).astype(np.int8)
    rowsum = q.astype(np.int64).sum(axis=1).astype(np.int32)
    return q, s_x.astype(np.float32), rowsum


def epilogue_bf16(acc: np.ndarray, s_x: np.ndarray, s_w: np.float32, bias_bits=None):
    """[FE-univ] BitLinear.forward after F.linear on a bf16 module: y =
    bf16(acc); d = bf16(bf16(s_w) * s_x); y = bf16(y / d); y = bf16(y + bias).
    Returns (y32 float32 holding the bf16 values, y bf16 bits)."""
    y = _bf16(acc.astype(np.float32))
    d = _bf16(_bf16(np.float32(s_w)) * np.asarray(s_x, np.float32))
    y = _bf16(y / d[:, None])
    if bias_bits is not None:
        y = _bf16(y + bf16_to_f32(bias_bits)[None, :])
    y = y.astype(np.float32)
    return y, f32_to_bf16_rne(y)


def forward_bf16(x_bits: np.ndarray, packed: np.ndarray, s_w: np.float32, bias_bits=None,
                 K: int | None = None):
    """BitLinear.forward with the listings' bf16 dtype semantics."""
    q, s_x, rowsum = act_quant_bf16(x_bits)
    acc = contract(q, unpack(packed, K))
    y32, y = epilogue_bf16(acc, s_x, s_w, bias_bits)
    return {"q": q, "s_x": s_x, "rowsum": rowsum, "acc": acc, "y32": y32, "y": y}


# ---------------------------------------------------------------------------
# bf16 export of the ternary weights
# ---------------------------------------------------------------------------

def dequant(packed: np.ndarray, s_w: np.float32, K: int | None = None) -> np.ndarray:
    """[FE-univ] state-dict loop: ``param_value = u / param_scale``, stored
    as bfloat16.  u comes from the packed codes; u / s_w is rounded to float32
    once, then to bfloat16 (RNE).  Returns uint16 bf16 bits [N, K]."""
    u = unpack(packed, K).astype(np.int64)
    num, den = np.float64(np.float32(s_w)).as_integer_ratio()   # s_w = num / den exactly
    inv = round_to_f32(den, num)                                  # RN_f32(1 / s_w)
    w32 = np.where(u > 0, inv, np.where(u < 0, -inv, np.float32(0.0))).astype(np.float32)
    return f32_to_bf16_rne(w32)

