"""Tensor-parallel BitLinear forward on the CPU: the oracle's steps, split
over the ranks of a torch.distributed process group, with the exchanges
such a split needs.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests may use
it.  It shows that the split design is exact before any GPU code exists
for it, and it is not that GPU code.

BitLinear.forward and _weight_quant of the Falcon-Edge blog (section
"Falcon-Edge, a series of universal models") reduce over whole tensors
twice: the activation scale takes each token's absmax over all of K, and
the weight scale takes mean |w| over the whole matrix.  A split has to
reproduce both exactly, and so it does:

* K-split (row parallel; rank r holds x[:, K_r] and W[:, K_r]):
  - the absmax is an all-reduce MAX of each token's partial absmax (max is
    exact in any order);
  - mean |w| comes from an all-reduce SUM of per-exponent significand sums,
    integers, so the sum is exact and independent of order; it is rounded
    once, as the unsplit oracle does;
  - each rank contracts its slice in int32; an all-reduce SUM of those
    partial sums is exact, and the epilogue runs on the total.
* N-split (column parallel; rank r holds W[N_r, :] and the whole x):
  - the same exponent-bin all-reduce gives the whole-tensor s_w;
  - each rank runs the forward of its rows; an all-gather joins the column
    blocks.

Either way every output equals the unsplit forward bit for bit.
"""

from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import (CLAMP_MIN, F32, QMAX, bf16_to_f32, contract, epilogue, forward, forward_bf16, pack,
               round_to_f32, ternarise, unpack)


def abs_bins(w: np.ndarray) -> np.ndarray:
    """Per-exponent sums of the significands of |w|: bins[e] = sum of m over
    the elements with biased exponent e, where |w| = m * 2^(max(e,1) - 150).
    int64; exact while the tensor has fewer than 2^29 elements."""
    bits = np.ascontiguousarray(w, dtype=np.float32).view(np.uint32).ravel() & np.uint32(0x7FFFFFFF)
    if bits.size >= (1 << 29):
        raise ValueError("shard too large for exact float64 bin sums")
    e = (bits >> np.uint32(23)).astype(np.int64)
    if bits.size and int(e.max()) == 255:
        raise ValueError("non-finite weight")
    m = (bits & np.uint32(0x7FFFFF)) | np.where(e > 0, np.uint32(0x800000), np.uint32(0))
    return np.bincount(e, weights=m.astype(np.float64), minlength=256).astype(np.int64)


def mean_from_bins(bins: np.ndarray, n: int) -> np.float32:
    """mean |w| from the exponent bins of the whole tensor, rounded once to
    float32 (ties to even, last place at least 2^-149)."""
    if n <= 0:
        raise ValueError("empty weight")
    S = 0
    for e in range(256):
        v = int(bins[e])
        if v:
            S += v << (max(e, 1) - 1)
    return round_to_f32(S, n << 149)


def _all_reduce(a: np.ndarray, op) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a).copy())
    dist.all_reduce(t, op=op)
    return t.numpy()


def global_weight_scale(w_shard: np.ndarray):
    """Whole-tensor (mean, s_w) from this rank's shard: one all-reduce SUM of
    the exponent bins and of the element count."""
    bins = _all_reduce(abs_bins(w_shard), dist.ReduceOp.SUM)
    n = int(_all_reduce(np.array([w_shard.size], np.int64), dist.ReduceOp.SUM)[0])
    mean = mean_from_bins(bins, n)
    return mean, F32(F32(1.0) / np.maximum(F32(mean), CLAMP_MIN))


def act_quant_given_absmax(x_bits: np.ndarray, a: np.ndarray):
    """activation_norm_quant with the token absmax supplied: s_x = 127 /
    max(a, 1e-5), q = clamp(round(x * s_x), -128, 127)."""
    x = bf16_to_f32(x_bits)
    s_x = (F32(QMAX) / np.maximum(np.asarray(a, np.float32), CLAMP_MIN)).astype(np.float32)
    q = np.clip(np.rint(x * s_x[:, None]), -128, 127).astype(np.int8)
    return q, s_x


def forward_ksplit(x_bits_shard: np.ndarray, w_shard: np.ndarray, bias_bits=None):
    """K-split forward: this rank's columns of x and W (the same K range;
    a multiple of 16 wide).  Every rank returns the full outputs."""
    x = bf16_to_f32(x_bits_shard)
    a_local = np.abs(x).max(axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    a = _all_reduce(a_local.astype(np.float32), dist.ReduceOp.MAX)
    q, s_x = act_quant_given_absmax(x_bits_shard, a)
    mean, s_w = global_weight_scale(w_shard)
    packed = pack(ternarise(w_shard, s_w))
    acc_local = contract(q, unpack(packed)).astype(np.int64)
    acc = _all_reduce(acc_local, dist.ReduceOp.SUM).astype(np.int32)
    y32, y = epilogue(acc, s_x, s_w, bias_bits)
    return {"q": q, "s_x": s_x, "mean": mean, "s_w": s_w, "packed": packed, "acc": acc, "y32": y32, "y": y}


def forward_nsplit(x_bits: np.ndarray, w_shard: np.ndarray, bias_bits_shard=None, bf16_mode: bool = False):
    """N-split forward: this rank's rows of W, the whole x.  Every rank
    returns the whole y, its column blocks gathered in rank order."""
    mean, s_w = global_weight_scale(w_shard)
    packed = pack(ternarise(w_shard, s_w))
    f = forward_bf16 if bf16_mode else forward
    out = f(x_bits, packed, s_w, bias_bits_shard)
    blocks = [None] * dist.get_world_size()
    dist.all_gather_object(blocks, (out["y32"], out["y"]))
    y32 = np.concatenate([b[0] for b in blocks], axis=1)
    y = np.concatenate([b[1] for b in blocks], axis=1)
    return {"mean": mean, "s_w": s_w, "packed": packed, "y32": y32, "y": y}
