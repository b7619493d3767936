"""Helpers for the GPU parity tests: run a workload case through the C ABI
(via the binding) and through the CPU oracle on the same seeded inputs."""

from __future__ import annotations

import functools

import numpy as np
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth

BIG = 50_000_000        # above this many weights, packing is compared on sampled rows


@functools.lru_cache(maxsize=8)
def _weights(case_key, make_w):
    return make_w()


def sample_rows(M: int, k: int = 61, seed: int = 5) -> np.ndarray:
    rng = np.random.default_rng(seed + M)
    extra = rng.choice(M, size=min(k, M), replace=False) if M > 0 else []
    return np.unique(np.concatenate([[0, 1, M - 1], extra]).clip(0, max(M - 1, 0))).astype(np.int64)


def gpu_pack(w: torch.Tensor):
    packed, s_w, mean = bl.bitlinear_pack_weights(w.cuda())
    return packed, s_w, mean


def oracle_weights(w: torch.Tensor, rows=None):
    """Oracle s_w and mean over the whole tensor; ternary u and packed bytes
    for all rows (or the given rows)."""
    wn = w.numpy()
    mean = oracle.absmean(wn)
    s_w = oracle.weight_scale(mean)
    sub = wn if rows is None else wn[rows]
    u = oracle.ternarise(sub, s_w)
    return {"mean": mean, "s_w": s_w, "u": u, "packed": oracle.pack(u)}


def oracle_forward_rows(x: torch.Tensor, u: np.ndarray, s_w, bias, rows):
    xb = synth.bf16_bits(x)[rows]
    q, s_x, _ = oracle.act_quant(xb)
    acc = oracle.contract(q, u)
    bb = None if bias is None else synth.bf16_bits(bias)
    y32, y = oracle.epilogue(acc, s_x, s_w, bb)
    return {"q": q, "s_x": s_x, "acc": acc, "y32": y32, "y": y}


def f32_bits(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32)


def assert_same_f32(got, want, what):
    g, w = f32_bits(got), f32_bits(want)
    bad = np.flatnonzero(g.ravel() != w.ravel())
    assert bad.size == 0, f"{what}: {bad.size} of {g.size} differ, first at {bad[:5]}: " \
        f"{np.asarray(got).ravel()[bad[:5]]} vs {np.asarray(want).ravel()[bad[:5]]}"


def assert_equal(got, want, what):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    bad = np.flatnonzero(got.ravel() != want.ravel())
    assert bad.size == 0, f"{what}: {bad.size} of {got.size} differ, first at {bad[:5]}: " \
        f"{got.ravel()[bad[:5]]} vs {want.ravel()[bad[:5]]}"


def check_y32_tolerance(got, want, acc, d_rows):
    """The stated bar for the float32 pre-cast output: relative error
    <= 1e-6 against the oracle (the kernels are in fact bit-exact; this is
    asserted separately)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    scale = np.maximum(np.abs(want), 1e-30)
    assert np.all(np.abs(got - want) <= 1e-6 * scale)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """|a - b| in units of bf16 ulps (both finite bf16 bit patterns)."""
    def ordered(v):
        v = v.astype(np.int64)
        return np.where(v & 0x8000, 0x8000 - (v & 0x7FFF), 0x8000 + v)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def run_and_compare(x, w, bias, engine=0, rows=None, check_pack_rows=None):
    """Runs pack + forward_debug on the GPU and compares every output with
    the oracle.  rows: token rows compared for acc/y (None = all)."""
    M, K = x.shape
    N = w.shape[0]
    prow = None
    if N * K > BIG:
        prow = sample_rows(N, 31, seed=11) if check_pack_rows is None else check_pack_rows
    ow = oracle_weights(w, prow)
    packed, s_w, mean = gpu_pack(w)
    assert_same_f32(mean.cpu().numpy(), [ow["mean"]], "mean |w|")
    assert_same_f32(s_w.cpu().numpy(), [ow["s_w"]], "s_w")
    gp = packed.cpu().numpy()
    assert_equal(gp if prow is None else gp[prow], ow["packed"], "packed weights")

    xd = x.cuda()
    bd = None if bias is None else bias.cuda()
    out = bl.bitlinear_forward_debug(xd, packed, s_w, bd, engine=engine)
    y_plain = bl.bitlinear_forward(xd, packed, s_w, bd) if engine == 0 else None
    torch.cuda.synchronize()
    assert bl.bitlinear_check_status(out["ws"]) == 0

    # activations: full compare (the oracle is fast here)
    q_all, sx_all, _ = oracle.act_quant(synth.bf16_bits(x))
    assert_equal(out["xq"].cpu().numpy(), q_all, "int8 activations")
    assert_same_f32(out["s_x"].cpu().numpy(), sx_all, "s_x")

    rows = np.arange(M) if rows is None else rows
    u = ow["u"] if prow is None else oracle.ternarise(w.numpy(), ow["s_w"])
    ref = oracle_forward_rows(x, u, ow["s_w"], bias, rows)
    acc = out["acc"].cpu().numpy()[rows]
    y32 = out["y32"].cpu().numpy()[rows]
    yb = out["y"].cpu().view(torch.int16).numpy().view(np.uint16)[rows]
    assert_equal(acc, ref["acc"], "int32 accumulators")
    check_y32_tolerance(y32, ref["y32"], acc, None)
    assert_same_f32(y32, ref["y32"], "y32 (bit-exact)")
    assert np.all(bf16_ulp_diff(yb, ref["y"]) <= 1)
    assert_equal(yb, ref["y"], "bf16 y (bit-exact)")
    if y_plain is not None:
        assert torch.equal(y_plain.cpu().view(torch.int16), out["y"].cpu().view(torch.int16))
    return out
