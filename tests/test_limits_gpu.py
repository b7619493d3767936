"""GPU parity at the edges of the shapes the C ABI accepts.

* K = 2^19, the largest K the header allows: there the exact sum |acc| can
  pass 2^24, so float(acc) is no longer exact and the epilogue's quotient
  starts from a rounded numerator (Falcon-Edge blog, section "Falcon-Edge, a
  series of universal models", post_quant_process: acc / (s_x * s_w)).  The
  inputs are built so that several rows do pass 2^24, on both engines.
* A grouped call at the 100B-class gate + up stack: N = 2 x 28672 rows,
  K = 8192, at M = 1 (decode engine) and M = 512 (prefill engine), sampled
  output columns and tokens.
* A very tall, narrow matrix: N = 2^23 - 1 rows (the largest N, ragged in
  every tile size) at K = 64, sampled columns.

Every expected value comes from the CPU oracle on its own packing of the
same seeded weights (or on the same seeded ternary codes); nothing the GPU
computes is fed to the oracle.
"""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from tests.gpu_util import assert_equal, assert_same_f32, sample_rows

pytestmark = pytest.mark.gpu

SEED = 0xB17E


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_columns(x_bits, opk_cols, s_w_cols, bias_bits_cols=None):
    """The oracle's forward for a subset of output columns: opk_cols are the
    oracle's packed rows of those columns, s_w_cols the scale of each
    column's layer."""
    q, s_x, _ = oracle.act_quant(x_bits)
    acc = oracle.contract(q, oracle.unpack(opk_cols))
    y32 = np.empty(acc.shape, np.float32)
    y = np.empty(acc.shape, np.uint16)
    for s in np.unique(s_w_cols):
        sel = np.flatnonzero(s_w_cols == s)
        b = None if bias_bits_cols is None else bias_bits_cols[sel]
        y32[:, sel], y[:, sel] = oracle.epilogue(acc[:, sel], s_x, np.float32(s), b)
    return {"q": q, "s_x": s_x, "acc": acc, "y32": y32, "y": y}


# ---------------------------------------------------------------------------
# K = 2^19: accumulators beyond 2^24
# ---------------------------------------------------------------------------

K_MAX = 1 << 19
N_K = 40                    # ragged for the 16-row units and the 128-row tiles


def _large_acc_inputs(M):
    """Weights whose first rows are (nearly) constant-sign, so that their
    ternary codes are all +1 or all -1, and positive activations of similar
    size, so that q is 64..127 on every k and |acc| reaches ~5e7 > 2^24."""
    w = synth.normal_f32(SEED, 1, (N_K, K_MAX), 0.3)
    w[0] = 1.0 + w[0] * 0.1
    w[1] = -1.0 + w[1] * 0.1
    w[2] = torch.where(torch.arange(K_MAX) % 3 == 0, -1.0, 1.0) * (1.0 + w[2] * 0.1)
    w[3] = 1.0 + w[3] * 0.1
    w[3, : K_MAX // 2] = 0.0
    # rows 4..10: constant sign (alternating +, -) with the first r - 3 weights
    # zeroed, so their sums differ from row 0's by a few small q values and
    # some of them are odd (float(acc) then rounds)
    for r in range(4, 11):
        w[r] = (1.0 if r % 2 == 0 else -1.0) + w[r] * 0.1
        w[r, : r - 3] = 0.0
    x = synth.normal_f32(SEED, 2, (M, K_MAX), 0.1).abs() + 0.6
    x[0, 7] = 2.0                              # one larger value: q = round(x * 63.5)
    return x.to(torch.bfloat16), w, synth.normal_bf16(SEED, 3, (N_K,), 0.01)


@pytest.fixture(scope="module")
def large_k_weights():
    _, w, _ = _large_acc_inputs(1)
    opk, osw, omean = oracle.pack_weights(w.numpy())
    packed, s_w, mean = bl.bitlinear_pack_weights(w.cuda())
    assert_same_f32(mean.cpu().numpy(), [omean], "mean |w| at K = 2^19")
    assert_same_f32(s_w.cpu().numpy(), [osw], "s_w at K = 2^19")
    assert_equal(packed.cpu().numpy(), opk, "packed weights at K = 2^19")
    return packed, s_w, opk, osw


@pytest.mark.parametrize("M,engine", [(1, 1), (1, 2), (16, 1), (16, 2), (64, 2)])
def test_k_max_accumulators_beyond_2_24(large_k_weights, M, engine):
    packed, s_w, opk, osw = large_k_weights
    x, _, bias = _large_acc_inputs(M)
    ref = oracle.forward(synth.bf16_bits(x), opk, osw, synth.bf16_bits(bias))
    # the case this test exists for: numerators that float32 cannot hold exactly
    big = np.abs(ref["acc"]) > (1 << 24)
    assert big.sum() >= 8 * M, "the inputs must drive |acc| past 2^24 (rows 0, 1 and 4..10 for every token)"
    assert np.any(ref["acc"][big] % 2 != 0), "some of them must be odd, so that float(acc) rounds"
    out = bl.bitlinear_forward_debug(x.cuda(), packed, s_w, bias.cuda(), engine=engine)
    torch.cuda.synchronize()
    assert bl.bitlinear_check_status(out["ws"]) == 0
    assert_equal(out["xq"].cpu().numpy(), ref["q"], "int8 activations")
    assert_same_f32(out["s_x"].cpu().numpy(), ref["s_x"], "s_x")
    assert_equal(out["acc"].cpu().numpy(), ref["acc"], "int32 accumulators")
    assert_same_f32(out["y32"].cpu().numpy(), ref["y32"], "y32")
    assert_equal(_u16(out["y"]), ref["y"], "bf16 y")


# ---------------------------------------------------------------------------
# grouped call at the 100B-class gate + up stack
# ---------------------------------------------------------------------------

H100B, F100B = 8192, 28672


@pytest.fixture(scope="module")
def gate_up():
    ws = [synth.normal_f32(SEED, 10 + g, (F100B, H100B), 0.01) for g in range(2)]
    gpu = [bl.bitlinear_pack_weights(w.cuda()) for w in ws]
    orc = [oracle.pack_weights(w.numpy()) for w in ws]
    cols = sample_rows(F100B, 200, seed=3)
    for (p, s, m), (opk, osw, om) in zip(gpu, orc):
        assert_same_f32(s.cpu().numpy(), [osw], "s_w")
        assert_equal(p.cpu().numpy()[cols], opk[cols], "packed rows")
    del ws
    packed = torch.cat([gpu[0][0], gpu[1][0]])
    scales = torch.cat([gpu[0][1], gpu[1][1]])
    return packed, scales, [o[0] for o in orc], [o[1] for o in orc]


@pytest.mark.parametrize("M", [1, 512])
def test_grouped_gate_up_100b(gate_up, M):
    packed, scales, opks, osws = gate_up
    x = synth.normal_bf16(SEED, 20 + M, (M, H100B))
    bias = synth.normal_bf16(SEED, 30, (2 * F100B,), 0.01)
    y = bl.bitlinear_forward_grouped(x.cuda(), packed, [F100B, F100B], scales, bias.cuda())
    torch.cuda.synchronize()
    # sampled output columns of both layers, including the boundary between them
    c0 = sample_rows(F100B, 150, seed=7)
    cols = np.unique(np.concatenate([c0, F100B + c0, [F100B - 1, F100B, 2 * F100B - 1]]))
    opk_cols = np.concatenate([opks[0][cols[cols < F100B]], opks[1][cols[cols >= F100B] - F100B]])
    s_cols = np.where(cols < F100B, osws[0], osws[1]).astype(np.float32)
    toks = np.arange(M) if M <= 16 else sample_rows(M, 40)
    xb = synth.bf16_bits(x)[toks]
    ref = _oracle_columns(xb, opk_cols, s_cols, synth.bf16_bits(bias)[cols])
    got = _u16(y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(cols).cuda()])
    assert_equal(got, ref["y"], f"grouped gate+up y at M = {M}")


# ---------------------------------------------------------------------------
# N = 2^23 - 1 rows at K = 64
# ---------------------------------------------------------------------------

N_MAX = (1 << 23) - 1


def _ternary_codes(seed, stream, shape):
    """Seeded ternary matrix u in {-1, 0, 1}: the sign of a normal draw, zero
    where |draw| < 0.43 (about a third of the entries)."""
    z = synth.normal_f32(seed, stream, shape)
    return (torch.sign(z) * (z.abs() >= 0.43)).to(torch.int8).numpy()


@pytest.fixture(scope="module")
def tall():
    u = _ternary_codes(SEED, 40, (N_MAX, 64))
    opk = oracle.pack(u)
    return torch.from_numpy(opk).cuda(), opk


@pytest.mark.parametrize("M,engine", [(3, 1), (16, 1), (40, 2)])
def test_tallest_matrix(tall, M, engine):
    packed, opk = tall
    s_w = np.float32(21.5)
    x = synth.normal_bf16(SEED, 50 + M, (M, 64))
    out = bl.bitlinear_forward_debug(x.cuda(), packed, torch.tensor([s_w], device="cuda"), engine=engine)
    torch.cuda.synchronize()
    assert bl.bitlinear_check_status(out["ws"]) == 0
    cols = np.unique(np.concatenate([sample_rows(N_MAX, 3000, seed=9), np.arange(N_MAX - 40, N_MAX)]))
    ref = _oracle_columns(synth.bf16_bits(x), opk[cols], np.full(cols.size, s_w, np.float32))
    ct = torch.from_numpy(cols).cuda()
    assert_equal(out["acc"][:, ct].cpu().numpy(), ref["acc"], "int32 accumulators")
    assert_same_f32(out["y32"][:, ct].cpu().numpy(), ref["y32"], "y32")
    assert_equal(_u16(out["y"][:, ct]), ref["y"], "bf16 y")
