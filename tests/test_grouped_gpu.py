"""bitlinear_forward_grouped (layers sharing one input: q/k/v, gate/up)
against the oracle, bit for bit, and against one bitlinear_forward call per
layer.  BitLinear.forward of the Falcon-Edge blog (section "Falcon-Edge, a
series of universal models"), once per layer of the stack."""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from tests.gpu_util import sample_rows

pytestmark = pytest.mark.gpu


def _stack(rows, K, seed, std=0.02):
    """The layers' weights packed by the GPU, and the same weights packed by
    the oracle (its own packing feeds its expected values)."""
    packs, scales, opks, oscales = [], [], [], []
    for g, n in enumerate(rows):
        w = synth.normal_f32(seed, 100 * g + n, (n, K), std * (1 + 0.5 * g))
        p, s, _ = bl.bitlinear_pack_weights(w.cuda())
        packs.append(p)
        scales.append(s)
        op, osw, _ = oracle.pack_weights(w.numpy())
        opks.append(op)
        oscales.append(osw)
    return torch.cat(packs), torch.cat(scales), packs, scales, np.concatenate(opks), oscales


def _check(M, K, rows, seed, with_bias, flags=0, sample=None):
    packed, s_ws, packs, scales, opk, oscales = _stack(rows, K, seed)
    N = sum(rows)
    x = synth.normal_bf16(seed, M + K, (M, K))
    b = synth.normal_bf16(seed, N, (N,), 0.05) if with_bias else None
    xd, bd = x.cuda(), (None if b is None else b.cuda())
    y = bl.bitlinear_forward_grouped(xd, packed, rows, s_ws, bd, flags=flags)
    # one call per layer gives the same columns
    off = 0
    for p, s, n in zip(packs, scales, rows):
        bb = None if bd is None else bd[off:off + n].clone()   # own 16-byte aligned buffer
        y1 = bl.bitlinear_forward(xd, p, s, bb)
        assert torch.equal(y[:, off:off + n].contiguous().view(torch.int16), y1.view(torch.int16)), f"layer at {off}"
        off += n
    torch.cuda.synchronize()
    mrows = np.arange(M) if sample is None else sample_rows(M, sample)
    xb = synth.bf16_bits(x)[mrows]
    want = oracle.forward_grouped(xb, opk, rows, oscales, None if b is None else synth.bf16_bits(b))
    got = y.cpu()[mrows].view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want["y"])


@pytest.mark.parametrize("M", [1, 4, 16])
def test_qkv_3b_decode(M):
    _check(M, 3200, [3200, 3200, 3200], 61, with_bias=False)


def test_qkv_3b_prefill_sampled():
    _check(2048, 3200, [3200, 3200, 3200], 62, with_bias=False, sample=24)


def test_gate_up_3b_decode_and_prefill():
    _check(4, 3200, [8640, 8640], 63, with_bias=False)
    _check(300, 3200, [8640, 8640], 64, with_bias=False, sample=16)


@pytest.mark.parametrize("M", [5, 40])
def test_ragged_groups_with_bias(M):
    _check(M, 640, [100, 37, 515], 65, with_bias=True)


def test_eight_groups_resident_flag():
    _check(3, 1088, [16, 48, 7, 130, 64, 1, 33, 250], 66, with_bias=True, flags=bl.WEIGHTS_RESIDENT)
    _check(70, 1088, [16, 48, 7, 130, 64, 1, 33, 250], 67, with_bias=True, flags=bl.WEIGHTS_RESIDENT)
