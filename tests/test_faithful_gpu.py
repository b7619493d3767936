"""bf16-faithful mode (BITLINEAR_BF16_FAITHFUL): the CUDA path against the
oracle's bf16 mode, bit for bit -- activation_norm_quant and
BitLinear.forward of the Falcon-Edge blog evaluated as a bfloat16 module
evaluates them (every tensor op rounded to bf16; 127.0 / t as
t.reciprocal() * 127)."""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from synth import workloads as wl
from tests.gpu_util import sample_rows

pytestmark = pytest.mark.gpu


def _compare(x, w, bias, engine, rows=None):
    packed, s_w, _ = bl.bitlinear_pack_weights(w.cuda())
    out = bl.bitlinear_forward_debug(x.cuda(), packed, s_w, None if bias is None else bias.cuda(),
                                     engine=engine, flags=bl.BF16_FAITHFUL)
    torch.cuda.synchronize()
    assert bl.bitlinear_check_status(out["ws"]) == 0
    M = x.shape[0]
    rows = np.arange(M) if rows is None else rows
    xb = synth.bf16_bits(x)
    # the oracle packs the same weights itself; nothing the GPU computed feeds it
    opk, osw, _ = oracle.pack_weights(w.numpy())
    want = oracle.forward_bf16(xb[rows], opk, osw, None if bias is None else synth.bf16_bits(bias))
    assert np.array_equal(out["xq"].cpu().numpy()[rows], want["q"])
    assert np.array_equal(out["s_x"].cpu().numpy()[rows], want["s_x"])
    assert np.array_equal(out["acc"].cpu().numpy()[rows], want["acc"])
    assert np.array_equal(out["y32"].cpu().numpy()[rows], want["y32"])
    assert np.array_equal(out["y"].cpu()[rows].view(torch.int16).numpy().view(np.uint16), want["y"])


@pytest.mark.parametrize("engine", [1, 2])
def test_workload1_both_engines(engine):
    (case,) = wl.workload1()
    _compare(case.x(), case.w(), case.bias(), engine)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 11008, 4096), (5, 97, 17472), (300, 520, 1088)])
def test_shapes_with_bias(M, N, K):
    x = synth.normal_bf16(88, M + K, (M, K))
    w = synth.normal_f32(88, N + K, (N, K), 0.02)
    b = synth.normal_bf16(88, N, (N,), 0.1)
    _compare(x, w, b, 0)


def test_prefill_3b_sampled():
    x = synth.student_t4_bf16(89, 1, (2048, 3200))
    w = synth.normal_f32(89, 2, (8640, 3200), 0.02)
    _compare(x, w, None, 0, rows=sample_rows(2048, 20))


def test_faithful_grouped_matches_single_calls():
    x = synth.normal_bf16(90, 3, (4, 640)).cuda()
    packs, scales = [], []
    for g, n in enumerate([100, 60]):
        p, s, _ = bl.bitlinear_pack_weights(synth.normal_f32(90, 10 + g, (n, 640), 0.02).cuda())
        packs.append(p)
        scales.append(s)
    y = bl.bitlinear_forward_grouped(x, torch.cat(packs), [100, 60], torch.cat(scales), flags=bl.BF16_FAITHFUL)
    y0 = bl.bitlinear_forward(x, packs[0], scales[0], flags=bl.BF16_FAITHFUL)
    y1 = bl.bitlinear_forward(x, packs[1], scales[1], flags=bl.BF16_FAITHFUL)
    assert torch.equal(y.view(torch.int16), torch.cat([y0, y1], 1).view(torch.int16))
