"""The failure path of the device-side bounded waits, driven without a real
hang: the test hook bitlinear_test_force_timeout makes every forward take
one wait on a barrier that nothing signals (1 ms limit).  Each engine must
then report BITLINEAR_ERR_TIMEOUT through the workspace status word, let
its in-flight copies and tensor-core work finish, and leave the context
usable: the next forward, with the hook off, must match the oracle."""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from tests.gpu_util import assert_equal

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = -6


@pytest.fixture(autouse=True)
def _hook_off():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    bl.bitlinear_test_force_timeout(False)


def _case(M, N, K, seed):
    w = synth.normal_f32(seed, 1, (N, K), 0.02)
    x = synth.normal_bf16(seed, 2, (M, K))
    bias = synth.normal_bf16(seed, 3, (N,), 0.01)
    return x, w, bias


@pytest.mark.parametrize("M,N,K,engine", [(1, 4096, 4096, 1), (16, 1000, 3200, 1), (300, 1000, 3200, 2),
                                          (64, 8640, 8640, 2)])
def test_forced_timeout_is_reported_and_the_next_call_is_correct(M, N, K, engine):
    x, w, bias = _case(M, N, K, 70 + M)
    opk, osw, _ = oracle.pack_weights(w.numpy())
    packed, s_w, _ = bl.bitlinear_pack_weights(w.cuda())
    xd, bd = x.cuda(), bias.cuda()
    assert bl.bitlinear_test_force_timeout(True) is False
    out = bl.bitlinear_forward_debug(xd, packed, s_w, bd, engine=engine)
    assert bl.bitlinear_check_status(out["ws"]) == ERR_TIMEOUT
    assert bl.bitlinear_test_force_timeout(False) is True
    # the same workspace, the same context: a normal forward again
    ws = out["ws"]
    good = bl.bitlinear_forward_debug(xd, packed, s_w, bd, engine=engine, ws=ws)
    assert bl.bitlinear_check_status(ws) == 0
    ref = oracle.forward(synth.bf16_bits(x), opk, osw, synth.bf16_bits(bias))
    assert_equal(good["acc"].cpu().numpy(), ref["acc"], "acc after a forced timeout")
    y = good["y"].cpu().view(torch.int16).numpy().view(np.uint16)
    assert_equal(y, ref["y"], "y after a forced timeout")


def test_forced_timeout_on_a_grouped_call():
    x, w, _ = _case(8, 3 * 512, 1024, 77)
    parts = [w[i * 512:(i + 1) * 512].contiguous() for i in range(3)]
    gp = [bl.bitlinear_pack_weights(p.cuda()) for p in parts]
    packed = torch.cat([g[0] for g in gp])
    scales = torch.cat([g[1] for g in gp])
    ws = bl.workspace(8, 3 * 512, 1024, "cuda")
    bl.bitlinear_test_force_timeout(True)
    bl.bitlinear_forward_grouped(x.cuda(), packed, [512] * 3, scales, ws=ws)
    assert bl.bitlinear_check_status(ws) == ERR_TIMEOUT
    bl.bitlinear_test_force_timeout(False)
    y = bl.bitlinear_forward_grouped(x.cuda(), packed, [512] * 3, scales, ws=ws)
    assert bl.bitlinear_check_status(ws) == 0
    orc = [oracle.pack_weights(p.numpy()) for p in parts]
    ref = oracle.forward_grouped(synth.bf16_bits(x), np.concatenate([o[0] for o in orc]), [512] * 3,
                                 [o[1] for o in orc])
    assert_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref["y"], "grouped y after a forced timeout")
