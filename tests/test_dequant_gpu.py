"""bf16 export of packed weights (bitlinear_dequant_weights) against the
oracle, bit for bit: the state-dict loop param_value / param_scale of the
Falcon-Edge blog (section on universal models), stored as bfloat16."""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from tests.gpu_util import sample_rows

pytestmark = pytest.mark.gpu

SHAPES = [(512, 256), (1, 64), (777, 2112), (3200, 8640), (8640, 3200)]


def _packed(N, K, seed, std=0.02):
    """The weights packed by the GPU, and by the oracle on its own."""
    w = synth.normal_f32(seed, N + K, (N, K), std)
    packed, s_w, _ = bl.bitlinear_pack_weights(w.cuda())
    opk, osw, _ = oracle.pack_weights(w.numpy())
    return packed, s_w, opk, osw


@pytest.mark.parametrize("N,K", SHAPES, ids=[f"N{n}K{k}" for n, k in SHAPES])
def test_dequant_matches_oracle(N, K):
    packed, s_w, opk, osw = _packed(N, K, 31)
    got = bl.bitlinear_dequant_weights(packed, s_w)
    torch.cuda.synchronize()
    want = oracle.dequant(opk, osw)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)


def test_dequant_100b_rows_sampled():
    # gate/up of the 100B-class FFN: 28672 x 8192 (235 M weights), rows sampled
    N, K = 28672, 8192
    packed, s_w, opk, osw = _packed(N, K, 32, 0.01)
    got = bl.bitlinear_dequant_weights(packed, s_w)
    torch.cuda.synchronize()
    rows = sample_rows(N, 40, seed=5)
    want = oracle.dequant(opk[rows], osw)
    assert np.array_equal(got[rows].view(torch.int16).cpu().numpy().view(np.uint16), want)


def test_dequant_all_zero_weights():
    # all-zero W: mean clamps to 1e-5, s_w = 1e5, every code is u = 0 -> +0
    packed, s_w = bl.bitlinear_pack_weights(torch.zeros(64, 128, device="cuda"))[:2]
    got = bl.bitlinear_dequant_weights(packed, s_w)
    assert torch.count_nonzero(got.view(torch.int16)).item() == 0
