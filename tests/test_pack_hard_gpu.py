"""GPU weight packing on weight tensors that stress the exact mean.

_weight_quant of the Falcon-Edge blog (section "Falcon-Edge, a series of
universal models") takes mean |w| over the whole tensor.  The library
computes it exactly: per-exponent significand sums, then one long division
and one rounding to float32.  These tensors stress each part against the
oracle:
- mixed exponents spanning 2^-140 .. 2^120;
- subnormal weights, and a subnormal or zero mean;
- values near the float32 maximum, which make s_w subnormal;
- exact ties of the mean, which must round to even.
The mean, s_w and the packed codes must match the oracle bit for bit.
"""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle

pytestmark = pytest.mark.gpu

N, K = 37, 192          # a ragged row count; K a multiple of 64


KINDS = ["mixed", "subnormal", "wide", "sparse_min_subnormal", "huge", "tie_even_down", "tie_even_up"]


def hard_weights(kind: str) -> np.ndarray:
    rng = np.random.default_rng(4100 + KINDS.index(kind))
    n = N * K
    if kind == "mixed":
        w = rng.standard_normal(n) * np.exp2(rng.integers(-140, 120, n))
    elif kind == "subnormal":
        w = rng.standard_normal(n) * 2.0 ** -140
    elif kind == "wide":
        w = rng.choice([3.0e38, 1e-38, 2.0 ** -149, 1.0, -7.5, 1e-3], n)
    elif kind == "sparse_min_subnormal":
        w = np.where(rng.random(n) < 0.01, 2.0 ** -149, 0.0)           # mean below 2^-149
    elif kind == "huge":
        w = rng.choice([3.4e38, -3.4e38, 1.0], n)                      # s_w is subnormal
    elif kind == "tie_even_down":
        one = np.float32(1.0)
        w = np.resize([one, np.nextafter(one, np.float32(2))], n)      # mean 1 + 2^-24: ties to 1
    elif kind == "tie_even_up":
        up1 = np.nextafter(np.float32(1.0), np.float32(2))
        w = np.resize([up1, np.nextafter(up1, np.float32(2))], n)      # mean 1 + 1.5*2^-23: ties up
    else:
        raise ValueError(kind)
    return np.asarray(w, dtype=np.float32).reshape(N, K)


@pytest.mark.parametrize("kind", KINDS)
def test_pack_hard_weights_match_oracle(kind):
    w = hard_weights(kind)
    assert np.all(np.isfinite(w))
    packed, s_w, mean = bl.bitlinear_pack_weights(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    om = np.float32(oracle.absmean(w))
    osw = np.float32(oracle.weight_scale(om))
    opk = oracle.pack(oracle.ternarise(w, osw))
    assert mean.cpu().numpy().view(np.uint32)[0] == om.view(np.uint32), (mean.item(), om)
    assert s_w.cpu().numpy().view(np.uint32)[0] == osw.view(np.uint32), (s_w.item(), osw)
    assert np.array_equal(packed.cpu().numpy(), opk)
    if kind == "tie_even_down":
        assert om == np.float32(1.0)
