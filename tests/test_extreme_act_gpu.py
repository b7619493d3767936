"""Activation quantisation at the edges of bf16, on both engines and in both
modes, against the oracle bit for bit.

activation_norm_quant of the Falcon-Edge blog (section "Falcon-Edge, a
series of universal models") scales each token by 127 / max(|x|, 1e-5).
These rows reach the parts of that formula that ordinary activations do
not:
- a row scaled by 1e30, so s_x is about 1e-28, and a row near the bf16
  maximum, whose 1 / absmax is subnormal (the bf16-faithful scale);
- a row of bf16 subnormals, and a row of tiny normal values, both below the
  clamp, so s_x = 127 / 1e-5;
- a single huge outlier in an otherwise ordinary row, so every other value
  quantises to 0;
- a row of -0.0;
- a row of exact .5 ties (absmax 127, s_x = 1).
The weights are ordinary, so every output stays finite.
"""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth

pytestmark = pytest.mark.gpu

K, N = 256, 160


def extreme_rows() -> np.ndarray:
    """Seven extreme rows, float32 values that bf16 holds exactly or rounds."""
    base = synth.normal_bf16(4200, 1, (7, K)).float().numpy()
    x = base.copy()
    x[0] = base[0] * np.float32(1e30)
    x[1] = base[1] * np.float32(2.0 ** -130)            # bf16 subnormals
    x[2] = base[2] * np.float32(1e-7)                    # normal, below the clamp
    x[3, 7] = np.float32(1e30)                           # one outlier
    x[4] = np.float32(-0.0)
    x[5] = np.resize(np.array([127.0, 2.5, 3.5, -0.5, 0.5, -2.5, 1.5, -63.5], np.float32), K)
    x[6] = base[6] / np.abs(base[6]).max() * np.float32(2e38)
    return x


def make_x(M: int) -> torch.Tensor:
    rows = extreme_rows()
    ordinary = synth.normal_bf16(4201, M, (M, K)).float().numpy()
    x = ordinary.copy()
    slots = range(M) if M <= 7 else range(0, M, 2)      # every second row past seven
    for j, i in enumerate(slots):
        x[i] = rows[j % 7]
    return torch.from_numpy(x).to(torch.bfloat16)


def oracle_out(x, packed, s_w, bias, faithful):
    xb = synth.bf16_bits(x)
    f = oracle.forward_bf16 if faithful else oracle.forward
    return f(xb, packed, np.float32(s_w), None if bias is None else synth.bf16_bits(bias))


CASES = [(7, 1), (16, 1), (7, 2), (40, 2)]      # (M, engine): 1 decode, 2 prefill


@pytest.mark.parametrize("faithful", [False, True], ids=["float32", "bf16_faithful"])
@pytest.mark.parametrize("M,engine", CASES, ids=[f"M{m}_engine{e}" for m, e in CASES])
def test_extreme_activations(M, engine, faithful):
    x = make_x(M)
    w = synth.normal_f32(4202, 1, (N, K), 0.02)
    bias = synth.normal_bf16(4202, 2, (N,), 0.1)
    packed, s_w, _ = bl.bitlinear_pack_weights(w.cuda())
    flags = bl.BF16_FAITHFUL if faithful else 0
    out = bl.bitlinear_forward_debug(x.cuda(), packed, s_w, bias.cuda(), engine=engine, flags=flags)
    torch.cuda.synchronize()
    assert bl.bitlinear_check_status(out["ws"]) == 0
    opk, osw, _ = oracle.pack_weights(w.numpy())               # the oracle's own packing
    want = oracle_out(x, opk, osw, bias, faithful)
    assert np.all(np.isfinite(want["y32"]))
    assert np.array_equal(out["xq"].cpu().numpy(), want["q"])
    assert np.array_equal(out["s_x"].cpu().numpy().view(np.uint32), want["s_x"].view(np.uint32))
    assert np.array_equal(out["acc"].cpu().numpy(), want["acc"])
    assert np.array_equal(out["y32"].cpu().numpy().view(np.uint32), want["y32"].view(np.uint32))
    assert np.array_equal(out["y"].cpu().view(torch.int16).numpy().view(np.uint16), want["y"])
