"""Pins of the CPU oracle to things other than itself.

Each test ties one oracle step to the pages' formulas by a route that does
not reuse the oracle's own code: a hand-worked example, exact rational
arithmetic, brute force over small domains, integer matrix products, closed
forms and invariants.  Sources: the Falcon-Edge blog (section "Falcon-Edge,
a series of universal models": activation_norm_quant, _weight_quant,
BitLinear) and the 2-bit storage remark in the Hacker News comments of
"BitNet: inference framework for 1-bit LLMs" (GeekNews).

Every pin runs twice: against the numpy oracle and against the C++ oracle
(``oracle.cpp``), two independent restatements of the same pages.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as numpy_oracle
import synth
from oracle import cpp as cpp_oracle
from tests.exact import f32_exact, nearest_bf16_bits, nearest_f32

RNG = np.random.default_rng(20260101)

ORACLES = {"numpy": numpy_oracle, "cpp": cpp_oracle}
oracle = numpy_oracle          # the oracle under test; set per test below


@pytest.fixture(params=sorted(ORACLES), autouse=True)
def which_oracle(request):
    global oracle
    saved, oracle = oracle, ORACLES[request.param]
    yield request.param
    oracle = saved


def bits_of_bf16(values):
    return synth.bf16_bits(torch.tensor(values, dtype=torch.bfloat16))


# --------------------------------------------------------------------------
# Hand-worked example (tests/golden/hand_worked_k4.json)
# --------------------------------------------------------------------------

def check_hand_worked(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "hand_worked_k4.json")))
    xb = bits_of_bf16([g["x"]])
    q, s_x, r = oracle.act_quant(xb)
    assert q.tolist() == [g["q"]]
    assert s_x[0] == np.float32(g["s_x"])
    assert int(r[0]) == g["rowsum"]
    w = np.array(g["w"], dtype=np.float32)
    mean = oracle.absmean(w)
    s_w = oracle.weight_scale(mean)
    assert mean == np.float32(g["mean"])
    assert s_w == np.float32(g["s_w"])
    u = oracle.ternarise(w, s_w)
    assert u.tolist() == g["u"]
    # K padded to 16 (the packing granule) with zero activations
    packed = oracle.pack(np.pad(u, ((0, 0), (0, 12))))
    out = oracle.forward(bits_of_bf16([g["x"] + [0.0] * 12]), packed, np.float32(g["s_w"]))
    assert out["acc"].tolist() == [g["acc"]]
    for n in range(2):
        want = nearest_f32(Fraction(g["y_exact_num"][n], g["y_exact_den"]))
        assert out["y32"][0, n] == want
        assert float(oracle.bf16_to_f32(out["y"][0, n])) == g["y_bf16"][n]


def test_hand_worked_example(golden_dir):
    check_hand_worked(golden_dir)


def test_pack_layout_fixture(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pack_layout.json")))
    u = np.array([g["u"]], dtype=np.int8)
    assert oracle.pack(u).ravel().tolist() == g["bytes"]
    assert oracle.unpack(np.array([g["bytes"]], dtype=np.uint8)).tolist() == [g["u"]]


# --------------------------------------------------------------------------
# Step 1: activation quantisation
# --------------------------------------------------------------------------

def test_act_quant_ties_round_half_even():
    # a = 127 so s_x = 1 and x*s_x = x exactly
    xb = bits_of_bf16([[127.0, 2.5, 3.5, -0.5, 0.5, -2.5, 1.5, -63.5]])
    q, s_x, _ = oracle.act_quant(xb)
    assert s_x[0] == np.float32(1.0)
    assert q.tolist() == [[127, 2, 4, 0, 0, -2, 2, -64]]


def test_act_quant_zero_row_and_clamp():
    xb = bits_of_bf16([[0.0] * 16, [1e-7] + [0.0] * 15])
    q, s_x, r = oracle.act_quant(xb)
    assert s_x[0] == np.float32(127.0) / np.float32(1e-5)
    assert s_x[1] == s_x[0]            # |x| below the clamp uses the clamp
    assert np.all(q[0] == 0) and r[0] == 0
    # 1e-7 (as bf16) * 12700000 ~ 1.27 -> 1
    assert q[1, 0] == 1


def test_act_quant_exact_against_rationals():
    """q and s_x from exact rationals with independent rounding."""
    x = synth.normal_bf16(7, 1, (6, 64))
    xb = synth.bf16_bits(x)
    q, s_x, r = oracle.act_quant(xb)
    xf = x.float().numpy()
    for m in range(6):
        a = max(abs(float(v)) for v in xf[m])
        s = nearest_f32(Fraction(127) / max(Fraction(a), f32_exact(1e-5)))
        assert s_x[m] == s
        for k in range(64):
            t = nearest_f32(Fraction(float(xf[m, k])) * Fraction(float(s)))
            tf = Fraction(float(t))
            fl = math.floor(tf)
            rnd = fl + 1 if (tf - fl > Fraction(1, 2) or (tf - fl == Fraction(1, 2) and fl % 2)) else fl
            assert int(q[m, k]) == max(-128, min(127, rnd))
        assert int(r[m]) == int(sum(int(v) for v in q[m]))


def test_act_quant_invariants():
    x = synth.normal_bf16(7, 2, (5, 128), 3.0)
    xb = synth.bf16_bits(x)
    q, s_x, _ = oracle.act_quant(xb)
    # absmax element maps to +-127
    xf = x.float().numpy()
    am = np.abs(xf).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(5), am]) == 127)
    assert np.all(np.abs(q.astype(int)) <= 127)
    # sign symmetry
    qn, sn, _ = oracle.act_quant(synth.bf16_bits(-x))
    assert np.array_equal(qn, -q) and np.array_equal(sn, s_x)
    # power-of-two scaling leaves q unchanged and scales s_x by 2**-k
    for k in (-3, 5):
        qk, sk, _ = oracle.act_quant(synth.bf16_bits(x * (2.0 ** k)))
        assert np.array_equal(qk, q)
        assert np.array_equal(sk, (s_x * np.float32(2.0 ** -k)).astype(np.float32))


def test_act_quant_approximates_x():
    """The int8 activations approximate x (the blog's x ~ x_quant / x_scale):
    q = round(fl(x * s_x)) with |fl(x * s_x)| <= 127 + ulp, so
    |x * s_x - q| <= 1/2 + 127 * 2^-24 for every element, in exact
    arithmetic (float64 holds x * s_x exactly: 8 + 24 significant bits)."""
    for seed, dist in ((11, "normal"), (12, "student"), (13, "outliers")):
        if dist == "normal":
            x = synth.normal_bf16(seed, 1, (9, 512), 3.0)
        elif dist == "student":
            x = synth.student_t4_bf16(seed, 1, (9, 512))
        else:
            x = synth.normal_with_outliers_bf16(seed, 1, (9, 512))
        q, s_x, _ = oracle.act_quant(synth.bf16_bits(x))
        xs = x.double().numpy() * s_x.astype(np.float64)[:, None]
        err = np.abs(xs - q.astype(np.float64))
        assert np.all(err <= 0.5 + 127 * 2.0 ** -24), err.max()
        # and the bound is not vacuous: errors fill most of [0, 1/2]
        assert err.max() > 0.45


# --------------------------------------------------------------------------
# Step 2: absmean scale, ternarisation, packing
# --------------------------------------------------------------------------

def exact_mean(w):
    return sum((abs(f32_exact(v)) for v in w.ravel()), Fraction(0)) / w.size


@pytest.mark.parametrize("case", ["gauss", "mixed", "denormal", "wide"])
def test_absmean_exact_vs_fraction(case):
    if case == "gauss":
        w = synth.normal_f32(3, 1, (37, 29), 0.02).numpy()
    elif case == "mixed":
        w = (RNG.standard_normal(500) * np.exp2(RNG.integers(-40, 40, 500))).astype(np.float32)
    elif case == "denormal":
        w = (RNG.standard_normal(300) * 2.0 ** -140).astype(np.float32)
        w[::7] = np.float32(3e-45)
    else:
        w = np.array([3.0e38, 1e-38, 2.0 ** -149, 1.0, -7.5, 1e-3] * 9, dtype=np.float32)
    assert oracle.absmean(w) == nearest_f32(exact_mean(w))


def test_absmean_ties_to_even():
    one = np.float32(1.0)
    up1 = np.nextafter(one, np.float32(2))
    up2 = np.nextafter(up1, np.float32(2))
    # mean of (1, 1+2^-23) is 1 + 2^-24: a tie, the even neighbour is 1
    assert oracle.absmean(np.array([one, up1], np.float32)) == one
    # mean of (1+2^-23, 1+2^-22) is 1 + 1.5*2^-23: a tie, the even neighbour is 1+2^-22
    assert oracle.absmean(np.array([up1, up2], np.float32)) == up2


def test_absmean_order_independent():
    w = synth.normal_f32(3, 2, (64, 64), 0.02).numpy()
    m = oracle.absmean(w)
    perm = RNG.permutation(w.size)
    assert oracle.absmean(w.ravel()[perm]) == m


def test_weight_scale_and_clamp():
    assert oracle.weight_scale(np.float32(0.2)) == np.float32(5.0)
    z = np.zeros((4, 16), np.float32)
    m = oracle.absmean(z)
    assert m == 0
    assert oracle.weight_scale(m) == np.float32(1.0) / np.float32(1e-5)
    assert np.all(oracle.ternarise(z, oracle.weight_scale(m)) == 0)


def test_ternarise_ties_and_clamp():
    w = np.array([0.5, -0.5, 1.5, -1.5, 0.49, 0.51, 7.0, -7.0, 0.0, -0.0], np.float32)
    assert oracle.ternarise(w, np.float32(1.0)).tolist() == [0, 0, 1, -1, 0, 1, 1, -1, 0, 0]


def test_ternarise_power_of_two_invariance():
    w = synth.normal_f32(3, 3, (32, 64), 0.02).numpy()
    _, s_w, _ = oracle.pack_weights(w)
    u = oracle.ternarise(w, s_w)
    for k in (-4, 6):
        wk = (w * np.float32(2.0 ** k)).astype(np.float32)
        _, s_k, _ = oracle.pack_weights(wk)
        assert s_k == np.float32(s_w * np.float32(2.0 ** -k))
        assert np.array_equal(oracle.ternarise(wk, s_k), u)


def test_zero_fraction_gaussian():
    """|w| <= mean|w|/2 has probability erf(1/(2 sqrt(pi))) ~ 0.3101 for
    Gaussian w (mean|w| = sigma sqrt(2/pi))."""
    w = synth.normal_f32(3, 4, (1000, 1024), 0.02).numpy()
    packed, s_w, _ = oracle.pack_weights(w)
    frac0 = float((oracle.ternarise(w, s_w) == 0).mean())
    assert abs(frac0 - math.erf(1.0 / (2.0 * math.sqrt(math.pi)))) < 2e-3


def test_pack_bruteforce_all_bytes():
    codes = np.array(list(itertools.product([-1, 0, 1], repeat=4)), dtype=np.int8)  # 81 x (i=0..3 at j=0)
    u = np.zeros((81, 16), np.int8)
    u[:, 0::4] = codes                      # k = 4i + 0 -> byte 0, bit pair i
    p = oracle.pack(u)
    want = ((codes.astype(int) + 1) * np.array([1, 4, 16, 64])).sum(axis=1)
    assert np.array_equal(p[:, 0], want)
    assert np.all(p[:, 1:] == 0x55)
    assert np.array_equal(oracle.unpack(p), u)


def test_pack_roundtrip_all_words():
    """All 3**16 ternary 16-tuples round-trip through pack/unpack (so the
    packing is injective) and no packed bit pair ever holds the code 3."""
    total = 3 ** 16
    step = 1 << 21
    digits = 3 ** np.arange(16, dtype=np.int64)
    for s in range(0, total, step):
        idx = np.arange(s, min(total, s + step), dtype=np.int64)
        u = ((idx[:, None] // digits[None, :]) % 3 - 1).astype(np.int8)
        p = oracle.pack(u)
        assert np.array_equal(oracle.unpack(p), u)
        words = np.ascontiguousarray(p).view("<u4").ravel()
        for i in range(4):
            pairs = ((words >> np.uint32(2 * i)) & np.uint32(0x03030303)).view(np.uint8)
            assert not np.any(pairs == 3)


def test_unpack_rejects_code3():
    bad = np.zeros((1, 4), np.uint8)
    bad[0, 2] = 0x0C                          # bit pair 1 of byte 2 holds 3
    with pytest.raises(ValueError):
        oracle.unpack(bad)


# --------------------------------------------------------------------------
# Step 3: contraction
# --------------------------------------------------------------------------

def test_contract_bruteforce_all_ternary_2x3():
    q = RNG.integers(-128, 128, (5, 3)).astype(np.int8)
    for t in itertools.product([-1, 0, 1], repeat=6):
        u = np.array(t, dtype=np.int8).reshape(2, 3)
        acc = oracle.contract(q, u)
        for m in range(5):
            for n in range(2):
                assert acc[m, n] == sum(int(q[m, k]) * int(u[n, k]) for k in range(3))


def test_contract_vs_int64_matmul():
    q = RNG.integers(-128, 128, (33, 1000)).astype(np.int8)
    u = RNG.integers(-1, 2, (2100, 1000)).astype(np.int8)
    want = np.matmul(q.astype(np.int64), u.astype(np.int64).T)
    assert np.array_equal(oracle.contract(q, u).astype(np.int64), want)


def test_contract_extreme_magnitude():
    K = 28672
    q = np.full((2, K), 127, np.int8)
    q[1] = -128
    u = np.ones((3, K), np.int8)
    u[1] = -1
    acc = oracle.contract(q, u)
    assert acc[0, 0] == 127 * K and acc[1, 1] == 128 * K and acc[0, 2] == 127 * K


def test_permutation_and_row_independence():
    x = synth.normal_bf16(9, 1, (4, 256))
    w = synth.normal_f32(9, 2, (48, 256), 0.02).numpy()
    packed, s_w, _ = oracle.pack_weights(w)
    out = oracle.forward(synth.bf16_bits(x), packed, s_w)
    perm = RNG.permutation(256)
    q, _, _ = oracle.act_quant(synth.bf16_bits(x))
    u = oracle.unpack(packed)
    assert np.array_equal(oracle.contract(q[:, perm], u[:, perm]), out["acc"])
    x2 = x.clone()
    x2[2] = x2[2] * 3 + 1
    out2 = oracle.forward(synth.bf16_bits(x2), packed, s_w)
    for key in ("q", "acc", "y32", "y"):
        assert np.array_equal(np.delete(out2[key], 2, axis=0), np.delete(out[key], 2, axis=0))


def test_dequant_invariant_float64_linear():
    """The integer path equals F.linear on the dequantised operands
    x ~ q/s_x and w ~ u/s_w, times s_x*s_w, up to float64 rounding."""
    x = synth.normal_bf16(9, 3, (8, 512))
    w = synth.normal_f32(9, 4, (64, 512), 0.02).numpy()
    packed, s_w, _ = oracle.pack_weights(w)
    out = oracle.forward(synth.bf16_bits(x), packed, s_w)
    q, s_x, _ = oracle.act_quant(synth.bf16_bits(x))
    u = oracle.unpack(packed)
    xd = torch.from_numpy(q.astype(np.float64) / s_x.astype(np.float64)[:, None])
    wd = torch.from_numpy(u.astype(np.float64) / np.float64(s_w))
    y = torch.nn.functional.linear(xd, wd).numpy()
    scale = s_x.astype(np.float64)[:, None] * np.float64(s_w)
    assert np.allclose(y * scale, out["acc"].astype(np.float64), rtol=0, atol=1e-6 * 127 * 512)
    # and the float32 epilogue is within float32 rounding of the float64 value
    rel = np.abs(out["y32"].astype(np.float64) - y) / np.maximum(np.abs(y), 1e-30)
    assert np.all(rel[np.abs(y) > 1e-6] < 3e-7)


# --------------------------------------------------------------------------
# Step 4: epilogue
# --------------------------------------------------------------------------

def test_epilogue_exact_rational():
    acc = RNG.integers(-400000, 400000, (7, 9)).astype(np.int32)
    s_x = (RNG.random(7) * 100 + 1).astype(np.float32)
    s_w = np.float32(37.125)
    bias = synth.bf16_bits(synth.normal_bf16(9, 5, (9,), 0.01))
    y32, y = oracle.epilogue(acc, s_x, s_w, bias)
    bf = oracle.bf16_to_f32(bias)
    for m in range(7):
        d = nearest_f32(f32_exact(s_x[m]) * f32_exact(s_w))
        for n in range(9):
            q = nearest_f32(Fraction(int(acc[m, n])) / Fraction(float(d)))
            want = nearest_f32(Fraction(float(q)) + Fraction(float(bf[n])))
            assert y32[m, n] == want
            assert int(y[m, n]) == nearest_bf16_bits(want)


def test_epilogue_large_accumulators_round_once():
    # beyond 2^24 (K > 132104) float(acc) is the float32 nearest to acc (ties
    # to even), then the division rounds once more
    acc = np.array([[(1 << 24) + 1, (1 << 24) + 3, -((1 << 25) + 2), (1 << 25) + 6, 127 * (1 << 19)]],
                   dtype=np.int32)
    s_x = np.array([3.5], np.float32)
    s_w = np.float32(21.25)
    y32, y = oracle.epilogue(acc, s_x, s_w)
    d = nearest_f32(f32_exact(s_x[0]) * f32_exact(s_w))
    for n in range(acc.shape[1]):
        a = nearest_f32(Fraction(int(acc[0, n])))
        want = nearest_f32(Fraction(float(a)) / Fraction(float(d)))
        assert y32[0, n] == want, n
        assert int(y[0, n]) == nearest_bf16_bits(want)
    # the ties: 2^24 + 1 -> 2^24 (even), 2^24 + 3 -> 2^24 + 4
    assert nearest_f32(Fraction((1 << 24) + 1)) == np.float32(1 << 24)
    assert nearest_f32(Fraction((1 << 24) + 3)) == np.float32((1 << 24) + 4)


def test_bf16_conversions():
    v = np.array([1.0, -2.5, 3.0e-39, 65504.0, 1.00390625, 1.005859375], np.float32)
    b = oracle.f32_to_bf16_rne(v)
    assert [int(t) for t in b] == [nearest_bf16_bits(t) for t in v]
    assert np.array_equal(oracle.bf16_to_f32(b), torch.tensor(v).to(torch.bfloat16).float().numpy())


# --------------------------------------------------------------------------
# The pins catch planted mistakes (mutations planted in the oracle, on CPU)
# --------------------------------------------------------------------------

def test_pins_catch_planted_mistakes(golden_dir, monkeypatch, tmp_path, which_oracle):
    if which_oracle == "cpp":
        # the same three mistakes, compiled into copies of the C++ oracle
        for mistake in (1, 2, 3):
            with cpp_oracle.planted(mistake, str(tmp_path)):
                with pytest.raises(AssertionError):
                    check_hand_worked(golden_dir)
                    test_pack_layout_fixture(golden_dir)
        check_hand_worked(golden_dir)
        return
    orig_act, orig_epi, orig_pack = oracle.act_quant, oracle.epilogue, oracle.pack

    def act_floor(xb):                      # floor instead of round
        q, s, r = orig_act(xb)
        x = oracle.bf16_to_f32(xb)
        qf = np.clip(np.floor(x * s[:, None]), -128, 127).astype(np.int8)
        return qf, s, qf.astype(np.int64).sum(1).astype(np.int32)

    def epi_mul(acc, s_x, s_w, bias_bits=None):  # multiply instead of divide
        y32 = acc.astype(np.float32) * (np.asarray(s_x, np.float32) * np.float32(s_w))[:, None]
        return y32, oracle.f32_to_bf16_rne(y32)

    def pack_swapped(u):                     # i and j swapped in the layout
        N, K = u.shape
        t = u.reshape(N, K // 16, 4, 4).transpose(0, 1, 3, 2).reshape(N, K)
        return orig_pack(t)

    for name, bad in (("act_quant", act_floor), ("epilogue", epi_mul), ("pack", pack_swapped)):
        monkeypatch.setattr(oracle, name, bad)
        with pytest.raises(AssertionError):
            check_hand_worked(golden_dir)
            if name == "pack":
                test_pack_layout_fixture(golden_dir)
        monkeypatch.undo()
    check_hand_worked(golden_dir)


# --------------------------------------------------------------------------
# bf16 export (state-dict loop: param_value / param_scale, stored as bf16)
# --------------------------------------------------------------------------

def test_dequant_hand_worked():
    # s_w = 50: 1/50 = 0.02; the float32 nearest to 0.02 is 0x3CA3D70A; its
    # upper half 0x3CA3 with 0xD70A > 0x8000 below rounds up to bf16 0x3CA4.
    u = np.array([[1, 0, -1, 1, -1, 0, 0, 1, 1, 1, -1, -1, 0, 1, 0, -1]], dtype=np.int8)
    got = oracle.dequant(oracle.pack(u), np.float32(50.0))
    want = np.array([{1: 0x3CA4, 0: 0x0000, -1: 0xBCA4}[int(v)] for v in u[0]], dtype=np.uint16)
    assert np.array_equal(got[0], want)


def test_dequant_against_exact_rationals():
    # for arbitrary float32 scales the exported +-1 weight is the bf16 nearest
    # to the float32 nearest to 1/s_w, computed here from fractions
    for s in RNG.uniform(0.5, 4000.0, size=200).astype(np.float32).tolist() + [1e5, 1.0, 3.0, 1e-3]:
        s32 = np.float32(s)
        inv = nearest_f32(Fraction(1) / f32_exact(s32))
        pos = nearest_bf16_bits(inv)
        u = np.array([[1, -1, 0, 0] * 4], dtype=np.int8)
        got = oracle.dequant(oracle.pack(u), s32)[0]
        assert int(got[0]) == pos and int(got[1]) == (pos ^ 0x8000) and int(got[2]) == 0, s


def test_dequant_invariants_on_packed_weights():
    w = synth.normal_f32(7, 1, (48, 320), 0.02)
    packed, s_w, _ = oracle.pack_weights(w.numpy())
    u = oracle.unpack(packed)
    deq = oracle.dequant(packed, s_w)
    assert deq.shape == u.shape and deq.dtype == np.uint16
    assert np.all(deq[u == 0] == 0)                          # +0, never -0
    mags = np.unique(deq[u != 0] & 0x7FFF)
    assert mags.size == 1                                    # one magnitude, 1/s_w
    assert np.all((deq[u > 0] >> 15) == 0) and np.all((deq[u < 0] >> 15) == 1)
    v = float(oracle.bf16_to_f32(mags.astype(np.uint16))[0])
    assert abs(v * float(s_w) - 1.0) < 2.0 ** -8              # bf16 keeps 8 significant bits


# --------------------------------------------------------------------------
# Grouped forward (layers sharing one input)
# --------------------------------------------------------------------------

def test_grouped_forward_scaled_copy_closed_form():
    # Group 2 holds 2*W of group 1: same ternary codes, mean doubled, so
    # s_w2 = s_w1 / 2 exactly, and y2 = acc / (s_x * s_w1 / 2) = 2 * y1.
    # Doubling commutes with float32 and bf16 rounding, so every nonzero
    # bf16 output of group 2 has the exponent of group 1's plus one.
    w1 = synth.normal_f32(41, 3, (24, 128), 0.02).numpy()
    p1, s1, _ = oracle.pack_weights(w1)
    p2, s2, _ = oracle.pack_weights(2.0 * w1)
    assert np.array_equal(p1, p2) and s2 == np.float32(s1 / 2)
    x = synth.normal_bf16(41, 4, (5, 128))
    xb = synth.bf16_bits(x)
    out = oracle.forward_grouped(xb, np.concatenate([p1, p2]), [24, 24], [s1, s2])
    y1, y2 = out["y"][:, :24].astype(np.int32), out["y"][:, 24:].astype(np.int32)
    nz = (y1 & 0x7FFF) != 0
    assert np.array_equal(y2[nz], y1[nz] + (1 << 7))          # exponent field + 1
    assert np.array_equal(y2[~nz], y1[~nz])
    # and group 1 alone is the single-layer forward
    assert np.array_equal(out["y"][:, :24], oracle.forward(xb, p1, s1)["y"])


def test_grouped_forward_acc_is_one_integer_matmul():
    # the contraction of all groups at once is the integer product with the
    # stacked ternary matrix, whatever the group split
    u = RNG.integers(-1, 2, size=(40, 64)).astype(np.int8)
    x = synth.normal_bf16(42, 1, (3, 64))
    xb = synth.bf16_bits(x)
    out = oracle.forward_grouped(xb, oracle.pack(u), [7, 30, 3], [np.float32(1.5), np.float32(2.0), np.float32(0.25)])
    q = oracle.act_quant(xb)[0].astype(np.int64)
    assert np.array_equal(out["acc"], (q @ u.astype(np.int64).T).astype(np.int32))


# --------------------------------------------------------------------------
# bf16-faithful mode: the listings executed by PyTorch on bf16 tensors
# --------------------------------------------------------------------------

def _listing_on_bf16_module(x, u, s_w, bias):
    """activation_norm_quant and BitLinear.forward of the Falcon-Edge blog,
    run by PyTorch (CPU) on a module whose dtype is bfloat16; the weight
    scale is the module's bf16 copy of s_w."""
    scale = 127.0 / x.abs().max(dim=-1, keepdim=True).values.clamp_(min=1e-5)
    xq = (x * scale).round().clamp_(-128, 127)
    w_quant = torch.tensor(u, dtype=torch.bfloat16)
    y = torch.nn.functional.linear(xq.to(torch.bfloat16), w_quant)
    weight_scale = torch.tensor(float(s_w), dtype=torch.float32).to(torch.bfloat16)
    y = y / (weight_scale * scale)          # post_quant_process(y, weight_scale, input_scale)
    if bias is not None:
        y += bias.view(1, -1).expand_as(y)
    return xq, scale, y


@pytest.mark.parametrize("seed", range(6))
def test_bf16_mode_matches_pytorch_bf16_execution(seed):
    rng = np.random.default_rng(900 + seed)
    M, K, N = int(rng.integers(1, 9)), int(rng.choice([64, 128, 256])), int(rng.integers(1, 65))
    x = synth.normal_bf16(300 + seed, 1, (M, K), float(rng.choice([0.01, 1.0, 30.0])))
    x[0, : K // 2] = 0 if M > 1 else x[0, : K // 2]
    if M > 2:
        x[2] = 0                                             # an all-zero row: the clamp decides
    w = synth.normal_f32(300 + seed, 2, (N, K), 0.02).numpy()
    packed, s_w, _ = oracle.pack_weights(w)
    u = oracle.unpack(packed)
    bias = synth.normal_bf16(300 + seed, 3, (N,), 0.5) if seed % 2 else None
    xq_t, scale_t, y_t = _listing_on_bf16_module(x, u.astype(np.float32), s_w, bias)
    out = oracle.forward_bf16(synth.bf16_bits(x), packed, s_w, None if bias is None else synth.bf16_bits(bias))
    assert np.array_equal(out["q"], xq_t.float().numpy().astype(np.int8))
    assert np.array_equal(out["s_x"], scale_t.float().numpy()[:, 0])
    assert np.array_equal(out["y"], synth.bf16_bits(y_t))


def test_bf16_mode_matches_pytorch_on_extreme_rows():
    # the listings on a bf16 module, run by PyTorch, for rows at the edges of
    # bf16: a 1e30 row, a row near the bf16 maximum (1 / absmax is subnormal),
    # a subnormal row and a tiny row (both below the clamp), one huge
    # outlier, -0.0, .5 ties
    K, N = 128, 48
    base = synth.normal_bf16(4300, 1, (7, K)).float()
    x = base.clone()
    x[0] = base[0] * 1e30
    x[1] = base[1] * 2.0 ** -130
    x[2] = base[2] * 1e-7
    x[3, 5] = 1e30
    x[4] = -0.0
    x[5] = torch.tensor([127.0, 2.5, 3.5, -0.5, 0.5, -2.5, 1.5, -63.5] * (K // 8))
    x[6] = base[6] / base[6].abs().max() * 2e38
    x = x.to(torch.bfloat16)
    assert 0 < 1.0 / float(x[6].float().abs().max()) < 1.1754944e-38      # a subnormal reciprocal
    w = synth.normal_f32(4300, 2, (N, K), 0.02).numpy()
    packed, s_w, _ = oracle.pack_weights(w)
    u = oracle.unpack(packed)
    bias = synth.normal_bf16(4300, 3, (N,), 0.5)
    xq_t, scale_t, y_t = _listing_on_bf16_module(x, u.astype(np.float32), s_w, bias)
    out = oracle.forward_bf16(synth.bf16_bits(x), packed, s_w, synth.bf16_bits(bias))
    assert np.array_equal(out["q"], xq_t.float().numpy().astype(np.int8))
    assert np.array_equal(out["s_x"], scale_t.float().numpy()[:, 0])
    assert np.array_equal(out["y"], synth.bf16_bits(y_t))


def test_bf16_mode_differs_from_float32_mode_only_by_rounding():
    # the two modes read the same pages; they differ only in where rounding
    # happens, so the outputs agree to within a few bf16 ulps
    x = synth.normal_bf16(77, 5, (6, 512))
    w = synth.normal_f32(77, 6, (96, 512), 0.02).numpy()
    packed, s_w, _ = oracle.pack_weights(w)
    xb = synth.bf16_bits(x)
    a = oracle.bf16_to_f32(oracle.forward(xb, packed, s_w)["y"]).astype(np.float64)
    b = oracle.bf16_to_f32(oracle.forward_bf16(xb, packed, s_w)["y"]).astype(np.float64)
    # per row, relative to the row's norm (single outputs near zero can move
    # by more: bf16 rounding of the integer sum and a different s_x)
    rel = np.linalg.norm(a - b, axis=1) / np.linalg.norm(a, axis=1)
    assert np.all(rel < 0.02), rel
