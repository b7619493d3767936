"""The C++ oracle against the numpy oracle, bit for bit, plus its errors.

Both restate the Falcon-Edge blog's BitLinear listings (section
"Falcon-Edge, a series of universal models") independently; each is pinned
on its own by ``test_oracle_pins.py``.  Here they must agree on every
intermediate (q, s_x, rowsum, acc, y32, y; packed bytes, s_w, mean; the
bf16 export) on seeded inputs with the workloads' shapes and distributions,
ragged edges and the degenerate cases.
"""

import numpy as np
import pytest

import oracle as numpy_oracle
import synth
from oracle import cpp as cpp_oracle
from synth import workloads as wl

KEYS = ("q", "s_x", "rowsum", "acc", "y32", "y")


def same_forward(a, b):
    for k in KEYS:
        assert a[k].dtype == b[k].dtype and np.array_equal(a[k], b[k]), k


def both_pack(w):
    pa, sa, ma = numpy_oracle.pack_weights(w)
    pb, sb, mb = cpp_oracle.pack_weights(w)
    assert np.array_equal(pa, pb) and sa == sb and ma == mb
    return pa, sa


@pytest.mark.parametrize("mode", ["forward", "forward_bf16"])
def test_workload1_single_layer(mode):
    case = wl.workload1()[0]
    packed, s_w = both_pack(case.w().numpy())
    xb = synth.bf16_bits(case.x())
    same_forward(getattr(numpy_oracle, mode)(xb, packed, s_w), getattr(cpp_oracle, mode)(xb, packed, s_w))


@pytest.mark.parametrize("mode", ["forward", "forward_bf16"])
def test_decode_shape_with_outliers_and_bias(mode):
    # the decode sweep's first shape and distribution: K = N = 4096, 1% of
    # the channels x20, a bias; M = 4
    case = [c for c in wl.workload2() if c.M == 4 and c.N == 4096][0]
    packed, s_w = both_pack(case.w().numpy())
    xb, bias = synth.bf16_bits(case.x()), synth.bf16_bits(case.bias())
    same_forward(getattr(numpy_oracle, mode)(xb, packed, s_w, bias),
                 getattr(cpp_oracle, mode)(xb, packed, s_w, bias))


@pytest.mark.parametrize("seed", range(8))
def test_ragged_shapes_and_degenerate_rows(seed):
    rng = np.random.default_rng(5000 + seed)
    M, N, K = int(rng.integers(0, 20)), int(rng.integers(1, 300)), 16 * int(rng.integers(1, 40))
    x = synth.student_t4_bf16(5000 + seed, 1, (M, K)) if seed % 2 else synth.normal_bf16(5000 + seed, 1, (M, K))
    if M > 1:
        x[1] = 0                                   # all-zero row: the clamp decides s_x
    if M > 3:
        x[3] = x[3] * 1e-30                        # tiny row, below the clamp
    w = synth.normal_f32(5000 + seed, 2, (N, K), float(rng.choice([0.02, 1e-20, 3.0]))).numpy()
    packed, s_w = both_pack(w)
    xb = synth.bf16_bits(x)
    bias = synth.bf16_bits(synth.normal_bf16(5000 + seed, 3, (N,), 0.5)) if seed % 3 else None
    for mode in ("forward", "forward_bf16"):
        same_forward(getattr(numpy_oracle, mode)(xb, packed, s_w, bias),
                     getattr(cpp_oracle, mode)(xb, packed, s_w, bias))


def test_grouped_three_layers_with_bias():
    x = synth.normal_bf16(6001, 1, (5, 320))
    rows = [64, 48, 100]
    ws = [synth.normal_f32(6001, 10 + g, (r, 320), 0.02 * (g + 1)).numpy() for g, r in enumerate(rows)]
    packs = [both_pack(w) for w in ws]
    packed = np.concatenate([p for p, _ in packs])
    s_ws = [s for _, s in packs]
    bias = synth.bf16_bits(synth.normal_bf16(6001, 2, (sum(rows),), 0.1))
    xb = synth.bf16_bits(x)
    same_forward(numpy_oracle.forward_grouped(xb, packed, rows, s_ws, bias),
                 cpp_oracle.forward_grouped(xb, packed, rows, s_ws, bias))


@pytest.mark.parametrize("kind", ["gauss", "mixed", "denormal", "wide", "zeros"])
def test_absmean_and_scale(kind):
    rng = np.random.default_rng(7000)
    for trial in range(20):
        n = int(rng.integers(1, 5000))
        if kind == "gauss":
            w = rng.standard_normal(n) * 0.02
        elif kind == "mixed":
            w = rng.standard_normal(n) * np.exp2(rng.integers(-60, 60, n))
        elif kind == "denormal":
            w = rng.standard_normal(n) * 2.0 ** -140
        elif kind == "wide":
            w = rng.choice([3.0e38, 1e-38, 2.0 ** -149, 1.0, -7.5, 1e-3], n)
        else:
            w = np.zeros(n)
        w = w.astype(np.float32)
        m = numpy_oracle.absmean(w)
        assert cpp_oracle.absmean(w) == m
        assert cpp_oracle.weight_scale(m) == numpy_oracle.weight_scale(m)
        s = numpy_oracle.weight_scale(m)
        assert np.array_equal(cpp_oracle.ternarise(w, s), numpy_oracle.ternarise(w, s))


def test_dequant_export():
    w = synth.normal_f32(8001, 1, (96, 512), 0.02).numpy()
    packed, s_w = both_pack(w)
    assert np.array_equal(cpp_oracle.dequant(packed, s_w), numpy_oracle.dequant(packed, s_w))
    rng = np.random.default_rng(8001)
    for s in rng.uniform(1e-3, 1e5, 100).astype(np.float32):
        assert np.array_equal(cpp_oracle.dequant(packed[:2], s), numpy_oracle.dequant(packed[:2], s))


def test_bf16_storage_conversions():
    rng = np.random.default_rng(9001)
    v = (rng.standard_normal(100000) * np.exp2(rng.integers(-130, 120, 100000))).astype(np.float32)
    assert np.array_equal(cpp_oracle.f32_to_bf16_rne(v), numpy_oracle.f32_to_bf16_rne(v))
    bits = rng.integers(0, 0x7F80, 100000).astype(np.uint16) | (rng.integers(0, 2, 100000) << 15).astype(np.uint16)
    assert np.array_equal(cpp_oracle.bf16_to_f32(bits).view(np.uint32), numpy_oracle.bf16_to_f32(bits).view(np.uint32))


def test_errors():
    with pytest.raises(ValueError):
        cpp_oracle.unpack(np.array([[0, 0, 0x0C, 0]], np.uint8))          # code 3
    with pytest.raises(ValueError):
        cpp_oracle.pack(np.zeros((1, 20), np.int8))                        # K % 16
    with pytest.raises(ValueError):
        cpp_oracle.pack(np.full((1, 16), 2, np.int8))                      # not ternary
    with pytest.raises(ValueError):
        cpp_oracle.absmean(np.array([1.0, np.inf], np.float32))            # non-finite
    with pytest.raises(ValueError):
        cpp_oracle.absmean(np.zeros(0, np.float32))                        # empty
    with pytest.raises(ValueError):
        cpp_oracle.forward_grouped(np.zeros((1, 16), np.uint16), np.full((3, 4), 0x55, np.uint8),
                                   [1, 1], [np.float32(1), np.float32(1)])   # rows != N
    with pytest.raises(ValueError):
        bad = np.full((2, 4), 0x55, np.uint8)
        bad[1, 3] = 0xFF
        cpp_oracle.forward(np.zeros((1, 16), np.uint16), bad, np.float32(1))
