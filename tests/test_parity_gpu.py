"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs, for all five workloads and the edge cases.

Integer stages (int8 activations, s_x, packed weights, s_w, the exact mean,
int32 accumulators) must match bit for bit.  The stated bar for floats is
relative error <= 1e-6 on the float32 pre-cast output and <= 1 bf16 ulp on
y; both engines in fact reproduce the oracle's IEEE operations exactly, and
that is asserted too.  Large workloads compare every activation and scale
and a seeded sample of token rows (plus the first and last) for acc and y.
"""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from synth import workloads as wl
from tests.gpu_util import run_and_compare, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


# ---------------- workload 1: single small layer -------------------------

@pytest.mark.parametrize("engine", [0, 1, 2])
def test_w1_single_layer(engine):
    c = wl.workload1()[0]
    run_and_compare(c.x(), c.w(), c.bias(), engine=engine)


# ---------------- workload 2: decode sweep --------------------------------

_W2 = wl.workload2()


@pytest.mark.parametrize("case", _W2, ids=[c.name for c in _W2])
def test_w2_decode(case):
    run_and_compare(case.x(), case.w(), case.bias(), engine=0)


def test_w2_decode_matches_prefill_engine():
    c = _W2[2]   # M = 16, 4096 x 4096
    a = run_and_compare(c.x(), c.w(), c.bias(), engine=1)
    b = run_and_compare(c.x(), c.w(), c.bias(), engine=2)
    assert torch.equal(a["acc"], b["acc"])


# ---------------- workload 3: prefill ---------------------------------------

_W3 = wl.workload3()


@pytest.mark.parametrize("case", _W3, ids=[c.name for c in _W3])
def test_w3_prefill(case):
    rows = None if case.M <= 512 else sample_rows(case.M)
    run_and_compare(case.x(), case.w(), case.bias(), engine=0, rows=rows)


# ---------------- workload 4: 3B-class projection stack ---------------------

@pytest.mark.parametrize("M", [1, 2048])
@pytest.mark.parametrize("layer", [0, 25])
def test_w4_stack3b(M, layer):
    for case in wl.workload4(M, layers=[layer]):
        if M > 1 and case.tags["proj"] not in ("q", "gate", "down"):
            continue
        rows = None if M <= 16 else sample_rows(M, 24)
        run_and_compare(case.x(), case.w(), case.bias(), engine=0, rows=rows)


# ---------------- workload 5: 100B-class FFN layer --------------------------

@pytest.mark.parametrize("M", wl.MS100B)
def test_w5_ffn100b(M):
    for case in wl.workload5(M, layers=[0]):
        if case.tags["proj"] == "up":
            continue
        rows = None if M <= 64 else sample_rows(M, 12)
        run_and_compare(case.x(), case.w(), case.bias(), engine=0, rows=rows)


# ---------------- edge cases ------------------------------------------------

EDGE = [
    (17, 256, 64), (129, 300, 192), (1, 1, 64), (16, 517, 320), (33, 1000, 640),
    (2, 130, 128), (9, 129, 448), (300, 520, 1088), (16, 8, 64), (255, 777, 2112),
    # K above the decode engine's 8192-k activation chunk, with a ragged last chunk
    (5, 97, 17472), (12, 40, 8640),
]


@pytest.mark.parametrize("M,N,K", EDGE, ids=[f"M{m}N{n}K{k}" for m, n, k in EDGE])
@pytest.mark.parametrize("with_bias", [False, True])
def test_edge_shapes(M, N, K, with_bias):
    x = synth.normal_bf16(77, M * 7 + K, (M, K), 2.0)
    w = synth.normal_f32(77, N * 3 + K, (N, K), 0.05)
    b = synth.normal_bf16(77, N, (N,), 0.1) if with_bias else None
    for engine in ([0, 1, 2] if M <= 16 else [0, 2]):
        run_and_compare(x, w, b, engine=engine)


def test_zero_activation_rows_and_zero_weights():
    x = synth.normal_bf16(78, 1, (20, 256))
    x[3] = 0
    x[17] = 0
    w = synth.normal_f32(78, 2, (96, 256), 0.02)
    run_and_compare(x, w, None, engine=0)
    run_and_compare(x[:8].clone(), w, None, engine=1)
    wz = torch.zeros(64, 256)
    b = synth.normal_bf16(78, 3, (64,), 0.5)
    out = run_and_compare(x, wz, b, engine=0)
    # all-zero weights: s_w = 1/1e-5, u = 0, so y is the bias in every row
    assert torch.equal(out["y"].cpu()[5].view(torch.int16), b.view(torch.int16))


def test_tie_values_round_half_even():
    # rows whose absmax is 127 make s_x = 1, so x * s_x hits exact .5 ties
    vals = [127.0, 2.5, 3.5, -0.5, 0.5, -2.5, 1.5, -63.5] * 8
    x = torch.tensor([vals, [-v for v in vals]], dtype=torch.bfloat16)
    w = synth.normal_f32(79, 1, (128, 64), 0.02)
    out = run_and_compare(x, w, None, engine=0)
    assert out["xq"].cpu()[0, :8].tolist() == [127, 2, 4, 0, 0, -2, 2, -64]


def test_deterministic_repeat():
    c = _W2[5]
    x, w, b = c.x().cuda(), c.w().cuda(), c.bias().cuda()
    outs = []
    for _ in range(3):
        packed, s_w, _ = bl.bitlinear_pack_weights(w)
        outs.append((packed.cpu(), s_w.cpu(), bl.bitlinear_forward(x, packed, s_w, b).cpu()))
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1])
        assert torch.equal(o[2].view(torch.int16), outs[0][2].view(torch.int16))


def test_deterministic_repeat_prefill():
    # the persistent tcgen05 GEMM has a static tile schedule and exact int32
    # sums: three runs give the same bytes (races would show up here)
    c = [c for c in _W3 if c.M == 2048 and c.K == 3200][0]
    x, w = c.x().cuda(), c.w().cuda()
    packed, s_w, _ = bl.bitlinear_pack_weights(w)
    ys = [bl.bitlinear_forward(x, packed, s_w).cpu() for _ in range(3)]
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))


def test_quant_act_standalone():
    x = synth.student_t4_bf16(80, 1, (300, 3200))
    xq, s_x, rs = bl.bitlinear_quant_act(x.cuda())
    q, s, r = oracle.act_quant(synth.bf16_bits(x))
    assert np.array_equal(xq.cpu().numpy(), q)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(rs.cpu().numpy(), r)


def test_forward_host_matches_device():
    c = _W2[4]
    w, b = c.w().cuda(), c.bias().cuda()
    packed, s_w, _ = bl.bitlinear_pack_weights(w)
    x = c.x()
    y_dev = bl.bitlinear_forward(x.cuda(), packed, s_w, b).cpu()
    y_host = bl.bitlinear_forward_host(x.pin_memory(), packed, s_w, b)
    assert torch.equal(y_dev.view(torch.int16), y_host.view(torch.int16))
    # the stream-ordered variant: several calls in flight, each with its own
    # workspace and output, one synchronisation at the end
    xs = [synth.normal_bf16(55, i, tuple(x.shape)).pin_memory() for i in range(3)]
    outs = [bl.bitlinear_forward_host_async(xi, packed, s_w, b, flags=bl.WEIGHTS_RESIDENT) for xi in xs]
    torch.cuda.current_stream().synchronize()
    for xi, yi in zip(xs, outs):
        want = bl.bitlinear_forward(xi.cuda(), packed, s_w, b).cpu()
        assert torch.equal(yi.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("M", [4, 16, 40])
def test_forward_q8_matches_forward(M):
    """Quantise once, contract against several weight matrices (q/k/v)."""
    x = synth.normal_bf16(81, M, (M, 3200))
    xq, s_x, rs = bl.bitlinear_quant_act(x.cuda())
    for proj in range(3):
        w = synth.normal_f32(81, 100 + proj, (3200, 3200), 0.02).cuda()
        packed, s_w, _ = bl.bitlinear_pack_weights(w)
        y_q8 = bl.bitlinear_forward_q8(xq, s_x, rs, packed, s_w).cpu()
        y = bl.bitlinear_forward(x.cuda(), packed, s_w).cpu()
        assert torch.equal(y_q8.view(torch.int16), y.view(torch.int16))


def test_device_argument_errors():
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((64, 32), dtype=torch.uint8, device="cuda")
    s_w = torch.ones(1, device="cuda")
    y = torch.empty((4, 64), dtype=torch.bfloat16, device="cuda")
    ws = bl.workspace(4, 64, 128, "cuda")
    lib = bl.lib()
    st = torch.cuda.current_stream().cuda_stream
    # misaligned activations
    assert lib.bitlinear_forward(x.data_ptr() + 2, 4, 128, packed.data_ptr(), 64, s_w.data_ptr(), None,
                                 y.data_ptr(), ws.data_ptr(), ws.numel(), st) == -3
    # workspace too small
    assert lib.bitlinear_forward(x.data_ptr(), 4, 128, packed.data_ptr(), 64, s_w.data_ptr(), None,
                                 y.data_ptr(), ws.data_ptr(), 64, st) == -4
    # a valid call succeeds and leaves the status word clear
    assert lib.bitlinear_forward(x.data_ptr(), 4, 128, packed.data_ptr(), 64, s_w.data_ptr(), None,
                                 y.data_ptr(), ws.data_ptr(), ws.numel(), st) == 0
    assert bl.bitlinear_check_status(ws) == 0


def test_forward_ex_resident_flag_matches():
    """Weights packed earlier on the stream, then a chain of forwards with the
    resident-weights flag (weights streamed before the dependency wait)."""
    c = _W2[1]
    w, b = c.w().cuda(), c.bias().cuda()
    packed, s_w, _ = bl.bitlinear_pack_weights(w)
    torch.cuda.synchronize()
    xs = [synth.normal_bf16(82, i, (c.M, c.K)).cuda() for i in range(4)]
    want = [bl.bitlinear_forward(x, packed, s_w, b).cpu() for x in xs]
    got = [bl.bitlinear_forward(x, packed, s_w, b, flags=bl.WEIGHTS_RESIDENT) for x in xs]
    for g_, w_ in zip(got, want):
        assert torch.equal(g_.cpu().view(torch.int16), w_.view(torch.int16))
