"""The tensor-parallel K-split pieces on one GPU: x and W are cut into
K-shards, each shard goes through bitlinear_absmean_bins /
bitlinear_pack_weights_from_bins / bitlinear_act_absmax /
bitlinear_forward_partial, the exchanges are done with plain tensor ops (the
sum of the bins, the max of the absmax, the list of partial sums), and
bitlinear_epilogue_sum finishes.  Every output must equal the unsplit CPU
oracle bit for bit (BitLinear.forward and _weight_quant of the Falcon-Edge
blog, section "Falcon-Edge, a series of universal models", reduce over the
whole K and the whole tensor; the exchanges keep those reductions exact)."""

import numpy as np
import pytest
import torch

import bitlinear_fwd_b200 as bl
import oracle
import synth
from tests.gpu_util import assert_equal, assert_same_f32

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("M,N,K,cuts,faithful", [
    (4, 1000, 4096, [1536], False),          # decode engine, two uneven shards
    (16, 520, 3200, [64, 1600], False),      # three shards, one of them thin
    (300, 1000, 3200, [1280], False),        # prefill engine
    (300, 700, 8640, [4096, 6400], True),    # prefill, bf16-faithful scale and epilogue
    (1, 4096, 4096, [2048], True),
])
def test_ksplit_equals_unsplit(M, N, K, cuts, faithful):
    seed = 6200 + M + len(cuts)
    x = synth.normal_with_outliers_bf16(seed, 1, (M, K))
    x[0] = 0                                            # a zero row: the clamp decides s_x
    w = synth.normal_f32(seed, 2, (N, K), 0.02)
    bias = synth.normal_bf16(seed, 3, (N,), 0.1)
    bounds = [0] + cuts + [K]
    shards = [(bounds[i], bounds[i + 1]) for i in range(len(bounds) - 1)]
    flags = bl.BF16_FAITHFUL if faithful else 0

    # packing: bins of every shard added, then each shard packed with the whole s_w
    wd = w.cuda()
    bins = sum(bl.bitlinear_absmean_bins(wd[:, a:b].contiguous()) for a, b in shards)
    packs = [bl.bitlinear_pack_weights_from_bins(wd[:, a:b].contiguous(), bins, N * K) for a, b in shards]
    opk, osw, omean = oracle.pack_weights(w.numpy())
    for (a, b), (p, s, m) in zip(shards, packs):
        assert_same_f32(s.cpu().numpy(), [osw], "s_w of a shard")
        assert_same_f32(m.cpu().numpy(), [omean], "mean |w| of a shard")
        assert_equal(p.cpu().numpy(), opk[:, a // 4:b // 4], "packed shard")

    # forward: max of the absmax, partial sums, epilogue on their sum
    xd = x.cuda()
    absmax = torch.stack([bl.bitlinear_act_absmax(xd[:, a:b].contiguous()) for a, b in shards]).amax(0)
    xf = synth.bf16_bits(x).astype(np.uint32) << 16
    want_a = np.abs(xf.view(np.float32)).max(axis=1)
    assert_same_f32(absmax.cpu().numpy(), want_a, "absmax")
    parts = [bl.bitlinear_forward_partial(xd[:, a:b].contiguous(), absmax, p, flags=flags)
             for (a, b), (p, _, _) in zip(shards, packs)]
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_epilogue_sum(parts, absmax, packs[0][1], bias.cuda(), flags=flags, acc_out=acc)
    y1 = bl.bitlinear_epilogue_sum(sum(parts), absmax, packs[0][1], bias.cuda(), flags=flags)
    torch.cuda.synchronize()
    f = oracle.forward_bf16 if faithful else oracle.forward
    ref = f(synth.bf16_bits(x), opk, osw, synth.bf16_bits(bias))
    assert_equal(acc.cpu().numpy(), ref["acc"], "summed partial accumulators")
    for (a, b), part in zip(shards, parts):
        q = ref["q"][:, a:b].astype(np.int64)
        u = oracle.unpack(opk[:, a // 4:b // 4]).astype(np.int64)
        assert_equal(part.cpu().numpy(), (q @ u.T).astype(np.int32), "one shard's partial sums")
    assert_equal(_u16(y), ref["y"], "y from the partial sums")
    assert_equal(_u16(y1), ref["y"], "y from the pre-summed accumulators")


def test_epilogue_sum_takes_up_to_eight_parts():
    M, N = 5, 300
    rng = np.random.default_rng(6300)
    parts = [rng.integers(-2000, 2000, (M, N), dtype=np.int32) for _ in range(8)]
    absmax = np.float32([0.5, 3.0, 0.0, 1e-6, 7.25])
    s_w = np.float32(31.0)
    y = bl.bitlinear_epilogue_sum([torch.from_numpy(p).cuda() for p in parts], torch.from_numpy(absmax).cuda(),
                                  torch.tensor([s_w], device="cuda"))
    acc = np.sum(parts, axis=0, dtype=np.int64).astype(np.int32)
    s_x = (np.float32(127.0) / np.maximum(absmax, np.float32(1e-5))).astype(np.float32)
    _, want = oracle.epilogue(acc, s_x, s_w)
    assert_equal(_u16(y), want, "y of eight partial sums")
