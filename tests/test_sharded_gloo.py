"""Tensor-parallel splits of the BitLinear forward (K-split and N-split),
run as two gloo ranks on the CPU through ``oracle.sharded``: every output
must equal the unsplit oracle forward bit for bit.  The split design keeps
the whole-tensor reductions of the Falcon-Edge blog's BitLinear (section
"Falcon-Edge, a series of universal models") exact: MAX of the token
absmax, SUM of integer exponent bins for mean |w|, SUM of int32 partial
accumulators."""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from oracle import sharded

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

M, K, N = 7, 512, 160
K_SPLIT = [192, 320]          # uneven, multiples of 64
N_SPLIT = [100, 60]


def _inputs():
    x = synth.normal_with_outliers_bf16(6100, 1, (M, K))
    x[2] = 0                                                 # a zero row: the clamp decides s_x
    w = synth.normal_f32(6100, 2, (N, K), 0.02).numpy()
    bias = synth.bf16_bits(synth.normal_bf16(6100, 3, (N,), 0.1))
    return synth.bf16_bits(x), w, bias


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        xb, w, bias = _inputs()
        k0 = sum(K_SPLIT[:rank])
        k1 = k0 + K_SPLIT[rank]
        ks = sharded.forward_ksplit(np.ascontiguousarray(xb[:, k0:k1]), np.ascontiguousarray(w[:, k0:k1]), bias)
        n0 = sum(N_SPLIT[:rank])
        n1 = n0 + N_SPLIT[rank]
        ns = sharded.forward_nsplit(xb, np.ascontiguousarray(w[n0:n1]), bias[n0:n1])
        nsb = sharded.forward_nsplit(xb, np.ascontiguousarray(w[n0:n1]), bias[n0:n1], bf16_mode=True)
        q.put((rank, ks, ns, nsb))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return out


def test_ksplit_equals_unsplit(results):
    xb, w, bias = _inputs()
    packed, s_w, mean = oracle.pack_weights(w)
    want = oracle.forward(xb, packed, s_w, bias)
    for rank, ks, _, _ in results:
        assert ks["mean"] == mean and ks["s_w"] == s_w
        assert np.array_equal(ks["s_x"].view(np.uint32), want["s_x"].view(np.uint32))
        k0 = sum(K_SPLIT[:rank])
        assert np.array_equal(ks["q"], want["q"][:, k0:k0 + K_SPLIT[rank]])
        assert np.array_equal(ks["packed"], packed[:, k0 // 4:(k0 + K_SPLIT[rank]) // 4])
        assert np.array_equal(ks["acc"], want["acc"])
        assert np.array_equal(ks["y32"].view(np.uint32), want["y32"].view(np.uint32))
        assert np.array_equal(ks["y"], want["y"])


def test_nsplit_equals_unsplit(results):
    xb, w, bias = _inputs()
    packed, s_w, mean = oracle.pack_weights(w)
    want = oracle.forward(xb, packed, s_w, bias)
    want_b = oracle.forward_bf16(xb, packed, s_w, bias)
    for rank, _, ns, nsb in results:
        assert ns["mean"] == mean and ns["s_w"] == s_w
        n0 = sum(N_SPLIT[:rank])
        assert np.array_equal(ns["packed"], packed[n0:n0 + N_SPLIT[rank]])
        assert np.array_equal(ns["y32"].view(np.uint32), want["y32"].view(np.uint32))
        assert np.array_equal(ns["y"], want["y"])
        assert np.array_equal(nsb["y"], want_b["y"])


def test_bins_reproduce_the_exact_mean():
    # the exponent bins of any split add up to the whole tensor's, and give
    # the oracle's exactly rounded mean (pinned against exact rationals)
    rng = np.random.default_rng(6101)
    for kind in range(4):
        n = int(rng.integers(1, 4000))
        w = (rng.standard_normal(n) * np.exp2(rng.integers(-140, 100, n) if kind == 1 else 0)
             * (0.02 if kind == 0 else 1.0)).astype(np.float32)
        if kind == 2:
            w = (w * np.float32(2.0 ** -140)).astype(np.float32)
        if kind == 3:
            w[:] = 0
        cut = int(rng.integers(0, n + 1))
        bins = sharded.abs_bins(w[:cut]) + sharded.abs_bins(w[cut:])
        assert np.array_equal(bins, sharded.abs_bins(w))
        assert sharded.mean_from_bins(bins, n) == oracle.absmean(w)


def test_local_scales_would_be_wrong():
    # without the exchanges each shard would use its own absmax and mean, and
    # both scales (and so q) would differ from the unsplit forward's
    xb, w, _ = _inputs()
    q, s_x, _ = oracle.act_quant(xb)
    k1 = K_SPLIT[0]
    q0, s0, _ = oracle.act_quant(np.ascontiguousarray(xb[:, :k1]))
    assert not np.array_equal(s0, s_x) and not np.array_equal(q0, q[:, :k1])
    assert oracle.absmean(w[:, :k1]) != oracle.absmean(w)
    assert oracle.absmean(w[:N_SPLIT[0]]) != oracle.absmean(w)
