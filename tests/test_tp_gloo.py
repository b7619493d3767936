"""The exchange logic of bitlinear_fwd_b200.tp (tensor-parallel K-split) on
two gloo ranks on the CPU.  The local steps come from a host stand-in built
on the CPU oracle (the kernels need a GPU); the all-reduces, their order,
dtypes and operands are tp.py's own.  Every rank must end with the unsplit
oracle forward's bits."""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

M, K, N = 6, 512, 200
K_SPLIT = [320, 192]


def _inputs():
    import synth
    x = synth.normal_with_outliers_bf16(6400, 1, (M, K))
    x[3] = 0
    w = synth.normal_f32(6400, 2, (N, K), 0.02)
    bias = synth.normal_bf16(6400, 3, (N,), 0.1)
    return x, w, bias


class OracleOps:
    """Host stand-in for the library's local K-split steps, from the oracle."""

    def absmean_bins(self, w):
        from oracle import sharded
        return torch.from_numpy(np.concatenate([sharded.abs_bins(w.numpy()), np.zeros(64, np.int64)]))

    def pack_from_bins(self, w, bins, n_total):
        import oracle
        from oracle import sharded
        b = bins.numpy()
        assert not b[256:].any()
        mean = sharded.mean_from_bins(b[:256], n_total)
        s_w = oracle.weight_scale(mean)
        return torch.from_numpy(oracle.pack(oracle.ternarise(w.numpy(), s_w))), torch.tensor([s_w]), \
            torch.tensor([mean])

    def act_absmax(self, x):
        import synth
        xf = (synth.bf16_bits(x).astype(np.uint32) << 16).view(np.float32)
        return torch.from_numpy(np.abs(xf).max(axis=1).astype(np.float32))

    def forward_partial(self, x, absmax, packed, flags):
        import oracle
        import synth
        from oracle import sharded
        assert flags == 0
        q, _ = sharded.act_quant_given_absmax(synth.bf16_bits(x), absmax.numpy())
        return torch.from_numpy(oracle.contract(q, oracle.unpack(packed.numpy())).astype(np.int32))

    def epilogue(self, acc, absmax, w_scale, bias, flags):
        import oracle
        import synth
        s_x = (np.float32(127.0) / np.maximum(absmax.numpy(), np.float32(1e-5))).astype(np.float32)
        _, y = oracle.epilogue(acc.numpy(), s_x, np.float32(w_scale.item()),
                               None if bias is None else synth.bf16_bits(bias))
        return torch.from_numpy(y.view(np.int16)).view(torch.bfloat16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from bitlinear_fwd_b200 import tp
        x, w, bias = _inputs()
        k0 = sum(K_SPLIT[:rank])
        k1 = k0 + K_SPLIT[rank]
        ops = OracleOps()
        packed, s_w, mean = tp.pack_ksplit(w[:, k0:k1].contiguous(), ops=ops)
        y = tp.forward_ksplit(x[:, k0:k1].contiguous(), packed, s_w, bias, ops=ops)
        q.put((rank, packed.numpy(), float(s_w.item()), y.view(torch.int16).numpy().view(np.uint16)))
    finally:
        dist.destroy_process_group()


def test_tp_ksplit_on_two_gloo_ranks():
    sys.path.insert(0, ROOT)
    import oracle
    import synth
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
    x, w, bias = _inputs()
    opk, osw, _ = oracle.pack_weights(w.numpy())
    want = oracle.forward(synth.bf16_bits(x), opk, osw, synth.bf16_bits(bias))
    for rank, packed, s_w, y in out:
        k0 = sum(K_SPLIT[:rank])
        assert np.float32(s_w) == osw
        assert np.array_equal(packed, opk[:, k0 // 4:(k0 + K_SPLIT[rank]) // 4])
        assert np.array_equal(y, want["y"])
