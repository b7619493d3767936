"""Host-only checks of the C ABI: the library loads, exports every function
that include/bitlinear.h declares, answers size queries, and rejects bad
arguments before touching the GPU.  On a machine without a GPU, valid
arguments are also shown to pass every host check and stop at the device
check; that test is skipped wherever a GPU is visible, because its fake
pointers would then reach a kernel launch."""

import ctypes
import os
import re

import pytest

import bitlinear_fwd_b200 as bl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(bl.LIB_PATH):
        from bitlinear_fwd_b200 import build
        build.build()
    return bl.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(bl.exported_symbols()) == names


def test_version_and_status_strings(lib):
    assert lib.bitlinear_version() >> 16 == 1
    for st in range(-7, 1):
        assert bl.status_string(st).startswith("BITLINEAR")
    assert "unknown" in bl.status_string(-99)


def test_size_queries(lib):
    assert bl.packed_bytes(512, 256) == 512 * 64
    assert bl.packed_bytes(512, 100) == 0
    assert bl.pack_workspace_bytes(1, 64) >= 256 + 256 * 8
    ws = bl.workspace_bytes(8, 512, 256)
    assert ws >= 8 * 256 + 8 * 4 * 2
    assert bl.workspace_bytes(8, 512, 100) == 0
    assert bl.host_workspace_bytes(8, 512, 256) >= ws + 2 * 8 * 256 + 2 * 8 * 512


def _fwd(lib, x=16, M=8, K=256, w=16, N=512, s=16, b=None, y=16, ws=16, wsb=1 << 20):
    return lib.bitlinear_forward(x, M, K, w, N, s, b, y, ws, wsb, None)


def test_argument_errors_without_gpu(lib):
    assert _fwd(lib, x=None) == -1
    assert _fwd(lib, w=None) == -1
    assert _fwd(lib, y=None) == -1
    assert _fwd(lib, K=100) == -2
    assert _fwd(lib, K=0) == -2
    assert _fwd(lib, N=0) == -2
    assert _fwd(lib, M=-1) == -2
    assert _fwd(lib, x=18) == -3
    assert _fwd(lib, b=20) == -3
    assert _fwd(lib, ws=None) == -4
    assert _fwd(lib, wsb=16) == -4
    assert lib.bitlinear_pack_weights(16, 512, 100, 16, 16, None, 16, 4096, None) == -2
    assert lib.bitlinear_pack_weights(None, 512, 256, 16, 16, None, 16, 4096, None) == -1
    assert lib.bitlinear_pack_weights(16, 512, 256, 16, 16, None, 16, 8, None) == -4
    assert lib.bitlinear_quant_act(16, 4, 96, 16, 16, None, None) == -2
    assert lib.bitlinear_quant_act(16, 0, 64, 16, 16, None, None) == 0   # M == 0: nothing to do
    assert lib.bitlinear_forward_debug(16, 32, 256, 16, 512, 16, None, 16, None, None, None, None, 1, 16,
                                       1 << 20, None) == -2               # decode engine needs M <= 16
    assert lib.bitlinear_check_status(None, 0, None) == -1
    # bf16 export: shape, null and alignment checks come before any device work
    assert lib.bitlinear_dequant_weights(16, 512, 100, 16, 16, None) == -2
    assert lib.bitlinear_dequant_weights(16, 0, 256, 16, 16, None) == -2
    assert lib.bitlinear_dequant_weights(None, 512, 256, 16, 16, None) == -1
    assert lib.bitlinear_dequant_weights(16, 512, 256, None, 16, None) == -1
    assert lib.bitlinear_dequant_weights(16, 512, 256, 16, 18, None) == -3
    # grouped forward: group list checks come first
    rows = (ctypes.c_int64 * 3)(100, 200, 212)
    bad = (ctypes.c_int64 * 2)(100, 0)
    g = lib.bitlinear_forward_grouped
    assert g(16, 8, 256, 16, None, 3, 16, None, 16, 0, 16, 1 << 20, None) == -1    # no group list
    assert g(16, 8, 256, 16, rows, 0, 16, None, 16, 0, 16, 1 << 20, None) == -2    # no groups
    assert g(16, 8, 256, 16, rows, 9, 16, None, 16, 0, 16, 1 << 20, None) == -2    # too many groups
    assert g(16, 8, 256, 16, bad, 2, 16, None, 16, 0, 16, 1 << 20, None) == -2     # empty group
    assert g(16, 8, 256, 16, rows, 3, None, None, 16, 0, 16, 1 << 20, None) == -1  # no scales
    assert g(16, 8, 256, 16, rows, 3, 16, None, 16, 4, 16, 1 << 20, None) == -2    # unknown flag
    assert g(16, 8, 256, 16, rows, 3, 16, None, 16, 0, 16, 16, None) == -4         # workspace too small
    # debug with flags: only the bf16-faithful flag is accepted
    assert lib.bitlinear_forward_debug_ex(16, 8, 256, 16, 512, 16, None, 16, None, None, None, None, 0, 1, 16,
                                          1 << 20, None) == -2
    assert lib.bitlinear_forward_debug_ex(None, 8, 256, 16, 512, 16, None, 16, None, None, None, None, 0, 2, 16,
                                          1 << 20, None) == -1
    # stream-ordered host forward: flag check first, then the host argument checks
    assert lib.bitlinear_forward_host_async(16, 8, 256, 16, 512, 16, None, 16, 4, 16, 1 << 20, None) == -2
    assert lib.bitlinear_forward_host_async(None, 8, 256, 16, 512, 16, None, 16, 0, 16, 1 << 20, None) == -1


def test_more_argument_errors_without_gpu(lib):
    """Every entry point rejects bad shapes, NULL and misaligned pointers and
    short workspaces on the host, before any CUDA call."""
    # sizes beyond the documented limits
    assert _fwd(lib, N=(1 << 23) + 1) == -2
    assert _fwd(lib, K=(1 << 19) + 64) == -2
    assert _fwd(lib, M=(1 << 23) + 1) == -2
    assert lib.bitlinear_pack_weights(16, 1 << 23, 1 << 19, 16, 16, None, 16, 4096, None) == -2   # N*K >= 2^39
    assert lib.bitlinear_pack_weights(16, 1 << 20, 1 << 19, 16, 16, None, 16, 4096, None) == -2   # N*K = 2^39
    # misaligned scale, workspace and output
    assert _fwd(lib, s=20) == -3
    assert _fwd(lib, ws=24) == -3
    assert _fwd(lib, y=18) == -3
    # M == 0 is a valid empty call that touches nothing
    assert _fwd(lib, M=0) == 0
    # flags
    assert lib.bitlinear_forward_ex(16, 8, 256, 16, 512, 16, None, 16, 4, 16, 1 << 20, None) == -2
    # pre-quantised activations
    q8 = lib.bitlinear_forward_q8
    assert q8(None, 16, 16, 8, 256, 16, 512, 16, None, 16, 16, 256, None) == -1
    assert q8(16, 16, None, 8, 256, 16, 512, 16, None, 16, 16, 256, None) == -1
    assert q8(16, 18, 16, 8, 256, 16, 512, 16, None, 16, 16, 256, None) == -3
    assert q8(16, 16, 16, 8, 100, 16, 512, 16, None, 16, 16, 256, None) == -2
    assert q8(16, 16, 16, 8, 256, 16, 512, 16, None, 16, 16, 128, None) == -4
    assert q8(16, 16, 16, 0, 256, 16, 512, 16, None, 16, 16, 256, None) == 0
    # host buffers: no alignment rule for host x and y, but a larger workspace
    dev_ws = bl.workspace_bytes(8, 512, 256)
    host = lib.bitlinear_forward_host
    assert host(16, 8, 256, 16, 512, 16, None, 16, 16, dev_ws, None) == -4
    assert host(16, 8, 256, 16, 512, 16, None, None, 16, 1 << 20, None) == -1
    assert host(16, 8, 256, 18, 512, 16, None, 16, 16, 1 << 20, None) == -3     # packed weights are on the device
    # the no-allocation forward: its fixed scratch bounds M*K
    na = lib.bitlinear_forward_noalloc
    assert na(16, 64, 1 << 19, 16, 512, 16, None, 16, None) == -4
    assert na(16, 8, 100, 16, 512, 16, None, 16, None) == -2
    # quantisation alone
    assert lib.bitlinear_quant_act(None, 4, 256, 16, 16, None, None) == -1
    assert lib.bitlinear_quant_act(16, 4, 256, 16, 18, None, None) == -3


def _no_cuda_device():
    import torch
    return not torch.cuda.is_available() and torch.cuda.device_count() == 0


@pytest.mark.skipif(not _no_cuda_device(),
                    reason="the fake pointers of this test would reach a kernel launch on a GPU")
def test_valid_arguments_pass_every_host_check(lib):
    """Valid arguments get through every host check of each entry point and
    stop only at the device check (no GPU here: BITLINEAR_ERR_CUDA or
    BITLINEAR_ERR_DEVICE), so the checks reject nothing the header allows."""
    no_device = (-5, -7)
    rows = (ctypes.c_int64 * 3)(100, 200, 212)
    host_ws = bl.host_workspace_bytes(8, 512, 256)
    calls = {
        "forward": _fwd(lib),
        "forward_ex resident": lib.bitlinear_forward_ex(16, 8, 256, 16, 512, 16, None, 16, 1, 16, 1 << 20, None),
        "forward_ex both flags": lib.bitlinear_forward_ex(16, 8, 256, 16, 512, 16, 32, 16, 3, 16, 1 << 20, None),
        "forward M=16": _fwd(lib, M=16),
        "forward M=17": _fwd(lib, M=17),
        "grouped": lib.bitlinear_forward_grouped(16, 8, 256, 16, rows, 3, 16, None, 16, 2, 16, 1 << 20, None),
        "q8": lib.bitlinear_forward_q8(16, 16, 16, 8, 256, 16, 512, 16, None, 16, 16, 256, None),
        "debug engine 1": lib.bitlinear_forward_debug(16, 16, 256, 16, 512, 16, None, 16, None, None, None,
                                                      None, 1, 16, 1 << 20, None),
        "debug_ex engine 2": lib.bitlinear_forward_debug_ex(16, 8, 256, 16, 512, 16, None, 16, 16, 16, 16, 16,
                                                            2, 2, 16, 1 << 20, None),
        "host": lib.bitlinear_forward_host(18, 8, 256, 16, 512, 16, None, 18, 16, host_ws, None),
        "host_async": lib.bitlinear_forward_host_async(18, 8, 256, 16, 512, 16, None, 18, 3, 16, host_ws, None),
        "noalloc": lib.bitlinear_forward_noalloc(16, 8, 256, 16, 512, 16, None, 16, None),
        "noalloc status": lib.bitlinear_noalloc_check_status(None),
        "absmean bins": lib.bitlinear_absmean_bins(16, 512, 256, 16, None),
        "pack from bins": lib.bitlinear_pack_weights_from_bins(16, 512, 256, 16, 1024 * 256, 16, 16, 16, 16, 4096,
                                                               None),
        "act absmax": lib.bitlinear_act_absmax(16, 4, 256, 16, None),
        "forward partial": lib.bitlinear_forward_partial(16, 8, 256, 16, 16, 512, 16, 0, 16, 1 << 20, None),
        "forward partial M=40": lib.bitlinear_forward_partial(16, 40, 256, 16, 16, 512, 16, 2, 16, 1 << 20, None),
        "epilogue sum": lib.bitlinear_epilogue_sum((ctypes.c_void_p * 2)(16, 32), 2, 8, 512, 16, 16, 16, 16, None,
                                                   0, None),
        "i8 peak": lib.bitlinear_measure_i8_peak(10, ctypes.byref(ctypes.c_int(0)), 16, 256, None),
        "pack": lib.bitlinear_pack_weights(16, 512, 256, 16, 16, 16, 16, 4096, None),
        "quant_act": lib.bitlinear_quant_act(16, 4, 256, 16, 16, 16, None),
        "dequant": lib.bitlinear_dequant_weights(16, 512, 256, 16, 16, None),
    }
    wrong = {k: v for k, v in calls.items() if v not in no_device}
    assert not wrong, wrong


def test_ksplit_entry_points_reject_bad_arguments(lib):
    """The tensor-parallel K-split calls check shapes, pointers, alignment and
    workspace before anything is enqueued."""
    bins = lib.bitlinear_absmean_bins
    assert bins(16, 512, 100, 16, None) == -2
    assert bins(None, 512, 256, 16, None) == -1
    assert bins(16, 512, 256, 18, None) == -3
    pfb = lib.bitlinear_pack_weights_from_bins
    assert pfb(16, 512, 256, 16, 512 * 256 - 1, 16, 16, None, 16, 4096, None) == -2   # n_total below N*K
    assert pfb(16, 512, 256, 16, 1 << 39, 16, 16, None, 16, 4096, None) == -2
    assert pfb(16, 512, 256, None, 512 * 256, 16, 16, None, 16, 4096, None) == -1
    assert pfb(16, 512, 256, 16, 512 * 256, 16, 16, None, 16, 100, None) == -4
    am = lib.bitlinear_act_absmax
    assert am(16, 4, 100, 16, None) == -2
    assert am(16, 0, 256, None, None) == 0
    assert am(16, 4, 256, 20, None) == -3
    part = lib.bitlinear_forward_partial
    assert part(16, 8, 256, None, 16, 512, 16, 0, 16, 1 << 20, None) == -1
    assert part(16, 8, 256, 16, 16, 512, 16, 4, 16, 1 << 20, None) == -2        # unknown flag
    assert part(16, 8, 256, 16, 16, 512, 16, 0, 16, 64, None) == -4
    assert part(16, 8, 256, 16, 16, 512, 24, 0, 16, 1 << 20, None) == -3
    assert part(16, 0, 256, 16, 16, 512, 16, 0, 16, 1 << 20, None) == 0
    ep = lib.bitlinear_epilogue_sum
    two = (ctypes.c_void_p * 2)(16, 32)
    assert ep(two, 0, 8, 512, 16, 16, None, 16, None, 0, None) == -2
    assert ep(two, 9, 8, 512, 16, 16, None, 16, None, 0, None) == -2
    assert ep(None, 2, 8, 512, 16, 16, None, 16, None, 0, None) == -1
    assert ep((ctypes.c_void_p * 2)(16, None), 2, 8, 512, 16, 16, None, 16, None, 0, None) == -1
    assert ep((ctypes.c_void_p * 2)(16, 20), 2, 8, 512, 16, 16, None, 16, None, 0, None) == -3
    assert ep(two, 2, 8, 512, 16, 16, None, 16, None, 8, None) == -2
    assert ep(two, 2, 0, 512, 16, 16, None, 16, None, 0, None) == 0


def test_i8_peak_rejects_bad_arguments(lib):
    g = ctypes.c_int(0)
    assert lib.bitlinear_measure_i8_peak(0, ctypes.byref(g), 16, 256, None) == -2
    assert lib.bitlinear_measure_i8_peak((1 << 24) + 1, ctypes.byref(g), 16, 256, None) == -2
    assert lib.bitlinear_measure_i8_peak(10, None, 16, 256, None) == -1
    assert lib.bitlinear_measure_i8_peak(10, ctypes.byref(g), 16, 128, None) == -4
    assert lib.bitlinear_measure_i8_peak(10, ctypes.byref(g), 20, 256, None) == -3
