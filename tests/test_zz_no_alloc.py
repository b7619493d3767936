"""bitlinear_forward_noalloc: the forward for callers that cannot allocate
device memory (code inside someone else's graph capture, plugins without an
allocator, paths that must never allocate).  It uses the library's fixed
device scratch array instead of a caller workspace; its output must equal
bitlinear_forward's, call after call, because every call reuses that array.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""

import ctypes

import pytest
import torch

import bitlinear_fwd_b200 as bl
import synth

pytestmark = pytest.mark.gpu


def _noalloc(x, packed, s_w, bias, y):
    M, K = x.shape
    N = packed.shape[0]
    st = torch.cuda.current_stream().cuda_stream
    return bl.lib().bitlinear_forward_noalloc(
        ctypes.c_void_p(x.data_ptr()), M, K, ctypes.c_void_p(packed.data_ptr()), N,
        ctypes.c_void_p(s_w.data_ptr()), None if bias is None else ctypes.c_void_p(bias.data_ptr()),
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(st))


@pytest.mark.parametrize("M,N,K,with_bias", [(300, 1000, 3200, True), (4, 4096, 4096, False), (17, 520, 640, True)])
def test_noalloc_matches_forward_twice(M, N, K, with_bias):
    assert torch.cuda.is_available()
    w = synth.normal_f32(90, N + K, (N, K), 0.02).cuda()
    packed, s_w, _ = bl.bitlinear_pack_weights(w)
    bias = synth.normal_bf16(90, N, (N,), 0.01).cuda() if with_bias else None
    for call in range(2):                      # two calls in a row share the scratch
        x = synth.normal_bf16(91 + call, M * K, (M, K)).cuda()
        want = bl.bitlinear_forward(x, packed, s_w, bias)
        y = torch.full((M, N), -1.0, dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        assert _noalloc(x, packed, s_w, bias, y) == 0
        torch.cuda.synchronize()
        if call == 1:                          # its kernels are loaded by now: no device memory taken
            assert torch.cuda.mem_get_info()[0] == free_before
        # same tolerance as the other parity tests: bit-exact bf16 output
        assert torch.equal(y.view(torch.int16), want.view(torch.int16)), f"call {call} differs"
        assert bl.bitlinear_noalloc_check_status() == 0


def test_noalloc_rejects_sizes_beyond_scratch():
    x = torch.empty(8, dtype=torch.bfloat16, device="cuda")
    packed = torch.empty(16, dtype=torch.uint8, device="cuda")
    s_w = torch.ones(1, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    M, K, N = 4096, 8192, 64                   # M*K = 32 MiB > the 16 MiB scratch
    assert bl.lib().bitlinear_forward_noalloc(ctypes.c_void_p(x.data_ptr()), M, K,
                                              ctypes.c_void_p(packed.data_ptr()), N,
                                              ctypes.c_void_p(s_w.data_ptr()), None,
                                              ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(st)) == -4


@pytest.mark.parametrize("M", [4, 40])
def test_noalloc_reports_a_timeout(M):
    """A device-side wait that gives up inside a noalloc call is visible to
    the caller through bitlinear_noalloc_check_status (the status word sits in
    the fixed scratch, which the caller cannot name); the next call is normal."""
    N, K = 512, 1024
    w = synth.normal_f32(95, N + K, (N, K), 0.02).cuda()
    packed, s_w, _ = bl.bitlinear_pack_weights(w)
    x = synth.normal_bf16(96, M * K, (M, K)).cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    bl.bitlinear_test_force_timeout(True)
    try:
        assert _noalloc(x, packed, s_w, None, y) == 0
        assert bl.bitlinear_noalloc_check_status() == -6
    finally:
        bl.bitlinear_test_force_timeout(False)
    assert _noalloc(x, packed, s_w, None, y) == 0
    assert bl.bitlinear_noalloc_check_status() == 0
    want = bl.bitlinear_forward(x, packed, s_w)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), want.view(torch.int16))
