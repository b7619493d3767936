"""Host-only checks of the Python binding: it fails loudly when the CUDA
library is missing (there is no fallback of any kind), and it rejects wrong
dtypes and invalid shapes before anything reaches the GPU."""

import pytest
import torch

import bitlinear_fwd_b200 as bl


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(bl, "_lib", None)
    monkeypatch.setattr(bl, "LIB_PATH", str(tmp_path / "libbitlinear.so"))
    with pytest.raises(ImportError):
        bl.lib()
    with pytest.raises(ImportError):
        bl.bitlinear_forward(torch.zeros((1, 64), dtype=torch.bfloat16), torch.zeros((16, 16), dtype=torch.uint8),
                             torch.ones(1))


def test_wrong_dtypes_raise_type_error():
    x32 = torch.zeros((2, 64))
    packed = torch.zeros((16, 16), dtype=torch.uint8)
    with pytest.raises(TypeError):
        bl.bitlinear_forward(x32, packed, torch.ones(1))
    with pytest.raises(TypeError):
        bl.bitlinear_pack_weights(torch.zeros((16, 64), dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        bl.bitlinear_pack_weights(torch.zeros(64))
    with pytest.raises(TypeError):
        bl.bitlinear_quant_act(x32)


def test_invalid_shapes_raise_before_the_gpu():
    # K = 100 is not a multiple of 64
    with pytest.raises(bl.BitLinearError) as e:
        bl.bitlinear_forward(torch.zeros((2, 100), dtype=torch.bfloat16), torch.zeros((16, 25), dtype=torch.uint8),
                             torch.ones(1))
    assert e.value.status == -2
    with pytest.raises(bl.BitLinearError):
        bl.workspace(2, 16, 100, "cpu")


def _args(M=2, N=16, K=64):
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    packed = torch.zeros((N, K // 4), dtype=torch.uint8)
    return x, packed, torch.ones(1)


@pytest.mark.parametrize("case", ["packed_dtype", "packed_cols", "packed_1d", "scale_dtype", "scale_empty",
                                  "bias_dtype", "bias_len", "out_dtype", "out_shape", "ws_dtype", "x_3d"])
def test_forward_argument_errors_raise_on_the_host(case):
    """Every forward argument is checked before the library is called: a
    packed matrix whose column count does not match K would make the TMA
    descriptor read past the allocation, and a short output would be written
    out of bounds."""
    x, packed, s = _args()
    kw = {}
    if case == "packed_dtype":
        packed = packed.to(torch.int8)
    elif case == "packed_cols":
        packed = torch.zeros((16, 15), dtype=torch.uint8)
    elif case == "packed_1d":
        packed = torch.zeros(256, dtype=torch.uint8)
    elif case == "scale_dtype":
        s = torch.ones(1, dtype=torch.float64)
    elif case == "scale_empty":
        s = torch.ones(0)
    elif case == "bias_dtype":
        kw["bias"] = torch.zeros(16)
    elif case == "bias_len":
        kw["bias"] = torch.zeros(15, dtype=torch.bfloat16)
    elif case == "out_dtype":
        kw["out"] = torch.zeros((2, 16))
    elif case == "out_shape":
        kw["out"] = torch.zeros((2, 15), dtype=torch.bfloat16)
    elif case == "ws_dtype":
        kw["ws"] = torch.zeros(4096, dtype=torch.float32)
    elif case == "x_3d":
        x = torch.zeros((1, 2, 64), dtype=torch.bfloat16)
    with pytest.raises((TypeError, ValueError)):
        bl.bitlinear_forward(x, packed, s, **kw)


def test_noalloc_and_debug_share_the_checks():
    x, _, s = _args()
    bad = torch.zeros((16, 15), dtype=torch.uint8)
    with pytest.raises(ValueError):
        bl.bitlinear_forward_noalloc(x, bad, s)
    with pytest.raises(ValueError):
        bl.bitlinear_forward_debug(x, bad, s)
    with pytest.raises(ValueError):
        bl.bitlinear_forward_grouped(x, torch.zeros((16, 16), dtype=torch.uint8), [8, 7], torch.ones(2))
    with pytest.raises(ValueError):        # one scale for two groups
        bl.bitlinear_forward_grouped(x, torch.zeros((16, 16), dtype=torch.uint8), [8, 8], torch.ones(1))


def test_device_mismatch_raises():
    """Host tensors never reach a kernel: the packed weights must be on a GPU,
    and the host entry points want host activations."""
    x, packed, s = _args()
    with pytest.raises(ValueError):
        bl.bitlinear_forward(x, packed, s)
    with pytest.raises(ValueError):
        bl.bitlinear_forward_host(x, packed, s)
    with pytest.raises(ValueError):
        bl.bitlinear_dequant_weights(packed, s)


def test_q8_argument_errors():
    xq = torch.zeros((2, 64), dtype=torch.int8)
    packed = torch.zeros((16, 16), dtype=torch.uint8)
    with pytest.raises(TypeError):
        bl.bitlinear_forward_q8(xq, torch.ones(2, dtype=torch.float64), torch.zeros(2, dtype=torch.int32), packed,
                                torch.ones(1))
    with pytest.raises(ValueError):
        bl.bitlinear_forward_q8(xq, torch.ones(3), torch.zeros(2, dtype=torch.int32), packed, torch.ones(1))
