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
    # K = 100 is not a multiple of 64: the workspace query fails first
    with pytest.raises(bl.BitLinearError) as e:
        bl.bitlinear_forward(torch.zeros((2, 100), dtype=torch.bfloat16), torch.zeros((16, 25), dtype=torch.uint8),
                             torch.ones(1))
    assert e.value.status == -2
    with pytest.raises(bl.BitLinearError):
        bl.workspace(2, 16, 100, "cpu")
