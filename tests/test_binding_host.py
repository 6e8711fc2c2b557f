"""The Python binding on the CPU: it has no fallback.  A missing libzmoe.so fails loudly at load time,
and every call rejects host (CPU) tensors before it reaches the library, so no step of the path can run
anywhere but in the CUDA kernels."""
import pytest
import torch

from sparse_moe_decoder_b200 import zmoe as Z


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(Z, "LIB_PATH", str(tmp_path / "libzmoe.so"))
    monkeypatch.setattr(Z, "_lib", None)
    with pytest.raises(ImportError, match="libzmoe.so not found"):
        Z.lib()


def _cpu(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype)


@pytest.mark.parametrize("call", [
    lambda: Z.zmoe_delay_shear(_cpu(4, 9, dtype=torch.int32)),
    lambda: Z.zmoe_delay_unshear(_cpu(12, 9, dtype=torch.int32)),
    lambda: Z.zmoe_embed_sum_rmsnorm(_cpu(2, 9, dtype=torch.int32), _cpu(9, 1025, 16, dtype=torch.bfloat16),
                                     _cpu(16)),
    lambda: Z.zmoe_rmsnorm(_cpu(2, 16), _cpu(16)),
    lambda: Z.zmoe_route(_cpu(4, 64, dtype=torch.bfloat16), _cpu(16, 64, dtype=torch.bfloat16), 1),
    lambda: Z.zmoe_permute(_cpu(4, 1, dtype=torch.int32), _cpu(4, 64, dtype=torch.bfloat16), 16),
    lambda: Z.zmoe_grouped_swiglu(_cpu(4, 256, dtype=torch.bfloat16), _cpu(17, dtype=torch.int32),
                                  _cpu(16, 256, 256, dtype=torch.bfloat16), _cpu(16, 256, 256, dtype=torch.bfloat16),
                                  _cpu(16, 256, 256, dtype=torch.bfloat16)),
    lambda: Z.zmoe_combine(_cpu(4, 64), _cpu(4, 1, dtype=torch.int32), _cpu(4, 1)),
    lambda: Z.zmoe_moe_layer(_cpu(16, 256, dtype=torch.bfloat16), _cpu(16, 256, 256, dtype=torch.bfloat16),
                             _cpu(16, 256, 256, dtype=torch.bfloat16), _cpu(16, 256, 256, dtype=torch.bfloat16), 1,
                             x=_cpu(4, 256, dtype=torch.bfloat16)),
    lambda: Z.zmoe_output_heads(_cpu(1, 64), _cpu(9, 1025, 64, dtype=torch.bfloat16)),
    lambda: Z.zmoe_speaker_prefix(_cpu(1, 1024), _cpu(64, 1024, dtype=torch.bfloat16)),
    lambda: Z.zmoe_prepare_w_down_f16(_cpu(4, 256, 256, dtype=torch.bfloat16)),
])
def test_host_tensors_are_rejected(call):
    with pytest.raises(TypeError, match="must be a CUDA tensor"):
        call()
