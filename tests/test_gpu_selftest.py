"""The hardware conversions the kernels use (cvt.rn.satfinite to E2M1 pairs
and to E4M3 pairs, and the decodes of E2M1 and E4M3 pairs to f16 pairs)
agree with the library's software encoders and decoders on every input. The software encoders are the ones the parity tests pin to
the oracle, so this extends that pin to the hardware path over all inputs."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_hardware_conversion_matches_encoder_on_all_fp32(dev, lib, which):
    bad = torch.full((1,), -1, dtype=torch.int64, device=dev)
    lib.selftest(which, bad)
    torch.cuda.synchronize()
    assert bad.item() == 0
