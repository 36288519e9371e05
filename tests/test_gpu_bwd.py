"""GPU parity of the SwiGLU backward against the oracle.

The kernel works in fp32 (IEEE division, expf) and rounds once to bf16; the
oracle works in fp64. Every output is within one bf16 ulp of the oracle's,
and almost all are bit-identical (the two differ only where the exact value
lies within the fp32 error of a bf16 rounding boundary).
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import dev_bf16, host_bits, sync

pytestmark = pytest.mark.gpu


def _ulp(v):
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-38))) - 7)


@pytest.mark.parametrize("rows,f", [(1000, 2560), (37, 8), (128, 512)])
def test_swiglu_bwd_matches_oracle(dev, lib, orc, rows, f):
    gu_bits = synth.rows_np(4, synth.TAG_ACT, 0, rows, 2 * f, 2.0)
    gu_bits[0, :8] = synth.f32_to_bf16_bits(np.array([-100, -30, -8, 0, 8, 30, 100, 1e-3],
                                                     np.float32))
    dh_bits = synth.rows_np(5, synth.TAG_ACT, 0, rows, f, 0.5)
    dh_bits[1, :] = 0
    out = torch.full((rows, 2 * f), -1.0, dtype=torch.bfloat16, device=dev)
    lib.swiglu_bwd(dev_bf16(gu_bits, dev), dev_bf16(dh_bits, dev), out)
    sync()
    got_bits = host_bits(out)
    ref_bits = orc.swiglu_bwd(gu_bits, dh_bits)
    got = synth.bf16_bits_to_f32(got_bits).astype(np.float64)
    ref = synth.bf16_bits_to_f32(ref_bits).astype(np.float64)
    assert np.all(np.abs(got - ref) <= _ulp(ref) + 1e-38)
    same = np.mean((got_bits == ref_bits) | ((got == 0) & (ref == 0)))
    assert same >= 0.99, same


def test_swiglu_bwd_no_rows(dev, lib):
    e = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    lib.swiglu_bwd(torch.empty(0, 128, dtype=torch.bfloat16, device=dev), e,
                   torch.empty(0, 128, dtype=torch.bfloat16, device=dev))
    sync()
