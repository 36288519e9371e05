"""GPU parity of moe_combine_rht (the combine read straight from the RHT32-
quantized payload) against the oracle, through the C ABI.

The payload is quantized by the oracle; routing is the oracle's on Zipf-skewed
logits. The GPU sums in fp32 (slot order, fused multiply-adds) and transforms
in fp32; the oracle in fp64. Bar per element: one bf16 ulp of the result plus
1e-5 of M = (1/sqrt(32)) sum_i sum_j |w_j v_j,i| over the element's 32-block,
which bounds the fp32 rounding of the sums and of the five butterfly stages.
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import dev_f32, dev_u8, host_bits, sync

pytestmark = pytest.mark.gpu


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _magnitude(orc, codes, scales, ts, fmt, pos, w, d):
    """M per (token, 32-block): the payload decoded by the oracle (fp32 rows
    through an identity-sign inverse would mix blocks, so decode directly)."""
    R = codes.shape[0]
    if fmt == 0:
        v = orc.nvfp4_dequantize(codes, scales, ts, R, d).astype(np.float64)
    else:
        v = orc.mxfp8_dequantize(codes, scales).astype(np.float64)
    T, k = pos.shape
    M = np.zeros((T, d // 32))
    for j in range(k):
        M += np.abs(w[:, j:j + 1]) * np.abs(v[pos[:, j]]).reshape(T, d // 32, 32).sum(axis=2)
    return np.repeat(M / np.sqrt(32.0), 32, axis=1)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("T,E,k,d", [(384, 16, 4, 512), (97, 8, 3, 96)])
def test_combine_rht_matches_oracle(dev, lib, orc, fmt, T, E, k, d):
    logits = synth.logits_zipf_np(9, T, E)
    idx, w = orc.route(logits, k)
    off, pos, tok = orc.permute(idx, E)
    R = len(tok)
    x = _f32(synth.payload_rows_np(10, 0, R, d, synth.outlier_channels(10, d, 2)))
    codes, scales, ts = orc.rht32_quantize(x, 11, fmt)
    wf = w.astype(np.float32)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    ts_dev = dev_f32([ts if ts is not None else 0.0], dev)
    lib.moe_combine_rht(dev_u8(codes, dev), dev_u8(scales, dev), ts_dev, fmt, 11,
                        torch.tensor(pos, device=dev), dev_f32(wf, dev), out)
    sync()
    got = _f32(host_bits(out)).astype(np.float64)
    ref = orc.combine_rht(codes, scales, ts, fmt, 11, pos, wf.astype(np.float64), f64=True)
    M = _magnitude(orc, codes, scales, ts, fmt, pos, wf.astype(np.float64), d)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-38))) - 7)
    err = np.abs(got - ref)
    bad = err > ulp + 1e-5 * M
    assert not bad.any(), (int(bad.sum()), got[bad][:4], ref[bad][:4])


def test_combine_rht_empty(dev, lib):
    out = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    z = torch.empty(0, dtype=torch.int32, device=dev).reshape(0, 2)
    lib.moe_combine_rht(None, None, None, 0, 11, z, torch.empty(0, 2, device=dev), out)
    sync()
