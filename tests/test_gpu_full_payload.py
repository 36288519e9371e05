"""Full-size parity of the combine-payload quantizer: the routed rows of the
full layer, [T*k x d] = [131072 x 4096] bf16, heavy-tailed (Student-t-like,
3 degrees of freedom) with 16 outlier channels x 50, through the 32-point
random Hadamard transform (sign seed 11) and block-scaled NVFP4 or MXFP8
quantization, as the benchmark runs it.

  tensor scale  the NVFP4 payload's tensor scale equals amax / 2688 with the
                amax of all 537M transformed values, which the oracle
                computes a slice of rows at a time;
  codes         64 rows spread over the tensor: codes and scales bit-exact
                for both formats (the NVFP4 rows quantized by the oracle with
                that tensor amax);
  round trip    the GPU's dequantization and inverse transform of those rows
                equals the oracle's bit for bit.
The input tensor comes from the seeded generator (on the device; the same
bits as its numpy twin), never from a kernel under test.
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import dev_f32, host_bits, host_u8, sync

pytestmark = pytest.mark.gpu

SHAPE = synth.SHAPES["full_moe"]
SIGN_SEED = 11
SAMPLE = 64


@pytest.fixture(scope="module")
def payload(dev, orc):
    R, d = SHAPE.T * SHAPE.k, SHAPE.d
    chans = synth.outlier_channels(5, d, 16)
    x = synth.payload_rows_torch(5, 0, R, d, chans, dev)
    sync()
    amax = np.float32(0.0)
    step = 8192
    for r0 in range(0, R, step):
        xs = synth.bf16_bits_to_f32(host_bits(x[r0:r0 + step]))
        amax = max(amax, orc.rht32_amax(xs, SIGN_SEED))
    rows = np.sort(np.random.default_rng(13).choice(R, size=SAMPLE, replace=False))
    rows[0], rows[-1] = 0, R - 1
    xr = synth.bf16_bits_to_f32(host_bits(x[torch.from_numpy(rows).to(dev)]))
    yield {"x": x, "amax": np.float32(amax), "rows": rows, "xr": xr}
    del x
    torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt", [0, 1])
def test_full_rht32_payload(payload, dev, lib, orc, fmt):
    x, rows, xr = payload["x"], payload["rows"], payload["xr"]
    R, d = x.shape
    if fmt == 0:
        codes = torch.empty(R, d // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(R, d // 16, dtype=torch.uint8, device=dev)
    else:
        codes = torch.empty(R, d, dtype=torch.uint8, device=dev)
        scales = torch.empty(R, d // 32, dtype=torch.uint8, device=dev)
    ts = torch.empty(1, device=dev)
    lib.rht32_quantize(x, SIGN_SEED, fmt, codes, scales, ts_out=ts if fmt == 0 else None)
    sync()
    amax_in = payload["amax"] if fmt == 0 else None
    rc, rs, rts = orc.rht32_quantize(xr, SIGN_SEED, fmt, amax_in=amax_in)
    if fmt == 0:
        assert ts.item() == np.float32(payload["amax"] / np.float32(2688.0))
        assert ts.item() == rts
    ridx = torch.from_numpy(rows).to(dev)
    gc = codes[ridx]
    gs = scales[ridx]
    assert np.array_equal(host_u8(gc), rc)
    assert np.array_equal(host_u8(gs), rs)
    # round trip of the sampled rows: dequantize + inverse transform
    out = torch.empty(len(rows), d, device=dev)
    lib.rht32_dequantize(gc.contiguous(), gs.contiguous(), dev_f32([rts or 0.0], dev), len(rows), d,
                         SIGN_SEED, fmt, out)
    sync()
    ref = orc.rht32_dequantize(rc, rs, rts, len(rows), d, SIGN_SEED, fmt)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
