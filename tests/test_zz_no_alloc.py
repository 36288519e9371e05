"""moe_route_permute_noalloc: routing and dispatch for callers that cannot
allocate device memory (their memory is reserved up front by another
allocator, they run inside a framework that forbids allocating, or they cannot
afford cudaMalloc's implicit synchronisation). It uses a 4 MiB array built
into the library instead of a caller-provided workspace.

Checked through the C ABI against moe_route_permute with a workspace, on two
calls in a row with different inputs, so a stale scratch from the first call
would show up in the second. Integer outputs, codes and scales must be
bit-exact; the router weights are held to the tolerance of the routing tests.
The size limit is enforced before anything is launched."""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import dev_bf16, dev_f32, sync

pytestmark = pytest.mark.gpu


def _outputs(dev, T, E, k, d):
    R = int((T * k + E * 127 + 127) // 128 * 128)
    return {
        "idx": torch.empty(T, k, dtype=torch.int32, device=dev),
        "w": torch.empty(T, k, dtype=torch.float32, device=dev),
        "off": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "pos": torch.empty(T, k, dtype=torch.int32, device=dev),
        "tok": torch.empty(R, dtype=torch.int32, device=dev),
        "xq": torch.full((R, d // 2), 0x5A, dtype=torch.uint8, device=dev),
        "xq_sc": torch.full((R * d // 16,), 0x5A, dtype=torch.uint8, device=dev),
        "x_ts": torch.empty(1, device=dev),
    }


def _compare(a, b):
    used = int(a["off"][-1].item())
    assert torch.equal(a["off"], b["off"])
    assert torch.equal(a["idx"], b["idx"])
    assert torch.equal(a["pos"], b["pos"])
    assert torch.equal(a["tok"], b["tok"])
    assert torch.equal(a["xq"][:used], b["xq"][:used])
    assert torch.equal(a["xq_sc"][:used * a["xq"].shape[1] // 8],
                      b["xq_sc"][:used * b["xq"].shape[1] // 8])
    assert torch.equal(a["x_ts"], b["x_ts"])
    assert np.allclose(a["w"].cpu().numpy(), b["w"].cpu().numpy(), rtol=4e-6, atol=1e-30)


def test_noalloc_matches_workspace_entry_point_on_two_calls(dev, lib):
    cases = [("uniform", 2048, 32, 4, 1024, 2), ("zipf", 1000, 384, 8, 256, 3)]
    for router, T, E, k, d, seed in cases:
        logits = (synth.logits_uniform_np(seed, T, E) if router == "uniform"
                  else synth.logits_zipf_np(seed, T, E))
        lg = dev_f32(logits, dev)
        x = dev_bf16(synth.rows_np(seed, synth.TAG_X, 0, T, d, 1.0), dev)
        ref = _outputs(dev, T, E, k, d)
        ws = torch.empty(lib.moe_route_permute_workspace_size(T, E, k), dtype=torch.uint8,
                         device=dev)
        lib.moe_route_permute(lg, x, k, 1, ref["idx"], ref["w"], ref["off"], ref["pos"],
                              ref["tok"], ref["xq"], ref["xq_sc"], ref["x_ts"], ws)
        got = _outputs(dev, T, E, k, d)
        lib.moe_route_permute_noalloc(lg, x, k, 1, got["idx"], got["w"], got["off"], got["pos"],
                                      got["tok"], got["xq"], got["xq_sc"], got["x_ts"])
        sync()
        _compare(ref, got)
    st, code = lib.device_error()
    assert st == 0 and code == 0


def test_noalloc_rejects_more_than_its_scratch(dev, lib):
    L = lib.lib()
    T, E, k, d = 1 << 20, 384, 8, 64  # needs about 34 MiB of scratch
    assert lib.moe_route_permute_workspace_size(T, E, k) > (4 << 20)
    P = 1 << 20  # never dereferenced: the size check fails before any launch
    st = L.moe_route_permute_noalloc(P, P, T, E, k, d, 1, None, P, P, P, P, P, P, P, P, None)
    assert st == 4  # NVFP4MOE_ERR_WORKSPACE
    assert b"4194304" in L.nvfp4moe_last_error()


def test_noalloc_given_amax_and_no_tokens(dev, lib):
    """The two paths of the built-in scratch the first test does not reach: a
    caller-supplied tensor amax (the scratch's amax slot is then not used; half
    the true amax also saturates blocks), and T = 0 (only the expert offsets
    and the padding of the token map are written). Each is compared with the
    workspace entry point, run right after a call that left the scratch
    dirty."""
    T, E, k, d = 700, 48, 6, 512
    logits = synth.logits_zipf_np(5, T, E)
    lg = dev_f32(logits, dev)
    xb = synth.rows_np(5, synth.TAG_X, 0, T, d, 1.0)
    x = dev_bf16(xb, dev)
    amax = dev_f32([np.abs(synth.bf16_bits_to_f32(xb)).max() * 0.5], dev)
    for renorm in (1, 0):
        ref = _outputs(dev, T, E, k, d)
        ws = torch.empty(lib.moe_route_permute_workspace_size(T, E, k), dtype=torch.uint8,
                         device=dev)
        lib.moe_route_permute(lg, x, k, renorm, ref["idx"], ref["w"], ref["off"], ref["pos"],
                              ref["tok"], ref["xq"], ref["xq_sc"], ref["x_ts"], ws, x_amax_in=amax)
        got = _outputs(dev, T, E, k, d)
        lib.moe_route_permute_noalloc(lg, x, k, renorm, got["idx"], got["w"], got["off"],
                                      got["pos"], got["tok"], got["xq"], got["xq_sc"],
                                      got["x_ts"], x_amax_in=amax)
        sync()
        _compare(ref, got)
    # T = 0 right after a call with tokens
    T0 = 0
    e = torch.empty(0, dtype=torch.int32, device=dev)
    ref = _outputs(dev, T0, E, k, d)
    got = _outputs(dev, T0, E, k, d)
    ref["off"].fill_(-5)
    got["off"].fill_(-5)
    lg0 = torch.empty(0, E, device=dev)
    x0 = torch.empty(0, d, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(16, lib.moe_route_permute_workspace_size(T0, E, k)), dtype=torch.uint8,
                     device=dev)
    lib.moe_route_permute(lg0, x0, k, 1, e, torch.empty(0, device=dev), ref["off"], e, ref["tok"],
                          ref["xq"], ref["xq_sc"], ref["x_ts"], ws)
    lib.moe_route_permute_noalloc(lg0, x0, k, 1, e, torch.empty(0, device=dev), got["off"], e,
                                  got["tok"], got["xq"], got["xq_sc"], got["x_ts"])
    sync()
    assert torch.equal(ref["off"], got["off"]) and not got["off"].any()
    assert torch.equal(ref["tok"], got["tok"]) and (got["tok"] == -1).all()
    assert torch.equal(ref["x_ts"], got["x_ts"])
    st, code = lib.device_error()
    assert st == 0 and code == 0
