"""The C ABI library loads without a GPU, exports every entry point the header
declares, and rejects bad arguments on the host before launching anything."""
import ctypes as C
import os
import re

import pytest

from precision_moe_numerics_quantize_b200 import build as B
from precision_moe_numerics_quantize_b200 import nvfp4moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4moe.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return M.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_0-9]+)\s*\(", src,
                       flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["nvfp4_quantize", "mxfp8_quantize_sr", "rht32_quantize", "moe_route_permute",
              "moe_expert_fwd", "moe_expert_fwd_mxfp8", "moe_combine", "nvfp4_grouped_gemm",
              "mxfp8_grouped_gemm"]:
        assert n in names
    assert set(names) == set(M.EXPORTED), set(names) ^ set(M.EXPORTED)


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_host_only_queries(L):
    assert L.nvfp4moe_version() == 100
    assert L.nvfp4moe_max_rows(16384, 8, 384) == (16384 * 8 + 384 * 127 + 127) // 128 * 128
    assert L.nvfp4moe_max_rows(0, 1, 1) == 128
    assert L.moe_route_permute_workspace_size(16384, 384, 8) > 0
    assert L.moe_route_permute_workspace_size(10, 0, 1) == 0


P = 1 << 20  # a fake, 16-byte aligned "device pointer"; validation fails before any use


@pytest.mark.parametrize("call,status", [
    (lambda L: L.nvfp4_quantize(P, 4, 48, 48, None, P, P, P + 16, 0, None), 2),      # cols % 64
    (lambda L: L.nvfp4_quantize(P, 100, 64, 64, None, P, P, P + 16, 1, None), 2),    # MMA rows
    (lambda L: L.nvfp4_quantize(P + 2, 4, 64, 64, None, P, P, P + 16, 0, None), 3),  # align
    (lambda L: L.nvfp4_quantize(None, 4, 64, 64, None, P, P, P + 16, 0, None), 1),   # null
    (lambda L: L.nvfp4_quantize(P, 4, 64, 64, P + 16, P, P, P + 16, 0, None), 1),    # alias
    (lambda L: L.nvfp4_quantize(P, 4, 64, 64, None, P, P, P + 16, 7, None), 1),      # layout
    (lambda L: L.mxfp8_quantize_sr(P, 4, 64, 64, 2, None, 0, 0, 0, 1, P, P, 0, None), 1),  # axis
    (lambda L: L.mxfp8_quantize_sr(P, 40, 64, 64, 1, None, 0, 0, 0, 1, P, P, 0, None), 2), # rows % 32
    (lambda L: L.mxfp8_quantize_sr(P, 4, 64, 64, 0, None, 0, 0, 0, 5, P, P, 0, None), 1),  # rounding
    (lambda L: L.mxfp8_quantize_sr(P, 40, 64, 64, 0, P, 2, 0, 0, 1, P, P, 0, None), 1),    # seg + axis 0
    (lambda L: L.mxfp8_quantize_sr(P, 40, 64, 64, 1, P, 0, 0, 0, 1, P, P, 0, None), 1),    # nseg 0
    (lambda L: L.mxfp8_quantize_sr(P, 40, 64, 64, 1, P, 1025, 0, 0, 1, P, P, 0, None), 1), # nseg > 1024
    (lambda L: L.mxfp8_quantize_sr(P, 40, 96, 96, 1, P, 2, 0, 0, 1, P, P, 0, None), 2),    # cols % 64
    (lambda L: L.mxfp8_quantize_sr(P, 40, 64, 64, 1, P + 2, 2, 0, 0, 1, P, P, 0, None), 3),  # seg_off align
    (lambda L: L.rht32_quantize(P, 4, 48, 48, 0, 0, None, P, P, P, 0, None), 2),     # cols % 32
    (lambda L: L.rht32_quantize(P, 4, 64, 64, 0, 0, None, P, P, P, 1, None), 7),     # MMA layout
    (lambda L: L.moe_route_permute(P, P, 8, 4, 5, 64, 1, None, P, P, P, P, P, P, P, P, P,
                                   1 << 20, None), 1),                               # k > E
    (lambda L: L.moe_route_permute(P, P, 8, 4, 2, 64, 1, None, P, P, P, P, P, P, P, P, P,
                                   4, None), 4),                                     # workspace
    (lambda L: L.moe_route_permute(P, P, 8, 4, 2, 96, 1, None, P, P, P, P, P, P, P, P, P,
                                   1 << 20, None), 2),                               # d % 64
    (lambda L: L.moe_expert_fwd(P, P, P, P, 4, 384, 256, P, P, P, P, P, P, P, P, P, P, P, P,
                                128, None), 2),                                      # d % 256
    (lambda L: L.moe_expert_fwd_fused_requant(P, P, P, P, 4, 256, 256, P, P, P, P, P, P, P, P,
                                              P, P, P, P, 128, P, 16, None), 4),     # workspace
    (lambda L: L.moe_expert_fwd_mxfp8(P, P, P, 4, 384, 256, P, P, P, P, P, P, P, P, P, 128,
                                      None), 2),                                     # d % 256
    (lambda L: L.moe_expert_fwd_mxfp8(P, P, P, 4, 256, 256, P, P, P, P, P, P, P, P, P, 100,
                                      None), 2),                                     # rows % 128
    (lambda L: L.moe_expert_fwd_mxfp8(P, P, P, 0, 256, 256, P, P, P, P, P, P, P, P, P, 128,
                                      None), 1),                                     # E
    (lambda L: L.moe_expert_fwd_mxfp8(P, P, P, 4, 256, 256, P, P, None, P, P, P, P, P, P, 128,
                                      None), 1),                                     # null w2
    (lambda L: L.moe_expert_fwd_mxfp8(P, P, P, 4, 256, 256, P, P, P, P, P + 2, P, P, P, P, 128,
                                      None), 3),                                     # align h
    (lambda L: L.swiglu_bwd(P, P, 4, 12, P + 4096, None), 2),                         # f % 8
    (lambda L: L.swiglu_bwd(P, P + 4096, 4, 64, P, None), 1),                        # alias
    (lambda L: L.swiglu_bwd(P, P + 8, 4, 64, P + 4096, None), 3),                    # align
    (lambda L: L.moe_expert_bwd_gemm1(P, P, P, 4, 384, 128, P, P, 0, 0, P, P, P, P, P, P, P, P,
                                      128, None), 2),                                # d % 256
    (lambda L: L.moe_expert_bwd_gemm1(P, P, P, 4, 256, 64, P, P, 0, 0, P, P, P, P, P, P, P, P,
                                      128, None), 2),                                # f % 128
    (lambda L: L.moe_expert_bwd_gemm1(P, P, P, 4, 256, 128, P, P, 0, 0, P, P, P, None, P, P, P,
                                      P, 128, None), 1),                             # null gt_sc
    (lambda L: L.moe_combine(P, P, P, 4, 2, 12, P, None), 2),                        # d % 8
    (lambda L: L.nvfp4_grouped_gemm(P, P, P, 2, P, P, P, P, 1, 128, 256, 256, P, 0, None), 1),
    (lambda L: L.nvfp4_grouped_gemm(P, P, P, 0, P, P, P, P, 1, 128, 256, 128, P, 0, None), 2),
    (lambda L: L.mxfp8_grouped_gemm(P, P, P, P, P, 1, 3, 128, 256, 128, P, 1, None), 1),
    (lambda L: L.mxfp8_grouped_gemm(P, P, P, P, P, 2000, 0, 128, 256, 128, P, 1, None), 1),
])
def test_validation_rejects_before_launch(L, call, status):
    assert call(L) == status
    assert L.nvfp4moe_last_error().decode()


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        M.nvfp4_quantize(x, x, x, x)


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "nvfp4moe.h"
int main(void) {
    if (nvfp4moe_max_rows(16384, 8, 384) != 179840) return 2;
    /* cols = 48 is not a multiple of 64: rejected on the host, nothing launched */
    nvfp4moe_status st = nvfp4_quantize((const uint16_t *)0x100000, 4, 48, 48, NULL,
                                        (uint8_t *)0x100000, (uint8_t *)0x100000,
                                        (float *)0x100010, NVFP4MOE_LAYOUT_ROWMAJOR, NULL);
    if (st != NVFP4MOE_ERR_SHAPE) return 3;
    if (strlen(nvfp4moe_last_error()) == 0) return 4;
    printf("%s\n", nvfp4moe_last_error());
    return 0;
}
"""


def test_plain_c_program_links_and_validates(L, tmp_path):
    """A C99 program compiled with gcc links against the library and gets the
    documented status and error text back, with no GPU involved."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(M.LIB_PATH)
    exe = tmp_path / "prog"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), f"-L{libdir}", "-l:libnvfp4moe.so",
                           f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert "nvfp4_quantize" in out.stdout
