"""The C ABI from C: a program that includes include/gdn.h, compiled by the host C
compiler (no CUDA headers, no torch) and linked against libgdn_b200.so, calls the entry
points that need no device (version, status strings, workspace sizes, argument checks)."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "gated_deltanet_05_b200")

PROGRAM = r'''
#include <stdio.h>
#include <string.h>
#include "gdn.h"

int main(void)
{
    int32_t cu[3] = {0, 64, 100};
    if (gdn_version() <= 0) return 1;
    if (strcmp(gdn_status_string(GDN_ERR_TIMEOUT), "GDN_ERR_TIMEOUT") != 0) return 2;
    /* one 64-token chunk per chain: two 16 x 16 states, U~ and dU~ (64 x 16), the chunk's
       cache and one block of sums */
    if (gdn_backward_workspace_bytes(cu, 2, 2, 16, 16) !=
        (size_t)2 * 2 * 1 * (2 * 16 * 16 + 2 * 64 * 16 + 64 * (3 * 64 + 16) + (64 * (2 * 64 + 3 * 16 + 1) + 1 + 3) / 4 * 4) * 4)
        return 3;
    /* rejected before any launch: an unsupported head size, an unknown dtype */
    if (gdn_decode_step(0, 0, 0, GDN_F32, 0, 0, 0, 1, 1, 48, 16, 1.f, 0, GDN_F32, 0) != GDN_ERR_UNSUPPORTED) return 4;
    if (gdn_gate_norm(0, (gdn_dtype)7, 0, GDN_F32, 0, 4, 16, 1e-6f, 0, GDN_F32, 0) != GDN_ERR_INVALID_ARG) return 5;
    printf("ok %d\n", gdn_version());
    return 0;
}
'''


def test_header_compiles_as_c_and_links(tmp_path):
    lib = os.path.join(LIBDIR, "libgdn_b200.so")
    if not os.path.exists(lib):
        pytest.skip("libgdn_b200.so not built")
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe), "-L", LIBDIR, "-lgdn_b200", "-Wl,-rpath," + LIBDIR], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok ")
