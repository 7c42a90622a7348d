"""include/moe.h is a C header: a plain C99 program compiles against it with gcc,
links to libmoe_b200.so and calls the entry points that need no GPU (status
strings, workspace sizes, argument checks that fail before any launch)."""
import os
import shutil
import subprocess

import pytest

import sparse_moe_ffn_sigmoid_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <stdint.h>
#include <string.h>
#include "moe.h"

int main(void) {
    /* status strings and sizes: pure host logic */
    if (strlen(moe_status_string(MOE_OK)) == 0) return 1;
    if (moe_workspace_size(64, 7168, 384, 8, 2048) == 0) return 2;
    if (moe_workspace_size_w8a8(64, 7168, 384, 8, 2048) <= moe_workspace_size(64, 7168, 384, 8, 2048))
        return 3;
    if (moe_workspace_size(64, 7100, 384, 8, 2048) != 0) return 4;   /* d not a multiple of 64 */
    /* argument checks reject before any launch */
    uint16_t dummy[8] __attribute__((aligned(16)));
    if (moe_layer_forward(NULL, dummy, (const float*)dummy, dummy, dummy, dummy, dummy,
                          64, 7168, 384, 8, 2048, 2.827f, dummy, NULL) != MOE_ERR_INVALID_ARG)
        return 5;
    if (moe_layer_forward(dummy, dummy, (const float*)dummy, dummy, dummy, dummy, dummy,
                          64, 7168, 384, 40, 2048, 2.827f, dummy, NULL) != MOE_ERR_UNSUPPORTED_SHAPE)
        return 6;
    if (moe_layer_forward(dummy, dummy, (const float*)dummy, dummy, dummy, dummy, dummy,
                          0, 7168, 384, 8, 2048, 2.827f, dummy, NULL) != MOE_OK)
        return 7;
    printf("noalloc scratch bytes %lu\n", (unsigned long)MOE_NOALLOC_SCRATCH_BYTES);
    printf("c abi ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_links(tmp_path):
    lib = moe.lib()._name
    src = tmp_path / "use_moe.c"
    exe = tmp_path / "use_moe"
    src.write_text(C_PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), lib,
                    "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert "c abi ok" in out.stdout
    # the binding's copy of the scratch array's size is the header's macro
    line = [ln for ln in out.stdout.splitlines() if ln.startswith("noalloc scratch bytes")][0]
    assert int(line.split()[-1]) == moe.NOALLOC_SCRATCH_BYTES
