"""The boundary from plain C: a C99 program that includes only include/gdn2.h, links libgdn2.so
and calls entry points that need no GPU (status strings, workspace sizes, argument checks).
This checks that the header is valid C and that the ABI is usable without Python or C++."""
import os
import shutil
import subprocess

import pytest

import gated_delta_rule_96_b200 as g

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "gdn2.h"

int main(void) {
    int fails = 0;
    void *fake = (void *)0x10000;   /* never dereferenced: every call below fails its checks first */
    size_t ws = gdn2_chunk_fwd_workspace_bytes(8, 16, 4096, 128, 128, 64, GDN2_BF16);
    if (ws < 256) { printf("workspace %zu\n", ws); ++fails; }
    if (gdn2_chunk_fwd_path(8, 16, 4096, 128, 128, 64, GDN2_BF16) != 2) ++fails;
    if (gdn2_chunk_fwd_path(1, 16, 65536, 128, 128, 64, GDN2_BF16) != 2) ++fails;
    if (gdn2_chunk_fwd_path(1, 16, 1024, 128, 128, 64, GDN2_BF16) != 1) ++fails;
    if (gdn2_chunk_fwd_path(1, 2, 256, 64, 64, 64, GDN2_F32) != 0) ++fails;
    if (gdn2_chunk_fwd(fake, fake, fake, (const float *)fake, fake, fake, NULL, fake, (float *)fake, 1, 1, 8, 96,
                       128, 64, GDN2_BF16, fake, ws, NULL) != GDN2_ERR_UNSUPPORTED) ++fails;
    if (gdn2_decode_step(NULL, fake, fake, (const float *)fake, fake, fake, (float *)fake, fake, 1, 1, 128, 128,
                         GDN2_BF16, NULL) != GDN2_ERR_NULL) ++fails;
    if (strcmp(gdn2_status_str(GDN2_OK), "ok") != 0) ++fails;
    if (gdn2_chunk_bwd_workspace_bytes(1, 1, 8, 96, 128) != 0) ++fails;
    printf("%s %d\n", gdn2_status_str(GDN2_ERR_ALIGN), fails);
    return fails;
}
"""


def test_c99_client(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = g.library_path()
    if not os.path.exists(lib):
        pytest.skip("libgdn2.so not built")
    src = tmp_path / "client.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "client"
    libdir = os.path.dirname(lib)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", libdir, "-lgdn2", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "a pointer is not 16-byte aligned 0"
