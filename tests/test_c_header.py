"""The boundary as a C caller sees it: include/bi.h compiles as C99 with
warnings as errors, and a C program linked against the library gets the
host-side answers (build flavour, status strings, argument rejections,
workspace sizes) without Python in between.  CPU only: nothing here
reaches a device."""
import os
import shutil
import subprocess

import pytest

import invariant_bi_rmsnorm_03_b200 as bi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "bi.h"

static int fails = 0;
#define EXPECT(cond) do { if (!(cond)) { printf("failed: %s\n", #cond); ++fails; } } while (0)

int main(void)
{
    void *fake = (void *)0x10000;  /* 16-byte aligned, never dereferenced */
    bi_paged_kv kv;
    memset(&kv, 0, sizeof kv);
    kv.k_cache = fake; kv.v_cache = fake; kv.block_table = fake;
    kv.max_pages_per_seq = 4; kv.num_pages = 8; kv.page_size = 8;  /* not 16 */
    kv.num_kv_heads = 2; kv.head_dim = 128;

    EXPECT(bi_build_invariant() == EXPECTED_FLAVOUR);
    EXPECT(strcmp(bi_status_string(BI_OK), "ok") == 0);
    EXPECT(bi_status_string(BI_ERR_TIMEOUT) != NULL);
    EXPECT(bi_rmsnorm(fake, fake, fake, 4, 12, 1e-6f, BI_BF16, NULL) == BI_ERR_INVALID);
    EXPECT(bi_rmsnorm(NULL, NULL, NULL, 0, 64, 1e-6f, BI_BF16, NULL) == BI_OK);
    EXPECT(bi_matmul(fake, fake, fake, 4, 64, 12, BI_BF16, NULL, 0, NULL) == BI_ERR_INVALID);
    EXPECT(bi_kv_write(&kv, fake, fake, (const int64_t *)fake, 4, NULL) == BI_ERR_INVALID);
    EXPECT(bi_rmsnorm_matmul(fake, fake, fake, 4, 64, 64, -1.0f, BI_BF16, fake, 256, NULL) ==
           BI_ERR_INVALID);
    EXPECT(bi_rmsnorm_matmul_workspace_bytes(5) == 256);
    EXPECT(bi_swiglu_backward(fake, fake, fake, 4, 12, BI_BF16, NULL) == BI_ERR_INVALID);
    EXPECT(bi_attention_backward_workspace_bytes(8, 10) == 640);
    EXPECT(bi_transpose(fake, fake, 8, 4, 7, NULL) == BI_ERR_INVALID);
    EXPECT(bi_matmul_backward_workspace_bytes(5, 64, 32) == 4096 + 1024 + 512);
    EXPECT(bi_matmul_workspace_bytes(2048, 4096, 4096) == 0 || !EXPECTED_FLAVOUR);
    printf("%s\n", fails ? "FAIL" : "PASS");
    return fails != 0;
}
"""


@pytest.mark.parametrize("variant", [False, True], ids=["invariant", "variant_off"])
def test_c_program_against_the_library(tmp_path, variant):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    lib = bi.load(variant=variant).path
    src = tmp_path / "caller.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "caller"
    flavour = "0" if variant else "1"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-DEXPECTED_FLAVOUR=" + flavour, "-I", INCLUDE, str(src), lib,
                    "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "PASS" in r.stdout, r.stdout + r.stderr
