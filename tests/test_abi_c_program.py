"""The C ABI from C: include/qsa.h compiles as C99 with warnings as errors,
and a C program links against libqsa.so and gets host-side validation
results on a machine without a GPU (no compute runs here)."""
import os
import shutil
import subprocess

import pytest

from sparse_attention_block_qsa_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "qsa.h"

int main(void) {
    /* fake device addresses: validation never dereferences them */
    const uintptr_t A = (uintptr_t)0x7f0000000000ull, S = (uintptr_t)1 << 28;
    const void *q = (const void *)A, *k = (const void *)(A + S);
    const int32_t *pt = (const int32_t *)(A + 2 * S), *sl = (const int32_t *)(A + 3 * S);
    float *out = (float *)(A + 4 * S);
    int fails = 0;
    /* an empty batch is a no-op that succeeds */
    if (qsa_mqa_decode(q, 2048, 512, 128, k, 100, 64, 64 * 128, 128, pt, 10, 10, sl, 0, 4, 0.088f,
                       out, 4000, 1000, 1000, NULL) != QSA_OK) fails |= 1;
    /* an unsupported query count and page size are rejected with a reason */
    if (qsa_mqa_decode(q, 2048, 512, 128, k, 100, 64, 64 * 128, 128, pt, 10, 10, sl, 4, 5, 0.088f,
                       out, 4000, 1000, 1000, NULL) != QSA_ERR_UNSUPPORTED) fails |= 2;
    if (strlen(qsa_last_error_detail()) == 0) fails |= 4;
    /* the fp8 entry rejects a non-positive dequantisation scale */
    if (qsa_mqa_decode_fp8(q, 2048, 512, 128, k, 0.0f, 100, 64, 64 * 128, 128, pt, 10, 10, sl, 4, 4,
                           0.088f, out, 4000, 1000, 1000, NULL) != QSA_ERR_INVALID_ARG) fails |= 8;
    /* a misaligned prefill query is an alignment error */
    if (qsa_mqa_prefill((const void *)(A + 2), 512, 128, k, 128, 1000, pt, sl, 100, 0.088f, out, 1000,
                        1000, NULL) != QSA_ERR_ALIGNMENT) fails |= 16;
    if (qsa_prefill_topk_workspace_size(64, 1000) < (size_t)64 * 1000 * 4) fails |= 32;
    printf("%s %d\n", qsa_status_string(QSA_ERR_ALIGNMENT), fails);
    return fails;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(tmp_path):
    src = tmp_path / "abi_check.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(_abi.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:libqsa.so", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.split()[-1] == "0"
