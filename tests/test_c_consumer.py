"""The boundary from plain C: a C99 program that includes include/moda.h, links against
libmoda_b200.so and calls the host-side entry points, with no Python or torch in between.

It compiles with -std=c99 -pedantic -Werror, so the header is valid C. It checks the
workspace sizes, the status strings, and that bad arguments are refused before any device
work. Those calls touch no GPU, so the program runs here as it would on a B200.
"""
import os
import shutil
import subprocess

import pytest

import depth_aware_attention_b200 as moda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moda.h"

static int fails = 0;
#define EXPECT(c) do { if (!(c)) { printf("FAILED line %d: %s\n", __LINE__, #c); ++fails; } } while (0)

int main(void) {
    /* workspace sizes: defined for valid sizes, 0 for invalid ones */
    size_t ws = moda_backward_workspace_size(1, 8, 2, 1000, 6, 128);
    EXPECT(ws >= (size_t)1 * 8 * 1000 * 128 * 4);     /* holds the fp32 dq accumulator */
    EXPECT(moda_backward_workspace_size(1, 8, 3, 1000, 6, 128) == 0);  /* Hq % Hkv != 0 */
    EXPECT(moda_decode_workspace_size(2, 8, 2, 300, 5, 128) > 0);
    EXPECT(moda_decode_workspace_size(2, 8, 2, 300, 5, 96) == 0);     /* d not supported */

    /* status strings and the last message */
    EXPECT(strcmp(moda_status_string(MODA_OK), "success") == 0);
    EXPECT(strlen(moda_status_string(MODA_ERR_TIMEOUT)) > 0);

    /* argument checks run before any device work */
    float *lse = NULL;
    moda_status_t s = moda_forward(NULL, NULL, NULL, NULL, NULL, NULL, lse, 1, 8, 2, 64, 4,
                                   128, 0.088f, 1, NULL);
    EXPECT(s == MODA_ERR_INVALID_ARGUMENT);
    EXPECT(strlen(moda_last_error_message()) > 0);
    s = moda_forward((void *)16, (void *)32, (void *)48, NULL, NULL, (void *)64, (float *)80,
                     1, 8, 2, 64, 0, 96, 0.1f, 1, NULL);
    EXPECT(s == MODA_ERR_UNSUPPORTED);                              /* d = 96 */
    s = moda_backward_stages(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                             NULL, NULL, NULL, 0, 1, 8, 2, 64, 4, 128, 0.1f, 1, 8u, NULL);
    EXPECT(s == MODA_ERR_INVALID_ARGUMENT);                         /* stage bit 8 */
    s = moda_depth_kv_write(NULL, NULL, NULL, NULL, 1, 64, 256, 2, 128, 4, 4, NULL);
    EXPECT(s == MODA_ERR_INVALID_ARGUMENT);                         /* slot == L */

    printf("%s\n", fails ? "C consumer: FAILED" : "C consumer: ok");
    return fails ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_uses_the_boundary(tmp_path):
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(moda.LIB_PATH)
    cc = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
          "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
          "-L", libdir, "-l:" + os.path.basename(moda.LIB_PATH), "-Wl,-rpath," + libdir]
    r = subprocess.run(cc, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "C consumer: ok" in r.stdout
