"""The boundary is a C ABI: a plain C program (gcc, no C++) includes
include/nvfp4w4a4.h, links libnvfp4w4a4.so and calls the entry points that
need no GPU -- size helpers, status strings, argument validation and the
launch-plan diagnostic -- and gets the documented results."""
import os
import subprocess

import pytest

from nvfp4_w4a4_quantized_06_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "nvfp4w4a4.h"

int main(void) {
    int out[8];
    if (nvfp4_codes_bytes(64, 256) != 64 * 128) return 1;
    if (nvfp4_sf_bytes(129, 5120) != 256 * 320) return 2;
    if (strncmp(nvfp4_status_string(NVFP4_ERR_SHAPE), "", 1) == 0) return 3;
    /* K % 64 != 0 is refused before anything touches a device */
    if (nvfp4_quantize((const void *)16, NVFP4_IN_BF16, 4, 100, 100, (const float *)16, (uint8_t *)16,
                       (uint8_t *)16, 0, 4, NULL) != NVFP4_ERR_SHAPE) return 4;
    if (nvfp4_plan_for(32, 5120, 5120, 148, 74, NULL, out) != NVFP4_OK) return 5;
    if (out[0] != 0 || out[1] != 32 || out[2] != 1) return 6;      /* single-CTA kernel, MMA N 32, swapped */
    if (nvfp4_plan_for(32768, 34816, 5120, 148, 74, NULL, out) != NVFP4_OK || out[0] != 1) return 7;
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_program_uses_the_library(work_dir):
    lib = build.build()
    src = os.path.join(work_dir, "consumer.c")
    exe = os.path.join(work_dir, "consumer")
    with open(src, "w") as f:
        f.write(PROGRAM)
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe,
           "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
