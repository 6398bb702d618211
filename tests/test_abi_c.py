"""The boundary from C itself: include/bq.h compiles as strict C99, and a
plain C program links against libbq.so and calls the host-only entry points
(no GPU needed)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "dequantize_absmax_reduce_b200")

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "bq.h"

int main(void) {
    int32_t lo = 0, hi = 0;
    if (bq_default_q_range(BQ_S8, &lo, &hi) != BQ_OK || lo != -128 || hi != 127) return 1;
    if (bq_default_q_range(BQ_U4X2, &lo, &hi) != BQ_OK || lo != 0 || hi != 15) return 2;
    if (bq_packed_transpose_stride(4097, 16) != 4112) return 3;
    if (strcmp(bq_granularity_name(BQ_GRAN_CHANNEL), "channel") != 0) return 4;
    if (strcmp(bq_status_string(BQ_OK), "ok") != 0) return 5;
    if (bq_diag_wait_timeout(0, NULL) != BQ_ERR_INVALID_ARG) return 6;
    puts("c abi ok");
    return 0;
}
"""


def test_header_is_strict_c99():
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-x", "c", os.path.join(ROOT, "include", "bq.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_links_and_calls_host_entry_points(tmp_path):
    src, exe = tmp_path / "abi.c", tmp_path / "abi"
    src.write_text(PROGRAM)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", PKG, "-lbq", f"-Wl,-rpath,{PKG}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "c abi ok", (run.returncode, run.stderr)
