"""The boundary is a C ABI: a plain C99 program includes include/osc.h, links libosc.so and
calls the host-only entry points (sizes, table width, grouped plan, tier rule, argument
checks). No device is touched, so this runs on the CPU."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "osc.h"

int main(void) {
  int fails = 0;
#define CHECK(c) do { if (!(c)) { printf("failed: %s\n", #c); ++fails; } } while (0)
  CHECK(strstr(osc_version(), "sm_100a") != NULL);
  CHECK(osc_scale_bytes(2048, 4096, 32) == (size_t)16 * 32 * 512);
  CHECK(osc_scale_bytes(1, 4096, 0) == (size_t)32 * 512);
  CHECK(osc_scale_bytes(16, 256, 24) == 0);
  int8_t L[8] = {-1, 5, 0, -1, 31, -1, -1, 9};
  CHECK(osc_table_kl(L, 8) == 16);
  int counts[3] = {130, 0, 1}, off[4], poff[4], mbe[3];
  CHECK(osc_grouped_plan(counts, 3, off, poff, NULL, 0) == 384);
  CHECK(osc_grouped_plan(counts, 3, off, poff, mbe, 3) == 384);
  CHECK(off[3] == 131 && poff[1] == 256 && mbe[0] == 0 && mbe[1] == 0 && mbe[2] == 2);
  int hit[2] = {3, 1}, tot[2] = {5, 4};
  double c = 0.0;
  CHECK(osc_select_tier(hit, tot, 2, &c) == OSC_TIER_MID && fabs(c - 0.425) < 1e-12);
  CHECK(osc_quantize(NULL, 4, 256, 24, NULL, 1, 0, NULL, NULL, NULL, NULL) == OSC_ERR_G);
  CHECK(osc_set_tile_n(96) == OSC_ERR_ARG);
  CHECK(strcmp(osc_error_string(OSC_ERR_TABLE), "table entry out of range or more entries than K_L") == 0);
  printf("%s\n", fails ? "C consumer: FAILED" : "C consumer: ok");
  return fails != 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    from w4a4_outlier_separated_b200 import build
    return os.path.dirname(build.build())


def test_header_compiles_as_c99_and_links(libdir, tmp_path):
    src = tmp_path / "consumer.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-losc", "-lm", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "C consumer: ok" in r.stdout
