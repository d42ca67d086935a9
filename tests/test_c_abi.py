"""The boundary is a plain C ABI: include/ratp.h compiles as C99 and a C
program links against libratp.so and calls it (host-only entry points, so
this runs without a GPU)."""
import os
import subprocess

from recurrence_augmented_dilated_chunked_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "ratp.h"

int main(void) {
  size_t ws = 0, ring = 0;
  ratp_cache c;
  int line = -1;
  memset(&c, 0, sizeof(c));
  if (ratp_scan_workspace_bytes(2, 1000, 2, 64, RATP_BF16, &ws) != RATP_OK) return 1;
  if (ratp_cache_window_bytes(2, 3, 128, 64, &ring) != RATP_OK) return 2;
  if (ratp_cache_set_chunk_local(&c, 16) != RATP_OK || c.reset_L != 16) return 3;
  if (ratp_scan_prefill_kv_window(0, 0, 0, 0, 0, 1, 8, 1, 64, RATP_BF16, 48, 0) != RATP_ERR_UNSUPPORTED) return 4;
  if (ratp_guard_line(&line) != RATP_ERR_UNSUPPORTED || line != 0) return 5;
  printf("%s|%zu|%zu\n", ratp_status_string(RATP_ERR_ALIGN), ws, ring);
  return 0;
}
"""


def test_header_is_c99_and_library_links_from_c(tmp_path):
    lib = B.build_library()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), "-L", libdir, "-l:libratp.so",
                           "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    msg, ws, ring = out.stdout.strip().split("|")
    assert "aligned" in msg
    assert int(ws) > 256 and int(ring) == 3 * 2 * 3 * 64 * 128 * 2
