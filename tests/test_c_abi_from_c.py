"""The boundary is a C ABI: a C99 program that includes include/osdn.h compiles with gcc under
-std=c99 -pedantic -Wall -Werror, links against libosdn.so and calls the library without a GPU
(the version, every status string, the workspace sizes and an argument error that is reported
before anything reaches CUDA).  Its answers equal the Python binding's."""
import os
import shutil
import subprocess

import pytest

osdn = pytest.importorskip("delta_rule_recurrent_osdn_b200.osdn")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "delta_rule_recurrent_osdn_b200")

PROGRAM = r"""
#include <stdio.h>
#include "osdn.h"

int main(void) {
    int s;
    size_t ws;
    osdn_status_t bad;
    printf("abi %d\n", (int)osdn_abi_version());
    for (s = 0; s <= 6; ++s) printf("status %d %s\n", s, osdn_status_string((osdn_status_t)s));
    ws = osdn_fwd_workspace_bytes(4, 4096, 16, 128, OSDN_BF16);
    printf("fwd_ws %lu\n", (unsigned long)ws);
    ws = osdn_bwd_workspace_bytes(0, 4, 4096, 16, 128, 128, OSDN_BF16);
    printf("bwd_ws %lu\n", (unsigned long)ws);
    /* an unsupported head size: rejected on the host, nothing is enqueued */
    bad = osdn_chunk_fwd((const void*)0x10000000, (const void*)0x11000000, (const void*)0x12000000,
                         (const void*)0x13000000, (const float*)0x14000000, NULL, 0, 1.0f, NULL,
                         (void*)0x15000000, NULL, NULL, 0, 1, 8, 1, 96, 128, 64, OSDN_BF16, NULL);
    printf("bad %d\n", (int)bad);
    return 0;
}
"""


def test_c_program_links_and_agrees_with_the_binding(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc is not installed")
    src = tmp_path / "use_osdn.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_osdn"
    cmd = [gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", PKG, "-losdn", f"-Wl,-rpath,{PKG}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines() if not line.startswith("status"))
    assert int(lines["abi"]) == osdn.LIB.osdn_abi_version()
    status = [line.split(" ", 2)[2] for line in out.splitlines() if line.startswith("status")]
    assert status == [osdn.status_string(s) for s in range(7)]
    assert int(lines["fwd_ws"]) == osdn.osdn_fwd_workspace_bytes(4, 4096, 16, 128)
    assert int(lines["bwd_ws"]) == osdn.LIB.osdn_bwd_workspace_bytes(0, 4, 4096, 16, 128, 128,
                                                                    osdn.OSDN_BF16) > 0
    assert int(lines["bad"]) == osdn.OSDN_ERR_UNSUPPORTED
