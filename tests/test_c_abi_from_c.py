"""The C ABI used from plain C99, on the CPU: a small program written here includes
include/dynconv.h, links libdynconv.so and calls the host-only entry points
(version, workspace sizing, kernel-family query, status strings, the validation
of a bad descriptor).  Nothing is launched: there is no GPU here."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "dynamic_short_convolutions_b200")
LIB = os.path.join(PKG, "libdynconv.so")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "dynconv.h"

int main(void) {
    dynconv_desc d;
    memset(&d, 0, sizeof d);
    d.kind = DYNCONV_LOWRANK;
    d.dtype = DYNCONV_BF16;
    d.batch = 8;
    d.seqlen = 2048;
    d.d_model = 768;
    d.channels = 2304;
    d.ksize = 3;
    d.rank = 32;
    d.algo = DYNCONV_ALGO_AUTO;
    d.layout = DYNCONV_TOKEN_MAJOR;
    printf("version %d\n", (int)dynconv_version());
    size_t ws = dynconv_workspace_bytes(&d);
    printf("workspace %zu\n", ws);
    int32_t f = 0, b = 0;
    dynconv_status s = dynconv_query_family(&d, &f, &b);
    printf("query %s %d %d\n", dynconv_status_string(s), (int)f, (int)b);
    d.ksize = 0;                                   /* invalid: validated before any launch */
    printf("bad_workspace %zu\n", dynconv_workspace_bytes(&d));
    s = dynconv_query_family(&d, &f, &b);
    printf("bad_query %s [%s]\n", dynconv_status_string(s), dynconv_last_error());
    s = dynconv_fwd(&d, 0, 0, 0, 0, 0, 0, 0, 0, 0);
    printf("bad_fwd %s\n", dynconv_status_string(s));
    return 0;
}
"""


def test_c_program_uses_the_library(tmp_path):
    if not os.path.exists(LIB):
        pytest.skip("library not built")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), "-L", PKG, "-ldynconv", f"-Wl,-rpath,{PKG}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60, check=True).stdout
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(lines["version"]) > 0
    assert int(lines["workspace"]) > 0
    status, fwd, bwd = lines["query"].split()
    assert status == "DYNCONV_OK" and int(fwd) in (1, 2) and int(bwd) in (1, 2)
    assert lines["bad_workspace"] == "0"
    assert lines["bad_query"].startswith("DYNCONV_ERR_INVALID [") and "ksize" in lines["bad_query"]
    assert lines["bad_fwd"] == "DYNCONV_ERR_INVALID"
