"""The boundary is a plain C ABI: include/eaga.h compiles as C99 with gcc
(no CUDA or torch headers), and a C program linked against libeaga.so calls
the host-only entry points (sizes, dispatch, error strings) without a GPU."""
import os
import subprocess

import pytest

from edge_aware_graph_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include "eaga.h"

int main(void) {
    eaga_dims d = {32, 192, 256, 64, 64, 8, 32, EAGA_BF16};
    size_t wf = eaga_workspace_size(&d, 0), wb = eaga_workspace_size(&d, 1), sv = eaga_saved_size(&d);
    int lf = eaga_kernel_launches(&d, 0), lb = eaga_kernel_launches(&d, 1);
    eaga_dims bad = d;
    bad.n = 4096;
    eaga_status s = eaga_forward(&bad, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0);
    printf("%zu %zu %zu %d %d %d %s\n", wf, wb, sv, lf, lb, (int)s, eaga_strerror(EAGA_ERR_TIMEOUT));
    return 0;
}
"""


def test_header_is_c99_and_host_calls_work(tmp_path):
    lib = B.build()
    src = tmp_path / "use_eaga.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_eaga"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", os.path.dirname(lib), "-leaga", "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    wf, wb, sv, lf, lb, s, msg = r.stdout.split(maxsplit=6)
    assert int(wf) > 0 and int(wb) > int(wf) and int(sv) > 0
    assert (int(lf), int(lb)) == (5, 12)              # the tcgen05 path for these dims
    assert int(s) == 2                                # n beyond the limits: EAGA_ERR_UNSUPPORTED, nothing launched
    assert msg.strip()
