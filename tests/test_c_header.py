"""The boundary from C: include/tk_route.h compiles as strict C99 and as C++17, and a C program
links against libtk_route.so and makes host-only calls (sizes, strings, argument rejections that
return before anything touches a GPU). No GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "token_routing_gate_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "tk_route.h"

int main(void) {
    int fake = 0;
    tk_status st;
    printf("abi %d\n", tk_abi_version());
    printf("max_rows %lld\n", (long long)tk_max_rows(8192, 256, 8, 128));
    printf("ok_str %s\n", tk_status_str(TK_OK));
    /* logits NULL with T > 0: rejected on the host */
    st = tk_gate_topk(NULL, NULL, 4, 16, 2, TK_SCORE_SOFTMAX, 1, (int32_t*)&fake, (float*)&fake, NULL);
    printf("gate %d %s\n", (int)st, strstr(tk_last_error_detail(), "NULL") ? "detail" : "nodetail");
    /* k = 0: rejected on the host */
    st = tk_reduce(&fake, 1, (const int32_t*)&fake, NULL, 4, 0, 256, &fake, NULL, NULL);
    printf("reduce %d %s\n", (int)st, strstr(tk_last_error_detail(), "k=0") ? "detail" : "nodetail");
    /* softmax with a selection bias: rejected */
    st = tk_gate_topk((const float*)&fake, (const float*)&fake, 4, 16, 2, TK_SCORE_SOFTMAX, 1,
                      (int32_t*)&fake, (float*)&fake, NULL);
    printf("bias %d\n", (int)st);
    return 0;
}
"""


@pytest.fixture(scope="module")
def lib():
    from token_routing_gate_b200 import build

    return build.build()


def test_header_is_strict_c99_and_cxx17(tmp_path, lib):
    if shutil.which("gcc") is None or shutil.which("g++") is None:
        pytest.skip("no host compiler")
    probe = tmp_path / "probe.c"
    probe.write_text('#include "tk_route.h"\nint tk_probe(void) { return TK_OK; }\n')
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        lang = ["-x", "c++"] if cc == "g++" else []
        r = subprocess.run([cc, std, *lang, "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                            "-I", INCLUDE, str(probe)], capture_output=True, text=True)
        assert r.returncode == 0, (cc, r.stderr)


def test_c_program_links_and_calls_the_library(tmp_path, lib):
    if shutil.which("gcc") is None:
        pytest.skip("no host compiler")
    src = tmp_path / "prog.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "prog"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE,
                        str(src), "-L", PKG, "-ltk_route", f"-Wl,-rpath,{PKG}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    out = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    assert int(out["abi"]) >> 16 == 1
    assert int(out["max_rows"]) == 8192 * 8 + 256 * 127
    assert out["ok_str"] == "TK_OK"
    assert out["gate"] == "1 detail"          # TK_ERR_INVALID_ARG with a detail naming the NULL
    assert out["reduce"] == "1 detail"
    assert out["bias"] == "1"
