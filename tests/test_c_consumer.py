"""The boundary is a C ABI: a plain C99 program (no CUDA headers, no torch) can
include awq_b200.h, link libawq_b200.so and call it.

Only calls that need no device are made here: the version and status strings,
the workspace sizes, and calls whose arguments are refused on the host before
anything is launched (the pointers are never dereferenced).  The header must
also compile as C++, where its declarations keep C linkage.
"""
import os
import shutil
import subprocess

import pytest

import weight_only_quantization_quantize_b200 as awq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.dirname(awq.LIB_PATH)

C_PROGRAM = r"""
#include <stdio.h>
#include "awq_b200.h"

int main(void)
{
    const uint16_t *h = (const uint16_t *)(uintptr_t)0x7f0000000000ull;  /* never dereferenced */
    const int32_t *q = (const int32_t *)(uintptr_t)0x7f0000000000ull;
    uint16_t *y = (uint16_t *)(uintptr_t)0x7f0000000000ull;
    printf("version %d\n", awq_abi_version());
    printf("status %s\n", awq_status_string(AWQ_ERR_SHAPE));
    printf("ws_gemv %zu\n", awq_w4a16_gemv_workspace_size(4096, 4096));
    printf("ws_gemm %zu\n", awq_w4a16_gemm_workspace_size(4096, 4096, 6144));
    printf("ws_bad %zu\n", awq_w4a16_gemm_workspace_size(4, 100, 4096));
    /* K not a multiple of 128, a NULL output, a missing workspace */
    printf("shape %d\n", (int)awq_w4a16_gemm(h, h, q, h, q, 4, 100, 4096, y, (void *)y, 1u << 20, NULL, NULL));
    printf("null %d\n", (int)awq_w4a16_gemm(h, h, q, h, q, 4, 4096, 4096, NULL, (void *)y, 1u << 20, NULL, NULL));
    printf("workspace %d\n", (int)awq_w4a16_gemm(h, h, q, h, q, 4, 4096, 4096, y, NULL, 0, NULL, NULL));
    printf("noalloc %d\n", (int)awq_w4a16_gemm_noalloc(h, h, q, h, q, 4096, 4096, 4096, y, NULL, NULL));
    return 0;
}
"""


def _compiler(name):
    path = shutil.which(name)
    if path is None:
        pytest.skip(f"{name} is not installed")
    return path


def test_plain_c_program_links_and_calls_the_library(tmp_path):
    from weight_only_quantization_quantize_b200 import _build
    _build.build()  # in-tree, if it is not built yet
    src = tmp_path / "consumer.c"
    exe = tmp_path / "consumer"
    src.write_text(C_PROGRAM)
    subprocess.run([_compiler("gcc"), "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", INCLUDE, str(src), "-o", str(exe), "-L", PKG, "-lawq_b200",
                    f"-Wl,-rpath,{PKG}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(got["version"]) == awq.ABI_VERSION
    assert got["status"].startswith("AWQ_ERR_SHAPE")
    assert int(got["ws_gemv"]) == awq.lib().awq_w4a16_gemv_workspace_size(4096, 4096) > 0
    assert int(got["ws_gemm"]) == awq.lib().awq_w4a16_gemm_workspace_size(4096, 4096, 6144) > 0
    assert int(got["ws_bad"]) == 0
    assert int(got["shape"]) == awq.ERR_SHAPE
    assert int(got["null"]) == awq.ERR_NULL
    assert int(got["workspace"]) == awq.ERR_WORKSPACE
    assert int(got["noalloc"]) == awq.ERR_WORKSPACE


def test_header_compiles_as_cplusplus_with_c_linkage(tmp_path):
    src = tmp_path / "consumer.cpp"
    src.write_text('#include "awq_b200.h"\n'
                   'extern "C" int awq_abi_version(void);\n'   # redeclaration must agree in linkage
                   'int main() { return awq_abi_version() < 0; }\n')
    subprocess.run([_compiler("g++"), "-std=c++17", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-fsyntax-only", "-I", INCLUDE, str(src)], check=True)
