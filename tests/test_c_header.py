"""The boundary is a C ABI: include/flexq.h compiles as plain C11 (no C++ and no torch
types in any signature), and a C program linked against libflexq.so calls the library
with no Python in between. The program uses only host-side entry points (size queries,
status strings, struct layouts and argument checks that return before any CUDA call),
so it runs without a GPU."""
import os
import shutil
import subprocess

import pytest

import group_wise_int4_b200 as fq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <stdint.h>
#include "flexq.h"

int main(void) {
    flexq_config cfg = {4, 64, 1, 0};
    int64_t shape[2] = {4096, 4096};
    printf("codes %lld\n", (long long)flexq_codes_bytes(2, shape, cfg));
    printf("meta %lld\n", (long long)flexq_meta_bytes(2, shape, cfg));
    flexq_config bad = {5, 64, 1, 0};
    printf("bad_bits %lld\n", (long long)flexq_codes_bytes(2, shape, bad));
    int64_t small[2] = {4, 128};
    printf("null_input %d\n", flexq_compress(NULL, 2, small, cfg, (void*)4096, (void*)8192, NULL));
    printf("gemm_ws_small %lld\n", (long long)flex_gemm_ws_bytes(1, 256, 256));
    printf("status %s\n", flex_status_string(FLEX_ERR_TIMEOUT));
    printf("sizeof_config %lld %d\n", (long long)flex_abi_layout(0, -1), (int)sizeof(flexq_config));
    printf("sizeof_tensor %lld %d\n", (long long)flex_abi_layout(1, -1), (int)sizeof(flexq_tensor));
    printf("sizeof_layer %lld %d\n", (long long)flex_abi_layout(2, -1), (int)sizeof(flex_layer));
    printf("sizeof_cache %lld %d\n", (long long)flex_abi_layout(3, -1), (int)sizeof(flex_kv_cache));
    return 0;
}
"""


def test_header_compiles_as_c_and_a_c_program_calls_the_library(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = fq.LIB_PATH
    if not os.path.exists(lib):
        pytest.skip("libflexq.so not built")
    src = tmp_path / "use_flexq.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_flexq"
    libdir = os.path.dirname(lib)
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(lib),
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    out = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    assert int(out["codes"]) == 4096 * 4096 // 2
    assert int(out["meta"]) == 4096 * 64 * 4
    assert int(out["bad_bits"]) == fq.FLEX_ERR_UNSUPPORTED
    assert int(out["null_input"]) == fq.FLEX_ERR_INVALID_ARG
    assert int(out["gemm_ws_small"]) >= 0
    assert "timed out" in out["status"]
    for k in ("sizeof_config", "sizeof_tensor", "sizeof_layer", "sizeof_cache"):
        lib_size, c_size = (int(v) for v in out[k].split())
        assert lib_size == c_size, (k, lib_size, c_size)
