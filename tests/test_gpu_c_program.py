"""A plain C host program drives the codec on the GPU through the C ABI alone: it reads a
seeded fp16 tensor from a file, moves it to memory from cudaMalloc, calls flexq_compress
and flexq_decompress, reads the status word with flex_get_status and writes codes,
metadata and the decompressed tensor back to files. The codes, metadata and fp16 output
must equal the oracle's bit for bit (the same check as the Python-driven codec tests),
so the boundary works without torch or the binding."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import group_wise_int4_b200 as fq
import synth
from oracle import codec as oc

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

C_PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <stdint.h>
#include <cuda_runtime.h>
#include "flexq.h"

static void* read_file(const char* path, size_t n) {
    void* p = malloc(n);
    FILE* f = fopen(path, "rb");
    if (!p || !f || fread(p, 1, n, f) != n) { fprintf(stderr, "read %s\n", path); exit(2); }
    fclose(f);
    return p;
}
static void write_file(const char* path, const void* p, size_t n) {
    FILE* f = fopen(path, "wb");
    if (!f || fwrite(p, 1, n, f) != n) { fprintf(stderr, "write %s\n", path); exit(2); }
    fclose(f);
}

int main(int argc, char** argv) {
    if (argc != 5) return 2;
    const int64_t rows = atoll(argv[2]), cols = atoll(argv[3]);
    const char* dir = argv[4];
    int64_t shape[2] = {rows, cols};
    flexq_config cfg = {4, 64, 1, 0};
    const int64_t cb = flexq_codes_bytes(2, shape, cfg), mb = flexq_meta_bytes(2, shape, cfg);
    const size_t xb = (size_t)(rows * cols * 2);
    if (cb <= 0 || mb <= 0) return 3;
    void* hx = read_file(argv[1], xb);
    void *dx, *dc, *dm, *dy;
    if (cudaMalloc(&dx, xb) || cudaMalloc(&dc, (size_t)cb) || cudaMalloc(&dm, (size_t)mb) || cudaMalloc(&dy, xb))
        return 4;
    if (cudaMemcpy(dx, hx, xb, cudaMemcpyHostToDevice)) return 5;
    int rc = flexq_compress(dx, 2, shape, cfg, dc, dm, NULL);
    if (rc != FLEX_OK) { fprintf(stderr, "compress %s\n", flex_status_string(rc)); return 6; }
    rc = flexq_decompress(dc, dm, 2, shape, cfg, dy, NULL);
    if (rc != FLEX_OK) { fprintf(stderr, "decompress %s\n", flex_status_string(rc)); return 7; }
    rc = flex_get_status(NULL);
    if (rc != FLEX_OK) { fprintf(stderr, "status %s\n", flex_status_string(rc)); return 8; }
    void* hc = malloc((size_t)cb); void* hm = malloc((size_t)mb); void* hy = malloc(xb);
    if (cudaMemcpy(hc, dc, (size_t)cb, cudaMemcpyDeviceToHost) || cudaMemcpy(hm, dm, (size_t)mb, cudaMemcpyDeviceToHost) ||
        cudaMemcpy(hy, dy, xb, cudaMemcpyDeviceToHost))
        return 9;
    char path[4096];
    snprintf(path, sizeof path, "%s/codes.bin", dir); write_file(path, hc, (size_t)cb);
    snprintf(path, sizeof path, "%s/meta.bin", dir); write_file(path, hm, (size_t)mb);
    snprintf(path, sizeof path, "%s/y.bin", dir); write_file(path, hy, xb);
    cudaFree(dx); cudaFree(dc); cudaFree(dm); cudaFree(dy);
    free(hx); free(hc); free(hm); free(hy);
    printf("ok\n");
    return 0;
}
"""


def test_c_program_codec_round_trip_bit_exact(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None or not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")):
        pytest.skip("no C compiler or CUDA headers")
    lib = fq.LIB_PATH
    libdir = os.path.dirname(lib)
    src = tmp_path / "codec.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "codec"
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(CUDA, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir,
                        "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    rows, cols = 96, 1088                      # several groups per row and a ragged row count
    x = synth.codec_tensor((rows, cols), 1, 64, 77).numpy()
    xin = tmp_path / "x.bin"
    xin.write_bytes(np.ascontiguousarray(x).tobytes())
    r = subprocess.run([str(exe), str(xin), str(rows), str(cols), str(tmp_path)], capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
    rc, rm = oc.compress(x, 4, 64, 1)
    codes = np.frombuffer((tmp_path / "codes.bin").read_bytes(), dtype=np.uint8).reshape(rc.shape)
    meta = np.frombuffer((tmp_path / "meta.bin").read_bytes(), dtype=np.uint16).reshape(rm.shape)
    y = np.frombuffer((tmp_path / "y.bin").read_bytes(), dtype=np.uint16).reshape(x.shape)
    assert np.array_equal(codes, rc), "codes differ from the oracle"
    assert np.array_equal(meta, rm.view(np.uint16)), "metadata differs from the oracle"
    assert np.array_equal(y, oc.decompress(rc, rm, x.shape, 4, 64, 1).view(np.uint16)), "decompressed values differ"
