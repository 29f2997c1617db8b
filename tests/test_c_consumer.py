"""The C ABI from plain C: include/grinqh.h compiles as strict C99 (gcc -pedantic,
warnings as errors), a C program links libgrinqh.so and calls the host-only entry
points (layout, status strings, maximum-entropy distribution, table construction),
and its results agree with the oracle's. No GPU is touched."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from activation_graded_bit_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "activation_graded_bit_b200")

C_SRC = r"""
#include <stdio.h>
#include <stdlib.h>
#include "grinqh.h"

int main(int argc, char** argv) {
  grinqh_layout L, L6;
  if (argc != 5) return 1;
  if (grinqh_layout_init(4096, 14336, &L) != GRINQH_OK) return 2;
  if (grinqh_layout_init_bmax(4096, 14336, 6, &L6) != GRINQH_OK) return 3;
  if (grinqh_layout_init_bmax(4096, 14336, 5, &L6) != GRINQH_ERR_INVALID_ARG) return 4;
  printf("layout %d %d %d %d %d %lld\n", L.K, L.N, L.n_groups, L.n_tiles, L.record_bytes, (long long)L.packed_bytes);
  size_t lb = 0;
  if (grinqh_lut_bytes(&L, &lb) != GRINQH_OK) return 5;
  printf("lut_bytes %zu\n", lb);
  printf("status %s|%s\n", grinqh_status_string(GRINQH_OK), grinqh_status_string(GRINQH_ERR_WORKSPACE));
  const uint8_t classes[5] = {0, 2, 3, 4, 8};
  double P[5];
  if (grinqh_maxent_distribution(classes, 5, 3.0, P) != GRINQH_OK) return 6;
  printf("maxent %.17g %.17g %.17g %.17g %.17g\n", P[0], P[1], P[2], P[3], P[4]);
  /* table construction of the weights in argv[1] (K x N float32, raw) */
  int K = atoi(argv[2]), N = atoi(argv[3]);
  float* W = malloc(sizeof(float) * (size_t)K * N);
  uint8_t* q = malloc((size_t)K * N);
  uint16_t* lut = malloc(sizeof(uint16_t) * (size_t)K * 512);
  FILE* f = fopen(argv[1], "rb");
  if (!f || fread(W, sizeof(float), (size_t)K * N, f) != (size_t)K * N) return 7;
  fclose(f);
  if (grinqh_lut_build(W, K, N, 8, q, lut) != GRINQH_OK) return 8;
  f = fopen(argv[4], "wb");
  fwrite(q, 1, (size_t)K * N, f);
  fwrite(lut, sizeof(uint16_t), (size_t)K * 512, f);
  fclose(f);
  free(W); free(q); free(lut);
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib():
    from activation_graded_bit_b200 import build
    return build.build()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_uses_the_abi(lib, orc, tmp_path):
    src = tmp_path / "consumer.c"
    src.write_text(C_SRC)
    exe = tmp_path / "consumer"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), str(src), "-L", PKG, "-lgrinqh",
                           "-Wl,-rpath," + PKG, "-o", str(exe)])
    K, N = 6, 700
    W = wl.weights_gaussian(K, N, key=(701,))
    wpath, opath = tmp_path / "w.bin", tmp_path / "out.bin"
    W.tofile(wpath)
    out = subprocess.run([str(exe), str(wpath), str(K), str(N), str(opath)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    lines = dict(l.split(" ", 1) for l in out.stdout.strip().splitlines())
    assert lines["layout"].split() == ["4096", "14336", "112", "14", "1024", str(4096 * 14 * (1024 + 32))]
    assert int(lines["lut_bytes"]) == 4096 * 1024
    assert lines["status"] == "ok|workspace missing or too small"
    P = np.array([float(v) for v in lines["maxent"].split()])
    assert np.allclose(P, orc.maxent_distribution(np.array([0, 2, 3, 4, 8], np.uint8), 3.0), rtol=0, atol=1e-12)
    raw = np.fromfile(opath, np.uint8)
    q = raw[:K * N].reshape(K, N)
    lut = raw[K * N:].view(np.uint16).reshape(K, 512)
    q_ref, lut_ref, _ = orc.lut_build(W, 8)
    assert np.array_equal(q, q_ref) and np.array_equal(lut, lut_ref)
