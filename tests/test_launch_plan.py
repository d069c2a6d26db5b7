"""Host logic of the attention launch (CPU): the slice grouping of causal
grids, compiled from the library's own header with the host compiler and
checked against a brute-force search."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_attention_sub_b200", "csrc")
CUDA_INC = "/usr/local/cuda/include"

DRIVER = r"""
#include <cstdio>
#include "sage_internal.h"
int main() {
  int bh; double bytes, budget;
  while (std::scanf("%d %lf %lf", &bh, &bytes, &budget) == 3)
    std::printf("%d\n", sage::causal_slice_group(bh, bytes, budget));
  return 0;
}
"""

CASES = [(1, 1e6, 80e6), (32, 2097152.0, 80e6), (128, 2097152.0, 80e6), (128, 8388608.0, 80e6),
         (128, 524288.0, 80e6), (12, 25e6, 80e6), (7, 1e9, 80e6), (97, 1e5, 80e6), (36, 3e6, 50e6),
         (65535, 100.0, 80e6)]


def brute(bh, nbytes, budget):
    ok = [g for g in range(1, bh + 1) if bh % g == 0 and g * nbytes <= budget]
    return max(ok) if ok else 1


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    if shutil.which("g++") is None or not os.path.isdir(CUDA_INC):
        pytest.skip("host compiler or CUDA headers missing")
    d = tmp_path_factory.mktemp("plan")
    src, exe = d / "plan.cpp", d / "plan"
    src.write_text(DRIVER)
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-I", CUDA_INC, str(src), "-o", str(exe)], check=True)
    return str(exe)


def test_causal_slice_group_is_the_largest_fitting_divisor(driver):
    stdin = "".join("%d %r %r\n" % c for c in CASES)
    out = subprocess.run([driver], input=stdin, capture_output=True, text=True, check=True).stdout.split()
    got = [int(x) for x in out]
    for (bh, nbytes, budget), g in zip(CASES, got):
        assert bh % g == 0 and g >= 1, (bh, g)
        assert g == brute(bh, nbytes, budget), (bh, nbytes, budget, g)
        # the whole group's K and V codes fit the budget unless one slice alone exceeds it
        assert g * nbytes <= budget or g == 1
