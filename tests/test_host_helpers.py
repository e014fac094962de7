"""Host-side helpers of the CUDA library, compiled into a small host program
(no GPU call) and checked against the properties their comments state.

probe_stride (csrc/work_items.cuh) picks which work items the sampled probe
covers: every stride-th item.  It must be prime and not 37, so that the
sampled items fall on every CTA of a persistent grid of 148 (items b, b + 148,
... go to CTA b), and it must keep the sample near 256 items once a chunk has
more than 7 * 256 items."""
import math
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "exact_certified_top_b200", "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

PROGRAM = r"""
#include <cstdio>
#include "work_items.cuh"
int main() {
  for (int n = 1; n <= 40000; ++n) std::printf("%d %d\n", n, dosa::probe_stride(n));
  return 0;
}
"""


@pytest.fixture(scope="module")
def strides(tmp_path_factory):
    if not (os.path.exists(NVCC) or shutil.which("nvcc")):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("host_helpers")
    src, exe = d / "probe_stride.cu", d / "probe_stride"
    src.write_text(PROGRAM)
    r = subprocess.run([NVCC, "-O1", "-std=c++17", "-Wno-deprecated-gpu-targets", "-I", CSRC, "-I", INCLUDE, str(src),
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    return {int(a): int(b) for a, b in (line.split() for line in out.split("\n") if line)}


def _is_prime(p):
    return p > 1 and all(p % i for i in range(2, int(math.isqrt(p)) + 1))


def test_stride_is_prime_and_coprime_to_the_persistent_grid(strides):
    for n, s in strides.items():
        assert _is_prime(s) and s != 37 and math.gcd(s, 148) == 1, (n, s)


def test_sampled_items_reach_every_cta_of_a_148_grid(strides):
    # a chunk of 148 * s items or more puts a sampled item on every CTA
    for n in (148 * 7, 26214, 40000):
        s = strides[n]
        hit = {i % 148 for i in range(0, n, s)}
        if n >= 148 * s:
            assert len(hit) == 148, (n, s, len(hit))


def test_stride_keeps_the_sample_near_256_items(strides):
    for n, s in strides.items():
        assert s >= 7
        if n <= 7 * 256:
            assert s == 7, (n, s)
        want = -(-n // 256)
        if want <= 113:
            # the smallest admissible prime at or above the wanted stride
            assert s >= want, (n, s)
            assert not any(_is_prime(p) and p != 37 and p >= 7 for p in range(want, s)), (n, s)
            sample = -(-n // s)
            assert sample <= 256, (n, s)
            if n > 7 * 256:
                assert sample >= 128, (n, s)


def test_headline_chunk_samples_every_13th_item(strides):
    # 26,214-row chunks of 8-query items hold 3,277 items: the stride is 13
    items = -(-26214 // 8)
    assert strides[items] == 13
    assert 240 <= -(-items // 13) <= 256
