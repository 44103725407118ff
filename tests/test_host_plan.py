"""Host-side launch planning (vq_compressed_linear_b200/csrc/hxq_plan.h) on
the CPU: the grouped GEMV's stream-K shares, compiled with the host C++
compiler and checked over many random groups.

For a group of layers with W[i] stages each and a grid of G CTAs
(n <= G <= sum W), every layer must get at least one CTA and no more CTAs
than stages (each CTA needs a stage), the shares must add up to G exactly,
and each share must stay within n CTAs of the proportional G W[i] / sum W.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vq_compressed_linear_b200", "csrc")

DRIVER = r"""
#include <cstdio>
#include <cstdlib>
#include "hxq_plan.h"
int main() {
  long long W[4];
  int n, G, Gl[4];
  while (scanf("%d %d", &n, &G) == 2) {
    for (int i = 0; i < n; ++i) scanf("%lld", &W[i]);
    int64_t W64[4];
    for (int i = 0; i < n; ++i) W64[i] = W[i];
    hxq::group_shares(W64, n, G, Gl);
    for (int i = 0; i < n; ++i) printf("%d ", Gl[i]);
    printf("\n");
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def shares(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("plan")
    src, exe = d / "driver.cpp", d / "driver"
    src.write_text(DRIVER)
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True)

    def run(cases):
        inp = "".join(f"{len(W)} {G} " + " ".join(map(str, W)) + "\n" for W, G in cases)
        out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True).stdout
        return [list(map(int, line.split())) for line in out.splitlines()]
    return run


def test_known_groups(shares):
    # Qwen2.5-3B q|k|v (16 + 2 + 2 tiles of 32 stages) and gate|up (86 + 86 tiles) on 148 SMs
    assert shares([([512, 64, 64], 148), ([2752, 2752], 148)]) == [[118, 15, 15], [74, 74]]
    # small layers: fewer stages than SMs, so the grid is the stage count and every CTA gets one stage
    assert shares([([12, 8, 8], 28)]) == [[12, 8, 8]]
    assert shares([([1, 1, 1, 1], 4)]) == [[1, 1, 1, 1]]


def test_random_groups_hold_the_invariants(shares):
    import numpy as np
    rng = np.random.default_rng(0)
    cases = []
    for _ in range(20000):
        n = int(rng.integers(1, 5))
        W = [int(rng.integers(1, 9)) if rng.random() < 0.3 else int(rng.integers(1, 300000)) for _ in range(n)]
        G = int(max(n, min(148, sum(W))))
        cases.append((W, G))
    for (W, G), Gl in zip(cases, shares(cases)):
        assert len(Gl) == len(W)
        assert sum(Gl) == G, (W, G, Gl)
        for w, g in zip(W, Gl):
            assert 1 <= g <= w, (W, G, Gl)
            assert abs(g - G * w / sum(W)) <= len(W), (W, G, Gl)
