"""Host logic shared by the library's launchers and kernels: the streaming
passes share one wave of CTAs among (batch row, kv head) units in proportion to
their work (row_items, unit_ctas).  The same integer arithmetic runs on the host,
which sizes the grid, and on the device, where each CTA finds its run of blocks;
this compiles it host-only (no GPU needed) and checks its invariants."""

import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "certified_quantized_kv_int8_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include "cqa_internal.cuh"
int main() {
  int target, units, cap;
  while (std::scanf("%d %d %d", &target, &units, &cap) == 3) {
    int nb[64], r[64];
    long long sum = 0;
    for (int u = 0; u < units; ++u) {
      std::scanf("%d %d", &nb[u], &r[u]);
      sum += cqa::row_items(nb[u], r[u]);
    }
    for (int u = 0; u < units; ++u)
      std::printf("%d ", cqa::unit_ctas(target, cqa::row_items(nb[u], r[u]), sum, cap));
    std::printf("\n");
  }
  return 0;
}
'''


@pytest.fixture(scope="module")
def tool(tmp_path_factory):
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    if not os.path.exists(nvcc):
        pytest.skip("nvcc is not available")
    d = tmp_path_factory.mktemp("grid")
    src = d / "grid.cu"
    src.write_text(PROGRAM)
    exe = d / "grid"
    subprocess.run([nvcc, "-std=c++17", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    "-o", str(exe), str(src)], check=True)
    return exe


def _share(tool, target, cap, rows):
    inp = f"{target} {len(rows)} {cap}\n" + "\n".join(f"{nb} {r}" for nb, r in rows) + "\n"
    out = subprocess.run([str(tool)], input=inp, capture_output=True, text=True, check=True)
    return [int(x) for x in out.stdout.split()]


def test_row_items_counts_the_residual_as_two_blocks():
    # restated here (not imported): sealed blocks plus 2 for a non-empty residual, else 1
    def row_items(nb, r):
        return nb + (2 if r > 0 else 1)
    assert row_items(512, 0) == 513 and row_items(512, 63) == 514 and row_items(0, 1) == 2


@pytest.mark.parametrize("rows", [
    [(512, 0)] * 8,                                   # 32K, 8 kv heads
    [(2048, 5)] * 8,                                  # 128K
    [(1024, 0)] * 32,                                 # 64K x B4
    [(512, 7)] * 8 + [(64, 37)] * 8 + [(256, 5)] * 8 + [(128, 0)] * 8,  # ragged B4
    [(0, 1)] * 8,                                     # one token per row
])
def test_unit_ctas_invariants(tool, rows):
    target, cap = 148 * 4, 10_000
    got = _share(tool, target, cap, rows)
    items = [nb + (2 if r > 0 else 1) for nb, r in rows]
    total = sum(items)
    assert all(g >= 1 for g in got)
    # never more than one wave unless every unit already has its one CTA
    assert sum(got) <= max(target, len(rows))
    for g, it in zip(got, items):
        assert g == max(1, min(cap, target * it // total))  # floor share, clamped
    # equal work, equal CTAs; more work, no fewer CTAs
    for i in range(len(rows)):
        for j in range(len(rows)):
            if items[i] >= items[j]:
                assert got[i] >= got[j]


def test_unit_ctas_cap(tool):
    got = _share(tool, 592, 20, [(4096, 0)] * 2)
    assert got == [20, 20]
