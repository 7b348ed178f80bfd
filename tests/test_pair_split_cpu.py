"""Host-side check of the persistent Euler loop's split-K work division (dm0::pd_pairs in
denoise_persistent.cuh): compiled with nvcc as a host program and run on the CPU.  For every phase
shape of the DM0-base action expert on 148 SMs, and for small and odd shapes, each (weight tile,
k-block) pair belongs to exactly one CTA, ranges are contiguous and in CTA order, and with at least
as many CTAs as tiles no range crosses a tile boundary (one output segment per CTA)."""
import os
import shutil
import subprocess

import pytest

from vla_dual_expert_b200 import build as B

PROG = r"""
#include <cstdio>
#include "denoise_persistent.cuh"
int main() {
  const int shapes[][3] = {
      {32, 16, 148}, {8, 32, 148}, {48, 16, 148}, {8, 48, 148},   // DM0-base QKV, O, gate/up, down
      {32, 16, 132}, {48, 16, 100}, {8, 32, 8}, {8, 32, 9}, {7, 5, 3}, {3, 7, 10}, {1, 1, 4}, {5, 2, 40}};
  int bad = 0;
  for (const auto& sh : shapes) {
    const int tiles = sh[0], nkb = sh[1], n = sh[2];
    int expect = 0, longest = 0;
    for (int c = 0; c < n; ++c) {
      int p0, p1;
      dm0::pd_pairs(tiles, nkb, c, n, p0, p1);
      if (p0 != expect || p1 < p0) ++bad;        // contiguous, in CTA order, non-negative
      expect = p1;
      if (p1 > p0 && n >= tiles && p0 / nkb != (p1 - 1) / nkb) ++bad;   // one tile per CTA
      if (p1 - p0 > longest) longest = p1 - p0;
    }
    if (expect != tiles * nkb) ++bad;            // every pair exactly once
    if (n >= tiles) {
      const int base = n / tiles;
      if (longest != (nkb + base - 1) / base) ++bad;   // the longest range is ceil(nkb / base)
    }
    printf("%d %d %d %d\n", tiles, nkb, n, longest);
  }
  printf("bad %d\n", bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(not shutil.which(B.nvcc_path()) and not os.path.exists(B.nvcc_path()), reason="nvcc not found")
def test_pair_split_covers_every_pair_once_one_tile_per_cta(tmp_path):
    src = tmp_path / "pairs.cu"
    src.write_text(PROG)
    exe = tmp_path / "pairs"
    res = subprocess.run([B.nvcc_path(), "-std=c++17", "--expt-relaxed-constexpr", "-gencode",
                          "arch=compute_100a,code=sm_100a", "-I", B.INCLUDE, "-I", B.CSRC, "-o", str(exe), str(src)],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout
    lines = dict((tuple(map(int, l.split()[:3])), int(l.split()[3])) for l in out.stdout.splitlines()[:-1])
    # DM0-base on 148 SMs: at most 4 / 2 / 6 / 3 pairs (QKV / O / gate-up / down), the staging area's six
    assert [lines[(32, 16, 148)], lines[(8, 32, 148)], lines[(48, 16, 148)], lines[(8, 48, 148)]] == [4, 2, 6, 3]
