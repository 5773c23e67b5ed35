"""The kernels' unit order (unit_order in fa_common.cuh), compiled for the host with nvcc.

Every grid maps its CTA index u to a (head, level) unit through this function, so it must
be a bijection of [0, heads * levels) onto the units, or some unit is computed twice and
another never.  Beyond that the tests check the stated order: tiers of `tsz` levels run
heaviest first with one head's units consecutive inside a tier, and with tail > 0 the last
`tail` heads come after all the others, level by level.
"""
import itertools
import pathlib
import shutil
import subprocess

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]
HARNESS = r'''
#include <cstdio>
#include <cstdlib>
#include "fa_common.cuh"
int main(int argc, char **argv) {
  for (int a = 1; a + 3 < argc; a += 4) {
    const int heads = atoi(argv[a]), levels = atoi(argv[a + 1]), tsz = atoi(argv[a + 2]), tail = atoi(argv[a + 3]);
    for (int u = 0; u < heads * levels; ++u) {
      int h = -1, l = -1;
      fa::unit_order(u, heads, levels, tsz, tail, h, l);
      printf("%d %d ", h, l);
    }
    printf("\n");
  }
  return 0;
}
'''

CASES = [(h, l, t, k) for h, l in [(1, 1), (1, 7), (3, 1), (5, 4), (8, 16), (32, 64), (128, 16), (7, 9)]
         for t in sorted({1, 2, 3, l}) if t <= l
         for k in sorted({0, 1, h // 4, h // 2, h - 1}) if 0 <= k < h]


@pytest.fixture(scope="module")
def orders(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not pathlib.Path(nvcc).exists():
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("unit_order")
    src = d / "harness.cu"
    src.write_text(HARNESS)
    exe = d / "harness"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", str(ROOT / "include"),
                    "-I", str(ROOT / "exact_io_aware_83_b200" / "csrc"), "-o", str(exe), str(src)],
                   check=True, capture_output=True)
    args = [str(x) for c in CASES for x in c]
    out = subprocess.run([str(exe)] + args, check=True, capture_output=True, text=True).stdout.splitlines()
    res = {}
    for case, line in zip(CASES, out):
        v = list(map(int, line.split()))
        res[case] = list(zip(v[0::2], v[1::2]))
    assert len(res) == len(CASES)
    return res


def test_every_unit_exactly_once(orders):
    for (heads, levels, tsz, tail), seq in orders.items():
        assert sorted(seq) == list(itertools.product(range(heads), range(levels))), (heads, levels, tsz, tail)


def test_tiers_run_heaviest_first_with_heads_contiguous(orders):
    for (heads, levels, tsz, tail), seq in orders.items():
        front = seq[: (heads - tail) * levels]
        tiers = [[(h, l) for h, l in front if l // tsz == t] for t in range((levels + tsz - 1) // tsz)]
        assert sum(tiers, []) == front            # tier after tier
        for tier in tiers:
            hs = [h for h, _ in tier]
            assert hs == sorted(hs)               # one head's units together
            for h in set(hs):                     # inside a head, heaviest (lowest level) first
                ls = [l for hh, l in tier if hh == h]
                assert ls == sorted(ls)


def test_tail_heads_come_last_level_by_level(orders):
    for (heads, levels, tsz, tail), seq in orders.items():
        front, back = seq[: (heads - tail) * levels], seq[(heads - tail) * levels:]
        assert {h for h, _ in front} == set(range(heads - tail))
        assert {h for h, _ in back} == set(range(heads - tail, heads))
        assert back == [(h, l) for l in range(levels) for h in range(heads - tail, heads)]


def test_head_major_and_level_major_extremes(orders):
    for (heads, levels, tsz, tail), seq in orders.items():
        if tail:
            continue
        if tsz == levels:
            assert seq == [(h, l) for h in range(heads) for l in range(levels)]
        if tsz == 1:
            assert seq == [(h, l) for l in range(levels) for h in range(heads)]
