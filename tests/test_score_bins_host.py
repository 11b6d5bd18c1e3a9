"""Level-0 score bins of the top-k search, checked on the CPU.

The scoring kernels count candidate scores into kExpBins bins around the mean
score R / L_c (score_center, score_bin), and every rank of the cluster select
narrows the threshold to the key range of one bin (score_bin_range).  The
select is exact only if the bin index never decreases as the key grows and
every key lies inside its own bin's range.  Both functions are
__host__ __device__ in common.cuh; this test runs them in a host program
over the keys of every non-negative float around several centres.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rank_decode_attention_b200", "csrc")

PROG = r'''
#include <cstdio>
#include <cstdlib>
#include "common.cuh"
using namespace s4r;
// Exit status 0 when every check holds; prints the first failure otherwise.
int main(int argc, char **argv) {
  const int R = atoi(argv[1]);
  const long long L = atoll(argv[2]);
  const uint32_t c = score_center(R, L);
  int prev = -1;
  uint32_t prev_hi = 0;
  // every 97th key from 0 (+0.0) up to 0x7f800000 (+inf), then +inf itself;
  // bins are 2^15 keys wide, so no bin is skipped between two samples
  auto check = [&](uint32_t key) -> bool {
    const int b = score_bin(key, c);
    if (b < 0 || b >= kExpBins) { printf("bin out of range %u %d\n", key, b); return false; }
    if (b < prev) { printf("not monotone at %u\n", key); return false; }
    uint32_t lo, hi;
    score_bin_range(b, c, lo, hi);
    if (key < lo || key > hi) { printf("key %u outside bin %d [%u, %u]\n", key, b, lo, hi); return false; }
    if (b != prev && prev >= 0 && lo != prev_hi + 1) { printf("gap before bin %d\n", b); return false; }
    prev = b;
    prev_hi = hi;
    return true;
  };
  for (uint32_t key = 0; key < 0x7f800000u; key += 97)
    if (!check(key)) return 1;
  if (!check(0x7f800000u)) return 1;
  // the centre's own bin is the middle one
  if (score_bin(c, c) != kExpBins / 2) { printf("centre bin %d\n", score_bin(c, c)); return 1; }
  printf("ok %u\n", c);
  return 0;
}
'''


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("bins")
    src, out = d / "bins.cu", d / "bins"
    src.write_text(PROG)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    "-o", str(out), str(src)], check=True, capture_output=True)
    return str(out)


@pytest.mark.parametrize("R,L", [(64, 32764), (64, 8188), (64, 131068), (512, 32764), (8, 2044), (32, 1), (64, 0)])
def test_bins_are_monotone_and_hold_their_keys(exe, R, L):
    out = subprocess.run([exe, str(R), str(L)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout
