"""Index arithmetic of the GPU basis build, checked on the CPU.

The sample-row formula, the round-robin (circle) schedule, the block-pair
index map and the inner rounds of the block Jacobi method in k_basis.cuh are
__host__ __device__ functions.  This test
compiles them into a host-only program with nvcc (no GPU needed) and checks
them bit-exactly: the sampled rows against the basis oracle
(oracle/basis.py, an independent implementation of the 7:3 rule), and the
schedule against its definition (every pair of m players meets exactly once
in m - 1 rounds and the pairs of a round are disjoint).  The kernel uses the
schedule twice: over the 32 indices of a submatrix, and over the mp / 16
index blocks of the Gram matrix (mp a multiple of 32, so an even count).
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import basis as obasis

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rank_decode_attention_b200", "csrc")

PROG = r'''
#include <cstdio>
#include <cstdlib>
#include "umma.cuh"
#include "k_basis.cuh"
using namespace s4r;
int main(int argc, char **argv) {
  if (argv[1][0] == 'r') {            // r L s T: the sampled rows
    const long long L = atoll(argv[2]), s = atoll(argv[3]), T = atoll(argv[4]);
    const long long avail = L - s > 0 ? L - s : 0, n = avail < T ? avail : T;
    for (long long j = 0; j < n; ++j) printf("%lld\n", (long long)basis_sample_row(L, s, n, j));
    return 0;
  }
  if (argv[1][0] == 'i') {            // i: index pairs of the 31 inner rounds of a 32 x 32 submatrix
    for (int kk = 0; kk < kBjInner; ++kk)
      for (int u = 0; u < kBjBlock; ++u) {
        int x, y;
        bj_inner_pair(kk, u, x, y);
        printf("%d %d %d %d\n", kk, u, x, y);
      }
    return 0;
  }
  if (argv[1][0] == 'b') {            // b nb: global index of local l of block pair a in round k
    const int nb = atoi(argv[2]);
    for (int k = 0; k < nb - 1; ++k)
      for (int a = 0; a < nb / 2; ++a)
        for (int l = 0; l < kBjPair; ++l) printf("%d %d %d %d\n", k, a, l, bj_index(nb, k, a, l));
    return 0;
  }
  const int m = atoi(argv[2]);        // p m: players of every slot of every round
  for (int k = 0; k < m - 1; ++k)
    for (int u = 0; u < m; ++u) printf("%d %d %d\n", k, u, jac_player(m, k, u));
  return 0;
}
'''


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("basis_host")
    src, out = d / "idx.cu", d / "idx"
    src.write_text(PROG)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
                    "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    "-o", str(out), str(src)], check=True, capture_output=True)
    return str(out)


@pytest.mark.parametrize("L,s,T", [(20, 4, 10), (14, 4, 10), (100, 0, 5), (9, 4, 10), (50, 4, 1), (50, 4, 2),
                                   (50, 4, 3), (4, 4, 8), (1000, 4, 20), (32768, 4, 256), (8192, 4, 512),
                                   (700, 4, 512), (131072, 4, 256), (2048, 4, 256), (5, 4, 3)])
def test_sample_rows_match_the_oracle(exe, L, s, T):
    out = subprocess.run([exe, "r", str(L), str(s), str(T)], capture_output=True, text=True, check=True).stdout
    gpu_rows = [int(v) for v in out.split()]
    assert gpu_rows == obasis.sample_rows(L, s, T).tolist()


@pytest.mark.parametrize("m", [2, 4, 6, 32, 38, 64, 1024])
def test_round_robin_schedule(exe, m):
    out = subprocess.run([exe, "p", str(m)], capture_output=True, text=True, check=True).stdout
    rec = np.array([[int(v) for v in line.split()] for line in out.splitlines()])
    assert rec.shape == ((m - 1) * m, 3)
    seen = set()
    for k in range(m - 1):
        r = rec[rec[:, 0] == k]
        players = r[np.argsort(r[:, 1]), 2]
        assert sorted(players.tolist()) == list(range(m))                  # a permutation of the players
        for a in range(m // 2):
            pair = tuple(sorted((int(players[2 * a]), int(players[2 * a + 1]))))
            assert pair not in seen
            seen.add(pair)
    assert len(seen) == m * (m - 1) // 2                                    # every pair once per sweep


def test_inner_rounds_meet_every_index_pair_once(exe):
    """The 31 inner rounds of a block-pair submatrix: rounds 0-14 pair the
    indices inside each 16-index block, rounds 15-30 pair the two blocks;
    every round pairs all 32 indices disjointly and every one of the 496
    index pairs meets exactly once (the first outer round of a sweep runs all
    31 rounds, the others the 16 across)."""
    out = subprocess.run([exe, "i"], capture_output=True, text=True, check=True).stdout
    rec = np.array([[int(v) for v in line.split()] for line in out.splitlines()])
    assert rec.shape == (31 * 16, 4)
    seen = set()
    for kk in range(31):
        r = rec[rec[:, 0] == kk]
        idx = sorted(r[:, 2].tolist() + r[:, 3].tolist())
        assert idx == list(range(32))                                     # disjoint, covering
        for x, y in r[:, 2:]:
            pair = (min(x, y), max(x, y))
            assert pair not in seen
            seen.add(pair)
            inside = (x < 16) == (y < 16)
            assert inside == (kk < 15)                                    # inside rounds first
    assert len(seen) == 32 * 31 // 2


@pytest.mark.parametrize("nb", [2, 4, 16, 64])
def test_block_pairs_cover_the_matrix_and_meet_once_per_sweep(exe, nb):
    """bj_index: in each round the nb / 2 submatrices partition the 16 nb
    indices; over the nb - 1 rounds of a sweep every two distinct blocks
    share a submatrix exactly once."""
    out = subprocess.run([exe, "b", str(nb)], capture_output=True, text=True, check=True).stdout
    rec = np.array([[int(v) for v in line.split()] for line in out.splitlines()])
    assert rec.shape == ((nb - 1) * (nb // 2) * 32, 4)
    met = set()
    for k in range(nb - 1):
        r = rec[rec[:, 0] == k]
        assert sorted(r[:, 3].tolist()) == list(range(16 * nb))           # a partition of the indices
        for a in range(nb // 2):
            g = r[r[:, 1] == a][:, 3]
            blocks = sorted(set((g // 16).tolist()))
            assert len(blocks) == 2 and sorted(g.tolist()) == sorted(
                [16 * blocks[0] + i for i in range(16)] + [16 * blocks[1] + i for i in range(16)])
            assert tuple(blocks) not in met
            met.add(tuple(blocks))
    assert len(met) == nb * (nb - 1) // 2
