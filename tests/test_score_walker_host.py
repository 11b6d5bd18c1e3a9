"""The persistent scoring kernel's tile walk, checked on the CPU.

Every role of a CTA of `score_tc_kernel` (TMA producer, MMA issuer,
epilogue, counter watcher) walks the same sequence of tiles with StcWalker,
and the watcher waits until stc_participants(...) CTAs have arrived on a
problem's counter.  Both are __host__ __device__ in k_score_tc.cuh; this test
compiles them into a host program (nvcc, no GPU) and checks them against a
brute-force enumeration over random batches, ragged lengths (empty problems
included), grid sizes and chunk sizes:
  * pass 1 visits every active 128-row tile exactly once over all CTAs, each
    CTA in increasing order, with k counting the CTA's tiles of a problem and
    `last` on its final one;
  * pass 2 revisits, in the same order, exactly the tiles with k >= kept;
  * the participant count equals the number of CTAs that own tiles of the
    problem (a larger one would leave the counter short of its target).
"""
import os
import random
import shutil
import subprocess
from collections import defaultdict

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rank_decode_attention_b200", "csrc")

PROG = r'''
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "k_score_tc.cuh"
using namespace s4r;
int main(int argc, char **argv) {
  const int batch = atoi(argv[1]), G = atoi(argv[3]), K = atoi(argv[4]), kept = atoi(argv[5]);
  const long long cap = atoll(argv[2]);
  std::vector<int32_t> len(batch);
  for (int p = 0; p < batch; ++p) len[p] = atoi(argv[6 + p]);
  for (int c = 0; c < G; ++c) {
    StcWalker w;
    w.start(len.data(), cap, batch, G, c, K, kept);
    StcTile t;
    while (w.next(t))
      printf("t %d %d %lld %d %d %d %d\n", c, t.p, (long long)t.row0, t.k, t.last ? 1 : 0, t.pass2 ? 1 : 0,
             t.pass2 ? -1 : stc_participants(w.S, t.T, K, G));
  }
  return 0;
}
'''


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("walker")
    src, out = d / "walk.cu", d / "walk"
    src.write_text(PROG)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    "-o", str(out), str(src)], check=True, capture_output=True)
    return str(out)


def _cases():
    rng = random.Random(11)
    cases = [(1, 131072, [131068], 148, 1, 4), (16, 8192, [8188] * 16, 148, 2, 4), (8, 40000, None, 148, 1, 4),
             (40, 3000, None, 40, 1, 4), (3, 1000, [0, 999, 1], 5, 2, 4), (5, 20000, None, 37, 2, 8)]
    for _ in range(24):
        b = rng.randint(1, 20)
        cap = rng.choice([128, 700, 4096, 20000, 65536])
        cases.append((b, cap, None, rng.choice([1, 3, 16, 64, 148]), rng.choice([1, 2, 3]), rng.choice([4, 8])))
    out = []
    for b, cap, L, G, K, kept in cases:
        if L is None:
            L = [rng.choice([0, rng.randint(0, cap)]) for _ in range(b)]
        out.append((b, cap, L, G, K, kept))
    return out


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}-cap{c[1]}-G{c[3]}-K{c[4]}-kept{c[5]}" for c in CASES])
def test_walk_covers_every_tile_and_counts_the_participants(exe, case):
    B, cap, L, G, K, kept = case
    out = subprocess.run([exe, str(B), str(cap), str(G), str(K), str(kept)] + [str(x) for x in L],
                         capture_output=True, text=True, check=True).stdout
    rec = [tuple(int(v) for v in line.split()[1:]) for line in out.splitlines()]
    T = [-(-l // 128) for l in L]
    S = [sum(T[:p]) for p in range(B)]
    owners = defaultdict(set)
    seen1 = set()
    for c in range(G):
        mine = [r for r in rec if r[0] == c]
        p1 = [r for r in mine if r[5] == 0]
        p2 = [r for r in mine if r[5] == 1]
        # brute force: the CTA owns global tiles g with (g // K) % G == c, in increasing order
        expect = [g for g in range(sum(T)) if (g // K) % G == c]
        glob = [S[r[1]] + r[2] // 128 for r in p1]
        assert glob == expect
        count = defaultdict(int)
        for i, (cc, p, row0, k, last, _, parts) in enumerate(p1):
            assert row0 % 128 == 0 and row0 < L[p]
            assert k == count[p]
            count[p] += 1
            later = [r for r in p1[i + 1:] if r[1] == p]
            assert last == (1 if not later else 0)
            owners[p].add(c)
            seen1.add((p, row0))
        assert [(r[1], r[2]) for r in p2] == [(r[1], r[2]) for r in p1 if r[3] >= kept]
    assert seen1 == {(p, 128 * i) for p in range(B) for i in range(T[p])}
    for r in rec:
        if r[5] == 0:
            assert r[6] == len(owners[r[1]])
