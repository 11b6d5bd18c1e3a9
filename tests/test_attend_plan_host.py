"""Launch plans of the two attention kernels, checked on the CPU.

The per-group kernel (k_attend.cuh) and the row-split kernel
(k_attend_rows.cuh) take their cluster size, chunk capacity, output slices
and shared-memory layout from host functions that the kernels trust without
checking again.  This test compiles those functions into a host program
(nvcc, no GPU) and checks, for the configurations' shapes and a few edge
shapes, the properties the kernels rely on:
  * per group: the ranks' output items partition the G * d_h outputs in
    order, a rank's items span at most two heads (its receive buffers hold
    two), its B^V rows fit the staged rows, the chunk capacity is a multiple
    of 32 within the staging limit and the shared memory within budget;
  * row split: the heads split evenly over the cluster, a CTA's heads span
    the planned number of kv groups, the plan is accepted exactly when a
    CTA's three split terms fill one 16-row tile and span at most two
    groups, the chunk capacity is a multiple of 16 within the limit, and the
    shared-memory regions are 16-byte aligned and in order.
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
#include "k_attend_rows.cuh"
using namespace s4r;
int main(int argc, char **argv) {
  Shape s{};
  s.batch = atoi(argv[1]); s.n_heads_q = atoi(argv[2]); s.n_heads_kv = atoi(argv[3]); s.head_dim = atoi(argv[4]);
  s.rank_k = atoi(argv[5]); s.rank_v = atoi(argv[6]); s.n_sink = atoi(argv[7]); s.local_window = atoi(argv[8]);
  s.top_k = atoi(argv[9]); s.query_window = 16; s.d_model = s.n_heads_kv * s.head_dim;
  s.group = s.n_heads_q / s.n_heads_kv; s.n_rows = 16 * s.group; s.cache_rows = 32768;
  const int esize = 2;
  const int nr = att_ranks(s, 148);
  AttPlan pl = att_plan(s, esize, nr);
  if (att_smem_bytes(s, esize, pl) > kAttSmemBudget) pl = att_plan(s, esize);
  printf("G %d %d %d %d %zu %zu %d %d\n", pl.n_ranks, pl.e_cap, pl.bv_rows, kAttEntriesMax,
         att_smem_bytes(s, esize, pl), (size_t)kAttSmemBudget, kAttCluster, s.group);
  for (int c = 0; c < pl.n_ranks; ++c) {
    const AttItems it = att_items(s.group, s.head_dim, pl.n_ranks, c);
    printf("I %d %d %d %d %d\n", c, it.t0, it.t1, it.e_lo, it.e_hi);
  }
  printf("S %d\n", ar_supported(s, esize) ? 1 : 0);
  for (int nc : {16, 8, 4, 2, 1}) {
    if (s.n_heads_q % nc != 0) continue;
    const ArPlan p = ar_plan(s, nc);
    const ArLayout l = ar_layout(s, p);
    int grp = 1;
    for (int c = 0; c < nc; ++c) grp = smax(grp, ar_groups_of(s.group, p.hpc, c));
    printf("R %d %d %d %d %d %d %d %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", nc, p.hpc, p.e_cap, p.n_grp,
           p.late_bv, grp, ar_plan_ok(p) ? 1 : 0, l.qb, l.rows, l.part, l.bv, l.pb, l.recv, l.ob, l.oacc, l.fl,
           l.rows_idx, l.total, (size_t)kArSmemBudget);
  }
  return 0;
}
'''


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("attend_plan")
    src, out = d / "plan.cu", d / "plan"
    src.write_text(PROG)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    "-o", str(out), str(src)], check=True, capture_output=True)
    return str(out)


# (batch, H_q, H_kv, d_h, r_k, r_v, s, w, k): the configurations' shapes, then edge shapes
SHAPES = [(1, 32, 8, 128, 192, 192, 4, 128, 1024), (16, 32, 8, 128, 128, 128, 4, 128, 512),
          (1, 32, 8, 128, 256, 256, 4, 256, 2048), (8, 32, 8, 128, 256, 256, 4, 128, 1024),
          (2, 32, 8, 128, 128, 192, 4, 128, 1024), (40, 32, 8, 128, 192, 192, 4, 128, 1024),
          (2, 32, 8, 128, 256, 256, 4, 512, 3000), (1, 4, 2, 64, 32, 32, 4, 64, 128),
          (3, 16, 16, 64, 64, 64, 0, 8, 40), (2, 8, 1, 128, 64, 64, 16, 32, 300)]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_attention_plans_hold_what_the_kernels_assume(exe, shape):
    out = subprocess.run([exe] + [str(v) for v in shape], capture_output=True, text=True, check=True).stdout
    lines = [l.split() for l in out.splitlines()]
    B, Hq, Hkv, dh, rk, rv, ns, w, k = shape
    G = Hq // Hkv
    g = next(l for l in lines if l[0] == "G")
    n_ranks, e_cap, bv_rows, e_max, smem, budget, cl_max, grp = map(int, g[1:])
    assert grp == G and 1 <= n_ranks <= cl_max and n_ranks & (n_ranks - 1) == 0
    assert e_cap % 32 == 0 and 32 <= e_cap <= e_max and smem <= budget
    items = [tuple(map(int, l[1:])) for l in lines if l[0] == "I"]
    assert [it[0] for it in items] == list(range(n_ranks))
    t_next = 0
    for c, t0, t1, e_lo, e_hi in items:
        if t1 <= t0:
            continue                                               # an idle rank
        assert t0 == t_next                                        # in order, no gap, no overlap
        t_next = t1
        assert (t1 - 1) // dh - t0 // dh + 1 <= 2                  # at most two heads per rank
        assert 0 <= e_lo < e_hi <= dh and e_hi - e_lo <= bv_rows
        if t0 // dh == (t1 - 1) // dh:
            assert (e_lo, e_hi) == (t0 % dh, (t1 - 1) % dh + 1)
    assert t_next == G * dh
    supported = int(next(l for l in lines if l[0] == "S")[1])
    assert supported == int(rk % 16 == 0 and rv % 16 == 0 and Hq <= 32 and ns <= 16 and dh % 8 == 0)
    for l in (l for l in lines if l[0] == "R"):
        nc, hpc, cap, n_grp, late, grp_max, ok = map(int, l[1:8])
        qb, rows, part, bv, pb, recv, ob, oacc, fl, rows_idx, total, ar_budget = map(int, l[8:])
        assert hpc * nc == Hq and n_grp == grp_max
        assert cap % 16 == 0 and 16 <= cap <= 128
        assert ok == int(hpc >= 1 and 3 * hpc <= 16 and n_grp <= 2)
        for off in (qb, rows, part, bv, pb, recv, ob, oacc, fl, rows_idx, total):
            assert off % 16 == 0
        assert qb <= rows <= pb <= recv <= fl <= rows_idx <= total      # regions in order
        assert rows_idx + cap * 8 == total
