"""Host logic of the persistent decode grid, on the CPU.

The planning header (online_rank_kv_b200/csrc/decode_plan.h) is plain C++: it
is compiled here with the host compiler into a small driver that prints the
runs for a list of shapes.  Checked against what the plan must satisfy: the
runs are contiguous and cover every tile once, there are at most as many runs
as CTAs, no run costs more than the bisected bound (tiles plus the charge for
each head it enters after its first), one unit less is infeasible, and the
per-head run count matches a brute-force count.
"""

import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "online_rank_kv_b200", "csrc")

DRIVER = r"""
#include <cstdio>
#include "decode_plan.h"
using namespace iskv;
int main() {
    long long total, tph; int nmax;
    static int64_t st[4096];
    while (std::scanf("%lld %lld %d", &total, &tph, &nmax) == 3) {
        const int n = partition_decode_tiles(total, tph, nmax, st);
        // the bound the bisection settled on: the largest run cost
        long long bound = 0;
        for (int i = 0; i < n; ++i) {
            const long long segs = (st[i + 1] - 1) / tph - st[i] / tph + 1;
            const long long c = st[i + 1] - st[i] + kHeadSwitchTiles * (segs - 1);
            if (c > bound) bound = c;
        }
        static int64_t tmp[4096];
        const int tighter = bound > 1 ? fill_decode_runs(total, tph, nmax, bound - 1, tmp) : nmax + 1;
        const int heads = (int)((total + tph - 1) / tph);
        std::printf("%d %lld %d %d", n, bound, tighter, max_runs_per_head(st, n, heads, tph));
        for (int i = 0; i <= n; ++i) std::printf(" %lld", (long long)st[i]);
        std::printf("\n");
    }
    // the memoized grid plan: a head cap forces fewer runs; same inputs reuse
    DecodeGridPlan p;
    const bool ok1 = plan_decode_grid(4000, 4000, 1, 148, 20, 2, &p);
    const int n1 = p.nruns, s1 = p.slots;
    const int64_t* before = p.start.data();
    const bool ok2 = plan_decode_grid(4000, 4000, 1, 148, 20, 2, &p);
    const bool same = p.start.data() == before && p.nruns == n1;
    const bool ok3 = plan_decode_grid(64 * 280, 280, 64, 148, 256, 2, &p);
    std::printf("memo %d %d %d %d %d %d %d\n", ok1, n1, s1, ok2, same, ok3, p.nruns);
}
"""

SHAPES = [
    (64 * 264, 264, 148),     # 64 heads, 32K context, 64-row exact tiles
    (64 * 280, 280, 148),     # the same with 32-row exact tiles
    (8 * 2064, 2064, 148),    # batch 1: eight heads, many CTAs per head
    (256 * 2064, 2064, 148),  # 256 heads, 256K context
    (40, 40, 148),            # one head, fewer tiles than CTAs
    (15, 5, 148),             # three tiny heads
    (7, 7, 1),                # one CTA
    (3 * 1000, 1000, 7),
    (5 * 3, 3, 4),
]


@pytest.fixture(scope="module")
def driver():
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tempfile.mkdtemp()
    src = os.path.join(d, "plan.cpp")
    exe = os.path.join(d, "plan")
    with open(src, "w") as fh:
        fh.write(DRIVER)
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", CSRC, src, "-o", exe], check=True)
    yield exe
    shutil.rmtree(d)


def _run(exe, shapes):
    inp = "".join(f"{t} {h} {n}\n" for t, h, n in shapes)
    out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout
    return [list(map(int, line.split())) for line in out.strip().splitlines()
            if not line.startswith("memo")]


def test_grid_plan_caps_slots_and_is_reused(driver):
    out = subprocess.run([driver], input="", capture_output=True, text=True, check=True).stdout
    memo = [line for line in out.splitlines() if line.startswith("memo")][0].split()[1:]
    ok1, n1, s1, ok2, same, ok3, n3 = map(int, memo)
    # one head of 4000 tiles, at most 20 slots: at most 10 runs share it
    assert ok1 == 1 and 2 * s1 <= 20 and n1 == s1 <= 10
    assert ok2 == 1 and same == 1          # same inputs: the stored plan, untouched
    assert ok3 == 1 and n3 == 148          # new inputs: planned afresh


def test_runs_cover_every_tile_within_the_bound(driver):
    S = 4  # the per-head charge in tiles (kHeadSwitchTiles)
    for (total, tph, nmax), row in zip(SHAPES, _run(driver, SHAPES)):
        n, bound, tighter, most = row[:4]
        st = row[4:]
        assert len(st) == n + 1 and 1 <= n <= nmax
        assert st[0] == 0 and st[-1] == total
        assert all(st[i] < st[i + 1] for i in range(n))
        # every run within the bound; one less is infeasible
        for i in range(n):
            heads_entered = (st[i + 1] - 1) // tph - st[i] // tph
            assert st[i + 1] - st[i] + S * heads_entered <= bound
        assert tighter > nmax
        # runs per head, brute force
        brute = 1
        for h in range((total + tph - 1) // tph):
            lo, hi = h * tph, min((h + 1) * tph, total)
            brute = max(brute, sum(1 for i in range(n) if st[i] < hi and st[i + 1] > lo))
        assert most == brute
