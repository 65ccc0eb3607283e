"""The router's grid schedule (csrc/route_schedule.cuh), compiled with the
host C++ compiler: how query blocks group into runs and how runs map to CTA
indices.  Pure index arithmetic, so it is checked here without a GPU: every
(run, KV head) unit is served exactly once, co-resident CTAs hold
complementary runs, and the run length is the one the schedule's rule picks
at the shapes the parity tests and the bench use."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "hierarchical_kv_routing_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "route_schedule.cuh"
using namespace hga;
int main(int argc, char **argv) {
    if (argc > 1) {            // pick_run NB units nmax sms per_sm
        std::printf("%d\n", pick_run(std::atoi(argv[1]), std::atoi(argv[2]), std::atoi(argv[3]),
                                     std::atoi(argv[4]), std::atoi(argv[5])));
        return 0;
    }
    long bad = 0;
    for (int R = 1; R <= 300; ++R)
        for (int U = 1; U <= 33; ++U) {
            const int N = R * U;
            std::vector<int> seen(N, 0);
            for (int l = 0; l < N; ++l) {
                int r, u;
                pair_slot(l, R, U, &r, &u);
                if (r < 0 || r >= R || u < 0 || u >= U) { ++bad; continue; }
                seen[r * U + u]++;
            }
            for (int k = 0; k < N; ++k) bad += seen[k] != 1;
            // partners N/2 apart hold runs r and R-1-r (complementary work);
            // in each half, neighbours 2m and 2m+1 hold runs summing to within
            // one of R-1
            for (int l = 0; l < N / 2; ++l) {
                int r1, u1, r2, u2;
                pair_slot(l, R, U, &r1, &u1);
                pair_slot(l + N / 2, R, U, &r2, &u2);
                bad += r1 + r2 != R - 1;
            }
            for (int half = 0; half < 2; ++half)
                for (int m = 0; 2 * m + 1 < N / 2; ++m) {
                    const int l = half * (N / 2) + 2 * m;
                    int r1, u1, r2, u2;
                    pair_slot(l, R, U, &r1, &u1);
                    pair_slot(l + 1, R, U, &r2, &u2);
                    bad += r1 + r2 < R - 2 || r1 + r2 > R;
                }
        }
    std::printf("%ld\n", bad);
    return 0;
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    d = tmp_path_factory.mktemp("sched")
    src, exe = d / "sched.cpp", d / "sched"
    src.write_text(HARNESS)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)])
    return str(exe)


def test_pair_layout_is_a_bijection_with_complementary_partners(harness):
    assert subprocess.check_output([harness]).decode().strip() == "0"


@pytest.mark.parametrize("NB,units,nmax,expect", [
    (512, 4, 8, 7),     # 32K Qwen3 prefill: 74 runs x 4 heads = 296 CTAs, two per SM
    (256, 4, 8, 7),     # 16K: 148 CTAs, one per SM
    (64, 64, 8, 8),     # SmallLM 8 x 4K, 8 heads: more than one wave whatever n, longest run
    (16, 1, 8, 1),      # tiny 1K: every block its own CTA
])
def test_run_length_at_the_workload_shapes(harness, NB, units, nmax, expect):
    out = subprocess.check_output([harness, str(NB), str(units), str(nmax), "148", "2"])
    assert int(out) == expect
