"""Host check of how the tensor-core GEMM deals a launch's tiles to its persistent CTAs.

The dealing (csrc/tile_deal.cuh) is compiled here with the host compiler and checked on the
CPU: every tile goes to exactly one CTA, each CTA's tiles come in increasing order (the
kernel's matrix cursor only moves forward), and on the Qwen2.5-0.5B decode set's launches
the busiest CTA carries at most 6 % more k-blocks than the mean (round robin: 26 %).
"""
import ctypes
import os
import shutil
import subprocess

import pytest

from bit_weight_quantized_unpack_b200 import workloads

CSRC = os.path.join(os.path.dirname(__file__), "..", "bit_weight_quantized_unpack_b200", "csrc")
SHIM = r"""
#include "tile_deal.cuh"
extern "C" int deal(int cta, int j, int ctas, int total, int r0, int b, int q) {
  return wq::dealt_tile(cta, j, ctas, total, wq::TileDeal{r0, b, q});
}
extern "C" void plan(int ctas, int n1, int c1, int c2, int* out) {
  const wq::TileDeal d = wq::plan_deal(ctas, n1, c1, c2);
  out[0] = d.r0; out[1] = d.b; out[2] = d.q;
}
"""


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("deal")
    src, so = d / "shim.cpp", d / "libdeal.so"
    src.write_text(SHIM)
    subprocess.run([cxx, "-O2", "-shared", "-fPIC", "-I", CSRC, str(src), "-o", str(so)], check=True)
    L = ctypes.CDLL(str(so))
    L.deal.restype = ctypes.c_int
    return L


def plan(lib, ctas, n1, c1, c2):
    out = (ctypes.c_int * 3)()
    lib.plan(ctas, n1, c1, c2, out)
    return tuple(out)


def lists_of(lib, ctas, total, d):
    lists = []
    for c in range(ctas):
        seq, j = [], 0
        while True:
            t = lib.deal(c, j, ctas, total, *d)
            if t < 0:
                break
            seq.append(t)
            j += 1
        lists.append(seq)
    return lists


@pytest.mark.parametrize("ctas", [1, 2, 7, 148])
@pytest.mark.parametrize("total", [1, 5, 148, 149, 1000])
@pytest.mark.parametrize("n1,c1,c2", [(0, 18, 0), (3, 80, 18), (56, 80, 18), (148, 80, 18),
                                      (300, 300, 60), (7, 18, 18), (999, 80, 18)])
def test_every_tile_once_in_order(lib, ctas, total, n1, c1, c2):
    n1 = min(n1, total)
    d = plan(lib, ctas, n1, c1, c2)
    lists = lists_of(lib, ctas, total, d)
    flat = sorted(t for l in lists for t in l)
    assert flat == list(range(total)), f"deal {d}: tiles not dealt exactly once"
    for l in lists:
        assert l == sorted(l), f"deal {d}: a CTA's tiles out of order"


def test_plain_round_robin_when_one_class(lib):
    assert plan(lib, 148, 1187, 18, 0) == (0, 0, 0)
    assert lists_of(lib, 3, 7, (0, 0, 0)) == [[0, 3, 6], [1, 4], [2, 5]]


def test_phases_by_hand(lib):
    # 4 CTAs, 2 large tiles (cost 4), then small tiles (cost 1): q = 4 rounds of the small
    # tiles go to CTAs 2 and 3 before round robin resumes over all four
    d = plan(lib, 4, 2, 4, 1)
    assert d == (0, 2, 4)
    assert lists_of(lib, 4, 16, d) == [[0, 10, 14], [1, 11, 15], [2, 4, 6, 8, 12], [3, 5, 7, 9, 13]]


@pytest.mark.parametrize("M", [33, 64, 512])
def test_balance_on_the_05b_set(lib, M):
    """The launches wq_linear_set makes for the 0.5B set's 169 matrices at M tokens: up to
    80 matrices per launch, ordered by K (largest first) and dealt to launches round robin;
    tiles of 128 weight rows x min(16 * ceil(M / 16), 256) tokens costing K / 64 + 4."""
    mats = workloads.workload_mats(1)
    bn = min((M + 15) // 16 * 16, 256)
    tm = (M + bn - 1) // bn
    order = sorted(range(len(mats)), key=lambda i: -mats[i].K)  # stable: ties keep set order
    launches = (len(mats) + 79) // 80
    worst, worst_rr = 0.0, 0.0
    for l in range(launches):
        costs = []
        for i in order[l::launches]:
            m = mats[i]
            costs += [m.K // 64 + 4] * ((m.N + 127) // 128 * tm)
        ctas = min(148, len(costs))
        c1 = costs[0]
        n1 = sum(1 for c in costs if c == c1)
        c2 = costs[n1] if n1 < len(costs) else 0
        d = plan(lib, ctas, n1, c1, c2)
        loads = [sum(costs[t] for t in seq) for seq in lists_of(lib, ctas, len(costs), d)]
        mean = sum(costs) / ctas
        worst = max(worst, max(loads) / mean)
        rr = [sum(costs[c::ctas]) for c in range(ctas)]
        worst_rr = max(worst_rr, max(rr) / mean)
    assert worst <= 1.06, f"busiest CTA {worst:.3f} x the mean"
    assert worst < worst_rr
