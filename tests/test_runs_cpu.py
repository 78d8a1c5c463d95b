"""Host-side check (CPU only) of how the fused tensor-core prefill splits its work: the unit
ranges of the persistent CTAs, the runs they cut from each chain (a head pair's blocks along
one sequence) and the slots the runs' states go to (mamba_ssd_b200/csrc/runs.cuh).

The header is compiled by the host C++ compiler into a small program that enumerates the runs
twice -- the way the run-state and scan kernels see them (walking each CTA's range) and the
way the pass kernel sees them (walking each chain's CTAs through cta_of) -- and checks:
  - every unit belongs to exactly one CTA, and cta_of agrees with first();
  - the runs of a CTA tile its range, each inside one chain;
  - every run's slot is unique and below slots();
  - the pass kernel's list of runs per chain equals the CTAs' list, in order, with the same slots.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "mamba_ssd_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <map>
#include <set>
#include <vector>
#include "runs.cuh"
using namespace ssd;
static int fail(const char *what, int U, int grid, int nk) {
    std::printf("FAIL %s U=%d grid=%d nk=%d\n", what, U, grid, nk);
    return 1;
}
int main() {
    int cases = 0;
    for (int nch = 1; nch <= 300; nch += (nch < 20 ? 1 : 37))
        for (int nk : {1, 2, 3, 7, 16, 32, 33, 256})
            for (int sms : {1, 2, 7, 148, 160}) {
                RunLayout lay;
                lay.nk = nk;
                lay.nch = nch;
                lay.U = nch * nk;
                lay.grid = lay.U < sms ? lay.U : sms;
                const int U = lay.U, grid = lay.grid;
                ++cases;
                // ranges tile [0, U); every CTA has at least one unit
                if (lay.first(0) != 0 || lay.first(grid) != U) return fail("range ends", U, grid, nk);
                for (int c = 0; c < grid; ++c) {
                    if (lay.first(c + 1) <= lay.first(c)) return fail("empty range", U, grid, nk);
                    for (int u = lay.first(c); u < lay.first(c + 1); ++u)
                        if (lay.cta_of(u) != c) return fail("cta_of", U, grid, nk);
                }
                // runs as the CTAs walk them: (chain, start, end, slot)
                std::map<int, std::vector<std::vector<int>>> by_chain;
                std::set<int> slots;
                for (int c = 0; c < grid; ++c) {
                    const int u0 = lay.first(c), u1 = lay.first(c + 1);
                    int rs = u0;
                    while (rs < u1) {
                        const int re = u1 < (rs / nk + 1) * nk ? u1 : (rs / nk + 1) * nk;
                        if (re <= rs || (re - 1) / nk != rs / nk) return fail("run crosses a chain", U, grid, nk);
                        const int s = lay.slot(rs, c);
                        if (s < 0 || s >= lay.slots() || !slots.insert(s).second) return fail("slot", U, grid, nk);
                        by_chain[rs / nk].push_back({rs, re, s});
                        rs = re;
                    }
                }
                if ((int)by_chain.size() != nch) return fail("chains", U, grid, nk);
                // runs as the pass kernel finds them
                for (int ch = 0; ch < nch; ++ch) {
                    const int c_lo = lay.cta_of(ch * nk), c_hi = lay.cta_of(ch * nk + nk - 1);
                    const std::vector<std::vector<int>> &runs = by_chain[ch];
                    if ((int)runs.size() != c_hi - c_lo + 1) return fail("run count", U, grid, nk);
                    int expect_start = ch * nk;
                    for (int c = c_lo; c <= c_hi; ++c) {
                        const std::vector<int> &r = runs[c - c_lo];
                        const int slot = c == c_lo ? ch : lay.nch + c;
                        if (r[0] != expect_start || r[2] != slot) return fail("pass order", U, grid, nk);
                        expect_start = r[1];
                    }
                    if (expect_start != ch * nk + nk) return fail("chain coverage", U, grid, nk);
                }
            }
    std::printf("OK %d\n", cases);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs the host C++ compiler")
def test_run_layout_invariants(tmp_path):
    src = tmp_path / "runs_check.cpp"
    exe = tmp_path / "runs_check"
    src.write_text(PROGRAM)
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-I", HEADER_DIR, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr
