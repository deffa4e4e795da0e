"""The far-update schedule behind the tensor-core sweep, compiled as plain C++ on the CPU
(no GPU).

csrc/update_plan.h is the schedule gptq_quantize_layer runs: super-blocks of S
coordinates (512, or 256 with the GPTAQ row term), and far updates by pairs of
super-blocks. A C++ program checks, for every K the tensor-core sweep takes (multiples
of 4) up to 20,000 and beyond, with both super-block lengths:
  - the errors of each coordinate reach each column of a later super-block exactly once
    ([GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": a block's errors reach everything
    after it through the delayed product), and never a column of its own or an earlier
    super-block;
  - when super-block m's sweep starts, its columns hold the errors of every super-block
    before m (each update runs after the sweep named in `after`, before the next sweep);
  - an update's errors are whole super-blocks starting at an even one, read from E column 0:
    its inner length is S or 2S, a multiple of 64 (the update's K-major A boxes), the
    super-blocks it reads wrote their errors at columns 0 and S (sweep_error_column), and
    2S fits the E rows' pitch of 1024.
"""

import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "post_weight_quantization_solve_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "update_plan.h"
using namespace gptq;

static int check(int K, int S) {
    const int nsb = (K + S - 1) / S;
    auto sb_of = [&](int x) { return x / S; };
    const std::vector<FarUpdate> plan = far_update_plan(K, S);
    // coverage[(super-block of the errors) * nsb + super-block of the column] counted per
    // (error coordinate, column) pair, checked as whole super-block pairs
    std::vector<long long> cover((size_t)nsb * nsb, 0);
    int last_after = -1;
    for (const FarUpdate &u : plan) {
        if (u.after < last_after) return 1;              // in sweep order
        last_after = u.after;
        if (u.after < 0 || u.after >= nsb - 1) return 2;  // never after the last sweep
        if (!(0 <= u.k0 && u.k0 < u.k1 && u.k1 <= K)) return 3;
        if (!(u.col0 < u.col1 && u.col1 <= K)) return 4;
        const int L = u.k1 - u.k0;
        if (L % 64 != 0 || (L != S && L != 2 * S) || L > 1024) return 5;
        if (u.k0 % S != 0 || sb_of(u.k0) % 2 != 0) return 6;   // starts at an even super-block
        // the E rows: the super-blocks read are at columns 0 (and S), as the sweep wrote them
        for (int i = sb_of(u.k0); i <= sb_of(u.k1 - 1); ++i)
            if (sweep_error_column(i, S) != (i - sb_of(u.k0)) * S) return 7;
        // the errors applied come from sweeps already run
        if (sb_of(u.k1 - 1) > u.after) return 8;
        // the columns lie after the errors' super-blocks
        if (sb_of(u.col0) <= sb_of(u.k1 - 1)) return 9;
        for (int i = sb_of(u.k0); i <= sb_of(u.k1 - 1); ++i)
            for (int c = u.col0; c < u.col1; ++c) cover[(size_t)i * nsb + sb_of(c)]++;
    }
    // every (error super-block i, column super-block m > i) pair once per column of m
    for (int i = 0; i < nsb; ++i)
        for (int m = 0; m < nsb; ++m) {
            const long long cols = std::min(K, (m + 1) * S) - m * S;
            const long long want = m > i ? cols : 0;
            if (cover[(size_t)i * nsb + m] != want) return 10;
        }
    // before sweep m: every update touching m's columns with errors of i < m ran earlier
    for (int m = 1; m < nsb; ++m)
        for (int i = 0; i < m; ++i) {
            long long before = 0;
            for (const FarUpdate &u : plan) {
                if (u.after >= m) continue;
                if (sb_of(u.k0) > i || sb_of(u.k1 - 1) < i) continue;
                const int a = std::max(u.col0, m * S), b = std::min(u.col1, std::min(K, (m + 1) * S));
                if (b > a) before += b - a;
            }
            if (before != std::min(K, (m + 1) * S) - m * S) return 11;
        }
    return 0;
}

int main() {
    int bad = 0;
    for (int S : {512, 256}) {
        for (int K = 4; K <= 20000; K += 4) {
            const int r = check(K, S);
            if (r) { std::printf("K=%d S=%d fails %d\n", K, S, r); if (++bad > 10) return 1; }
        }
        for (int K : {28672, 28704, 65504}) {
            const int r = check(K, S);
            if (r) { std::printf("K=%d S=%d fails %d\n", K, S, r); ++bad; }
        }
    }
    if (!bad) std::printf("ok\n");
    return bad ? 1 : 0;
}
"""


def test_far_update_plan(tmp_path):
    src = tmp_path / "plan.cpp"
    exe = tmp_path / "plan"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
