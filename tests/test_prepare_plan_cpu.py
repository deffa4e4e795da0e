"""The factorisation's host-side plan, compiled as plain C++ on the CPU (no GPU).

csrc/prepare_plan.h is the plan the library's prepare runs: the diagonal blocks of the
factorisation and the tree of the triangular inverse U = V^-1, cut into launch rounds
of at most one item table. A C++ program checks, for every K the tensor-core path
takes up to the ABI's largest (multiples of 32 from 256 to 65,504) and for ragged K:
  - the blocks partition [0, K), each CH_NB wide but the first;
  - every pair of blocks (i < j) is produced by exactly one node of the tree, and
    that node splits them (i below its split point, j above), so the inverse fills
    every off-diagonal block once;
  - the nodes of one depth touch disjoint ranges (they may run in one launch);
  - a depth's rounds hold at most the item-table size, cover its nodes in order, and
    each round's T^T fits the depth scratch the workspace reserves.
"""

import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "post_weight_quantization_solve_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "prepare_plan.h"
using namespace gptq;

static int check(int K, int max_items) {
    const Blocks bk = blocks_of(K);
    // blocks partition [0, K)
    if (bk.start(0) != 0) return 1;
    for (int t = 0; t < bk.T; ++t) {
        const int a = bk.start(t), b = t + 1 < bk.T ? bk.start(t + 1) : K;
        if (b <= a) return 2;
        if (t > 0 && b - a != CH_NB) return 3;
        if (t == 0 && b - a > CH_NB) return 4;
    }
    std::vector<std::vector<InvNode>> levels;
    inv_nodes(bk, K, 0, bk.T, 0, levels);
    // block index of a coordinate
    auto blk = [&](int x) { int t = 0; while (t + 1 < bk.T && bk.start(t + 1) <= x) ++t; return t; };
    std::vector<int> seen((size_t)bk.T * bk.T, 0);
    const size_t tsz = inverse_scratch_floats(K);
    for (const auto &lv : levels) {
        // disjoint ranges within a depth
        for (size_t i = 0; i < lv.size(); ++i)
            for (size_t j = i + 1; j < lv.size(); ++j)
                if (!(lv[i].b <= lv[j].a || lv[j].b <= lv[i].a)) return 5;
        for (const InvNode &nd : lv) {
            if (!(nd.a < nd.m && nd.m < nd.b)) return 6;
            for (int i = blk(nd.a); i < blk(nd.m); ++i)
                for (int j = blk(nd.m); j <= blk(nd.b - 1); ++j) seen[(size_t)i * bk.T + j]++;
        }
        // rounds
        const std::vector<InvRound> rounds = inv_rounds(lv, max_items);
        size_t k = 0;
        for (const InvRound &r : rounds) {
            if (r.nodes.empty() || (int)r.nodes.size() > max_items) return 7;
            int rows = 0;
            for (size_t n = 0; n < r.nodes.size(); ++n, ++k) {
                const InvNode &nd = r.nodes[n];
                if (k >= lv.size() || nd.a != lv[k].a || nd.m != lv[k].m || nd.b != lv[k].b) return 8;
                if (r.trow0[n] != rows || nd.m - nd.a > r.pitch) return 9;
                rows += nd.b - nd.m;
            }
            if (rows != r.trows || (size_t)r.trows * r.pitch > tsz) return 10;
        }
        if (k != lv.size()) return 11;
    }
    for (int i = 0; i < bk.T; ++i)
        for (int j = 0; j < bk.T; ++j)
            if (seen[(size_t)i * bk.T + j] != (i < j ? 1 : 0)) return 12;
    return 0;
}

int main() {
    int bad = 0, count = 0, max_round = 0;
    std::vector<int> Ks;
    for (int K = 256; K <= 65504; K += 32) Ks.push_back(K);
    const int ragged[] = {1, 2, 100, 127, 128, 129, 200, 255, 300, 4097, 14335, 28673};
    for (int K : ragged) Ks.push_back(K);
    for (int K : Ks) {
        const int rc = check(K, 96);
        ++count;
        if (rc) { std::printf("K=%d code %d\n", K, rc); ++bad; }
        std::vector<std::vector<InvNode>> levels;
        inv_nodes(blocks_of(K), K, 0, blocks_of(K).T, 0, levels);
        for (const auto &lv : levels)
            for (const InvRound &r : inv_rounds(lv, 96)) max_round = r.nodes.size() > (size_t)max_round ? (int)r.nodes.size() : max_round;
    }
    std::vector<std::vector<InvNode>> l28;
    inv_nodes(blocks_of(28672), 28672, 0, blocks_of(28672).T, 0, l28);
    size_t one_round = 0;
    for (const auto &lv : l28) one_round += inv_rounds(lv, 96).size() == 1;
    std::printf("checked %d bad %d max_round %d k28672_single_round_levels %zu of %zu\n", count, bad,
                max_round, one_round, l28.size());
    return bad ? 1 : 0;
}
"""


def test_prepare_plan(tmp_path):
    src = tmp_path / "plan.cc"
    src.write_text(PROGRAM)
    exe = tmp_path / "plan"
    cc = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Wextra", "-Werror", "-I", CSRC,
                         str(src), "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    out = run.stdout.split()
    assert out[0] == "checked" and int(out[1]) > 2000 and out[3] == "0"
    assert int(out[5]) == 96                      # the largest K needs full item tables
    # up to K = 28,672 every depth is a single round: the launches are one per depth
    assert out[7] == out[9]
