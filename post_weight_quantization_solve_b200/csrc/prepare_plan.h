// Host-side plan of the factorisation and of the triangular inverse (plain C++17, no
// CUDA: the CPU tests compile it on its own).
//
// [GPTQ blog] "为什么 Cholesky Factor 不能当作原始逆矩阵": the sweep reads H^-1 through the
// upper factor U with U^T U = H^-1. The library factors H_d = V V^T with V upper from
// the bottom-right corner in diagonal blocks of CH_NB coordinates, then forms U = V^-1
// by a triangular inverse laid out as a tree over the block range: a node (a, m, b)
// splits [a, b) at m and computes the off-diagonal block U[a:m, m:b] from the two
// diagonal inverses below it, so every pair of blocks (i < j) is produced by exactly
// one node, and the nodes of one depth touch disjoint ranges.
#pragma once

#include <algorithm>
#include <cstddef>
#include <vector>

namespace gptq {

constexpr int CH_NB = 128;

struct Blocks {
    int K, T;  // T blocks; block t covers [start(t), start(t+1))
    int start(int t) const {
        // blocks are aligned to the bottom-right corner: the first may be short
        const int first = K - (T - 1) * CH_NB;
        return t == 0 ? 0 : first + (t - 1) * CH_NB;
    }
};

inline Blocks blocks_of(int K) { return Blocks{K, (K + CH_NB - 1) / CH_NB}; }

// Scratch of one depth of the inverse: the largest T^T a depth needs fits in it.
inline size_t inverse_scratch_floats(int K) {
    const int T = (K + CH_NB - 1) / CH_NB;
    const size_t half = (size_t)((T + 1) / 2) * CH_NB;
    return half * half;
}

struct InvNode {
    int a, m, b;
};

// The recursion [A B; 0 D]^-1 = [A^-1, -A^-1 B D^-1; 0, D^-1] over block ranges
// [bl, br): levels[d] holds the nodes of depth d.
inline void inv_nodes(const Blocks &bk, int K, int bl, int br, int depth,
                      std::vector<std::vector<InvNode>> &levels) {
    if (br - bl <= 1) return;
    const int mid = (bl + br) / 2;
    if ((int)levels.size() <= depth) levels.resize(depth + 1);
    levels[depth].push_back({bk.start(bl), bk.start(mid), br == bk.T ? K : bk.start(br)});
    inv_nodes(bk, K, bl, mid, depth + 1, levels);
    inv_nodes(bk, K, mid, br, depth + 1, levels);
}

// One launch round of a depth: at most max_items nodes, and the layout of their
// T^T = (R_ab U_bb)^T blocks, (b - m) x (m - a) each, stacked at a common pitch.
struct InvRound {
    std::vector<InvNode> nodes;
    std::vector<int> trow0;   // first row of each node's block
    int pitch = 0, trows = 0;
};

inline std::vector<InvRound> inv_rounds(const std::vector<InvNode> &level, int max_items) {
    std::vector<InvRound> out;
    for (size_t c0 = 0; c0 < level.size(); c0 += (size_t)max_items) {
        InvRound r;
        r.nodes.assign(level.begin() + c0,
                       level.begin() + std::min(level.size(), c0 + (size_t)max_items));
        for (const InvNode &nd : r.nodes) {
            r.pitch = std::max(r.pitch, nd.m - nd.a);
            r.trow0.push_back(r.trows);
            r.trows += nd.b - nd.m;
        }
        out.push_back(r);
    }
    return out;
}

}  // namespace gptq
