// Host-side schedule of the far updates behind the tensor-core sweep (plain C++, no CUDA,
// so that a CPU test can check it).
//
// [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": the errors of a block of coordinates reach
// the coordinates after it through one delayed (lazy) product. The sweep runs super-blocks
// of S coordinates; the errors of super-block i must reach every column after it, and the
// columns of super-block m must hold the errors of every super-block before m when m's
// sweep starts. Far updates go by pairs of super-blocks: after an even super-block only
// the next super-block's columns take its errors; after the odd one every column after the
// pair takes both super-blocks' errors as one product (inner length 2S), so the rest of W
// is read and written once per pair. The E rows hold a pair side by side: super-block i
// writes its errors at column (i % 2) S of them.
#pragma once

#include <algorithm>
#include <vector>

namespace gptq {

// One far update, launched after the sweep of super-block `after`.
struct FarUpdate {
    int after;          // super-block whose sweep precedes it
    int col0, col1;     // columns of W it updates
    int k0, k1;         // coordinates whose errors it applies (U rows), from E column 0
};

// Column of the E rows at which super-block i writes its errors.
inline int sweep_error_column(int i, int S) { return (i & 1) * S; }

inline std::vector<FarUpdate> far_update_plan(int K, int S) {
    std::vector<FarUpdate> plan;
    for (int i = 0, sb0 = 0; sb0 < K; sb0 += S, ++i) {
        const int sb1 = std::min(K, sb0 + S);
        if (sb1 >= K) break;                      // nothing after the last super-block
        if (i & 1)
            plan.push_back({i, sb1, K, sb0 - S, sb1});
        else
            plan.push_back({i, sb1, std::min(K, sb1 + S), sb0, sb1});
    }
    return plan;
}

}  // namespace gptq
