// Shared declarations of the fp32-accurate tensor-core GEMM (gemm_tc32.cu).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace gptq {

constexpr int TC32_MAX_ITEMS = 96;

// One product of a launch. Both operands are K-major tf32 pairs: A origin
// (x = k index, y = row i), B origin (x = k index, y = column j, i.e. B is stored as
// B^T rows), C = p.C + c_off with row pitch ldc.
struct Tc32Item {
    int m, n, k;
    int a_x0, a_y0, b_x0, b_y0;
    int parts, unit0;       // filled by launch_gemm_tc32
    int64_t c_off, ldc;
};

struct Tc32Params {
    float *C;
    float alpha;
    int accumulate;         // C += alpha AB (else C = alpha AB; split items need C zeroed first)
    int upper_tiles, a_upper, b_upper, mask_strict_upper;
    int a_lower;            // A(i,k) == 0 for k > i: the k range ends at the row tile
    int b_lower;            // B(k,j) == 0 for k < j: the k range starts at the column tile
    int nitems, units;
    int max_grid;           // > 0: at most this many CTAs (leaves SMs to other streams)
    int pdl;                // launch as a programmatic dependent of the stream's previous kernel
    // Optional (one item, overwrite mode, unsplit inner range): the stored values also
    // as tf32 pairs, element (i, j) of the item at pair_hi / pair_lo[i * pair_ld + j].
    float *pair_hi, *pair_lo;
    int64_t pair_ld;
    // Elements addressable from C and from each pair array (0: not given); the
    // index-checking build skips any store beyond them.
    int64_t c_extent, pair_extent;
    int32_t *status;
    Tc32Item item[TC32_MAX_ITEMS];
};

bool tc32_available();
gptq_status make_f32_map(CUtensorMap *m, const float *base, int64_t cols, int64_t rows, int64_t ld,
                         int box_cols, int box_rows);
gptq_status split_tf32(const float *in, int64_t ld_in, int rows, int cols, float *hi, float *lo,
                       int64_t ld_out, int batch, int64_t batch_in, int64_t batch_out,
                       cudaStream_t st);
gptq_status split_tf32_t(const float *in, int64_t ld_in, int rows, int cols, float *hi, float *lo,
                         int64_t ld_out, int batch, int64_t batch_in, int64_t batch_out,
                         cudaStream_t st);
gptq_status launch_gemm_tc32(const CUtensorMap maps[4], Tc32Params &p, cudaStream_t st);
int tc32_sms();

}  // namespace gptq
