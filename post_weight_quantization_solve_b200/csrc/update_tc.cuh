// Shared declarations of the tensor-core lazy update (update_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace gptq {

// Product group g uses A operands a[2g] (hi), a[2g+1] (lo) and B operands b[2g],
// b[2g+1]: group 0 is E with U, group 1 (GPTAQ) the pre-rounding weights with P1.
struct UpdateMaps {
    CUtensorMap a[4];   // A operands: [rows j][n] bf16 (a_kmajor: [rows n][j], 64 x 128 boxes)
    CUtensorMap b[4];   // B operands: [rows j][k], bf16
};

struct UpdateParams {
    float *C;
    int64_t ldc;
    int M, Ncols, L;        // output rows, output columns, inner rows (multiple of 16)
    int a_x0, a_y0;         // A: column (n) origin, row (j) origin
    int b_x0, b_y0;         // B: column (k) origin, row (j) origin
    int ngroups;            // 1, or 2 with the GPTAQ group
    int neg[2];             // subtract group g's product
    int vec4;               // C rows 16-byte aligned: float4 reductions
    int a_kmajor;           // A stored with the channel index as rows (k contiguous); L % 64 == 0
    int64_t c_extent;       // elements addressable from C (0: not given; index-checking build)
    int32_t *status;
};

bool update_tc_available();
gptq_status make_bf16_map(CUtensorMap *m, const void *base, int64_t cols, int64_t rows,
                          int64_t ld, int box_rows);
gptq_status launch_update_tc(const UpdateMaps &maps, const UpdateParams &p, int box_rows,
                             cudaStream_t st);
gptq_status split_bf16(const float *in, int64_t ld_in, int rows, int cols, __nv_bfloat16 *hi,
                       __nv_bfloat16 *lo, int64_t ld_out, int batch, int64_t batch_in,
                       int64_t batch_out, cudaStream_t st);

}  // namespace gptq
