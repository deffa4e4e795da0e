// Streamed Gram / Hessian accumulation, H += 2 X^T diag(w) X, and the GPTAQ cross
// statistic C += 2 (X_fp - X_q)^T X_q.
//
// [GPTQ blog] "Calibration 让量化看见输入方向": one K x K statistic shared by every
// output channel, accumulated batch by batch; factor 2 from the two-weight example.
// [ResComp] item 3: the cross statistic dX X^T with dX = X~ - X.
//
// This file holds the fp32 SIMT path (every fp32 stream, and bf16 streams when the
// tensor-core path does not apply). Only the tiles that meet the upper triangle
// are computed; the lower triangle is mirrored afterwards.
#include "common.cuh"
#include "gemm_simt.cuh"

namespace gptq {

// H[i][j] = H[j][i] for i > j, per group.
__global__ void k_mirror_upper(float *H, int K) {
    const int g = blockIdx.z;
    H += (int64_t)g * K * K;
    // 32 x 32 tiles below the diagonal, transposed through shared memory
    const int bi = blockIdx.y, bj = blockIdx.x;
    if (bj > bi) return;
    __shared__ float t[32][33];
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int i = bj * 32 + r, j = bi * 32 + tx;  // source: upper element (i <= j)
        if (i < K && j < K) t[r][tx] = H[(int64_t)i * K + j];
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int i = bi * 32 + r, j = bj * 32 + tx;  // destination (i > j)
        if (i < K && j < K && i > j) H[(int64_t)i * K + j] = t[tx][r];
    }
}

gptq_status mirror_upper(float *H, int K, int g, cudaStream_t st) {
    const int nb = (K + 31) / 32;
    k_mirror_upper<<<dim3(nb, nb, g), dim3(32, 8), 0, st>>>(H, K);
    return launch_status();
}

gptq_status gram_simt(float *H, int K, int g, const void *X, int xdtype, int64_t M,
                      int64_t ldx, const float *w, int64_t ldw, const int32_t *status,
                      cudaStream_t st) {
    // H(i,j) += 2 sum_m X[m][i] w[m] X[m][j]: A(i,m) = X[m*ldx + i] (transposed view)
    GemmParams p = gemm_params(K, K, (int)M, X, ldx, X, ldx, H, K, 2.f, 1, status);
    p.upper_tiles = 1;
    p.kscale = w;
    p.sK = ldw;
    p.sC = (int64_t)K * K;
    gptq_status s = (xdtype == GPTQ_F32)
                        ? gemm_simt<float, float, true, false>(p, g, st)
                        : gemm_simt<__nv_bfloat16, __nv_bfloat16, true, false>(p, g, st);
    if (s != GPTQ_OK) return s;
    return mirror_upper(H, K, g, st);
}

gptq_status cross_simt(float *C, int K, const void *Xfp, const void *Xq, int xdtype, int64_t M,
                       int64_t ldx, const int32_t *status, cudaStream_t st) {
    GemmParams p = gemm_params(K, K, (int)M, Xfp, ldx, Xq, ldx, C, K, 2.f, 1, status);
    p.A2 = Xq;
    return (xdtype == GPTQ_F32) ? gemm_simt<float, float, true, false>(p, 1, st)
                                : gemm_simt<__nv_bfloat16, __nv_bfloat16, true, false>(p, 1, st);
}

}  // namespace gptq
