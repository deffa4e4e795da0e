// gptq_first_order_shift: the first-order (gradient) term of the compensation as a
// shifted starting point, W <- W - beta G H^-1 with H^-1 = U^T U.
//
// [G2PTQ] summary: the compensation keeps GPTQ's second-order update and adds the
// first-order term of an exact gradient G, scaled by a trust-region factor beta. The
// pages print no formula; the reading taken: per output channel the objective is the
// quadratic model beta g^T d + 1/2 d^T H d around the given weights, and sequential
// OBQ on that model is GPTQ started from its minimiser w - beta H^-1 g (each later
// step keeps the free coordinates at the model's conditional minimiser, which is what
// GPTQ's update does once the start is that minimiser). So the term costs one shift
// before the sweep:
//   T = G U^T        (N x K: the gradient in the factor's coordinates)
//   W -= beta T U    (U upper triangular: only k >= j contributes)
//   gamma = sum T^2 = sum_n g_n H^-1 g_n^T (the model's loss change along the step is
//                    -(beta - beta^2 / 2) gamma, which the trust region bounds)
// Both products run on the fp32 tiled GEMM (exact fp32 accumulation; the shift moves
// the values the sweep rounds, so it is kept at the working precision).
#include "common.cuh"
#include "gemm_simt.cuh"

namespace gptq {

// sum of squares of n floats into a double (one atomic per CTA)
__global__ void __launch_bounds__(256) k_sum_squares(const float *__restrict__ x, int64_t n,
                                                     double *out, const int32_t *status) {
    if (failed(status)) return;
    double acc = 0.0;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
        const double v = x[i];
        acc += v * v;
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ double red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int i = 0; i < 8; ++i) t += red[i];
        atomicAdd(out, t);
    }
}

size_t first_order_workspace(int K, int N) { return round_up((size_t)N * K * sizeof(float), 256); }

gptq_status first_order_shift(float *W, int N, int K, const float *U, const void *G, int gdtype,
                              float beta, double *gamma, void *ws, int32_t *status,
                              cudaStream_t st) {
    float *T = static_cast<float *>(ws);
    // T = G U^T: T[n][j] = sum_k G[n][k] U[j][k]
    GemmParams p1 = gemm_params(N, K, K, G, K, U, K, T, K, 1.f, 0, status);
    gptq_status s = (gdtype == GPTQ_F32) ? gemm_simt<float, float, false, true>(p1, 1, st)
                                         : gemm_simt<__nv_bfloat16, float, false, true>(p1, 1, st);
    if (s != GPTQ_OK) return s;
    if (gamma) {
        if (cudaMemsetAsync(gamma, 0, sizeof(double), st) != cudaSuccess) return GPTQ_ERR_CUDA;
        k_sum_squares<<<592, 256, 0, st>>>(T, (int64_t)N * K, gamma, status);
        if ((s = launch_status()) != GPTQ_OK) return s;
    }
    // W -= beta T U: W[n][k] -= beta sum_{j <= k} T[n][j] U[j][k]
    GemmParams p2 = gemm_params(N, K, K, T, K, U, K, W, K, -beta, 1, status);
    p2.b_upper = 1;
    return gemm_simt<float, float, false, false>(p2, 1, st);
}

}  // namespace gptq
