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
// Both products run as tf32x3 tensor-core GEMMs (every operand a tf32 hi + lo pair,
// three MMAs per step, ~2^-22 relative: the shift moves the values the sweep rounds, so
// it is kept near fp32 accuracy), with the structure of U used on both: T needs only
// k >= j of U's row j, the update only j <= k. Sizes the tensor-core kernel does not
// take (K not a multiple of 32, or below 256) run on the fp32 tiled SIMT GEMM.
#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc32.cuh"

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

static bool first_order_tc_eligible(int K) { return K % 32 == 0 && K >= 256; }

// T, plus on the tensor-core path the tf32 pairs of G (then of T) and of U and U^T
size_t first_order_workspace(int K, int N) {
    const size_t nk = (size_t)N * K, kk = (size_t)K * K;
    return round_up((first_order_tc_eligible(K) ? 3 * nk + 4 * kk : nk) * sizeof(float), 256);
}

__global__ void k_bf16_to_f32(const __nv_bfloat16 *__restrict__ in, float *__restrict__ out,
                              int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256)
        out[i] = __bfloat162float(in[i]);
}

static gptq_status first_order_tc(float *W, int N, int K, const float *U, const void *G,
                                  int gdtype, float beta, double *gamma, float *ws,
                                  int32_t *status, cudaStream_t st) {
    const int64_t NK = (int64_t)N * K, KK = (int64_t)K * K;
    float *T = ws, *Ah = T + NK, *Al = Ah + NK, *Uh = Al + NK, *Ul = Uh + KK, *Vh = Ul + KK,
          *Vl = Vh + KK;
    gptq_status s;
    const float *Gf = static_cast<const float *>(G);
    if (gdtype != GPTQ_F32) {       // bf16 -> fp32 (exact) through T, split below
        k_bf16_to_f32<<<592, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(G), T, NK);
        if ((s = launch_status()) != GPTQ_OK) return s;
        Gf = T;
    }
    if ((s = split_tf32(Gf, K, N, K, Ah, Al, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    if ((s = split_tf32(U, K, K, K, Uh, Ul, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    if ((s = split_tf32_t(U, K, K, K, Vh, Vl, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    static thread_local Tc32Params p;
    CUtensorMap m[4];
    // T = G U^T: A = rows of G, B^T = rows of U (U[j][k] = 0 for k < j)
    if ((s = make_f32_map(&m[0], Ah, K, N, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[1], Al, K, N, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[2], Uh, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[3], Ul, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if (cudaMemsetAsync(T, 0, sizeof(float) * (size_t)NK, st) != cudaSuccess) return GPTQ_ERR_CUDA;
    p = Tc32Params{};
    p.C = T; p.alpha = 1.f; p.accumulate = 1; p.b_lower = 1; p.status = status;
    p.c_extent = NK;
    p.nitems = 1;
    p.item[0].m = N; p.item[0].n = K; p.item[0].k = K;
    p.item[0].c_off = 0; p.item[0].ldc = K;
    if ((s = launch_gemm_tc32(m, p, st)) != GPTQ_OK) return s;
    if (gamma) {
        if (cudaMemsetAsync(gamma, 0, sizeof(double), st) != cudaSuccess) return GPTQ_ERR_CUDA;
        k_sum_squares<<<592, 256, 0, st>>>(T, NK, gamma, status);
        if ((s = launch_status()) != GPTQ_OK) return s;
    }
    // W -= beta T U: A = rows of T, B^T = rows of U^T (U[j][k] = 0 for j > k)
    if ((s = split_tf32(T, K, N, K, Ah, Al, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[2], Vh, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[3], Vl, K, K, K, 32, 128)) != GPTQ_OK) return s;
    p = Tc32Params{};
    p.C = W; p.alpha = -beta; p.accumulate = 1; p.b_upper = 1; p.status = status;
    p.c_extent = NK;
    p.nitems = 1;
    p.item[0].m = N; p.item[0].n = K; p.item[0].k = K;
    p.item[0].c_off = 0; p.item[0].ldc = K;
    return launch_gemm_tc32(m, p, st);
}

gptq_status first_order_shift(float *W, int N, int K, const float *U, const void *G, int gdtype,
                              float beta, double *gamma, void *ws, int32_t *status,
                              cudaStream_t st) {
    if (first_order_tc_eligible(K) && tc32_available() && aligned(W, 16) && aligned(U, 16))
        return first_order_tc(W, N, K, U, G, gdtype, beta, gamma, static_cast<float *>(ws), status,
                              st);
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
