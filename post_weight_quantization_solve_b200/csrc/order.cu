// act-order: the processing order of the input coordinates and the reordered
// Hessian (or cross statistic).
//
// [GPTQ blog] "Damping 与两个不同的分组参数": act-order reorders the input coordinates
// by the Hessian diagonal from large to small (an ordering heuristic); the
// coordinates are restored after quantisation. Ties keep the lower index first.
#include "common.cuh"

namespace gptq {

// perm[rank(k)] = k with rank(k) = #{i : d_i > d_k or (d_i == d_k and i < k)}; the
// diagonal is walked in shared-memory tiles.
__global__ void k_act_order(const float *__restrict__ H, int K, int32_t *__restrict__ perm) {
    __shared__ float tile[1024];
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    const float dk = k < K ? H[(int64_t)k * K + k] : 0.f;
    int rank = 0;
    for (int t0 = 0; t0 < K; t0 += 1024) {
        __syncthreads();
        for (int i = threadIdx.x; i < 1024; i += blockDim.x)
            tile[i] = (t0 + i < K) ? H[(int64_t)(t0 + i) * K + t0 + i] : 0.f;
        __syncthreads();
        const int n = min(1024, K - t0);
        for (int i = 0; i < n; ++i) {
            const float di = tile[i];
            rank += (di > dk) || (di == dk && t0 + i < k);
        }
    }
    if (k < K) perm[rank] = k;
}

// out[i][j] = H[perm[i]][perm[j]]; 32 x 32 output tiles, rows of H gathered.
__global__ void k_permute_square(float *__restrict__ out, const float *__restrict__ H, int K,
                                 const int32_t *__restrict__ perm) {
    const int j = blockIdx.x * 32 + threadIdx.x;
    const int pj = j < K ? perm[j] : 0;
    for (int r = threadIdx.y; r < 32; r += 8) {
        const int i = blockIdx.y * 32 + r;
        if (i < K && j < K) out[(int64_t)i * K + j] = H[(int64_t)perm[i] * K + pj];
    }
}

gptq_status act_order(const float *H, int K, int32_t *perm, cudaStream_t st) {
    k_act_order<<<(K + 255) / 256, 256, 0, st>>>(H, K, perm);
    return launch_status();
}

gptq_status permute_square(float *out, const float *H, int K, const int32_t *perm,
                           cudaStream_t st) {
    k_permute_square<<<dim3((K + 31) / 32, (K + 31) / 32), dim3(32, 8), 0, st>>>(out, H, K, perm);
    return launch_status();
}

}  // namespace gptq
