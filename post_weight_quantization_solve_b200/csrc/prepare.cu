// gptq_prepare: dead coordinates, damping, and the upper factor U with
// U^T U = H^-1, computed without forming H^-1.
//
// [GPTQ blog] "Damping 与两个不同的分组参数": dead coordinates (H_kk == 0) get
// their diagonal adjusted (to 1 here), then H += percdamp * mean(diag H) * I.
// [GPTQ blog] "为什么 Cholesky Factor 不能当作原始逆矩阵": GPTQ reads H^-1 through
// the upper triangular U with U^T U = H^-1.
//
// Route: H = R R^T with R upper triangular (a Cholesky factorisation that runs from
// the last coordinate to the first), then U = R^-1, since
// U^T U = R^-T R^-1 = (R R^T)^-1 = H^-1 and the upper factor with a positive
// diagonal is unique. Cost 1/3 K^3 + 1/3 K^3 multiply-adds.
//
// Blocked, NB coordinates per diagonal block, blocks taken from the bottom-right:
//   diag   : R_JJ R_JJ^T = H_JJ, and U_JJ = R_JJ^-1, in one CTA (shared memory)
//   panel  : R[0:j0, J] = H[0:j0, J] U_JJ^T
//   update : H[0:j0, 0:j0] -= R[0:j0, J] R[0:j0, J]^T   (upper tiles only)
// then the recursive triangular inverse
//   [A B; 0 D]^-1 = [A^-1, -A^-1 B D^-1; 0, D^-1]
// over the same block boundaries, whose leaves U_JJ the diag kernel already wrote.
#include <float.h>

#include "common.cuh"
#include "gemm_simt.cuh"

namespace gptq {

constexpr int CH_NB = 128;
constexpr int CH_THREADS = 512;
constexpr int CH_LD = CH_NB + 1;

__global__ void k_check_finite(const float *A, int64_t count, int32_t *status) {
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    bool bad = false;
    for (; i < count; i += stride) bad |= !isfinite(A[i]);
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(status, GPTQ_ERR_NONFINITE);
}

// One CTA per group: dead fix, damping, the damped diagonal kept for pivot tests.
__global__ void k_dead_damp(float *H, int K, float percdamp, uint8_t *dead_out, float *diag_d,
                            int32_t *status) {
    if (failed(status)) return;
    const int g = blockIdx.x;
    H += (int64_t)g * K * K;
    __shared__ double red[32];
    double sum = 0.0;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float d = H[(int64_t)k * K + k];
        sum += (d == 0.f) ? 1.0 : (double)d;
    }
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float damp = (float)((double)percdamp * red[0] / K);
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float d = H[(int64_t)k * K + k];
        const bool dead = d == 0.f;
        const float v = (dead ? 1.f : d) + damp;
        H[(int64_t)k * K + k] = v;
        diag_d[(int64_t)g * K + k] = v;
        if (dead_out) dead_out[(int64_t)g * K + k] = dead ? 1 : 0;
    }
}

// Factor one diagonal block H[J,J] (J = [j0, j0+nb)) as R R^T (R upper), then
// replace it by U_JJ = R^-1 (upper, strict lower zeroed). One CTA per group.
__global__ void __launch_bounds__(CH_THREADS) k_chol_diag(float *H, int K, int j0, int nb,
                                                          const float *diag_d, float tol,
                                                          int32_t *status) {
    if (failed(status)) return;
    const int g = blockIdx.x;
    H += (int64_t)g * K * K;
    diag_d += (int64_t)g * K;
    extern __shared__ float S[];  // [CH_NB][CH_LD]
    float *tmp = S + CH_NB * CH_LD;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = CH_THREADS / 32;
    for (int idx = tid; idx < nb * nb; idx += CH_THREADS) {
        const int r = idx / nb, c = idx % nb;
        S[r * CH_LD + c] = (r <= c) ? H[(int64_t)(j0 + r) * K + j0 + c]
                                    : H[(int64_t)(j0 + c) * K + j0 + r];
    }
    __syncthreads();
    // R R^T factorisation, last column first (upper triangle of S holds R).
    for (int j = nb - 1; j >= 0; --j) {
        if (tid == 0) {
            const float d = S[j * CH_LD + j];
            if (!(d > tol * diag_d[j0 + j])) set_status(status, GPTQ_ERR_NOT_PD);
            S[j * CH_LD + j] = sqrtf(fmaxf(d, FLT_MIN));
        }
        __syncthreads();
        const float r = S[j * CH_LD + j];
        for (int i = tid; i < j; i += CH_THREADS) S[i * CH_LD + j] = S[i * CH_LD + j] / r;
        __syncthreads();
        for (int i = warp; i < j; i += nwarps) {
            const float sij = S[i * CH_LD + j];
            for (int k = i + lane; k < j; k += 32) S[i * CH_LD + k] -= sij * S[k * CH_LD + j];
        }
        __syncthreads();
    }
    // In-place inverse of the upper triangular R, column by column:
    // U_jj = 1/R_jj, U[0:j, j] = -U_jj * U[0:j, 0:j] R[0:j, j].
    for (int j = 0; j < nb; ++j) {
        for (int k = tid; k < j; k += CH_THREADS) tmp[k] = S[k * CH_LD + j];
        __syncthreads();
        const float ujj = 1.f / S[j * CH_LD + j];
        for (int i = warp; i < j; i += nwarps) {
            float acc = 0.f;
            for (int k = i + lane; k < j; k += 32) acc += S[i * CH_LD + k] * tmp[k];
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) S[i * CH_LD + j] = -ujj * acc;
        }
        __syncthreads();
        if (tid == 0) S[j * CH_LD + j] = ujj;
        __syncthreads();
    }
    for (int idx = tid; idx < nb * nb; idx += CH_THREADS) {
        const int r = idx / nb, c = idx % nb;
        H[(int64_t)(j0 + r) * K + j0 + c] = (r <= c) ? S[r * CH_LD + c] : 0.f;
    }
}

__global__ void k_zero_lower(float *H, int K) {
    const int g = blockIdx.z;
    H += (int64_t)g * K * K;
    const int i = blockIdx.y;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < i; j += gridDim.x * blockDim.x)
        H[(int64_t)i * K + j] = 0.f;
}

struct Blocks {
    int K, T;  // T blocks; block t covers [start(t), start(t+1))
    int start(int t) const {
        // blocks are aligned to the bottom-right corner: the first may be short
        const int first = K - (T - 1) * CH_NB;
        return t == 0 ? 0 : first + (t - 1) * CH_NB;
    }
};

static size_t inverse_scratch_floats(int K) {
    const int T = (K + CH_NB - 1) / CH_NB;
    const size_t half = (size_t)((T + 1) / 2) * CH_NB;
    return half * half;
}

// Off-diagonal blocks of U = R^-1 over blocks [bl, br).
static gptq_status tri_inverse(float *H, int K, int g, const Blocks &bk, int bl, int br,
                               float *T, const int32_t *status, cudaStream_t st) {
    if (br - bl <= 1) return GPTQ_OK;
    const int mid = (bl + br) / 2;
    gptq_status s = tri_inverse(H, K, g, bk, bl, mid, T, status, st);
    if (s != GPTQ_OK) return s;
    s = tri_inverse(H, K, g, bk, mid, br, T, status, st);
    if (s != GPTQ_OK) return s;
    const int a = bk.start(bl), m = bk.start(mid), b = (br == bk.T) ? K : bk.start(br);
    const int64_t KK = (int64_t)K * K;
    const int64_t tsz = (int64_t)inverse_scratch_floats(K);
    // T = R[a:m, m:b] * U[m:b, m:b]   (U block upper triangular)
    GemmParams p1 = gemm_params(m - a, b - m, b - m, H + (int64_t)a * K + m, K,
                                H + (int64_t)m * K + m, K, T, b - m, 1.f, 0, status);
    p1.b_upper = 1;
    p1.sA = KK; p1.sB = KK; p1.sC = tsz;
    if ((s = gemm_simt<float, float, false, false>(p1, g, st)) != GPTQ_OK) return s;
    // U[a:m, m:b] = -U[a:m, a:m] * T
    GemmParams p2 = gemm_params(m - a, b - m, m - a, H + (int64_t)a * K + a, K, T, b - m,
                                H + (int64_t)a * K + m, K, -1.f, 0, status);
    p2.a_upper = 1;
    p2.sA = KK; p2.sB = tsz; p2.sC = KK;
    return gemm_simt<float, float, false, false>(p2, g, st);
}

size_t prepare_workspace(int K, int g) {
    Carver c(nullptr);
    c.take<float>((size_t)g * K);
    c.take<float>((size_t)g * inverse_scratch_floats(K));
    return round_up(c.off, 256);
}

gptq_status prepare(float *H, int K, int g, float percdamp, uint8_t *dead_out, void *ws,
                    int32_t *status, cudaStream_t st) {
    Carver c(ws);
    float *diag_d = c.take<float>((size_t)g * K);
    float *T = c.take<float>((size_t)g * inverse_scratch_floats(K));
    const int64_t KK = (int64_t)K * K;

    k_check_finite<<<592, 256, 0, st>>>(H, KK * g, status);
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    k_dead_damp<<<g, 1024, 0, st>>>(H, K, percdamp, dead_out, diag_d, status);
    if ((s = launch_status()) != GPTQ_OK) return s;

    const size_t smem = (size_t)(CH_NB * CH_LD + CH_NB) * sizeof(float);
    cudaFuncSetAttribute(k_chol_diag, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const float tol = (float)K * FLT_EPSILON;
    Blocks bk{K, (K + CH_NB - 1) / CH_NB};
    for (int t = bk.T - 1; t >= 0; --t) {
        const int j0 = bk.start(t);
        const int j1 = (t == bk.T - 1) ? K : bk.start(t + 1);
        const int nb = j1 - j0;
        k_chol_diag<<<g, CH_THREADS, smem, st>>>(H, K, j0, nb, diag_d, tol, status);
        if ((s = launch_status()) != GPTQ_OK) return s;
        if (j0 == 0) break;
        // panel: R[0:j0, J] = H[0:j0, J] U_JJ^T  (in place: each CTA owns whole rows)
        GemmParams pp = gemm_params(j0, nb, nb, H + j0, K, H + (int64_t)j0 * K + j0, K,
                                    H + j0, K, 1.f, 0, status);
        pp.sA = KK; pp.sB = KK; pp.sC = KK;
        if ((s = gemm_simt<float, float, false, true>(pp, g, st)) != GPTQ_OK) return s;
        // trailing update of the upper triangle: H11 -= R12 R12^T
        GemmParams ps = gemm_params(j0, j0, nb, H + j0, K, H + j0, K, H, K, -1.f, 1, status);
        ps.upper_tiles = 1;
        ps.sA = KK; ps.sB = KK; ps.sC = KK;
        if ((s = gemm_simt<float, float, false, true>(ps, g, st)) != GPTQ_OK) return s;
    }
    // The strict lower triangle still holds the input and update leftovers; the
    // inverse reads whole tiles of its triangular operands, so clear it first.
    k_zero_lower<<<dim3((K + 255) / 256 > 8 ? 8 : (K + 255) / 256, K, g), 256, 0, st>>>(H, K);
    if ((s = launch_status()) != GPTQ_OK) return s;
    return tri_inverse(H, K, g, bk, 0, bk.T, T, status, st);
}

}  // namespace gptq
