// Tiled fp32 SIMT GEMM used by the factorisation (SYRK, panel solves, triangular
// inversion), the GPTAQ residual and the fp32-input Gram.
//
//   C[i][j] = (accumulate ? C[i][j] : 0) + alpha * sum_k A(i,k) B(k,j)
//   A(i,k) = A_T ? A[k*lda + i] : A[i*lda + k]      (optionally minus A2(i,k),
//                                                     times kscale[k])
//   B(k,j) = B_T ? B[j*ldb + k] : B[k*ldb + j]
//
// 128 x 128 output tile per CTA, k-steps of 8 staged through double-buffered
// shared memory, 8 x 8 outputs per thread. Structural options skip work that is
// known to be zero: upper-only output tiles, A upper triangular (A(i,k) = 0 for
// k < i) and B upper triangular (B(k,j) = 0 for k > j). An epilogue mask can keep
// only the strict upper part (j > i) and write zeros elsewhere.
#pragma once

#include "common.cuh"

namespace gptq {

struct GemmParams {
    int m, n, k;
    const void *A;
    const void *A2;  // optional: A(i,k) - A2(i,k), same layout as A
    int64_t lda;
    const void *B;
    int64_t ldb;
    float *C;
    int64_t ldc;
    float alpha;
    int accumulate;
    const float *kscale;  // optional per-k multiplier of A
    int upper_tiles;      // compute only tiles that meet j >= i
    int a_upper;          // A(i,k) == 0 for k < i
    int b_upper;          // B(k,j) == 0 for k > j
    int mask_strict_upper;  // write alpha*acc for j > i, 0 for j <= i
    int64_t sA, sA2, sB, sC, sK;  // batch strides (gridDim.z)
    const int32_t *status;
};

constexpr int GB_M = 128, GB_N = 128, GB_K = 8, G_THREADS = 256;

// One 128 x 128 output tile (rows i0.., columns j0..) of the product described by p,
// with A, A2, B, C, ks already offset to this product.
template <typename TA, typename TB, bool AT, bool BT>
__device__ __forceinline__ void gemm_tile(const GemmParams &p, const TA *A, const TA *A2,
                                          const TB *B, float *C, const float *ks, int i0,
                                          int j0) {
    if (p.upper_tiles && i0 > j0 + GB_N - 1) return;
    int kbeg = 0, kend = p.k;
    if (p.a_upper) kbeg = (i0 / GB_K) * GB_K;
    if (p.b_upper) kend = min(kend, j0 + GB_N);

    __shared__ __align__(16) float As[2][GB_K][GB_M];
    __shared__ __align__(16) float Bs[2][GB_K][GB_N];

    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

    float ra[4], rb[4];
    auto load = [&](int k0) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int e = tid + t * G_THREADS;
            int ii, kk;
            if (AT) { ii = e % GB_M; kk = e / GB_M; } else { ii = e / GB_K; kk = e % GB_K; }
            const int gi = i0 + ii, gk = k0 + kk;
            float v = 0.f;
            if (gi < p.m && gk < kend) {
                const int64_t off = AT ? (int64_t)gk * p.lda + gi : (int64_t)gi * p.lda + gk;
                v = to_f32(A[off]);
                if (A2) v -= to_f32(A2[off]);
                if (ks) v *= ks[gk];
            }
            ra[t] = v;
            int jj, kb;
            if (BT) { jj = e / GB_K; kb = e % GB_K; } else { jj = e % GB_N; kb = e / GB_N; }
            const int gj = j0 + jj, gkb = k0 + kb;
            float w = 0.f;
            if (gj < p.n && gkb < kend) {
                const int64_t off = BT ? (int64_t)gj * p.ldb + gkb : (int64_t)gkb * p.ldb + gj;
                w = to_f32(B[off]);
            }
            rb[t] = w;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int e = tid + t * G_THREADS;
            int ii, kk;
            if (AT) { ii = e % GB_M; kk = e / GB_M; } else { ii = e / GB_K; kk = e % GB_K; }
            As[buf][kk][ii] = ra[t];
            int jj, kb;
            if (BT) { jj = e / GB_K; kb = e % GB_K; } else { jj = e % GB_N; kb = e / GB_N; }
            Bs[buf][kb][jj] = rb[t];
        }
    };

    if (kbeg < kend) {
        load(kbeg);
        store(0);
        __syncthreads();
        int buf = 0;
        for (int k0 = kbeg; k0 < kend; k0 += GB_K) {
            const bool more = k0 + GB_K < kend;
            if (more) load(k0 + GB_K);
#pragma unroll
            for (int kk = 0; kk < GB_K; ++kk) {
                const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4]);
                const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4 + 64]);
                const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4 + 64]);
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
            }
            if (more) {
                store(buf ^ 1);
                __syncthreads();
                buf ^= 1;
            }
        }
    }

#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int gi = i0 + ty * 4 + (a & 3) + (a >> 2) * 64;
        if (gi >= p.m) continue;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int gj = j0 + tx * 4 + (b & 3) + (b >> 2) * 64;
            if (gj >= p.n) continue;
            float v = p.alpha * acc[a][b];
            if (p.mask_strict_upper && gj <= gi) v = 0.f;
            float *dst = C + (int64_t)gi * p.ldc + gj;
            *dst = p.accumulate ? *dst + v : v;
        }
    }
}

template <typename TA, typename TB, bool AT, bool BT>
__global__ void __launch_bounds__(G_THREADS) gemm_simt_kernel(GemmParams p) {
    if (failed(p.status)) return;
    const int bz = blockIdx.z;
    const TA *A = static_cast<const TA *>(p.A) + bz * p.sA;
    const TA *A2 = p.A2 ? static_cast<const TA *>(p.A2) + bz * p.sA2 : nullptr;
    const TB *B = static_cast<const TB *>(p.B) + bz * p.sB;
    float *C = p.C + bz * p.sC;
    const float *ks = p.kscale ? p.kscale + bz * p.sK : nullptr;
    gemm_tile<TA, TB, AT, BT>(p, A, A2, B, C, ks, blockIdx.y * GB_M, blockIdx.x * GB_N);
}

// A group of independent products with their own sizes, offsets and leading
// dimensions (one per blockIdx.z); the structural flags are shared.
constexpr int GROUP_MAX = 128;
struct GroupItem {
    int m, n, k;
    int lda, ldb, ldc;
    int64_t offA, offB, offC;
};
struct GroupParams {
    GemmParams base;
    int nitems;
    GroupItem item[GROUP_MAX];
};

template <typename TA, typename TB, bool AT, bool BT>
__global__ void __launch_bounds__(G_THREADS) gemm_simt_grouped(const __grid_constant__ GroupParams gp) {
    if (failed(gp.base.status)) return;
    const GroupItem &it = gp.item[blockIdx.z];
    const int i0 = blockIdx.y * GB_M, j0 = blockIdx.x * GB_N;
    if (i0 >= it.m || j0 >= it.n) return;
    GemmParams p = gp.base;
    p.m = it.m; p.n = it.n; p.k = it.k;
    p.lda = it.lda; p.ldb = it.ldb; p.ldc = it.ldc;
    gemm_tile<TA, TB, AT, BT>(p, static_cast<const TA *>(p.A) + it.offA, nullptr,
                              static_cast<const TB *>(p.B) + it.offB, p.C + it.offC, nullptr, i0, j0);
}

template <typename TA, typename TB, bool AT, bool BT>
inline gptq_status gemm_simt(const GemmParams &p, int batch, cudaStream_t st) {
    if (p.m <= 0 || p.n <= 0) return GPTQ_OK;
    dim3 grid((p.n + GB_N - 1) / GB_N, (p.m + GB_M - 1) / GB_M, batch);
    gemm_simt_kernel<TA, TB, AT, BT><<<grid, G_THREADS, 0, st>>>(p);
    return launch_status();
}

template <typename TA, typename TB, bool AT, bool BT>
inline gptq_status gemm_simt_group(const GroupParams &gp, cudaStream_t st) {
    int mm = 0, nn = 0;
    for (int i = 0; i < gp.nitems; ++i) {
        mm = mm > gp.item[i].m ? mm : gp.item[i].m;
        nn = nn > gp.item[i].n ? nn : gp.item[i].n;
    }
    if (gp.nitems <= 0 || mm <= 0 || nn <= 0) return GPTQ_OK;
    dim3 grid((nn + GB_N - 1) / GB_N, (mm + GB_M - 1) / GB_M, gp.nitems);
    gemm_simt_grouped<TA, TB, AT, BT><<<grid, G_THREADS, 0, st>>>(gp);
    return launch_status();
}

inline GemmParams gemm_params(int m, int n, int k, const void *A, int64_t lda, const void *B,
                              int64_t ldb, float *C, int64_t ldc, float alpha, int accumulate,
                              const int32_t *status) {
    GemmParams p{};
    p.m = m; p.n = n; p.k = k;
    p.A = A; p.lda = lda; p.B = B; p.ldb = ldb; p.C = C; p.ldc = ldc;
    p.alpha = alpha; p.accumulate = accumulate; p.status = status;
    return p;
}

}  // namespace gptq
