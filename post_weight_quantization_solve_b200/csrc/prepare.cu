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

#include <algorithm>
#include <cstdlib>
#include <map>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc32.cuh"
#include "prepare_plan.h"
#include "tc_ptx.cuh"

namespace gptq {

gptq_status launch_chol_diag_blk(float *H, int K, int g, int j0, int nb, const float *diag_d,
                                 float tol, int32_t *status, cudaStream_t st, float *pairs,
                                 int64_t pstride);

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

// Factor one diagonal block H[J,J] (J = [j0, j0+nb), nb <= 128) and replace it by
// U_JJ. One CTA per group; the block is padded with the identity beyond nb.
// H_JJ = L D L^T with L unit upper, eliminated from the last pivot to the first,
// and V = L^-1 built in the same pass: once pivot j is eliminated, column j of L
// is final and so is row j of V (every later row has been applied to it), so
//   S[i][k] -= S[i][j] S[k][j] / d_j        (i, k < j)
//   V[i][c] -= (S[i][j] / d_j) V[j][c]      (i < j)
// share one published column. Then U_JJ = R^-1 = D^-1/2 V with R = L D^1/2.
// Each thread keeps a 4 x 8 tile of S and the same tile of V in registers; the 272
// tiles that meet the upper triangle are dealt row-major, so a warp whose rows all
// lie at or below pivot j skips the update. Column j of S, row j of V and d_j are
// published into buffers of their own (no reuse), one barrier per pivot.
constexpr int DG_TILES = 272;
constexpr int DG_T = 288;
constexpr int DG_N = CH_NB;

__global__ void __launch_bounds__(DG_T, 1) k_chol_diag(float *H, int K, int j0, int nb,
                                                    const float *diag_d, float tol,
                                                    int32_t *status) {
    if (failed(status)) return;
    const int g = blockIdx.x;
    H += (int64_t)g * K * K;
    diag_d += (int64_t)g * K;
    extern __shared__ __align__(16) float sm[];
    float *colb = sm;                      // [128][128]: column j of S, rows < j
    float *vrow = colb + DG_N * DG_N;      // [128][128]: row j of V
    float *dpiv = vrow + DG_N * DG_N;      // [128]
    float *rpiv = dpiv + DG_N;             // [128]
    float *dref = rpiv + DG_N;             // [128]
    const int tid = threadIdx.x;

    // this thread's tile (ti, tk): rows 4 ti .. 4 ti + 3, columns 8 tk .. 8 tk + 7
    int ti = 32, tk = 0;
    if (tid < DG_TILES) {
        int t = tid;
        for (int r = 0; r < 32; ++r) {
            const int cnt = 16 - (r >> 1);
            if (t < cnt) { ti = r; tk = (r >> 1) + t; break; }
            t -= cnt;
        }
    }
    const int wrow0 = 4 * __shfl_sync(0xffffffffu, ti, 0);   // lowest row of this warp
    const int i0 = 4 * ti, c0 = 8 * tk;

    for (int idx = tid; idx < 2 * DG_N * DG_N / 4; idx += DG_T)
        reinterpret_cast<float4 *>(colb)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < DG_N) dref[tid] = tid < nb ? diag_d[j0 + tid] : 1.f;
    // tiles entirely below the diagonal: zero in the output
    for (int idx = tid; idx < DG_N * DG_N; idx += DG_T) {
        const int r = idx >> 7, c = idx & 127;
        if (r < nb && c < nb && (r >> 2) > 2 * (c >> 3) + 1) H[(int64_t)(j0 + r) * K + j0 + c] = 0.f;
    }

    // tile rows as column pairs (c, c + 1): the updates run as packed fp32 FMAs
    float2 s[4][4], v[4][4];
    const bool vec = (nb == DG_N) && (K % 4 == 0) && ((reinterpret_cast<uintptr_t>(H) & 15) == 0) &&
                     (j0 % 4 == 0);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = i0 + r;
        if (ti < 32 && vec) {
            const float *src = H + (int64_t)(j0 + i) * K + j0 + c0;
            const float4 x0 = *reinterpret_cast<const float4 *>(src);
            const float4 x1 = *reinterpret_cast<const float4 *>(src + 4);
            s[r][0] = make_float2(x0.x, x0.y); s[r][1] = make_float2(x0.z, x0.w);
            s[r][2] = make_float2(x1.x, x1.y); s[r][3] = make_float2(x1.z, x1.w);
        } else {
            float e[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int k = c0 + c;
                e[c] = (i < nb && k < nb) ? H[(int64_t)(j0 + i) * K + j0 + k] : (i == k ? 1.f : 0.f);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) s[r][c] = make_float2(e[2 * c], e[2 * c + 1]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            v[r][c] = make_float2((i == c0 + 2 * c) ? 1.f : 0.f, (i == c0 + 2 * c + 1) ? 1.f : 0.f);
    }
    __syncthreads();

    for (int jb = DG_N / 8 - 1; jb >= 0; --jb) {
#pragma unroll
        for (int jj = 7; jj >= 0; --jj) {
            const int j = 8 * jb + jj;
            // publish column j of S (rows < j), d_j and row j of V
            if (tk == jb && i0 < j) {
                float4 o;
                o.x = (i0 + 0 < j) ? ((jj & 1) ? s[0][jj >> 1].y : s[0][jj >> 1].x) : 0.f;
                o.y = (i0 + 1 < j) ? ((jj & 1) ? s[1][jj >> 1].y : s[1][jj >> 1].x) : 0.f;
                o.z = (i0 + 2 < j) ? ((jj & 1) ? s[2][jj >> 1].y : s[2][jj >> 1].x) : 0.f;
                o.w = (i0 + 3 < j) ? ((jj & 1) ? s[3][jj >> 1].y : s[3][jj >> 1].x) : 0.f;
                *reinterpret_cast<float4 *>(colb + j * DG_N + i0) = o;
            }
            if (ti == (j >> 2)) {
                const int r = jj & 3;
                *reinterpret_cast<float4 *>(vrow + j * DG_N + c0) =
                    make_float4(v[r][0].x, v[r][0].y, v[r][1].x, v[r][1].y);
                *reinterpret_cast<float4 *>(vrow + j * DG_N + c0 + 4) =
                    make_float4(v[r][2].x, v[r][2].y, v[r][3].x, v[r][3].y);
                if (tk == jb) {
                    const float d = (jj & 1) ? s[r][jj >> 1].y : s[r][jj >> 1].x;
                    dpiv[j] = d;
                    rpiv[j] = 1.f / fmaxf(d, FLT_MIN);
                    if (j < nb && !(d > tol * dref[j])) set_status(status, GPTQ_ERR_NOT_PD);
                }
            }
            __syncthreads();
            if (wrow0 < j) {
                const float rd = rpiv[j];
                const float4 a = *reinterpret_cast<const float4 *>(colb + j * DG_N + i0 % DG_N);
                const float4 k0 = *reinterpret_cast<const float4 *>(colb + j * DG_N + c0);
                const float4 k1 = *reinterpret_cast<const float4 *>(colb + j * DG_N + c0 + 4);
                const float4 v0 = *reinterpret_cast<const float4 *>(vrow + j * DG_N + c0);
                const float4 v1 = *reinterpret_cast<const float4 *>(vrow + j * DG_N + c0 + 4);
                const float li[4] = {-a.x * rd, -a.y * rd, -a.z * rd, -a.w * rd};
                const float2 ak[4] = {make_float2(k0.x, k0.y), make_float2(k0.z, k0.w),
                                      make_float2(k1.x, k1.y), make_float2(k1.z, k1.w)};
                const float2 vk[4] = {make_float2(v0.x, v0.y), make_float2(v0.z, v0.w),
                                      make_float2(v1.x, v1.y), make_float2(v1.z, v1.w)};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float2 l2 = make_float2(li[r], li[r]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        s[r][c] = ffma2(l2, ak[c], s[r][c]);
                        v[r][c] = ffma2(l2, vk[c], v[r][c]);
                    }
                }
            }
        }
    }
    // U = D^-1/2 V on the tiles (zero below the diagonal)
    if (ti < 32) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = i0 + r;
            if (i >= nb) continue;
            const float sc = 1.f / sqrtf(fmaxf(dpiv[i], FLT_MIN));
            float o[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float vc = (c & 1) ? v[r][c >> 1].y : v[r][c >> 1].x;
                o[c] = (c0 + c >= i) ? vc * sc : 0.f;
            }
            float *dst = H + (int64_t)(j0 + i) * K + j0 + c0;
            if (vec) {
                *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(o[4], o[5], o[6], o[7]);
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (c0 + c < nb) dst[c] = o[c];
            }
        }
    }
}

// The same factor with two pivots per block barrier: for the pair (ja, ja - 1) both
// columns of S and both rows of V are published before pivot ja is applied, and every
// thread forms column ja - 1, row ja - 1 and d_{ja - 1} after pivot ja itself, so the
// 128 pivots of a block take 64 barriers.
__global__ void __launch_bounds__(DG_T, 1) k_chol_diag2(float *H, int K, int j0, int nb,
                                                    const float *diag_d, float tol,
                                                    int32_t *status) {
    if (failed(status)) return;
    const int g = blockIdx.x;
    H += (int64_t)g * K * K;
    diag_d += (int64_t)g * K;
    extern __shared__ __align__(16) float sm[];
    float *colb = sm;                      // [128][128]: column j of S, rows < j
    float *vrow = colb + DG_N * DG_N;      // [128][128]: row j of V
    float *dpiv = vrow + DG_N * DG_N;      // [128]
    float *rpiv = dpiv + DG_N;             // [128]
    float *dref = rpiv + DG_N;             // [128]
    const int tid = threadIdx.x;

    // this thread's tile (ti, tk): rows 4 ti .. 4 ti + 3, columns 8 tk .. 8 tk + 7
    int ti = 32, tk = 0;
    if (tid < DG_TILES) {
        int t = tid;
        for (int r = 0; r < 32; ++r) {
            const int cnt = 16 - (r >> 1);
            if (t < cnt) { ti = r; tk = (r >> 1) + t; break; }
            t -= cnt;
        }
    }
    const int wrow0 = 4 * __shfl_sync(0xffffffffu, ti, 0);   // lowest row of this warp
    const int i0 = 4 * ti, c0 = 8 * tk;

    for (int idx = tid; idx < 2 * DG_N * DG_N / 4; idx += DG_T)
        reinterpret_cast<float4 *>(colb)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < DG_N) dref[tid] = tid < nb ? diag_d[j0 + tid] : 1.f;
    // tiles entirely below the diagonal: zero in the output
    for (int idx = tid; idx < DG_N * DG_N; idx += DG_T) {
        const int r = idx >> 7, c = idx & 127;
        if (r < nb && c < nb && (r >> 2) > 2 * (c >> 3) + 1) H[(int64_t)(j0 + r) * K + j0 + c] = 0.f;
    }

    // tile rows as column pairs (c, c + 1): the updates run as packed fp32 FMAs
    float2 s[4][4], v[4][4];
    const bool vec = (nb == DG_N) && (K % 4 == 0) && ((reinterpret_cast<uintptr_t>(H) & 15) == 0) &&
                     (j0 % 4 == 0);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = i0 + r;
        if (ti < 32 && vec) {
            const float *src = H + (int64_t)(j0 + i) * K + j0 + c0;
            const float4 x0 = *reinterpret_cast<const float4 *>(src);
            const float4 x1 = *reinterpret_cast<const float4 *>(src + 4);
            s[r][0] = make_float2(x0.x, x0.y); s[r][1] = make_float2(x0.z, x0.w);
            s[r][2] = make_float2(x1.x, x1.y); s[r][3] = make_float2(x1.z, x1.w);
        } else {
            float e[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int k = c0 + c;
                e[c] = (i < nb && k < nb) ? H[(int64_t)(j0 + i) * K + j0 + k] : (i == k ? 1.f : 0.f);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) s[r][c] = make_float2(e[2 * c], e[2 * c + 1]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            v[r][c] = make_float2((i == c0 + 2 * c) ? 1.f : 0.f, (i == c0 + 2 * c + 1) ? 1.f : 0.f);
    }
    __syncthreads();

    for (int jb = DG_N / 8 - 1; jb >= 0; --jb) {
#pragma unroll
        for (int jp = 3; jp >= 0; --jp) {
            // pivots ja = 8 jb + 2 jp + 1 and jc = ja - 1 share a tile column pair, a
            // four-row block and one barrier
            const int ja = 8 * jb + 2 * jp + 1, jc = ja - 1;
            if (tk == jb && i0 < ja) {
                float4 o;
                o.x = (i0 + 0 < ja) ? s[0][jp].y : 0.f;
                o.y = (i0 + 1 < ja) ? s[1][jp].y : 0.f;
                o.z = (i0 + 2 < ja) ? s[2][jp].y : 0.f;
                o.w = (i0 + 3 < ja) ? s[3][jp].y : 0.f;
                *reinterpret_cast<float4 *>(colb + ja * DG_N + i0) = o;
                if (i0 < jc) {
                    o.x = (i0 + 0 < jc) ? s[0][jp].x : 0.f;
                    o.y = (i0 + 1 < jc) ? s[1][jp].x : 0.f;
                    o.z = (i0 + 2 < jc) ? s[2][jp].x : 0.f;
                    o.w = (i0 + 3 < jc) ? s[3][jp].x : 0.f;
                    *reinterpret_cast<float4 *>(colb + jc * DG_N + i0) = o;
                }
            }
            if (ti == (ja >> 2)) {
                const int ra = ja & 3, rc = jc & 3;
                *reinterpret_cast<float4 *>(vrow + ja * DG_N + c0) =
                    make_float4(v[ra][0].x, v[ra][0].y, v[ra][1].x, v[ra][1].y);
                *reinterpret_cast<float4 *>(vrow + ja * DG_N + c0 + 4) =
                    make_float4(v[ra][2].x, v[ra][2].y, v[ra][3].x, v[ra][3].y);
                *reinterpret_cast<float4 *>(vrow + jc * DG_N + c0) =
                    make_float4(v[rc][0].x, v[rc][0].y, v[rc][1].x, v[rc][1].y);
                *reinterpret_cast<float4 *>(vrow + jc * DG_N + c0 + 4) =
                    make_float4(v[rc][2].x, v[rc][2].y, v[rc][3].x, v[rc][3].y);
                if (tk == jb) {
                    // d_ja, and d_jc after pivot ja (the same product as the tile update)
                    const float da = s[ra][jp].y;
                    const float rda = 1.f / fmaxf(da, FLT_MIN);
                    const float sca = s[rc][jp].y;                 // S[jc][ja]
                    const float dc = fmaf(-sca * rda, sca, s[rc][jp].x);
                    dpiv[ja] = da;
                    rpiv[ja] = rda;
                    dpiv[jc] = dc;
                    rpiv[jc] = 1.f / fmaxf(dc, FLT_MIN);
                    if (ja < nb && !(da > tol * dref[ja])) set_status(status, GPTQ_ERR_NOT_PD);
                    if (jc < nb && !(dc > tol * dref[jc])) set_status(status, GPTQ_ERR_NOT_PD);
                }
            }
            __syncthreads();
            if (wrow0 < ja) {
                const float rda = rpiv[ja], rdc = rpiv[jc];
                const float m = colb[ja * DG_N + jc] * rda;        // l of row jc on pivot ja
                const float4 aa = *reinterpret_cast<const float4 *>(colb + ja * DG_N + i0 % DG_N);
                const float4 ka0 = *reinterpret_cast<const float4 *>(colb + ja * DG_N + c0);
                const float4 ka1 = *reinterpret_cast<const float4 *>(colb + ja * DG_N + c0 + 4);
                const float4 va0 = *reinterpret_cast<const float4 *>(vrow + ja * DG_N + c0);
                const float4 va1 = *reinterpret_cast<const float4 *>(vrow + ja * DG_N + c0 + 4);
                const float4 ac = *reinterpret_cast<const float4 *>(colb + jc * DG_N + i0 % DG_N);
                const float4 kc0 = *reinterpret_cast<const float4 *>(colb + jc * DG_N + c0);
                const float4 kc1 = *reinterpret_cast<const float4 *>(colb + jc * DG_N + c0 + 4);
                const float4 vc0 = *reinterpret_cast<const float4 *>(vrow + jc * DG_N + c0);
                const float4 vc1 = *reinterpret_cast<const float4 *>(vrow + jc * DG_N + c0 + 4);
                const float aav[4] = {aa.x, aa.y, aa.z, aa.w};
                const float kav[8] = {ka0.x, ka0.y, ka0.z, ka0.w, ka1.x, ka1.y, ka1.z, ka1.w};
                const float vav[8] = {va0.x, va0.y, va0.z, va0.w, va1.x, va1.y, va1.z, va1.w};
                const float acv[4] = {ac.x, ac.y, ac.z, ac.w};
                const float kcv[8] = {kc0.x, kc0.y, kc0.z, kc0.w, kc1.x, kc1.y, kc1.z, kc1.w};
                const float vcv[8] = {vc0.x, vc0.y, vc0.z, vc0.w, vc1.x, vc1.y, vc1.z, vc1.w};
                // column jc of S and row jc of V after pivot ja (entries at or past jc stay 0)
                float la[4], lc[4];
                float2 ka2[4], kc2[4], va2[4], vc2[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    la[r] = -aav[r] * rda;
                    const float acn = (i0 + r < jc) ? fmaf(-aav[r], m, acv[r]) : 0.f;
                    lc[r] = -acn * rdc;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int k = c0 + 2 * c;
                    ka2[c] = make_float2(kav[2 * c], kav[2 * c + 1]);
                    va2[c] = make_float2(vav[2 * c], vav[2 * c + 1]);
                    kc2[c] = make_float2((k < jc) ? fmaf(-kav[2 * c], m, kcv[2 * c]) : 0.f,
                                         (k + 1 < jc) ? fmaf(-kav[2 * c + 1], m, kcv[2 * c + 1]) : 0.f);
                    vc2[c] = make_float2(fmaf(-m, vav[2 * c], vcv[2 * c]),
                                         fmaf(-m, vav[2 * c + 1], vcv[2 * c + 1]));
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float2 l2a = make_float2(la[r], la[r]);
                    const float2 l2c = make_float2(lc[r], lc[r]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        s[r][c] = ffma2(l2a, ka2[c], s[r][c]);
                        v[r][c] = ffma2(l2a, va2[c], v[r][c]);
                        s[r][c] = ffma2(l2c, kc2[c], s[r][c]);
                        v[r][c] = ffma2(l2c, vc2[c], v[r][c]);
                    }
                }
            }
        }
    }
    // U = D^-1/2 V on the tiles (zero below the diagonal)
    if (ti < 32) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = i0 + r;
            if (i >= nb) continue;
            const float sc = 1.f / sqrtf(fmaxf(dpiv[i], FLT_MIN));
            float o[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float vc = (c & 1) ? v[r][c >> 1].y : v[r][c >> 1].x;
                o[c] = (c0 + c >= i) ? vc * sc : 0.f;
            }
            float *dst = H + (int64_t)(j0 + i) * K + j0 + c0;
            if (vec) {
                *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(o[4], o[5], o[6], o[7]);
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (c0 + c < nb) dst[c] = o[c];
            }
        }
    }
}

__global__ void k_zero_lower(float *H, int K, const int32_t *status) {
    if (failed(status)) return;
    const int g = blockIdx.z;
    H += (int64_t)g * K * K;
    const int i = blockIdx.y;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < i; j += gridDim.x * blockDim.x)
        H[(int64_t)i * K + j] = 0.f;
}

// Off-diagonal blocks of U = R^-1 (the tree of prepare_plan.h): all nodes of one depth
// are independent and run as grouped launches per product (deepest first):
// T = R[a:m, m:b] U[m:b, m:b], then U[a:m, m:b] = -U[a:m, a:m] T.

static gptq_status tri_inverse(float *H, int K, int g, const Blocks &bk, float *T,
                               const int32_t *status, cudaStream_t st) {
    std::vector<std::vector<InvNode>> levels;
    inv_nodes(bk, K, 0, bk.T, 0, levels);
    const int64_t KK = (int64_t)K * K;
    const int64_t tsz = (int64_t)inverse_scratch_floats(K);
    static thread_local GroupParams g1, g2;
    for (int d = (int)levels.size() - 1; d >= 0; --d) {
        const std::vector<InvNode> &lv = levels[d];
        // (node, group) items, in launches of at most GROUP_MAX
        std::vector<std::pair<int, int>> items;
        for (int gi = 0; gi < g; ++gi)
            for (int ni = 0; ni < (int)lv.size(); ++ni) items.push_back({gi, ni});
        // scratch offsets of this depth's nodes (disjoint, within the scratch)
        std::vector<int64_t> toff(lv.size());
        int64_t acc = 0;
        for (size_t ni = 0; ni < lv.size(); ++ni) {
            toff[ni] = acc;
            acc += (int64_t)(lv[ni].m - lv[ni].a) * (lv[ni].b - lv[ni].m);
        }
        for (size_t c0 = 0; c0 < items.size(); c0 += GROUP_MAX) {
            const int cnt = (int)std::min<size_t>(GROUP_MAX, items.size() - c0);
            g1.base = gemm_params(0, 0, 0, H, 0, H, 0, T, 0, 1.f, 0, status);
            g1.base.b_upper = 1;
            g2.base = gemm_params(0, 0, 0, H, 0, T, 0, H, 0, -1.f, 0, status);
            g2.base.a_upper = 1;
            g1.nitems = g2.nitems = cnt;
            for (int i = 0; i < cnt; ++i) {
                const int gi = items[c0 + i].first, ni = items[c0 + i].second;
                const InvNode &nd = lv[ni];
                const int rows = nd.m - nd.a, cols = nd.b - nd.m;
                const int64_t hb = gi * KK, tb = gi * tsz + toff[ni];
                g1.item[i] = {rows, cols, cols, K, K, cols, hb + (int64_t)nd.a * K + nd.m,
                              hb + (int64_t)nd.m * K + nd.m, tb};
                g2.item[i] = {rows, cols, rows, K, cols, K, hb + (int64_t)nd.a * K + nd.a, tb,
                              hb + (int64_t)nd.a * K + nd.m};
            }
            gptq_status s = gemm_simt_group<float, float, false, false>(g1, st);
            if (s != GPTQ_OK) return s;
            if ((s = gemm_simt_group<float, float, false, false>(g2, st)) != GPTQ_OK) return s;
        }
    }
    return GPTQ_OK;
}

// Compact workspace: damped diagonal + one level's inverse scratch T (fp32 SIMT path).
size_t prepare_workspace_compact(int K, int g) {
    Carver c(nullptr);
    c.take<float>((size_t)g * K);
    c.take<float>((size_t)g * inverse_scratch_floats(K));
    return round_up(c.off, 256);
}

static bool tc_inverse_eligible(int K) { return K % 32 == 0 && K >= 256; }

// Tensor-core path (one group at a time): tf32 pairs of H and of H^T (4 K^2) and of
// one level's T^T scratch (2 x the inverse scratch).
static size_t tc_extra_floats(int K) {
    return 4 * (size_t)K * K + 2 * inverse_scratch_floats(K) + 4 * 64;
}

// One Cholesky step on the tensor cores, for one group, split for lookahead:
//   panel : R[0:j0, J] = H[0:j0, J] U_JJ^T       (A = rows of the column block,
//                                                 B^T = U_JJ rows)
//   strip : H[0:j0, J'] -= R[0:j0, J] R[J', J]^T  (J' = the next diagonal block, the
//                                                 columns the next step reads first)
//   rest  : H[0:j0', 0:j0'] -= R R^T on the rows and columns before J' (upper tiles)
// with j0' = start of J'. The panel and strip run on the caller's stream (the
// critical path: next diagonal factor, next panel); the rest runs on a second
// stream and overlaps the next steps. The tf32 pairs of the column block live in a
// per-(group, step parity) buffer so that a rest still reading them is not
// overwritten by the next step.
static gptq_status chol_panel_strip_tc(float *H, int K, int j0, int j1, int j0n, float *buf,
                                       int32_t *status, cudaStream_t st, CUtensorMap (&m)[4],
                                       bool pairs_ready) {
    const int nb = j1 - j0;
    float *Ch = buf, *Cl = Ch + (size_t)j1 * nb;
    static thread_local Tc32Params pp, ps;
    gptq_status s;
    // the column block's pairs (rows 0 .. j1), unless the diagonal factor's launch wrote them
    if (!pairs_ready && (s = split_tf32(H + j0, K, j1, nb, Ch, Cl, nb, 1, 0, 0, st)) != GPTQ_OK)
        return s;
    if ((s = make_f32_map(&m[0], Ch, nb, j1, nb, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[1], Cl, nb, j1, nb, 32, 128)) != GPTQ_OK) return s;
    m[2] = m[0]; m[3] = m[1];
    pp = Tc32Params{};
    pp.C = H; pp.alpha = 1.f; pp.accumulate = 0; pp.status = status; pp.nitems = 1;
    pp.item[0].m = j0; pp.item[0].n = nb; pp.item[0].k = nb;
    pp.item[0].a_x0 = 0; pp.item[0].a_y0 = 0; pp.item[0].b_x0 = 0; pp.item[0].b_y0 = j0;
    pp.item[0].c_off = j0; pp.item[0].ldc = K;
    // the epilogue also writes the tf32 pairs of the new panel R over the front rows
    // (0..j0) of the block's pairs: each row tile is read (as A) and written by the
    // same unit, and the U_JJ rows read as B lie behind them
    pp.pair_hi = Ch; pp.pair_lo = Cl; pp.pair_ld = nb;
    pp.pdl = 1;         // its set-up overlaps the end of the kernel before it
    pp.c_extent = (int64_t)K * K; pp.pair_extent = (int64_t)j1 * nb;
    if ((s = launch_gemm_tc32(m, pp, st)) != GPTQ_OK) return s;
    // strip: every row above j0 against the rows of J' (entries below the diagonal of
    // H[J', J'] are updated too; nothing reads them)
    ps = Tc32Params{};
    ps.C = H; ps.alpha = -1.f; ps.accumulate = 1; ps.status = status; ps.nitems = 1;
    ps.item[0].m = j0; ps.item[0].n = j0 - j0n; ps.item[0].k = nb;
    ps.item[0].a_x0 = 0; ps.item[0].a_y0 = 0; ps.item[0].b_x0 = 0; ps.item[0].b_y0 = j0n;
    ps.item[0].c_off = j0n; ps.item[0].ldc = K;
    ps.c_extent = (int64_t)K * K;
    ps.pdl = 1;
    return launch_gemm_tc32(m, ps, st);
}

static gptq_status chol_rest_tc(float *H, int K, int j0n, const CUtensorMap (&m)[4],
                                int32_t *status, cudaStream_t st, int nb, int max_grid) {
    if (j0n <= 0) return GPTQ_OK;
    static thread_local Tc32Params pr;
    pr = Tc32Params{};
    pr.C = H; pr.alpha = -1.f; pr.accumulate = 1; pr.upper_tiles = 1; pr.status = status;
    pr.nitems = 1;
    pr.item[0].m = j0n; pr.item[0].n = j0n; pr.item[0].k = nb;
    pr.item[0].c_off = 0; pr.item[0].ldc = K;
    pr.max_grid = max_grid;
    pr.c_extent = (int64_t)K * K;
    return launch_gemm_tc32(m, pr, st);
}

// Second stream and events of the lookahead, one set per (device, caller stream),
// created on first use and kept until exit. Keying on the caller's stream keeps two
// host threads that enqueue prepare on different streams of one device apart: each
// has its own side stream and events, so neither can wait on the other's records, and
// a capture on one stream never pulls in another caller's side-stream work. `mu` is
// held for a whole enqueue, so calls on the same stream from several threads enqueue
// one after the other.
constexpr int LA_MAX_GROUPS = 8;
struct Lookahead {
    std::mutex mu;
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t panel[LA_MAX_GROUPS][2], rest[LA_MAX_GROUPS][2];
    bool ok = false;
};

static Lookahead *lookahead_for(cudaStream_t caller) {
    static std::mutex mu;
    static std::map<std::pair<int, cudaStream_t>, Lookahead *> table;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    Lookahead *&L = table[{dev, caller}];
    if (!L) L = new Lookahead();
    if (!L->ok) {
        bool good = cudaStreamCreateWithFlags(&L->side, cudaStreamNonBlocking) == cudaSuccess;
        good = good && cudaEventCreateWithFlags(&L->fork, cudaEventDisableTiming) == cudaSuccess;
        good = good && cudaEventCreateWithFlags(&L->join, cudaEventDisableTiming) == cudaSuccess;
        for (int gi = 0; gi < LA_MAX_GROUPS && good; ++gi)
            for (int b = 0; b < 2 && good; ++b)
                good = cudaEventCreateWithFlags(&L->panel[gi][b], cudaEventDisableTiming) == cudaSuccess &&
                       cudaEventCreateWithFlags(&L->rest[gi][b], cudaEventDisableTiming) == cudaSuccess;
        if (!good) {
            cudaGetLastError();
            return nullptr;
        }
        L->ok = true;
    }
    return L;
}

// Trailing sizes below this stay on the SIMT kernels.
constexpr int TC_STEP_MIN = 128;

size_t prepare_workspace(int K, int g) {
    size_t base = prepare_workspace_compact(K, g);
    if (!tc_inverse_eligible(K)) return base;
    return round_up(base + tc_extra_floats(K) * sizeof(float), 256);
}

// tf32 pairs of square blocks H[r0:r0+n, r0:r0+n] (one block per blockIdx.z), written
// at the same positions of the pair arrays; transposed pairs when `transposed`.
struct SplitBlocks {
    int n_items;
    int r0[TC32_MAX_ITEMS], n[TC32_MAX_ITEMS];
};

__global__ void k_split_blocks(const float *__restrict__ H, int K, float *__restrict__ hi,
                               float *__restrict__ lo, float *__restrict__ hit,
                               float *__restrict__ lot, const SplitBlocks sb) {
    // one read of each 32 x 32 tile; its pairs are written in place (hi, lo) and
    // transposed (hit, lot)
    __shared__ float t[32][33];
    const int r0 = sb.r0[blockIdx.z], n = sb.n[blockIdx.z];
    const int tr = blockIdx.y * 32, tcol = blockIdx.x * 32;
    if (tr >= n || tcol >= n) return;
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int r = tr + y, c = tcol + threadIdx.x;
        const float x = (r < n && c < n) ? H[(int64_t)(r0 + r) * K + r0 + c] : 0.f;
        t[y][threadIdx.x] = x;
        if (r < n && c < n) {
            uint32_t h;
            asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
            const float hf = __uint_as_float(h);
            const int64_t o = (int64_t)(r0 + r) * K + r0 + c;
            hi[o] = hf;
            lo[o] = x - hf;
        }
    }
    __syncthreads();
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int orow = tcol + y, ocol = tr + threadIdx.x;
        if (orow < n && ocol < n) {
            const float x = t[threadIdx.x][y];
            uint32_t h;
            asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
            const float hf = __uint_as_float(h);
            const int64_t o = (int64_t)(r0 + orow) * K + r0 + ocol;
            hit[o] = hf;
            lot[o] = x - hf;
        }
    }
}

__global__ void k_zero_blocks(float *C, const Tc32Params p) {
    if (failed(p.status)) return;
    const Tc32Item &I = p.item[blockIdx.z];
    const int r = blockIdx.y;
    if (r >= I.m) return;
    float *row = C + I.c_off + (int64_t)r * I.ldc;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < I.n; c += gridDim.x * blockDim.x)
        row[c] = 0.f;
}

// Level-batched inverse of one group on the tensor cores (the recursion of
// tri_inverse). Every operand is K-major: per level, with tf32 pairs of H and H^T,
//   T^T = U[m:b, m:b]^T R[a:m, m:b]^T      (A = rows of H^T, lower triangular)
//   U[a:m, m:b] = -U[a:m, a:m] T           (B^T = rows of T^T; A upper triangular)
static gptq_status tri_inverse_tc(float *H, int K, const Blocks &bk, float *Tt, float *ex,
                                  int32_t *status, cudaStream_t st) {
    std::vector<std::vector<InvNode>> levels;
    inv_nodes(bk, K, 0, bk.T, 0, levels);
    const int64_t KK = (int64_t)K * K;
    const int64_t tsz = (int64_t)inverse_scratch_floats(K);
    float *Hh = ex, *Hl = Hh + KK, *Gh = Hl + KK, *Gl = Gh + KK;   // H and H^T pairs
    float *Th = Gl + KK, *Tl = Th + tsz;
    static thread_local Tc32Params p1, p2;
    CUtensorMap mh[2], mg[2], m1[4], m2[4];
    gptq_status s;
    if ((s = make_f32_map(&mh[0], Hh, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&mh[1], Hl, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&mg[0], Gh, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&mg[1], Gl, K, K, K, 32, 128)) != GPTQ_OK) return s;
    // The nodes of one depth are independent; a depth with more nodes than one launch's
    // item table (K above 28,672) runs as several rounds of at most TC32_MAX_ITEMS nodes.
    for (int d = (int)levels.size() - 1; d >= 0; --d)
    for (const InvRound &round : inv_rounds(levels[d], TC32_MAX_ITEMS)) {
        const std::vector<InvNode> &lv = round.nodes;
        // T^T of this round: node blocks (b - m) x (m - a) stacked, common pitch
        const int pitch = round.pitch, trows = round.trows;
        const std::vector<int> &trow0 = round.trow0;
        if ((int64_t)trows * pitch > tsz) return GPTQ_ERR_WORKSPACE;
        {   // pairs of the node blocks [a, b) x [a, b) only (normal and transposed)
            static thread_local SplitBlocks sb;
            sb.n_items = (int)lv.size();
            int nmax = 0;
            for (size_t ni = 0; ni < lv.size(); ++ni) {
                sb.r0[ni] = lv[ni].a;
                sb.n[ni] = lv[ni].b - lv[ni].a;
                nmax = std::max(nmax, sb.n[ni]);
            }
            const dim3 grid((nmax + 31) / 32, (nmax + 31) / 32, sb.n_items);
            k_split_blocks<<<grid, dim3(32, 8), 0, st>>>(H, K, Hh, Hl, Gh, Gl, sb);
            if ((s = launch_status()) != GPTQ_OK) return s;
        }
        cudaMemsetAsync(Tt, 0, sizeof(float) * (size_t)trows * pitch, st);
        // T^T = (U_bb^T)(R_ab^T): A rows j of H^T at column m, B^T rows i of H at column m
        p1 = Tc32Params{};
        p1.C = Tt; p1.alpha = 1.f; p1.accumulate = 1; p1.a_lower = 1; p1.status = status;
        p1.c_extent = (int64_t)trows * pitch;
        p1.nitems = (int)lv.size();
        for (size_t ni = 0; ni < lv.size(); ++ni) {
            const InvNode &nd = lv[ni];
            Tc32Item &I = p1.item[ni];
            I.m = nd.b - nd.m; I.n = nd.m - nd.a; I.k = nd.b - nd.m;
            I.a_x0 = nd.m; I.a_y0 = nd.m;
            I.b_x0 = nd.m; I.b_y0 = nd.a;
            I.c_off = (int64_t)trow0[ni] * pitch;
            I.ldc = pitch;
        }
        m1[0] = mg[0]; m1[1] = mg[1]; m1[2] = mh[0]; m1[3] = mh[1];
        if ((s = launch_gemm_tc32(m1, p1, st)) != GPTQ_OK) return s;
        if ((s = split_tf32(Tt, pitch, trows, pitch, Th, Tl, pitch, 1, 0, 0, st)) != GPTQ_OK) return s;
        if ((s = make_f32_map(&m2[2], Th, pitch, trows, pitch, 32, 128)) != GPTQ_OK) return s;
        if ((s = make_f32_map(&m2[3], Tl, pitch, trows, pitch, 32, 128)) != GPTQ_OK) return s;
        m2[0] = mh[0]; m2[1] = mh[1];
        // U_ab = -U_aa T into zeroed blocks of H: A rows of H at column a, B^T rows of T^T
        p2 = Tc32Params{};
        p2.C = H; p2.alpha = -1.f; p2.accumulate = 1; p2.a_upper = 1; p2.status = status;
        p2.c_extent = KK;
        p2.nitems = (int)lv.size();
        int maxm = 0, maxn = 0;
        for (size_t ni = 0; ni < lv.size(); ++ni) {
            const InvNode &nd = lv[ni];
            Tc32Item &I = p2.item[ni];
            I.m = nd.m - nd.a; I.n = nd.b - nd.m; I.k = nd.m - nd.a;
            I.a_x0 = nd.a; I.a_y0 = nd.a;
            I.b_x0 = 0; I.b_y0 = trow0[ni];
            I.c_off = (int64_t)nd.a * K + nd.m;
            I.ldc = K;
            maxm = std::max(maxm, I.m);
            maxn = std::max(maxn, I.n);
        }
        k_zero_blocks<<<dim3(std::min(8, (maxn + 255) / 256), maxm, p2.nitems), 256, 0, st>>>(H, p2);
        if ((s = launch_status()) != GPTQ_OK) return s;
        if ((s = launch_gemm_tc32(m2, p2, st)) != GPTQ_OK) return s;
    }
    return GPTQ_OK;
}

gptq_status prepare(float *H, int K, int g, float percdamp, uint8_t *dead_out, void *ws,
                    size_t ws_bytes, int32_t *status, cudaStream_t st) {
    Carver c(ws);
    float *diag_d = c.take<float>((size_t)g * K);
    float *T = c.take<float>((size_t)g * inverse_scratch_floats(K));
    const bool use_tc = tc_inverse_eligible(K) && tc32_available() &&
                        ws_bytes >= prepare_workspace(K, g);
    float *ex = use_tc ? c.take<float>(tc_extra_floats(K)) : nullptr;
    const int64_t KK = (int64_t)K * K;

    k_check_finite<<<592, 256, 0, st>>>(H, KK * g, status);
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    k_dead_damp<<<g, 1024, 0, st>>>(H, K, percdamp, dead_out, diag_d, status);
    if ((s = launch_status()) != GPTQ_OK) return s;

    const float tol = (float)K * FLT_EPSILON;
    const int chol_smem = (int)((2 * DG_N * DG_N + 3 * DG_N) * sizeof(float));
    // diagonal blocks: the blocked factor (16-pivot sub-blocks, diag_blk.cu) by default;
    // GPTQ_DIAG=pairs or single selects the per-pivot kernels (two pivots or one per
    // block barrier), kept for comparisons
    const char *diag_env = getenv("GPTQ_DIAG");
    const int diag_mode = !diag_env ? 0 : (diag_env[0] == 'p' ? 1 : diag_env[0] == 's' ? 2 : 0);
    if (diag_mode > 0)
        cudaFuncSetAttribute(diag_mode == 1 ? k_chol_diag2 : k_chol_diag,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, chol_smem);
    Blocks bk{K, (K + CH_NB - 1) / CH_NB};
    // lookahead on the tensor-core steps (a second stream runs the bulk trailing
    // updates); without it every step runs in order on the caller's stream
    const size_t pair_floats = (size_t)K * CH_NB * 2;
    // the per-(group, parity) pair buffers use the front of the inverse's pair area
    Lookahead *la = (use_tc && g <= LA_MAX_GROUPS && (size_t)g * 2 * pair_floats <= 4 * (size_t)KK)
                        ? lookahead_for(st)
                        : nullptr;
    std::unique_lock<std::mutex> la_lock;
    if (la) la_lock = std::unique_lock<std::mutex>(la->mu);
    bool side_busy = false;         // work issued on the side stream not yet joined
    int rest_of[2] = {-1, -1};      // step whose rest was last recorded in parity slot
    auto join_side = [&]() -> gptq_status {
        if (!side_busy) return GPTQ_OK;
        if (cudaEventRecord(la->join, la->side) != cudaSuccess ||
            cudaStreamWaitEvent(st, la->join, 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        side_busy = false;
        return GPTQ_OK;
    };
    for (int t = bk.T - 1; t >= 0; --t) {
        const int j0 = bk.start(t);
        const int j1 = (t == bk.T - 1) ? K : bk.start(t + 1);
        const int nb = j1 - j0;
        // the diagonal block's last updates: the rest of step t + 2 (the rest of step
        // t + 1 does not reach it)
        if (la && t + 2 < bk.T && rest_of[(t + 2) & 1] == t + 2)
            for (int gi = 0; gi < g; ++gi)
                if (cudaStreamWaitEvent(st, la->rest[gi][(t + 2) & 1], 0) != cudaSuccess)
                    return GPTQ_ERR_CUDA;
        // with the lookahead's per-group pair buffers, the factor's launch also writes the
        // tf32 pairs of the column block that the step's panel product reads
        const bool tc_step = use_tc && j0 >= TC_STEP_MIN && nb % 32 == 0;
        const bool fused_pairs =
            la && tc_step && diag_mode == 0 && nb == CH_NB && K % 4 == 0 && aligned(H, 16);
        const int rec = prof_begin(GPTQ_PROF_DIAG, st);
        if (diag_mode == 0) {
            s = launch_chol_diag_blk(H, K, g, j0, nb, diag_d, tol, status, st,
                                     fused_pairs ? ex + (size_t)(t & 1) * pair_floats : nullptr,
                                     (int64_t)(2 * pair_floats));
        } else {
            if (diag_mode == 1)
                k_chol_diag2<<<g, DG_T, chol_smem, st>>>(H, K, j0, nb, diag_d, tol, status);
            else
                k_chol_diag<<<g, DG_T, chol_smem, st>>>(H, K, j0, nb, diag_d, tol, status);
            s = launch_status();
        }
        prof_end(rec, st);
        if (s != GPTQ_OK) return s;
        if (j0 == 0) break;
        if (tc_step) {
            if (la) {
                const int j0n = bk.start(t - 1);
                if (!side_busy) {
                    if (cudaEventRecord(la->fork, st) != cudaSuccess ||
                        cudaStreamWaitEvent(la->side, la->fork, 0) != cudaSuccess)
                        return GPTQ_ERR_CUDA;
                    side_busy = true;
                }
                for (int gi = 0; gi < g; ++gi) {
                    float *Hg = H + (int64_t)gi * KK;
                    float *buf = ex + (size_t)(gi * 2 + (t & 1)) * pair_floats;
                    CUtensorMap m[4];
                    if ((s = chol_panel_strip_tc(Hg, K, j0, j1, j0n, buf, status, st, m, fused_pairs)) !=
                        GPTQ_OK)
                        return s;
                    if (cudaEventRecord(la->panel[gi][t & 1], st) != cudaSuccess ||
                        cudaStreamWaitEvent(la->side, la->panel[gi][t & 1], 0) != cudaSuccess)
                        return GPTQ_ERR_CUDA;
                    if ((s = chol_rest_tc(Hg, K, j0n, m, status, la->side, nb, 0)) != GPTQ_OK)
                        return s;
                    if (cudaEventRecord(la->rest[gi][t & 1], la->side) != cudaSuccess)
                        return GPTQ_ERR_CUDA;
                }
                rest_of[t & 1] = t;
                continue;
            }
            for (int gi = 0; gi < g; ++gi) {
                float *Hg = H + (int64_t)gi * KK;
                CUtensorMap m[4];
                const int j0n = bk.start(t - 1);
                if ((s = chol_panel_strip_tc(Hg, K, j0, j1, j0n, ex, status, st, m, false)) != GPTQ_OK)
                    return s;
                if ((s = chol_rest_tc(Hg, K, j0n, m, status, st, nb, 0)) != GPTQ_OK) return s;
            }
            continue;
        }
        if ((s = join_side()) != GPTQ_OK) return s;
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
    if ((s = join_side()) != GPTQ_OK) return s;
    // The strict lower triangle still holds the input and update leftovers; the
    // inverse reads whole tiles of its triangular operands, so clear it first.
    k_zero_lower<<<dim3((K + 255) / 256 > 8 ? 8 : (K + 255) / 256, K, g), 256, 0, st>>>(H, K, status);
    if ((s = launch_status()) != GPTQ_OK) return s;
    if (use_tc) {
        for (int gi = 0; gi < g; ++gi)
            if ((s = tri_inverse_tc(H + (int64_t)gi * KK, K, bk, T, ex, status, st)) != GPTQ_OK)
                return s;
        return GPTQ_OK;
    }
    return tri_inverse(H, K, g, bk, T, status, st);
}

}  // namespace gptq
