// Factor of one diagonal block of gptq_prepare, blocked in 16-pivot sub-blocks.
//
// [GPTQ blog] "为什么 Cholesky Factor 不能当作原始逆矩阵": the sweep reads H^-1 through the
// upper factor U with U^T U = H^-1. prepare factors H_d = R R^T (R upper) from the
// bottom-right corner in diagonal blocks of 128 coordinates; for one block
// S = H_d[J, J] (already updated by the blocks after it) this kernel writes
// U_JJ = R_JJ^-1 = D^-1/2 V, where S = L D L^T with L unit upper (pivots eliminated
// from the last to the first) and V = L^-1.
//
// The 128 pivots run as eight sub-blocks of 16, from the last:
//   (A) one warp factors the sub-block S_bb = L_bb D_b L_bb^T and forms V_bb = L_bb^-1:
//       lanes 0-15 hold the rows of S_bb, lanes 16-31 the rows of V_bb, four pivots per
//       step, each step's pivot rows published in shared memory (no block barrier per
//       pivot);
//   (A') the sub-block's rows of V over the later columns: V_b,later = V_bb X, where X
//       holds what the later sub-blocks' eliminations left there;
//   (B) the panel above the sub-block: P = S_ab V_bb^T and L_ab = P D_b^-1;
//   (C) the trailing update S_aa' -= P L_a'b^T of the rows and columns before the
//       sub-block (upper triangle);
//   (D) the rows before the sub-block of V: V_a,c -= L_ab V_b,c for the columns c from
//       the sub-block on (right-looking elimination of L^-1).
// Two block barriers per sub-block: one warp's A runs beside the previous sub-block's
// C and D on six other warps, then A' and B. The products run from shared memory in
// 4 x 4 register tiles. The block arrives in two groups of asynchronous copies (the
// last sub-block's rows first, the rest during its factor), and the eighth warp, which
// shares the factoring warp's scheduler and takes no tiles, writes each sub-block's
// rows of U as soon as they are final. The pivot test is the same as the per-pivot
// kernels': refuse a pivot p_j <= tol * Hd_jj.
#include <float.h>

#include <algorithm>

#include "bounds.cuh"
#include "common.cuh"

namespace gptq {

namespace {
constexpr int DB_N = 128;        // block size (padded with the identity beyond nb)
constexpr int DB_SB = 16;        // pivots per sub-block
constexpr int DB_LD = 132;       // shared-memory row pitch (16-byte rows for float4 access)
constexpr int DB_T = 256;
}  // namespace

constexpr size_t diag_blk_smem() {
    return sizeof(float) * (2 * DB_N * DB_LD + 2 * DB_SB * DB_LD + 3 * DB_N + 4);
}

// x -> its tf32 pair (hi = x rounded to tf32, lo = x - hi), as the tf32x3 products read it.
__device__ __forceinline__ void tf32_pair(float x, float &hi, float &lo) {
    uint32_t b;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(b) : "f"(x));
    hi = __uint_as_float(b);
    lo = x - hi;
}

__device__ __forceinline__ void store_pair4(float *hi, float *lo, float4 v) {
    float4 h, l;
    tf32_pair(v.x, h.x, l.x);
    tf32_pair(v.y, h.y, l.y);
    tf32_pair(v.z, h.z, l.z);
    tf32_pair(v.w, h.w, l.w);
    *reinterpret_cast<float4 *>(hi) = h;
    *reinterpret_cast<float4 *>(lo) = l;
}

// Grid: g factor CTAs, then (with pairs) g * nsplit CTAs that write the tf32 pairs of
// the column block's rows above the diagonal block, H[0:j0, J], for the step's panel
// product. pairs: per group (stride pstride floats) hi rows then lo rows (at
// (j0 + nb) * nb), row pitch nb; the factor CTA adds U_JJ's rows j0 .. j0 + nb.
__global__ void __launch_bounds__(DB_T, 1) k_chol_diag_blk(float *H, int K, int j0, int nb,
                                                          const float *diag_d, float tol,
                                                          int32_t *status, float *pairs,
                                                          int64_t pstride, int nsplit) {
    if (pairs && (int)blockIdx.x >= (int)gridDim.x / (1 + nsplit)) {
        // a pair-split CTA: rows [r0, r1) of H[0:j0, J] of one group
        const int id = (int)blockIdx.x - (int)gridDim.x / (1 + nsplit);
        const int gi = id / nsplit, part = id - gi * nsplit;
        if (failed(status)) return;
        const int r0 = (int)((int64_t)j0 * part / nsplit), r1 = (int)((int64_t)j0 * (part + 1) / nsplit);
        const float *Hg = H + (int64_t)gi * K * K;
        float *ph = pairs + gi * pstride, *pl = ph + (int64_t)(j0 + nb) * nb;
        const int c4n = nb / 4;
        for (int idx = threadIdx.x; idx < (r1 - r0) * c4n; idx += DB_T) {
            const int r = r0 + idx / c4n, c = (idx % c4n) * 4;
            const float4 v = *reinterpret_cast<const float4 *>(Hg + (int64_t)r * K + j0 + c);
            store_pair4(ph + (int64_t)r * nb + c, pl + (int64_t)r * nb + c, v);
        }
        return;
    }
    extern __shared__ __align__(16) float sm[];
    float *S = sm;                          // [128][LD] the block, upper triangle
    float *V = S + DB_N * DB_LD;            // [128][LD] V = L^-1 (unit upper)
    float *PT = V + DB_N * DB_LD;           // [16][LD] P^T of the current sub-block
    float *LT = PT + DB_SB * DB_LD;         // [16][LD] L^T of the current sub-block
    float *dd = LT + DB_SB * DB_LD;         // [128] pivots
    float *rd = dd + DB_N;                  // [128] 1 / pivots
    float *dref = rd + DB_N;                // [128] damped diagonal, then D^-1/2
    int *skip = reinterpret_cast<int *>(dref + DB_N);
    __shared__ __align__(16) float rowb[32 * DB_SB];   // pivot rows of S (0-15) and V (16-31)
    const int tid = threadIdx.x;
    // one reading of the status word for the whole CTA
    if (tid == 0) {
        *skip = failed(status) ? 1 : 0;
        // the block lies inside H (nothing of it is read or written otherwise)
        if (!GQ_IN_BOUNDS(status, j0 >= 0 && nb >= 1 && nb <= DB_N && j0 + nb <= K, BS_DIAG, j0))
            *skip = 1;
    }
    __syncthreads();
    if (*skip) return;
    const int g = blockIdx.x;
    H += (int64_t)g * K * K;
    diag_d += (int64_t)g * K;
    // this group's pair rows of U_JJ (rows j0 .. j0 + nb of the column block's pairs)
    float *ph = pairs ? pairs + g * pstride : nullptr;
    float *pl = pairs ? ph + (int64_t)(j0 + nb) * nb : nullptr;

    // S = the block as stored; only its upper triangle is ever read (the lower one may
    // hold stale values). Beyond nb: the identity. V = I. A full block arrives as
    // coalesced 16-byte copies (a warp per row), others element by element.
    const bool vec = nb == DB_N && K % 4 == 0 && j0 % 4 == 0 &&
                     (reinterpret_cast<uintptr_t>(H) & 15) == 0;
    if (vec) {
        // two groups of copies: the last sub-block's rows (all the first factor step
        // reads), then the rest, which lands while that step runs
        auto copy = [&](int id) {
            const int r = id >> 5, c4 = (id & 31) * 4;
            const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(S + r * DB_LD + c4));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                         "l"(H + (int64_t)(j0 + r) * K + j0 + c4)
                         : "memory");
        };
        constexpr int LAST = (DB_N - DB_SB) * DB_N / 4;      // first copy of the last rows
#pragma unroll
        for (int it = 0; it < DB_SB * DB_N / 4 / DB_T; ++it) copy(LAST + tid + DB_T * it);
        asm volatile("cp.async.commit_group;" ::: "memory");
#pragma unroll 4
        for (int it = 0; it < LAST / DB_T; ++it) copy(tid + DB_T * it);
        asm volatile("cp.async.commit_group;" ::: "memory");
    } else {
        for (int idx = tid; idx < DB_N * DB_N; idx += DB_T) {
            const int r = idx >> 7, c = idx & 127;
            S[r * DB_LD + c] = (r < nb && c < nb) ? H[(int64_t)(j0 + r) * K + j0 + c]
                                                  : (r == c ? 1.f : 0.f);
        }
    }
    for (int idx = tid; idx < DB_N * DB_N / 4; idx += DB_T) {
        const int r = idx >> 5, c4 = (idx & 31) * 4;
        *reinterpret_cast<float4 *>(V + r * DB_LD + c4) =
            make_float4(r == c4 ? 1.f : 0.f, r == c4 + 1 ? 1.f : 0.f, r == c4 + 2 ? 1.f : 0.f,
                        r == c4 + 3 ? 1.f : 0.f);
    }
    asm volatile("cp.async.wait_group 1;" ::: "memory");   // this thread's last-rows copies
    if (tid < DB_N) dref[tid] = tid < nb ? diag_d[j0 + tid] : 1.f;
    __syncthreads();

    // Iteration b: stage 1 finishes step b + 1 (its trailing and V updates, C and D) on
    // warps 1-7 while warp 0 first updates sub-block b's own diagonal tiles and then
    // factors it (A); stage 2 forms sub-block b's V rows and panel (A', B). Warp 0's
    // factor thus overlaps the bulk of the previous step's updates.
    for (int b = DB_N / DB_SB - 1; b >= 0; --b) {
        const int o = DB_SB * b;                 // first coordinate of sub-block b
        // the step's panel product (launched as a programmatic dependent) may start its
        // set-up during the last sub-block; it waits for this grid's end before reading
        if (b == 0) asm volatile("griddepcontrol.launch_dependents;");
        {
            const int op = o + DB_SB;            // step b + 1 (none for the last sub-block)
            const int T = b + 1 < DB_N / DB_SB ? op / 4 : 0;
            const int nC = T * (T + 1) / 2;      // upper 4 x 4 tiles of [0, op)^2; the last
            const int ncol = (DB_N - op) / 4;    // ten are sub-block b's diagonal block
            const int nD = T * ncol;
            const int nCo = nC > 10 ? nC - 10 : 0;
            // one 4 x 4 tile of step b + 1: u < nC a trailing tile (C) of [0, op)^2, else
            // a tile of V (D): rows before op, columns from op on
            // one 4 x 4 tile: u < nC a trailing tile (C) of [0, o)^2, else a tile of V (D)
            auto tile = [&](int u) {
                float2 acc[4][2];        // row r, columns (2 h, 2 h + 1)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
                if (u < nC) {
                    int ti = 0, rem = u;
                    while (rem >= T - ti) { rem -= T - ti; ++ti; }
                    const int i0 = 4 * ti, k0 = 4 * (ti + rem);
#pragma unroll
                    for (int m = 0; m < DB_SB; ++m) {
                        const float4 a = *reinterpret_cast<const float4 *>(PT + m * DB_LD + i0);
                        const float4 q = *reinterpret_cast<const float4 *>(LT + m * DB_LD + k0);
                        const float av[4] = {a.x, a.y, a.z, a.w};
                        const float2 q0 = make_float2(q.x, q.y), q1 = make_float2(q.z, q.w);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float2 ar = make_float2(av[r], av[r]);
                            acc[r][0] = ffma2(ar, q0, acc[r][0]);
                            acc[r][1] = ffma2(ar, q1, acc[r][1]);
                        }
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        float *row = S + (i0 + r) * DB_LD + k0;
                        const float av[4] = {acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y};
                        if (i0 < k0) {
                            const float4 old = *reinterpret_cast<const float4 *>(row);
                            *reinterpret_cast<float4 *>(row) =
                                make_float4(old.x - av[0], old.y - av[1], old.z - av[2], old.w - av[3]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                if (r <= c) row[c] -= av[c];
                        }
                    }
                } else {
                    const int v = u - nC;
                    const int i0 = 4 * (v / ncol), c0 = op + 4 * (v % ncol);
#pragma unroll
                    for (int m = 0; m < DB_SB; ++m) {
                        const float4 a = *reinterpret_cast<const float4 *>(LT + m * DB_LD + i0);
                        const float4 q = *reinterpret_cast<const float4 *>(V + (op + m) * DB_LD + c0);
                        const float av[4] = {a.x, a.y, a.z, a.w};
                        const float2 q0 = make_float2(q.x, q.y), q1 = make_float2(q.z, q.w);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float2 ar = make_float2(av[r], av[r]);
                            acc[r][0] = ffma2(ar, q0, acc[r][0]);
                            acc[r][1] = ffma2(ar, q1, acc[r][1]);
                        }
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        float *row = V + (i0 + r) * DB_LD + c0;
                        const float4 o4 = *reinterpret_cast<const float4 *>(row);
                        *reinterpret_cast<float4 *>(row) =
                            make_float4(o4.x - acc[r][0].x, o4.y - acc[r][0].y, o4.z - acc[r][1].x,
                                        o4.w - acc[r][1].y);
                    }
                }
            };

            if (tid < 32) {
                if (T > 0 && tid < 10) tile(nCo + tid);
                __syncwarp();
                // (A) one warp: lanes 0-15 rows of S_bb, lanes 16-31 rows of V_bb, four pivots
                // per step. A step's pivot rows (published in shared memory by their lanes) are
                // read by every lane, which factors their 4 x 4 block itself (reverse LDL^T:
                // pivots p3 > p2 > p1 > p0, multipliers m_qt between pivot rows), forms the
                // transformed pivot rows Z_q' = Z_q - sum_{t > q} m_qt Z_t', and applies
                // z -= sum_q a_q Z_q' to its own row with a_q its row's multipliers (zero for the
                // rows at or past p_q). The V lanes take a_q from the S lane of the same row.
                {
                    const int half = tid >> 4, i = tid & 15;
                    float z[DB_SB];
        #pragma unroll
                    for (int k = 0; k < DB_SB; ++k)
                        z[k] = half == 0 ? S[(o + min(i, k)) * DB_LD + o + max(i, k)] : (k == i ? 1.f : 0.f);
                    float *myrow = rowb + tid * DB_SB;
                    if (i >= DB_SB - 4) {
        #pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<float4 *>(myrow + 4 * q) = make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
                    }
                    __syncwarp();
                    // a loop, not unrolled: the body is fetched once per sub-block and reused
        #pragma unroll 1
                    for (int st = DB_SB / 4 - 1; st >= 0; --st) {
                        const int p0 = 4 * st;
                        // the four pivot rows (S or V, by half) and the S pivot block P[q][t]
                        float Z[4][DB_SB], P[4][4];
        #pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float *zr = rowb + (half * 16 + p0 + q) * DB_SB;
        #pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const float4 v = *reinterpret_cast<const float4 *>(zr + 4 * c);
                                Z[q][4 * c] = v.x; Z[q][4 * c + 1] = v.y; Z[q][4 * c + 2] = v.z; Z[q][4 * c + 3] = v.w;
                            }
                            const float4 pv = *reinterpret_cast<const float4 *>(rowb + (p0 + q) * DB_SB + p0);
                            P[q][0] = pv.x; P[q][1] = pv.y; P[q][2] = pv.z; P[q][3] = pv.w;
                        }
                        // reverse LDL^T of the pivot block: d_q, r_q = 1 / d_q, m[q][t] (q < t)
                        float d[4], r[4], m[4][4];
        #pragma unroll
                        for (int t = 3; t >= 0; --t) {
                            d[t] = P[t][t];
                            // the pivot's reciprocal (hardware approximation, ~1 ulp): it only
                            // scales multipliers whose rounding is of the same order
                            asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r[t]) : "f"(fmaxf(d[t], FLT_MIN)));
        #pragma unroll
                            for (int q = 0; q < t; ++q) m[q][t] = P[q][t] * r[t];
        #pragma unroll
                            for (int q = 0; q < t; ++q)
        #pragma unroll
                                for (int u = 0; u < t; ++u) P[q][u] = fmaf(-m[q][t], P[t][u], P[q][u]);
                        }
                        if (tid == 0) {
        #pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                dd[o + p0 + q] = d[q];
                                rd[o + p0 + q] = r[q];
                            }
                        }
                        // this row's multipliers (S lanes: from its own pivot-column entries)
                        float a[4];
                        {
                            float zc[4];
        #pragma unroll
                            for (int q = 0; q < 4; ++q) {   // z[p0 + q], selected without indexing
                                float v = z[q];
                                v = st == 1 ? z[4 + q] : v;
                                v = st == 2 ? z[8 + q] : v;
                                v = st == 3 ? z[12 + q] : v;
                                zc[q] = v;
                            }
        #pragma unroll
                            for (int t = 3; t >= 0; --t) {
                                a[t] = i < p0 + t ? zc[t] * r[t] : 0.f;
        #pragma unroll
                                for (int q = 0; q < t; ++q) zc[q] = fmaf(-a[t], P[t][q], zc[q]);
                            }
                        }
        #pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const float at = __shfl_xor_sync(0xffffffffu, a[t], 16);
                            a[t] = half ? at : a[t];
                        }
                        // transformed pivot rows, then this row
        #pragma unroll
                        for (int t = 3; t >= 0; --t)
        #pragma unroll
                            for (int q = 0; q < t; ++q)
        #pragma unroll
                                for (int k = 0; k < DB_SB; ++k) Z[q][k] = fmaf(-m[q][t], Z[t][k], Z[q][k]);
        #pragma unroll
                        for (int t = 3; t >= 0; --t)
        #pragma unroll
                            for (int k = 0; k < DB_SB; ++k) z[k] = fmaf(-a[t], Z[t][k], z[k]);
                        __syncwarp();
                        if (st > 0 && i >= p0 - 4 && i < p0) {
        #pragma unroll
                            for (int q = 0; q < 4; ++q)
                                *reinterpret_cast<float4 *>(myrow + 4 * q) = make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
                        }
                        __syncwarp();
                    }
                    if (half == 1) {
        #pragma unroll
                        for (int k = 0; k < DB_SB; ++k) V[(o + i) * DB_LD + o + k] = z[k];
                    }
                    __syncwarp();
                    if (tid < DB_SB && o + tid < nb && !(dd[o + tid] > tol * dref[o + tid]))
                        set_status(status, GPTQ_ERR_NOT_PD);
                }
                // this warp's share of the block's other rows (the first factor step reads
                // only the last sub-block's; the tiles start from the next iteration)
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            } else if (tid < 128 || tid >= 160) {
                // the tiles on six warps: warp 4 shares warp 0's scheduler and stays off them
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                const int wi = tid < 128 ? tid - 32 : tid - 64;
                for (int u = wi; u < nCo + nD; u += DB_T - 64) tile(u < nCo ? u : u + 10);
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                // warp 4: sub-block b + 1's rows of U are final (nothing after its step
                // writes them): U = D^-1/2 V, zero below the diagonal, written out now
                if (vec && b + 1 < DB_N / DB_SB) {
                    const int lane = tid - 128;
#pragma unroll 4
                    for (int it = 0; it < DB_SB * DB_N / 4 / 32; ++it) {
                        const int id = lane + 32 * it, r = op + (id >> 5), c4 = (id & 31) * 4;
                        const float4 v = *reinterpret_cast<const float4 *>(V + r * DB_LD + c4);
                        const float sc = 1.f / sqrtf(fmaxf(dd[r], FLT_MIN));
                        const float4 u =
                            make_float4(c4 >= r ? v.x * sc : 0.f, c4 + 1 >= r ? v.y * sc : 0.f,
                                        c4 + 2 >= r ? v.z * sc : 0.f, c4 + 3 >= r ? v.w * sc : 0.f);
                        *reinterpret_cast<float4 *>(H + (int64_t)(j0 + r) * K + j0 + c4) = u;
                        if (ph) store_pair4(ph + (int64_t)(j0 + r) * DB_N + c4, pl + (int64_t)(j0 + r) * DB_N + c4, u);
                    }
                }
            }
        }
        __syncthreads();
        if (tid >= 128) {
            // (A') the sub-block's rows of V over the later columns c: V_bb X
            const int c = o + DB_SB + (tid - 128);
            if (c < DB_N) {
                float xm[DB_SB];
#pragma unroll
                for (int m = 0; m < DB_SB; ++m) xm[m] = V[(o + m) * DB_LD + c];
#pragma unroll
                for (int i = 0; i < DB_SB; ++i) {   // row i of V_bb from its diagonal chunk on
                    float y = 0.f;
#pragma unroll
                    for (int q = i / 4; q < DB_SB / 4; ++q) {
                        const float4 v = *reinterpret_cast<const float4 *>(V + (o + i) * DB_LD + o + 4 * q);
                        y = fmaf(v.x, xm[4 * q], y);
                        y = fmaf(v.y, xm[4 * q + 1], y);
                        y = fmaf(v.z, xm[4 * q + 2], y);
                        y = fmaf(v.w, xm[4 * q + 3], y);
                    }
                    V[(o + i) * DB_LD + c] = y;
                }
            }
        } else if (tid < o) {
            // (B) panel row i: P[i][k] = sum_m S[i][o + m] V_bb[k][m] (m >= k); L = P D^-1
            const int i = tid;
            float s16[DB_SB];
#pragma unroll
            for (int q = 0; q < DB_SB / 4; ++q) {
                const float4 v = *reinterpret_cast<const float4 *>(S + i * DB_LD + o + 4 * q);
                s16[4 * q] = v.x; s16[4 * q + 1] = v.y; s16[4 * q + 2] = v.z; s16[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int k = 0; k < DB_SB; ++k) {   // row k of V_bb (zero before its diagonal)
                float pk = 0.f;
#pragma unroll
                for (int q = k / 4; q < DB_SB / 4; ++q) {
                    const float4 v = *reinterpret_cast<const float4 *>(V + (o + k) * DB_LD + o + 4 * q);
                    pk = fmaf(s16[4 * q], v.x, pk);
                    pk = fmaf(s16[4 * q + 1], v.y, pk);
                    pk = fmaf(s16[4 * q + 2], v.z, pk);
                    pk = fmaf(s16[4 * q + 3], v.w, pk);
                }
                PT[k * DB_LD + i] = pk;
                LT[k * DB_LD + i] = pk * rd[o + k];
            }
        }
        __syncthreads();
    }

    // U_JJ = D^-1/2 V (zero below the diagonal)
    if (tid < DB_N) dref[tid] = 1.f / sqrtf(fmaxf(dd[tid], FLT_MIN));
    __syncthreads();
    if (vec) {      // rows 16 .. 127 were written during the later iterations
#pragma unroll
        for (int it = 0; it < DB_SB * DB_N / 4 / DB_T; ++it) {
            const int id = tid + DB_T * it, r = id >> 5, c4 = (id & 31) * 4;
            const float4 v = *reinterpret_cast<const float4 *>(V + r * DB_LD + c4);
            const float sc = dref[r];
            const float4 u = make_float4(c4 >= r ? v.x * sc : 0.f, c4 + 1 >= r ? v.y * sc : 0.f,
                                         c4 + 2 >= r ? v.z * sc : 0.f, c4 + 3 >= r ? v.w * sc : 0.f);
            *reinterpret_cast<float4 *>(H + (int64_t)(j0 + r) * K + j0 + c4) = u;
            if (ph) store_pair4(ph + (int64_t)(j0 + r) * DB_N + c4, pl + (int64_t)(j0 + r) * DB_N + c4, u);
        }
    } else {
        for (int idx = tid; idx < nb * nb; idx += DB_T) {
            const int r = idx / nb, c = idx - r * nb;
            const float u = c >= r ? V[r * DB_LD + c] * dref[r] : 0.f;
            H[(int64_t)(j0 + r) * K + j0 + c] = u;
            if (ph) tf32_pair(u, ph[(int64_t)(j0 + r) * nb + c], pl[(int64_t)(j0 + r) * nb + c]);
        }
    }
}

gptq_status launch_chol_diag_blk(float *H, int K, int g, int j0, int nb, const float *diag_d,
                                 float tol, int32_t *status, cudaStream_t st, float *pairs,
                                 int64_t pstride) {
    if (nb < 1 || nb > DB_N) return GPTQ_ERR_ARG;
    // the pairs are written with 16-byte stores over rows of nb = 128 floats
    if (pairs && (nb != DB_N || K % 4 != 0 || j0 % 4 != 0 || pstride % 4 != 0 ||
                  (reinterpret_cast<uintptr_t>(pairs) & 15) != 0 || (reinterpret_cast<uintptr_t>(H) & 15) != 0))
        return GPTQ_ERR_ARG;
    const int smem = (int)diag_blk_smem();
    if (cudaFuncSetAttribute(k_chol_diag_blk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return launch_status();
    // about 128 rows (64 KB of H) per split CTA
    const int nsplit = pairs ? std::max(1, std::min(64, (j0 + 127) / 128)) : 0;
    k_chol_diag_blk<<<g * (1 + nsplit), DB_T, smem, st>>>(H, K, j0, nb, diag_d, tol, status, pairs,
                                                          pstride, nsplit);
    return launch_status();
}

}  // namespace gptq
