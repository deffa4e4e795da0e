// Tensor-core Gram with a transformed left operand:
//   weighted (per output-channel group g):  H_g += 2 (diag(s_g) X)^T X
//   cross (GPTAQ):                          C   += 2 (X_fp - X_q)^T X_q
//
// [G2PTQ] output-channel groups each carry their own Hessian (here with per-token
// weights s_g); [ResComp] items 2-3: the cross statistic dX X^T with dX = X~ - X.
//
// The left operand is formed in fp32 from bf16 inputs (s * x, or x_fp - x_q, both
// exact or correctly rounded in fp32) and split into a bf16 pair a = hi + lo; the
// right operand X is bf16 and exact, so D += hi X + lo X keeps ~16 bits of the
// left factor, accumulated in fp32 in TMEM.
//
// Same MN-major TMA / 128-byte swizzle layout as the plain Gram (64-feature x
// 32-token boxes). A transform warpgroup (warps 6-9) reads the loaded left tile(s)
// and writes the hi / lo tiles in the same swizzled layout: the swizzle only
// permutes 16-byte units inside a 128-byte row, and a row is one token, so the
// transform is element-wise with the token index = byte offset / 128.
//
// Roles (320 threads): warp 0 TMA, warp 1 TMEM + MMA, warps 2-5 epilogue, 6-9
// transform. Work units (group, token part, tile) are dealt part-major to a
// persistent grid; the weighted Gram computes only tiles meeting the upper
// triangle (written in place and transposed by the epilogue's bulk reductions),
// the cross Gram every tile.
#include <cuda.h>

#include <algorithm>

#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {

namespace {
constexpr int GX_BM = 128, GX_BN = 256, GX_BK = 32, GX_STAGES = 4;
constexpr int GX_BOX = 64 * GX_BK * 2;                  // 4 KB
constexpr int GX_A = GX_BM * GX_BK * 2;                 // 8 KB (one 128-row bf16 tile)
constexpr int GX_B = GX_BN * GX_BK * 2;                 // 16 KB
// stage: src0 (A source), src1 (second A source, cross only), B, A_hi, A_lo
constexpr int GX_STAGE = 2 * GX_A + GX_B + 2 * GX_A;    // 48 KB
constexpr int GX_EPI = 4 * 32 * 32 * 4;                 // one 32 x 32 fp32 box per epilogue warp
constexpr int GX_SMEM = GX_STAGES * GX_STAGE + GX_EPI + 1024 + 512;
constexpr int GX_THREADS = 320;
constexpr uint32_t GX_TMEM_COLS = 512;
constexpr uint32_t GX_IDESC = tc::idesc_bf16_f32(GX_BM, GX_BN, 1, 1);
}  // namespace

struct GramXParams {
    float *H;
    const float *w;     // weighted: [g][ldw] per-token weights
    int64_t ldw;
    int64_t M;          // tokens in the chunk
    int K, S, T, P, ntm, ntn, groups, cross;
    float alpha;
    int32_t *status;
};

__device__ __forceinline__ void gx_unit(const GramXParams &p, int u, int &grp, int &ti, int &tj,
                                        int &k0, int &k1) {
    const int per_group = p.T * p.P;
    grp = u / per_group;
    u -= grp * per_group;
    const int part = u / p.T;
    int t = u - part * p.T;
    if (p.cross) {
        tj = t / p.ntm;
        ti = t - tj * p.ntm;
    } else {
        int j = 0;
        while (true) {
            const int cnt = min(p.ntm, 2 * (j + 1));
            if (t < cnt) break;
            t -= cnt;
            ++j;
        }
        tj = j;
        ti = t;
    }
    k0 = (int)((int64_t)p.S * part / p.P);
    k1 = (int)((int64_t)p.S * (part + 1) / p.P);
}

__global__ void __launch_bounds__(GX_THREADS, 1)
    k_gram_x_tc(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap hmap,
                const GramXParams p) {
    if (failed(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + GX_STAGES * GX_STAGE;       // 1 KB aligned
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + GX_STAGES * GX_STAGE + GX_EPI);
    uint64_t *xfull = full + GX_STAGES;      // transformed tiles ready
    uint64_t *empty = xfull + GX_STAGES;
    uint64_t *tfull = empty + GX_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *consumed = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int units = p.groups * p.T * p.P;
    const uint32_t src_bytes = (p.cross ? 2 * GX_A : GX_A) + GX_B;

    if (threadIdx.x == 0) {
        for (int s = 0; s < GX_STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&xfull[s], 128);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&tfull[b], 1);
            tc::mbar_init(&tempty[b], 128);
        }
        tc::mbar_init(drain, 1);
        *abort = 0;
        *consumed = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, GX_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // set-up done: wait for the previous kernel on the stream (when launched as its
    // programmatic dependent; at once otherwise) before any global access, and let the
    // next kernel start its own set-up
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
                int grp, ti, tj, k0, k1;
                gx_unit(p, u, grp, ti, tj, k0, k1);
                for (int k = k0; k < k1; ++k) {
                    // bf16 boxes: feature origins on 16-byte boundaries, token step inside the chunk
                    if (!GQ_IN_BOUNDS(p.status, grp >= 0 && grp < p.groups && k >= 0 && k < p.S && ti >= 0 &&
                                                    tj >= 0 && ti * GX_BM < p.K && tj * GX_BN < p.K &&
                                                    ((ti * GX_BM) & 7) == 0 && ((tj * GX_BN) & 7) == 0,
                                      BS_GRAM_TMA, (long long)k * GX_BK)) {
                        *abort = 1;
                        break;
                    }
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort)) break;
                    tc::mbar_arrive_expect_tx(&full[stage], src_bytes);
                    uint8_t *st = smem + stage * GX_STAGE;
                    const int y = k * GX_BK;
                    tc::tma_load_2d(st, &map_a0, &full[stage], ti * GX_BM, y);
                    tc::tma_load_2d(st + GX_BOX, &map_a0, &full[stage], ti * GX_BM + 64, y);
                    if (p.cross) {
                        tc::tma_load_2d(st + GX_A, &map_a1, &full[stage], ti * GX_BM, y);
                        tc::tma_load_2d(st + GX_A + GX_BOX, &map_a1, &full[stage], ti * GX_BM + 64, y);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        tc::tma_load_2d(st + 2 * GX_A + q * GX_BOX, &map_b, &full[stage],
                                        tj * GX_BN + 64 * q, y);
                    ++issued;
                    if (++stage == GX_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort) {
                for (int i = *reinterpret_cast<volatile int *>(consumed); i < issued; ++i) {
                    volatile int never = 0;
                    tc::mbar_wait(&full[i % GX_STAGES], (i / GX_STAGES) & 1, &never);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, acc = 0, n = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
                int grp, ti, tj, k0, k1;
                gx_unit(p, u, grp, ti, tj, k0, k1);
                if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
                tc::fence_after_sync();
                const uint32_t d = tmem + acc * GX_BN;
                bool ok = true;
                for (int k = k0; k < k1; ++k) {
                    if (!tc::mbar_wait(&xfull[stage], phase, abort)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t sbase = tc::smem_u32(smem + stage * GX_STAGE);
                    const uint32_t sb = sbase + 2 * GX_A, shi = sbase + 2 * GX_A + GX_B,
                                   slo = shi + GX_A;
#pragma unroll
                    for (int kk = 0; kk < GX_BK / 16; ++kk) {
                        const uint64_t bd = tc::desc_sw128(sb + kk * 2048, GX_BOX, 1024);
                        tc::mma_bf16(d, tc::desc_sw128(shi + kk * 2048, GX_BOX, 1024), bd, GX_IDESC,
                                     (k > k0 || kk > 0) ? 1u : 0u);
                        tc::mma_bf16(d, tc::desc_sw128(slo + kk * 2048, GX_BOX, 1024), bd, GX_IDESC, 1u);
                    }
                    tc::mma_commit(&empty[stage]);
                    *reinterpret_cast<volatile int *>(consumed) = ++n;
                    if (++stage == GX_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc::mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            tc::mma_commit(drain);
            volatile int never = 0;
            tc::mbar_wait(drain, 0, &never);
        }
    } else if (warp >= 6) {
        // transform: a = s[token] * x  or  a = x_fp - x_q, split into bf16 hi + lo
        const int t = threadIdx.x - 192;      // 0..127
        int stage = 0;
        uint32_t phase = 0;
        for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
            int grp, ti, tj, k0, k1;
            gx_unit(p, u, grp, ti, tj, k0, k1);
            const float *wg = p.w ? p.w + (int64_t)grp * p.ldw : nullptr;
            bool ok = true;
            for (int k = k0; k < k1; ++k) {
                // this stage's token weights (two distinct tokens per thread), requested
                // before the wait so that their latency overlaps it
                float swr[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int64_t m = (int64_t)k * GX_BK + (((t + 128 * r) * 16) % GX_BOX) / 128;
                    swr[r] = (wg && m < p.M) ? wg[m] : 0.f;     // rows past M are zero-filled
                }
                if (!tc::mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
                uint8_t *st = smem + stage * GX_STAGE;
                const uint4 *s0 = reinterpret_cast<const uint4 *>(st);
                const uint4 *s1 = reinterpret_cast<const uint4 *>(st + GX_A);
                uint4 *dhi = reinterpret_cast<uint4 *>(st + 2 * GX_A + GX_B);
                uint4 *dlo = reinterpret_cast<uint4 *>(st + 2 * GX_A + GX_B + GX_A);
                // 8 KB tile = 512 16-byte units; 4 per thread
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int unit = t + 128 * r;    // its token (box row): ((16 unit) % box) / 128
                    const uint4 xa = s0[unit];
                    const __nv_bfloat16 *xv = reinterpret_cast<const __nv_bfloat16 *>(&xa);
                    float a[8];
                    if (p.cross) {
                        const uint4 xb = s1[unit];
                        const __nv_bfloat16 *qv = reinterpret_cast<const __nv_bfloat16 *>(&xb);
#pragma unroll
                        for (int e = 0; e < 8; ++e) a[e] = __bfloat162float(xv[e]) - __bfloat162float(qv[e]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) a[e] = swr[r] * __bfloat162float(xv[e]);
                    }
                    // hi = bf16(a), lo = bf16(a - hi), two values per conversion (the
                    // one-value conversions saturated the conversion pipe)
                    uint4 ho, lo;
                    uint32_t *hw = reinterpret_cast<uint32_t *>(&ho);
                    uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(a[2 * e], a[2 * e + 1]);
                        const float2 hf = __bfloat1622float2(h2);
                        const __nv_bfloat162 l2 = __floats2bfloat162_rn(a[2 * e] - hf.x, a[2 * e + 1] - hf.y);
                        hw[e] = *reinterpret_cast<const uint32_t *>(&h2);
                        lw[e] = *reinterpret_cast<const uint32_t *>(&l2);
                    }
                    dhi[unit] = ho;
                    dlo[unit] = lo;
                }
                // generic-proxy writes must be visible to the MMA (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                tc::mbar_arrive(&xfull[stage]);
                if (++stage == GX_STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
        }
    } else {
        // alpha * D into H through bulk tensor reductions (H seen as [g K][K]): the
        // weighted Gram writes the entries on or above the diagonal and, transposed,
        // the strictly upper ones (H_g stays symmetric); the cross Gram every entry.
        const int quad = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        uint8_t *buf = epi + (warp - 2) * 4096;
        const float alpha = p.alpha;
        const bool sym = !p.cross;
        auto stage_out = [&](int x, int y) {
            tc::fence_async_shared();
            __syncwarp();
            // a reduction box starts inside the stack of H_g, its column on a 16-byte boundary
            if (lane == 0 && GQ_IN_BOUNDS(p.status, x >= 0 && y >= 0 && x < p.K && y < p.groups * p.K &&
                                                        (x & 3) == 0,
                                          BS_GRAM_RED, (long long)y * p.K + x)) {
                tc::tma_reduce_add_2d(&hmap, buf, x, y);
                tc::bulk_commit();
                tc::bulk_wait_read<0>();    // buf is free again
            }
            __syncwarp();
        };
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            int grp, ti, tj, k0, k1;
            gx_unit(p, u, grp, ti, tj, k0, k1);
            if (!tc::mbar_wait(&tfull[acc], acc_phase, abort)) break;
            tc::fence_after_sync();
            const int r0 = ti * GX_BM + quad * 32;      // this warp's 32 rows
            const int row = r0 + lane;
            const int gy = grp * p.K;                   // group offset in the [g K][K] view
#pragma unroll 1
            for (int c = 0; c < GX_BN / 32; ++c) {
                uint32_t r[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * GX_BN + c * 32 + ((uint32_t)(quad * 32) << 16), r);
                tc::tmem_ld_wait();
                const int col0 = tj * GX_BN + c * 32;
                if (r0 >= p.K || col0 >= p.K || (sym && r0 > col0 + 31)) continue;
                // row = lane, 16-byte chunk q at q ^ (lane & 7) (128-byte swizzle); rows or
                // columns past K fall outside the map (and H_g) and are dropped
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float x[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        x[e] = (!sym || row <= col0 + 4 * q + e) ? alpha * __uint_as_float(r[4 * q + e]) : 0.f;
                    *reinterpret_cast<float4 *>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                        make_float4(x[0], x[1], x[2], x[3]);
                }
                if (r0 + 32 > p.K) {
                    // keep the box inside H_g: zero the rows past K (the next group's)
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (row >= p.K)
                            *reinterpret_cast<float4 *>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                                make_float4(0.f, 0.f, 0.f, 0.f);
                }
                stage_out(col0, gy + r0);
                if (!sym || r0 >= col0 + 31) continue;     // no strictly upper entry
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float x = (row < col0 + q && row < p.K) ? alpha * __uint_as_float(r[q]) : 0.f;
                    *reinterpret_cast<float *>(buf + q * 128 + ((((lane >> 2) ^ (q & 7))) << 4) +
                                               (lane & 3) * 4) = x;
                }
                if (col0 + 32 > p.K) {
                    // box rows past K would land in the next group's rows: zero them
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (col0 + q >= p.K)
                            *reinterpret_cast<float *>(buf + q * 128 + ((((lane >> 2) ^ (q & 7))) << 4) +
                                                       (lane & 3) * 4) = 0.f;
                }
                stage_out(r0, gy + col0);
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (lane == 0) tc::bulk_wait_all();
    }

    __syncwarp();   // each role warp reconverges before the block barrier
    tc::fence_before_sync();
    __syncthreads();
    if (*abort && threadIdx.x == 0) set_status(p.status, GPTQ_ERR_TIMEOUT);
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, GX_TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------ host side

gptq_status make_f32_map(CUtensorMap *m, const float *base, int64_t cols, int64_t rows, int64_t ld,
                         int box_cols, int box_rows);
gptq_status make_bf16_map(CUtensorMap *m, const void *base, int64_t cols, int64_t rows,
                          int64_t ld, int box_rows);

static int gx_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Token parts: bounded TMEM accumulation chains first (see MAX_MMA_CHAIN), then the
// first P that fills the persistent grid to >= 97 % in the last wave.
static int gx_parts(long T, int S, int grid, int mma_per_step) {
    int best = 1;
    double best_eff = 0.0;
    const int pmin = std::max(1, (S * mma_per_step + tc::MAX_MMA_CHAIN - 1) / tc::MAX_MMA_CHAIN);
    const int pmax = std::max(pmin, std::min(std::max(64, pmin), S / 16));
    best = pmin;
    for (int P = pmin; P <= pmax; ++P) {
        const long units = T * P;
        const long waves = (units + grid - 1) / grid;
        const double eff = (double)units / (double)(waves * grid);
        if (eff > best_eff + 1e-9) { best_eff = eff; best = P; }
        if (eff >= 0.97) return P;
    }
    return best;
}

// Weighted (w != NULL, X2 == NULL, g >= 1) or cross (X2 = X_q, X = X_fp, g == 1).
gptq_status gram_x_tc(float *H, int K, int g, const void *X, const void *X2, int64_t M,
                      int64_t ldx, const float *w, int64_t ldw, int32_t *status,
                      cudaStream_t st, bool *used) {
    *used = false;
    if (K < 64 || K % 4 != 0 || !aligned(H, 16)) return GPTQ_OK;
    const bool cross = X2 != nullptr;
    CUtensorMap ma0, ma1, mb;
    // left source (x for weighted, x_fp for cross), second source (x_q), right operand
    const void *left = X, *right = cross ? X2 : X;
    gptq_status s = make_bf16_map(&ma0, left, K, M, ldx, GX_BK);
    if (s != GPTQ_OK) return GPTQ_OK;
    if ((s = make_bf16_map(&ma1, cross ? X2 : X, K, M, ldx, GX_BK)) != GPTQ_OK) return GPTQ_OK;
    if ((s = make_bf16_map(&mb, right, K, M, ldx, GX_BK)) != GPTQ_OK) return GPTQ_OK;

    GramXParams p{};
    p.H = H;
    p.w = w;
    p.ldw = ldw;
    p.M = M;
    p.K = K;
    p.S = (int)((M + GX_BK - 1) / GX_BK);
    p.ntm = (K + GX_BM - 1) / GX_BM;
    p.ntn = (K + GX_BN - 1) / GX_BN;
    p.cross = cross ? 1 : 0;
    p.groups = cross ? 1 : g;
    p.T = 0;
    if (cross) {
        p.T = p.ntm * p.ntn;
    } else {
        for (int j = 0; j < p.ntn; ++j) p.T += std::min(p.ntm, 2 * (j + 1));
    }
    const int grid_max = gx_sms();
    p.P = std::min(gx_parts((long)p.T * p.groups, p.S, grid_max, 2 * (GX_BK / 16)), p.S);
    p.alpha = 2.f;
    p.status = status;
    const int units = p.groups * p.T * p.P;
    const int grid = std::min(units, grid_max);
    // H as [groups K][K] fp32, 32 x 32 boxes with the 128-byte swizzle
    CUtensorMap hmap;
    if ((s = make_f32_map(&hmap, H, K, (int64_t)p.groups * K, K, 32, 32)) != GPTQ_OK) return s;
    cudaFuncSetAttribute(k_gram_x_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, GX_SMEM);
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(GX_THREADS);
        cfg.dynamicSmemBytes = GX_SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaLaunchKernelEx(&cfg, k_gram_x_tc, ma0, ma1, mb, hmap, p);
    }
    if ((s = launch_status()) != GPTQ_OK) return s;
    *used = true;
    return GPTQ_OK;
}

}  // namespace gptq
