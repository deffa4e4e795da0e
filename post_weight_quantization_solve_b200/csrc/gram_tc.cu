// Tensor-core Gram: H += alpha * X^T X for a bf16 token chunk X[M][ldx], fp32
// accumulation in TMEM (tcgen05), operands fed by TMA.
//
// [GPTQ blog] "Calibration 让量化看见输入方向": H = 2 X^T X, one K x K statistic for all
// output channels, accumulated chunk by chunk.
//
// Both MMA operands come straight from the row-major token chunk: for a tile of
// H rows [i0, i0+128) and columns [j0, j0+256) the A operand is X[m][i0:i0+128]
// and the B operand X[m][j0:j0+256] over the chunk's tokens m, both "MN-major"
// (the feature index is contiguous). TMA loads 64-feature x 64-token boxes with
// the 128-byte swizzle, which is exactly the canonical MN-major SW128 layout:
// 128-byte rows (one token each), 8-row swizzle atoms (SBO = 1024 B), 64-feature
// chunks one box apart (LBO = 8 KB).
//
// Work: only tiles that meet the upper triangle; the chunk's tokens are split into
// P equal parts and units (part, tile) are dealt part-major to a persistent grid of
// one CTA per SM, so CTAs running at the same time read the same token slab (L2
// reuse). Each unit ends with bulk tensor reductions of alpha * D into H, written
// both in place (on and above the diagonal) and transposed (strictly above), so H
// is complete and symmetric after every chunk.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 2-5 epilogue (TMEM lane quadrant = warp % 4). 4-stage smem ring, 2 TMEM
// accumulators of 256 columns.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {

namespace {
constexpr int GT_BM = 128, GT_BN = 256, GT_BK = 64, GT_STAGES = 4;
constexpr int GT_BOX = GT_BK * 64 * 2;                 // one 64 x 64 bf16 box = 8 KB
constexpr int GT_A_BYTES = GT_BM * GT_BK * 2;          // 16 KB
constexpr int GT_B_BYTES = GT_BN * GT_BK * 2;          // 32 KB
constexpr int GT_STAGE = GT_A_BYTES + GT_B_BYTES;      // 48 KB
constexpr int GT_EPI = 4 * 32 * 32 * 4;               // one 32 x 32 fp32 box per epilogue warp
constexpr int GT_SMEM = GT_STAGES * GT_STAGE + GT_EPI + 1024 + 256;
constexpr int GT_THREADS = 192;
constexpr uint32_t GT_TMEM_COLS = 512;
constexpr uint32_t GT_IDESC = tc::idesc_bf16_f32(GT_BM, GT_BN, 1, 1);
}  // namespace

struct GramTcParams {
    float *H;
    int K;
    int S;      // 64-token k-steps in the chunk
    int T;      // upper tiles
    int P;      // token parts
    int ntm;    // 128-row tile count
    float alpha;
    int32_t *status;
};

__device__ __forceinline__ void gt_unit(const GramTcParams &p, int u, int &ti, int &tj, int &k0,
                                        int &k1) {
    const int part = u / p.T;
    int t = u - part * p.T;
    int j = 0;
    while (true) {
        const int cnt = min(p.ntm, 2 * (j + 1));
        if (t < cnt) break;
        t -= cnt;
        ++j;
    }
    tj = j;
    ti = t;
    k0 = (int)((int64_t)p.S * part / p.P);
    k1 = (int)((int64_t)p.S * (part + 1) / p.P);
}

__global__ void __launch_bounds__(GT_THREADS, 1)
    k_gram_tc(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap hmap,
              const GramTcParams p) {
    if (failed(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + GT_STAGES * GT_STAGE;       // 1 KB aligned
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + GT_STAGES * GT_STAGE + GT_EPI);
    uint64_t *empty = full + GT_STAGES;
    uint64_t *tfull = empty + GT_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *consumed = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int units = p.T * p.P;

    if (threadIdx.x == 0) {
        for (int s = 0; s < GT_STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
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
        tc::prefetch_tmap(&tmap);
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, GT_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
                int ti, tj, k0, k1;
                gt_unit(p, u, ti, tj, k0, k1);
                for (int k = k0; k < k1; ++k) {
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort)) break;
                    tc::mbar_arrive_expect_tx(&full[stage], GT_STAGE);
                    uint8_t *a = smem + stage * GT_STAGE;
                    uint8_t *b = a + GT_A_BYTES;
                    const int y = k * GT_BK;
                    tc::tma_load_2d(a, &tmap, &full[stage], ti * GT_BM, y);
                    tc::tma_load_2d(a + GT_BOX, &tmap, &full[stage], ti * GT_BM + 64, y);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        tc::tma_load_2d(b + q * GT_BOX, &tmap, &full[stage], tj * GT_BN + 64 * q, y);
                    ++issued;
                    if (++stage == GT_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort) {
                // let every load still in flight land before the CTA can exit
                for (int i = *reinterpret_cast<volatile int *>(consumed); i < issued; ++i) {
                    volatile int never = 0;
                    tc::mbar_wait(&full[i % GT_STAGES], (i / GT_STAGES) & 1, &never);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, acc = 0, n = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
                int ti, tj, k0, k1;
                gt_unit(p, u, ti, tj, k0, k1);
                if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
                tc::fence_after_sync();
                const uint32_t d = tmem + acc * GT_BN;
                bool ok = true;
                for (int k = k0; k < k1; ++k) {
                    if (!tc::mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t sa = tc::smem_u32(smem + stage * GT_STAGE);
                    const uint32_t sb = sa + GT_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < GT_BK / 16; ++kk) {
                        const uint64_t ad = tc::desc_sw128(sa + kk * 2048, GT_BOX, 1024);
                        const uint64_t bd = tc::desc_sw128(sb + kk * 2048, GT_BOX, 1024);
                        tc::mma_bf16(d, ad, bd, GT_IDESC, (k > k0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&empty[stage]);
                    *reinterpret_cast<volatile int *>(consumed) = ++n;
                    if (++stage == GT_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc::mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            // all issued MMAs complete before TMEM can be released
            tc::mma_commit(drain);
            volatile int never = 0;
            tc::mbar_wait(drain, 0, &never);
        }
    } else {
        // alpha * D into H through bulk tensor reductions: the entries on or above the
        // diagonal as they are, the strictly upper ones also transposed into the lower
        // triangle, so H stays symmetric without a separate pass. Each warp stages one
        // 32 x 32 box at a time (128-byte swizzle) and lets the reduction read it.
        const int quad = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        uint8_t *buf = epi + (warp - 2) * 4096;
        const float alpha = p.alpha;
        auto stage_out = [&](int x, int y) {
            tc::fence_async_shared();
            __syncwarp();
            if (lane == 0) {
                tc::tma_reduce_add_2d(&hmap, buf, x, y);
                tc::bulk_commit();
                tc::bulk_wait_read<0>();    // buf is free again
            }
            __syncwarp();
        };
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            int ti, tj, k0, k1;
            gt_unit(p, u, ti, tj, k0, k1);
            if (!tc::mbar_wait(&tfull[acc], acc_phase, abort)) break;
            tc::fence_after_sync();
            const int r0 = ti * GT_BM + quad * 32;      // this warp's 32 rows
            const int row = r0 + lane;
#pragma unroll 1
            for (int c = 0; c < GT_BN / 32; ++c) {
                uint32_t r[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * GT_BN + c * 32 + ((uint32_t)(quad * 32) << 16), r);
                tc::tmem_ld_wait();
                const int col0 = tj * GT_BN + c * 32;
                if (r0 >= p.K || col0 >= p.K || r0 > col0 + 31) continue;   // nothing on or above
                // upper part (row <= col) in place: row = lane, chunk q at q ^ (lane & 7)
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float x[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        x[e] = (row <= col0 + 4 * q + e) ? alpha * __uint_as_float(r[4 * q + e]) : 0.f;
                    *reinterpret_cast<float4 *>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                        make_float4(x[0], x[1], x[2], x[3]);
                }
                stage_out(col0, r0);
                if (r0 + 1 > col0 + 31) continue;           // no strictly upper entry
                // strictly upper part transposed: box row q (column col0 + q), column lane
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float x = (row < col0 + q) ? alpha * __uint_as_float(r[q]) : 0.f;
                    *reinterpret_cast<float *>(buf + q * 128 + ((((lane >> 2) ^ (q & 7))) << 4) +
                                               (lane & 3) * 4) = x;
                }
                stage_out(r0, col0);
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
        tc::tmem_dealloc(tmem, GT_TMEM_COLS);
    }
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

static int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Token parts P: at least enough parts that no TMEM accumulation chain exceeds
// MAX_MMA_CHAIN MMAs, then the first P whose units (T * P) fill the persistent grid
// to >= 97 % in the last wave, keeping >= 16 k-steps per unit.
static int pick_parts(int T, int S, int grid, int mma_per_step) {
    int best = 1;
    double best_eff = 0.0;
    const int pmin = std::max(1, (S * mma_per_step + tc::MAX_MMA_CHAIN - 1) / tc::MAX_MMA_CHAIN);
    const int pmax = std::max(pmin, std::min(std::max(64, pmin), S / 16));
    best = pmin;
    for (int P = pmin; P <= pmax; ++P) {
        const long units = (long)T * P;
        const long waves = (units + grid - 1) / grid;
        const double eff = (double)units / (double)(waves * grid);
        if (eff > best_eff + 1e-9) { best_eff = eff; best = P; }
        if (eff >= 0.97) return P;
    }
    return best;
}

gptq_status gram_tc(float *H, int K, int g, const void *X, int64_t M, int64_t ldx, const float *w,
                    int64_t ldw, const void *X2, cudaStream_t st, int32_t *status, bool *used) {
    (void)ldw;
    *used = false;
    // tensor-core path: plain bf16 Gram (one Hessian, unit weights, no cross term)
    if (g != 1 || w != nullptr || X2 != nullptr || K < 64) return GPTQ_OK;
    if (!aligned(H, 16) || K % 4 != 0) return GPTQ_OK;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return GPTQ_OK;

    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
    const cuuint32_t box[2] = {64, GT_BK};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), gdim,
                     gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return GPTQ_ERR_CUDA;

    GramTcParams p{};
    p.H = H;
    p.K = K;
    p.S = (int)((M + GT_BK - 1) / GT_BK);
    p.ntm = (K + GT_BM - 1) / GT_BM;
    const int ntn = (K + GT_BN - 1) / GT_BN;
    p.T = 0;
    for (int j = 0; j < ntn; ++j) p.T += std::min(p.ntm, 2 * (j + 1));
    const int grid_max = sm_count();
    p.P = pick_parts(p.T, p.S, grid_max, GT_BK / 16);
    if (p.P > p.S) p.P = p.S;
    p.alpha = 2.f;
    p.status = status;
    const int units = p.T * p.P;
    const int grid = std::min(units, grid_max);

    // H as 32 x 32 fp32 boxes for the epilogue's reductions (rows 16-byte aligned)
    CUtensorMap hmap;
    {
        const cuuint64_t hdim[2] = {(cuuint64_t)K, (cuuint64_t)K};
        const cuuint64_t hstride[1] = {(cuuint64_t)K * 4};
        const cuuint32_t hbox[2] = {32, 32};
        r = enc(&hmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, H, hdim, hstride, hbox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return GPTQ_ERR_CUDA;
    }
    cudaFuncSetAttribute(k_gram_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, GT_SMEM);
    k_gram_tc<<<grid, GT_THREADS, GT_SMEM, st>>>(tmap, hmap, p);
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    *used = true;
    return GPTQ_OK;
}

}  // namespace gptq
