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
#include <cstdlib>

#include "bounds.cuh"
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
                int ti, tj, k0, k1;
                gt_unit(p, u, ti, tj, k0, k1);
                for (int k = k0; k < k1; ++k) {
                    // bf16 boxes: feature origins on 16-byte boundaries, token step inside the chunk
                    if (!GQ_IN_BOUNDS(p.status, k >= 0 && k < p.S && ti >= 0 && tj >= 0 && ti * GT_BM < p.K &&
                                                    tj * GT_BN < p.K && ((ti * GT_BM) & 7) == 0 && ((tj * GT_BN) & 7) == 0,
                                      BS_GRAM_TMA, (long long)k * GT_BK)) {
                        *abort = 1;
                        break;
                    }
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
            // a reduction box starts inside H, its column on a 16-byte boundary
            if (lane == 0 && GQ_IN_BOUNDS(p.status, x >= 0 && y >= 0 && x < p.K && y < p.K && (x & 3) == 0,
                                          BS_GRAM_RED, (long long)y * p.K + x)) {
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


// ---- CTA-pair form -------------------------------------------------------------------
//
// The same Gram with 256 x 256 tiles computed by a cluster of two CTAs (tcgen05
// cta_group::2): CTA r of the pair loads rows [i0 + 128 r, +128) of the A operand and
// columns [j0 + 128 r, +128) of B (32 KB per 64-token stage instead of 48 KB for a
// 128 x 256 tile), the even CTA issues 256 x 256 x 16 MMAs that read both CTAs' halves,
// and each CTA's TMEM receives its 128 rows of the tile. Per SM this cuts the operand
// traffic per MMA cycle by a third (64 instead of 96 bytes per clock) and leaves room
// for a 6-stage ring. Synchronisation (all bounded):
//   full[s]    even CTA only: its producer arms it with both halves' bytes; both
//              CTAs' loads complete on it (pair form of the tiled TMA load).
//   empty[s]   in each CTA: the even CTA's MMA thread commits to both after the
//              stage's MMAs, so each producer refills its own half.
//   tfull[b]   in each CTA: committed to both after a unit's last MMA.
//   tempty[b]  even CTA only: one arrival per epilogue warp of both CTAs.
namespace {
constexpr int G2_BM = 128;                              // rows per CTA (256 per pair)
constexpr int G2_BN = 256;                              // tile columns
constexpr int G2_BK = 64, G2_STAGES = 6;
constexpr int G2_BOX = 64 * 64 * 2;                     // 8 KB
constexpr int G2_A_BYTES = G2_BM * G2_BK * 2;           // 16 KB
constexpr int G2_B_BYTES = (G2_BN / 2) * G2_BK * 2;     // 16 KB: this CTA's half of B
constexpr int G2_STAGE = G2_A_BYTES + G2_B_BYTES;       // 32 KB
constexpr int G2_EPI = 4 * 32 * 32 * 4;
constexpr int G2_SMEM = G2_STAGES * G2_STAGE + G2_EPI + 1024 + 256;
constexpr int G2_THREADS = 192;
constexpr uint32_t G2_TMEM_COLS = 512;
constexpr uint32_t G2_IDESC = tc::idesc_bf16_f32(2 * G2_BM, G2_BN, 1, 1);
// after an abort, how long the odd CTA lets its last loads land before it leaves
constexpr long long G2_DRAIN_CYCLES = 20000000ll;
}  // namespace

// Unit u -> (row tile, column tile, k-step range) over square 256 tiles on or above the
// diagonal, part-major as in gt_unit.
__device__ __forceinline__ void g2_unit(const GramTcParams &p, int u, int &ti, int &tj, int &k0,
                                        int &k1) {
    const int part = u / p.T;
    int t = u - part * p.T;
    int j = 0;
    while (true) {
        const int cnt = min(p.ntm, j + 1);
        if (t < cnt) break;
        t -= cnt;
        ++j;
    }
    tj = j;
    ti = t;
    k0 = (int)((int64_t)p.S * part / p.P);
    k1 = (int)((int64_t)p.S * (part + 1) / p.P);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(G2_THREADS, 1)
    k_gram_tc2(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap hmap,
               const GramTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + G2_STAGES * G2_STAGE;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + G2_STAGES * G2_STAGE + G2_EPI);
    uint64_t *empty = full + G2_STAGES;
    uint64_t *tfull = empty + G2_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *consumed = reinterpret_cast<int *>(tmem_slot + 2);
    int *skip = consumed + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = tc::cluster_ctarank();
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G2_STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&tfull[b], 1);
            tc::mbar_init(&tempty[b], 8);
        }
        tc::mbar_init(drain, 1);
        *abort = 0;
        *consumed = 0;
        *skip = failed(p.status) ? 1 : 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tmap);
    }
    if (warp == 1) tc::tmem_alloc_pair(tmem_slot, G2_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();             // both CTAs' barriers exist before any remote use
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // set-up done: wait for the previous kernel on the stream (when launched as its
    // programmatic dependent; at once otherwise) before any global access, and let the
    // next kernel start its own set-up
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    // an earlier failure skips the work; both CTAs take the even CTA's reading of the
    // status, so the pair always agrees and meets at the final cluster barrier
    const int units =
        tc::ld_shared_cluster(tc::mapa_shared(tc::smem_u32(skip), 0)) ? 0 : p.T * p.P;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int u = cluster; u < units && !*abort; u += nclusters) {
                int ti, tj, k0, k1;
                g2_unit(p, u, ti, tj, k0, k1);
                const int ra = ti * 2 * G2_BM + (int)rank * G2_BM;   // this CTA's A rows
                const int cb = tj * G2_BN + (int)rank * (G2_BN / 2);  // this CTA's B columns
                for (int k = k0; k < k1; ++k) {
                    if (!GQ_IN_BOUNDS(p.status, k >= 0 && k < p.S && ra >= 0 && cb >= 0 && ra < p.K + G2_BM &&
                                                    cb < p.K + G2_BN && (ra & 7) == 0 && (cb & 7) == 0,
                                      BS_GRAM_TMA, (long long)k * G2_BK)) {
                        *abort = 1;
                        break;
                    }
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort)) break;
                    if (rank == 0) tc::mbar_arrive_expect_tx(&full[stage], 2 * G2_STAGE);
                    const uint32_t fb = tc::mapa_shared(tc::smem_u32(&full[stage]), 0);
                    uint8_t *a = smem + stage * G2_STAGE;
                    uint8_t *b = a + G2_A_BYTES;
                    const int y = k * G2_BK;
                    tc::tma_load_2d_pair(a, &tmap, fb, ra, y);
                    tc::tma_load_2d_pair(a + G2_BOX, &tmap, fb, ra + 64, y);
                    tc::tma_load_2d_pair(b, &tmap, fb, cb, y);
                    tc::tma_load_2d_pair(b + G2_BOX, &tmap, fb, cb + 64, y);
                    ++issued;
                    if (++stage == G2_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort) {
                if (rank == 0) {
                    // stages the MMA thread never consumed: let them land (or time out)
                    for (int i = *reinterpret_cast<volatile int *>(consumed); i < issued; ++i) {
                        volatile int never = 0;
                        tc::mbar_wait(&full[i % G2_STAGES], (i / G2_STAGES) & 1, &never);
                    }
                } else {
                    // the odd CTA's loads complete on the even CTA's barriers: give them
                    // a fixed, generous time to land in this CTA's shared memory
                    const long long t0 = clock64();
                    while (clock64() - t0 < G2_DRAIN_CYCLES) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            int stage = 0, acc = 0, n = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int u = cluster; u < units && !*abort; u += nclusters) {
                int ti, tj, k0, k1;
                g2_unit(p, u, ti, tj, k0, k1);
                if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
                tc::fence_after_sync();
                const uint32_t d = tmem + acc * G2_BN;
                bool ok = true;
                for (int k = k0; k < k1; ++k) {
                    if (!tc::mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t sa = tc::smem_u32(smem + stage * G2_STAGE);
                    const uint32_t sb = sa + G2_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < G2_BK / 16; ++kk) {
                        const uint64_t ad = tc::desc_sw128(sa + kk * 2048, G2_BOX, 1024);
                        const uint64_t bd = tc::desc_sw128(sb + kk * 2048, G2_BOX, 1024);
                        tc::mma_bf16_pair(d, ad, bd, G2_IDESC, (k > k0 || kk > 0) ? 1u : 0u);
                    }
                    const uint32_t eb = tc::smem_u32(&empty[stage]);
                    tc::mma_commit_pair(tc::mapa_shared(eb, 0));
                    tc::mma_commit_pair(tc::mapa_shared(eb, 1));
                    *reinterpret_cast<volatile int *>(consumed) = ++n;
                    if (++stage == G2_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                const uint32_t fb = tc::smem_u32(&tfull[acc]);
                tc::mma_commit_pair(tc::mapa_shared(fb, 0));
                tc::mma_commit_pair(tc::mapa_shared(fb, 1));
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            // every issued MMA completes before the pair's TMEM is released
            tc::mma_commit_pair(tc::mapa_shared(tc::smem_u32(drain), 0));
            volatile int never = 0;
            tc::mbar_wait(drain, 0, &never);
        }
    } else {
        // epilogue: this CTA's 128 rows of the tile, as in k_gram_tc
        const int quad = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        uint8_t *buf = epi + (warp - 2) * 4096;
        const float alpha = p.alpha;
        auto stage_out = [&](int x, int y) {
            tc::fence_async_shared();
            __syncwarp();
            if (lane == 0 && GQ_IN_BOUNDS(p.status, x >= 0 && y >= 0 && x < p.K && y < p.K && (x & 3) == 0,
                                          BS_GRAM_RED, (long long)y * p.K + x)) {
                tc::tma_reduce_add_2d(&hmap, buf, x, y);
                tc::bulk_commit();
                tc::bulk_wait_read<0>();
            }
            __syncwarp();
        };
        for (int u = cluster; u < units; u += nclusters) {
            int ti, tj, k0, k1;
            g2_unit(p, u, ti, tj, k0, k1);
            if (!tc::mbar_wait(&tfull[acc], acc_phase, abort)) break;
            tc::fence_after_sync();
            const int r0 = ti * 2 * G2_BM + (int)rank * G2_BM + quad * 32;
            const int row = r0 + lane;
#pragma unroll 1
            for (int c = 0; c < G2_BN / 32; ++c) {
                uint32_t r[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * G2_BN + c * 32 + ((uint32_t)(quad * 32) << 16), r);
                tc::tmem_ld_wait();
                const int col0 = tj * G2_BN + c * 32;
                if (r0 >= p.K || col0 >= p.K || r0 > col0 + 31) continue;
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
                if (r0 + 1 > col0 + 31) continue;
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float x = (row < col0 + q) ? alpha * __uint_as_float(r[q]) : 0.f;
                    *reinterpret_cast<float *>(buf + q * 128 + ((((lane >> 2) ^ (q & 7))) << 4) +
                                               (lane & 3) * 4) = x;
                }
                stage_out(r0, col0);
            }
            // this warp's TMEM reads are done: one arrival on the even CTA's tempty
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(&tempty[acc]), 0));
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (lane == 0) tc::bulk_wait_all();
    }

    __syncwarp();
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();             // neither CTA leaves while the pair still uses its memory
    if (*abort && threadIdx.x == 0) set_status(p.status, GPTQ_ERR_TIMEOUT);
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem, G2_TMEM_COLS);
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

    // CTA pairs for layers of at least one 256 x 256 tile (GPTQ_GRAM_PAIR=0 selects the
    // single-CTA kernel)
    const char *pair_env = getenv("GPTQ_GRAM_PAIR");
    const bool pair = K >= 256 && !(pair_env && pair_env[0] == '0');
    GramTcParams p{};
    p.H = H;
    p.K = K;
    p.S = (int)((M + GT_BK - 1) / GT_BK);
    p.alpha = 2.f;
    p.status = status;
    int grid;
    if (pair) {
        p.ntm = (K + 2 * G2_BM - 1) / (2 * G2_BM);
        p.T = 0;
        for (int j = 0; j < p.ntm; ++j) p.T += j + 1;
        const int clusters_max = sm_count() / 2;
        p.P = pick_parts(p.T, p.S, clusters_max, G2_BK / 16);
        if (p.P > p.S) p.P = p.S;
        grid = 2 * std::min(p.T * p.P, clusters_max);
    } else {
        p.ntm = (K + GT_BM - 1) / GT_BM;
        const int ntn = (K + GT_BN - 1) / GT_BN;
        p.T = 0;
        for (int j = 0; j < ntn; ++j) p.T += std::min(p.ntm, 2 * (j + 1));
        const int grid_max = sm_count();
        p.P = pick_parts(p.T, p.S, grid_max, GT_BK / 16);
        if (p.P > p.S) p.P = p.S;
        grid = std::min(p.T * p.P, grid_max);
    }

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
    if (pair) {
        cudaFuncSetAttribute(k_gram_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize, G2_SMEM);
        // programmatic dependents: a chunk's launch sets up while the previous one ends
        {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(G2_THREADS);
        cfg.dynamicSmemBytes = G2_SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaLaunchKernelEx(&cfg, k_gram_tc2, tmap, hmap, p);
    }
    } else {
        cudaFuncSetAttribute(k_gram_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, GT_SMEM);
        {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(GT_THREADS);
        cfg.dynamicSmemBytes = GT_SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaLaunchKernelEx(&cfg, k_gram_tc, tmap, hmap, p);
    }
    }
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    *used = true;
    return GPTQ_OK;
}

}  // namespace gptq
