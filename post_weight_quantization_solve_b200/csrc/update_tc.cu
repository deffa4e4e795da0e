// Tensor-core lazy update of the far coordinates (tcgen05, TMA):
//   C[n][k] += sum_t sign_t * sum_j A_t[j][n] * B_t[j][k]
// over j in a block (or super-block) of already-quantised coordinates.
//
// [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": after a block of B coordinates the
// far coordinates get W_far -= U[blk, far]^T E_blk in one matrix product; with the
// GPTAQ term ([ResComp] item 3) also W_far += P1[blk, far]^T W_pre,blk.
//
// Operands are fp32 values carried as bf16 pairs x = hi + lo; three products
// hi*hi + hi*lo + lo*hi keep about 16 bits of each factor (the dropped lo*lo term
// is ~2^-18 relative), accumulated in fp32 in TMEM. Both operands are MN-major
// (rows j, the n or k index contiguous), loaded as 64-wide x 16-row boxes with the
// 128-byte swizzle: LBO = one box (2 KB), SBO = 8 rows (1 KB).
//
// One CTA per 128 x 256 output tile (two CTAs fit on an SM): warp 0 issues TMA,
// warp 1 owns TMEM and issues the MMAs, warps 2-5 read TMEM and update C in place.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "update_tc.cuh"

namespace gptq {

namespace {
constexpr int UT_BM = 128, UT_BN = 256;
constexpr int UT_RING = 192 * 1024;                   // shared-memory ring for all stages
constexpr int UT_SMEM = UT_RING + 1024 + 512;   // ring + alignment + barriers
constexpr int UT_THREADS = 192;
constexpr uint32_t UT_TMEM_COLS = 512;                // two 256-column accumulators
}  // namespace

// Persistent: tiles (row tile fastest, so CTAs running together share the B rows)
// are dealt round-robin; each tile runs every term over the inner rows, then the
// epilogue adds the TMEM accumulator into C with vector reductions while the MMA
// warp already fills the other accumulator.
template <int BK>
__global__ void __launch_bounds__(UT_THREADS, 1)
    k_update_tc(const __grid_constant__ UpdateMaps maps, const UpdateParams p) {
    constexpr int BOX = 64 * BK * 2;
    constexpr int A_BYTES = UT_BM * BK * 2;
    constexpr int STAGE = A_BYTES + UT_BN * BK * 2;
    constexpr int STAGES = UT_RING / STAGE;
    if (failed(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + UT_RING);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *consumed = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nm = (p.M + UT_BM - 1) / UT_BM;
    const int tiles = nm * ((p.Ncols + UT_BN - 1) / UT_BN);
    const int ksteps = p.L / BK;
    const int per_tile = ksteps * p.nterms;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
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
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, UT_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                const int row0 = (tile % nm) * UT_BM, col0 = (tile / nm) * UT_BN;
                for (int it = 0; it < per_tile; ++it) {
                    const int t = it / ksteps, ks = it - t * ksteps;
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort)) break;
                    tc::mbar_arrive_expect_tx(&full[stage], STAGE);
                    uint8_t *a = smem + stage * STAGE;
                    uint8_t *b = a + A_BYTES;
                    const CUtensorMap *am = &maps.a[p.a_id[t]];
                    const CUtensorMap *bm = &maps.b[p.b_id[t]];
                    const int ay = p.a_y0 + ks * BK, by = p.b_y0 + ks * BK;
                    tc::tma_load_2d(a, am, &full[stage], p.a_x0 + row0, ay);
                    tc::tma_load_2d(a + BOX, am, &full[stage], p.a_x0 + row0 + 64, ay);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        tc::tma_load_2d(b + q * BOX, bm, &full[stage], p.b_x0 + col0 + 64 * q, by);
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort) {
                for (int i = *reinterpret_cast<volatile int *>(consumed); i < issued; ++i) {
                    volatile int never = 0;
                    tc::mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &never);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc_pos = tc::idesc_bf16_f32(UT_BM, UT_BN, 1, 1, 0);
            const uint32_t idesc_neg = tc::idesc_bf16_f32(UT_BM, UT_BN, 1, 1, 1);
            int stage = 0, n = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
                tc::fence_after_sync();
                const uint32_t d = tmem + acc * UT_BN;
                bool ok = true;
                for (int it = 0; it < per_tile; ++it) {
                    const int t = it / ksteps;
                    if (!tc::mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t sa = tc::smem_u32(smem + stage * STAGE);
                    const uint32_t idesc = p.neg[t] ? idesc_neg : idesc_pos;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad = tc::desc_sw128(sa + kk * 2048, BOX, 1024);
                        const uint64_t bd = tc::desc_sw128(sa + A_BYTES + kk * 2048, BOX, 1024);
                        tc::mma_bf16(d, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&empty[stage]);
                    *reinterpret_cast<volatile int *>(consumed) = ++n;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc::mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            tc::mma_commit(drain);
            volatile int never = 0;
            tc::mbar_wait(drain, 0, &never);
        }
    } else {
        const int quad = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int row0 = (tile % nm) * UT_BM, col0 = (tile / nm) * UT_BN;
            if (!tc::mbar_wait(&tfull[acc], acc_phase, abort)) break;
            tc::fence_after_sync();
            const int r = row0 + quad * 32 + lane;
            float *crow = p.C + (int64_t)r * p.ldc;
#pragma unroll 1
            for (int c = 0; c < UT_BN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * UT_BN + c * 32 + ((uint32_t)(quad * 32) << 16), v);
                tc::tmem_ld_wait();
                const int cb = col0 + c * 32;
                if (r >= p.M || cb >= p.Ncols) continue;
                if (p.vec4 && cb + 32 <= p.Ncols) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        atomicAdd(reinterpret_cast<float4 *>(crow + cb + 4 * q),
                                  make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                              __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (cb + q < p.Ncols) atomicAdd(crow + cb + q, __uint_as_float(v[q]));
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (*abort && threadIdx.x == 0) set_status(p.status, GPTQ_ERR_TIMEOUT);
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, UT_TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn update_encode_fn() {
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

bool update_tc_available() { return update_encode_fn() != nullptr; }

// bf16 matrix [rows][ld] (cols valid) as 64 x box_rows boxes with the 128-byte swizzle.
gptq_status make_bf16_map(CUtensorMap *m, const void *base, int64_t cols, int64_t rows,
                          int64_t ld, int box_rows) {
    EncodeTiledFn enc = update_encode_fn();
    if (!enc) return GPTQ_ERR_CUDA;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), gdim, gstride,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

static int update_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// box_rows of the maps must equal the kernel's BK: 64 when L % 64 == 0, else 16.
gptq_status launch_update_tc(const UpdateMaps &maps, const UpdateParams &p, int box_rows,
                             cudaStream_t st) {
    if (p.M <= 0 || p.Ncols <= 0 || p.L <= 0) return GPTQ_OK;
    if (p.L % box_rows != 0) return GPTQ_ERR_ARG;
    const int tiles = ((p.M + UT_BM - 1) / UT_BM) * ((p.Ncols + UT_BN - 1) / UT_BN);
    const int grid = std::min(tiles, update_sms());
    if (box_rows == 64) {
        cudaFuncSetAttribute(k_update_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, UT_SMEM);
        k_update_tc<64><<<grid, UT_THREADS, UT_SMEM, st>>>(maps, p);
    } else {
        cudaFuncSetAttribute(k_update_tc<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, UT_SMEM);
        k_update_tc<16><<<grid, UT_THREADS, UT_SMEM, st>>>(maps, p);
    }
    return launch_status();
}

// x -> (hi, lo) with hi = bf16(x), lo = bf16(x - hi); rows x cols fp32 (ld_in) to bf16
// pairs (ld_out, padded columns written as zero). One grid row per matrix row.
__global__ void k_split_bf16(const float *__restrict__ in, int64_t ld_in, int cols,
                             __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo,
                             int64_t ld_out, int64_t batch_in, int64_t batch_out) {
    const int64_t r = blockIdx.y;
    in += blockIdx.z * batch_in + r * ld_in;
    hi += blockIdx.z * batch_out + r * ld_out;
    lo += blockIdx.z * batch_out + r * ld_out;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < ld_out; c += gridDim.x * blockDim.x) {
        const float x = c < cols ? in[c] : 0.f;
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        hi[c] = h;
        lo[c] = __float2bfloat16_rn(x - __bfloat162float(h));
    }
}

gptq_status split_bf16(const float *in, int64_t ld_in, int rows, int cols, __nv_bfloat16 *hi,
                       __nv_bfloat16 *lo, int64_t ld_out, int batch, int64_t batch_in,
                       int64_t batch_out, cudaStream_t st) {
    const int bx = (int)std::min<int64_t>(8, (ld_out + 255) / 256);
    k_split_bf16<<<dim3(bx, rows, batch), 256, 0, st>>>(in, ld_in, cols, hi, lo, ld_out, batch_in,
                                                        batch_out);
    return launch_status();
}

}  // namespace gptq
