// Tensor-core lazy update of the far coordinates (tcgen05, TMA):
//   C[n][k] += sum_g sign_g * sum_j A_g[j][n] * B_g[j][k]
// over j in a block (or super-block) of already-quantised coordinates.
//
// [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": after a block of B coordinates the
// far coordinates get W_far -= U[blk, far]^T E_blk in one matrix product; with the
// GPTAQ term ([ResComp] item 3) also W_far += P1[blk, far]^T W_pre,blk.
//
// Operands are fp32 values carried as bf16 pairs x = hi + lo; three products
// hi*hi + hi*lo + lo*hi keep about 16 bits of each factor (the dropped lo*lo term
// is ~2^-18 relative), accumulated in fp32 in TMEM. Both operands are MN-major
// (rows j, the n or k index contiguous), loaded as 64-wide boxes with the 128-byte
// swizzle: LBO = one box, SBO = 8 rows (1 KB). One pipeline stage holds the hi and
// lo tiles of both operands for one k-step of one product group (E with U, or the
// pre-rounding weights with P1), so each tile is loaded once for its three MMAs.
//
// Persistent CTAs over 128 x 256 output tiles: warp 0 issues TMA, warp 1 owns TMEM
// and issues the MMAs, warps 2-5 drain the double-buffered TMEM accumulator. The
// epilogue adds into C with TMA tensor reductions (fp32 add performed in L2 on whole
// lines): each epilogue warp stages its 32 rows x 32 columns in a swizzled
// shared-memory buffer and issues one bulk reduction per chunk. Rows that are not
// 16-byte aligned fall back to per-thread vector reductions.
#include <cuda.h>

#include <algorithm>

#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"
#include "update_tc.cuh"

namespace gptq {

namespace {
constexpr int UT_BM = 128, UT_BN = 256;
constexpr int UT_RING = 192 * 1024;                   // shared-memory ring for all stages
constexpr int UT_EPI = 4 * 2 * 32 * 32 * 4;           // 4 warps x 2 buffers x 32 x 32 fp32
constexpr int UT_SMEM = UT_RING + UT_EPI + 1024 + 512;  // + alignment + barriers
constexpr int UT_THREADS = 192;
constexpr uint32_t UT_TMEM_COLS = 512;                // two 256-column accumulators
}  // namespace

template <int BK, bool TMA_EPI, bool AK>
__global__ void __launch_bounds__(UT_THREADS, 1)
    k_update_tc(const __grid_constant__ UpdateMaps maps, const __grid_constant__ CUtensorMap cmap,
                const UpdateParams p) {
    constexpr int BOX = 64 * BK * 2;                  // one 64-wide box of BK rows
    constexpr int A_BYTES = UT_BM * BK * 2;           // 2 boxes
    constexpr int B_BYTES = UT_BN * BK * 2;           // 4 boxes
    constexpr int STAGE = 2 * A_BYTES + 2 * B_BYTES;  // A hi, A lo, B hi, B lo
    constexpr int STAGES = UT_RING / STAGE;
    if (failed(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + UT_RING;                    // 1 KB aligned
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + UT_RING + UT_EPI);
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
    const int per_tile = ksteps * p.ngroups;

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
    // set-up done: wait for the previous kernel on the stream (when launched as its
    // programmatic dependent; at once otherwise) before any global access, and let the
    // next kernel start its own set-up
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            const int a_x0 = p.a_x0, a_y0 = p.a_y0, b_x0 = p.b_x0, b_y0 = p.b_y0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                const int row0 = (tile % nm) * UT_BM, col0 = (tile / nm) * UT_BN;
                for (int it = 0; it < per_tile; ++it) {
                    const int g = it / ksteps, ks = it - g * ksteps;
                    const int ay = a_y0 + ks * BK, by = b_y0 + ks * BK;
                    // bf16 boxes: innermost coordinates on 16-byte boundaries, the inner
                    // step and the tile inside the product
                    if (!GQ_IN_BOUNDS(p.status, g < p.ngroups && ks * BK < p.L && row0 < p.M && col0 < p.Ncols &&
                                                    ay >= 0 && by >= 0 && ((AK ? ay : a_x0 + row0) & 7) == 0 &&
                                                    ((b_x0 + col0) & 7) == 0,
                                      BS_UPDATE_TMA, AK ? ay : a_x0 + row0)) {
                        *abort = 1;
                        break;
                    }
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort)) break;
                    tc::mbar_arrive_expect_tx(&full[stage], STAGE);
                    uint8_t *st = smem + stage * STAGE;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {       // hi, lo
                        const CUtensorMap *am = &maps.a[2 * g + h];
                        const CUtensorMap *bm = &maps.b[2 * g + h];
                        uint8_t *a = st + h * A_BYTES;
                        uint8_t *b = st + 2 * A_BYTES + h * B_BYTES;
                        if (AK) {       // channel rows with j contiguous: one 64 x 128 box
                            tc::tma_load_2d(a, am, &full[stage], ay, a_x0 + row0);
                        } else {
                            tc::tma_load_2d(a, am, &full[stage], a_x0 + row0, ay);
                            tc::tma_load_2d(a + BOX, am, &full[stage], a_x0 + row0 + 64, ay);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            tc::tma_load_2d(b + q * BOX, bm, &full[stage], b_x0 + col0 + 64 * q, by);
                    }
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
            const uint32_t idesc_pos = tc::idesc_bf16_f32(UT_BM, UT_BN, AK ? 0 : 1, 1, 0);
            const uint32_t idesc_neg = tc::idesc_bf16_f32(UT_BM, UT_BN, AK ? 0 : 1, 1, 1);
            const bool neg0 = p.neg[0] != 0, neg1 = p.neg[1] != 0;
            int stage = 0, n = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
                tc::fence_after_sync();
                const uint32_t d = tmem + acc * UT_BN;
                bool ok = true;
                for (int it = 0; it < per_tile; ++it) {
                    const int g = it / ksteps;
                    if (!tc::mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t s0 = tc::smem_u32(smem + stage * STAGE);
                    const uint32_t idesc = (g ? neg1 : neg0) ? idesc_neg : idesc_pos;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // A K-major: the k step is 32 bytes inside the 128-byte rows
                        const uint64_t ah = AK ? tc::desc_sw128(s0 + kk * 32, 16, 1024)
                                               : tc::desc_sw128(s0 + kk * 2048, BOX, 1024);
                        const uint64_t al = AK ? tc::desc_sw128(s0 + A_BYTES + kk * 32, 16, 1024)
                                               : tc::desc_sw128(s0 + A_BYTES + kk * 2048, BOX, 1024);
                        const uint64_t bh = tc::desc_sw128(s0 + 2 * A_BYTES + kk * 2048, BOX, 1024);
                        const uint64_t bl = tc::desc_sw128(s0 + 2 * A_BYTES + B_BYTES + kk * 2048, BOX, 1024);
                        tc::mma_bf16(d, ah, bh, idesc, (it > 0 || kk > 0) ? 1u : 0u);
                        tc::mma_bf16(d, ah, bl, idesc, 1u);
                        tc::mma_bf16(d, al, bh, idesc, 1u);
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
        int acc = 0, nbuf = 0;
        uint32_t acc_phase = 0;
        uint8_t *mybuf = epi + (warp - 2) * 2 * 4096;
        float *const C = p.C;
        const int64_t ldc = p.ldc;
        const int M = p.M, Ncols = p.Ncols;
        const bool vec4 = p.vec4;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int row0 = (tile % nm) * UT_BM, col0 = (tile / nm) * UT_BN;
            if (!tc::mbar_wait(&tfull[acc], acc_phase, abort)) break;
            tc::fence_after_sync();
            const int r = row0 + quad * 32 + lane;
#pragma unroll 1
            for (int c = 0; c < UT_BN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * UT_BN + c * 32 + ((uint32_t)(quad * 32) << 16), v);
                tc::tmem_ld_wait();
                const int cb = col0 + c * 32;
                if (TMA_EPI) {
                    if (row0 + quad * 32 >= M || cb >= Ncols) continue;    // warp-uniform
                    uint8_t *buf = mybuf + (nbuf & 1) * 4096;
                    if (lane == 0) tc::bulk_wait_read<1>();   // the reduction that used buf is done reading
                    __syncwarp();
                    // row = lane, 16-byte chunk q stored at chunk q ^ (row & 7) (128-byte swizzle)
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4 *>(buf + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                            make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    tc::fence_async_shared();
                    __syncwarp();
                    if (lane == 0 && GQ_IN_BOUNDS(p.status, cb >= 0 && cb < Ncols && (cb & 3) == 0 &&
                                                                row0 + quad * 32 < M,
                                                  BS_UPDATE_C, (int64_t)(row0 + quad * 32) * ldc + cb)) {
                        tc::tma_reduce_add_2d(&cmap, buf, cb, row0 + quad * 32);
                        tc::bulk_commit();
                    }
                    ++nbuf;
                } else {
                    if (r >= M || cb >= Ncols) continue;
                    if (!GQ_IN_BOUNDS(p.status, p.c_extent == 0 || (int64_t)r * ldc + min(cb + 32, Ncols) <= p.c_extent,
                                      BS_UPDATE_C, (int64_t)r * ldc + cb))
                        continue;
                    float *crow = C + (int64_t)r * ldc;
                    if (vec4 && cb + 32 <= Ncols) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            atomicAdd(reinterpret_cast<float4 *>(crow + cb + 4 * q),
                                      make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                  __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            if (cb + q < Ncols) atomicAdd(crow + cb + q, __uint_as_float(v[q]));
                    }
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (TMA_EPI && lane == 0) tc::bulk_wait_all();
    }

    __syncwarp();   // each role warp reconverges before the block barrier
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

// The output C [M][ldc] fp32 as 32 x 32 boxes with the 128-byte swizzle (the target of
// the epilogue's bulk reductions).
static gptq_status make_out_map(CUtensorMap *m, float *C, int64_t cols, int64_t rows, int64_t ld) {
    EncodeTiledFn enc = update_encode_fn();
    if (!enc) return GPTQ_ERR_CUDA;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld * 4};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, C, gdim, gstride, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

static int update_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <int BK, bool TMA_EPI, bool AK>
static gptq_status launch_update(const UpdateMaps &maps, const CUtensorMap &cmap,
                                 const UpdateParams &p, int grid, cudaStream_t st) {
    cudaFuncSetAttribute(k_update_tc<BK, TMA_EPI, AK>, cudaFuncAttributeMaxDynamicSharedMemorySize, UT_SMEM);
    const int rec = prof_begin(GPTQ_PROF_UPDATE, st);
    // a programmatic dependent of the previous kernel on the stream (a sweep): its set-up
    // overlaps that kernel's end; griddepcontrol.wait orders its accesses
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(UT_THREADS);
    cfg.dynamicSmemBytes = UT_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, k_update_tc<BK, TMA_EPI, AK>, maps, cmap, p);
    const gptq_status s = launch_status();
    prof_end(rec, st);
    return s;
}

// box_rows of the maps must equal the kernel's BK: 64 when L % 64 == 0, else 16.
gptq_status launch_update_tc(const UpdateMaps &maps, const UpdateParams &p, int box_rows,
                             cudaStream_t st) {
    if (p.M <= 0 || p.Ncols <= 0 || p.L <= 0) return GPTQ_OK;
    if (p.L % box_rows != 0 || p.ngroups < 1 || p.ngroups > 2) return GPTQ_ERR_ARG;
    if (p.a_kmajor && box_rows != 64) return GPTQ_ERR_ARG;
    const int tiles = ((p.M + UT_BM - 1) / UT_BM) * ((p.Ncols + UT_BN - 1) / UT_BN);
    const int grid = std::min(tiles, update_sms());
    // bulk reductions need a 16-byte aligned base and row pitch
    CUtensorMap cmap;
    const bool tma_epi = (p.ldc % 4 == 0) && aligned(p.C, 16) &&
                         make_out_map(&cmap, p.C, p.Ncols, p.M, p.ldc) == GPTQ_OK;
    if (!tma_epi) memset(&cmap, 0, sizeof(cmap));
    if (p.a_kmajor)
        return tma_epi ? launch_update<64, true, true>(maps, cmap, p, grid, st)
                       : launch_update<64, false, true>(maps, cmap, p, grid, st);
    if (box_rows == 64)
        return tma_epi ? launch_update<64, true, false>(maps, cmap, p, grid, st)
                       : launch_update<64, false, false>(maps, cmap, p, grid, st);
    return tma_epi ? launch_update<16, true, false>(maps, cmap, p, grid, st)
                   : launch_update<16, false, false>(maps, cmap, p, grid, st);
}

// x -> (hi, lo) with hi = bf16(x), lo = bf16(x - hi); rows x cols fp32 (ld_in) to bf16
// pairs (ld_out, padded columns written as zero). One grid row per matrix row; eight
// columns per thread when the rows are 16-byte aligned.
__global__ void k_split_bf16(const float *__restrict__ in, int64_t ld_in, int cols,
                             __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo,
                             int64_t ld_out, int64_t batch_in, int64_t batch_out, int vec) {
    const int64_t r = blockIdx.y;
    in += blockIdx.z * batch_in + r * ld_in;
    hi += blockIdx.z * batch_out + r * ld_out;
    lo += blockIdx.z * batch_out + r * ld_out;
    if (vec) {
        for (int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8; c < ld_out;
             c += gridDim.x * blockDim.x * 8) {
            float x[8];
            if (c + 8 <= cols) {
                const float4 a = *reinterpret_cast<const float4 *>(in + c);
                const float4 b = *reinterpret_cast<const float4 *>(in + c + 4);
                x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = c + i < cols ? in[c + i] : 0.f;
            }
            uint32_t h[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
                const float2 hf = __bfloat1622float2(hh);
                const __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
                h[i] = *reinterpret_cast<const uint32_t *>(&hh);
                l[i] = *reinterpret_cast<const uint32_t *>(&ll);
            }
            *reinterpret_cast<uint4 *>(hi + c) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4 *>(lo + c) = make_uint4(l[0], l[1], l[2], l[3]);
        }
        return;
    }
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
    const int vec = (ld_in % 4 == 0 && ld_out % 8 == 0 && batch_in % 4 == 0 && batch_out % 8 == 0 &&
                     aligned(in, 16) && aligned(hi, 16) && aligned(lo, 16))
                        ? 1
                        : 0;
    const int bx = (int)std::min<int64_t>(vec ? 2 : 8, (ld_out + 255) / 256);
    const int rec = prof_begin(GPTQ_PROF_SPLIT, st);
    k_split_bf16<<<dim3(bx, rows, batch), 256, 0, st>>>(in, ld_in, cols, hi, lo, ld_out, batch_in,
                                                        batch_out, vec);
    prof_end(rec, st);
    return launch_status();
}

}  // namespace gptq
