// fp32-accurate tensor-core GEMM for the factorisation and the GPTAQ residual:
//   C[i][j] (+)= alpha * sum_k A[i][k] B(k, j)
// with every operand carried as a tf32 pair x = hi + lo (hi = tf32(x) rounded to
// nearest, lo = x - hi, exact in fp32). Three tcgen05 kind::tf32 products
// hi*hi + hi*lo + lo*hi keep ~21 bits of each factor (the dropped lo*lo term is
// ~2^-22 relative), enough for the 1e-4 bound on U at the conditioning the
// damping allows; fp32 accumulation in TMEM in chains of at most MAX_MMA_CHAIN
// MMAs, flushed with fp32 atomics when an item's inner range is split.
//
// Operands are read by TMA from pre-split copies (hi and lo arrays of the same
// shape), both K-major: A rows i and B^T rows j with k contiguous, 32 x 128 boxes,
// 128-byte swizzle (SBO = 1 KB, the MMA's k step = 32 bytes inside the atom). A
// product whose B is naturally row-major in k is given B^T by a transposing split.
//
// One launch runs a list of independent products ("items", e.g. every node of one
// level of the recursive inverse) on a persistent grid; structural flags skip work
// known to be zero: tiles below the diagonal, A upper triangular (k starts at the
// row tile), B upper triangular (k ends at the column tile).
#include <cuda.h>

#include <algorithm>
#include <vector>

#include "bounds.cuh"
#include "common.cuh"
#include "gemm_tc32.cuh"
#include "tc_ptx.cuh"

namespace gptq {

namespace {
constexpr int G32_BM = 128, G32_BN = 128, G32_BK = 32, G32_STAGES = 3;
constexpr int G32_TILE = G32_BM * G32_BK * 4;                  // 16 KB (A or B tile)
constexpr int G32_STAGE = 4 * G32_TILE;                        // A hi, A lo, B hi, B lo
constexpr int G32_SMEM = G32_STAGES * G32_STAGE + 1024 + 512;
constexpr int G32_THREADS = 192;
constexpr uint32_t G32_TMEM_COLS = 256;                        // two 128-column accumulators
constexpr int G32_MMA_PER_KSTEP = (G32_BK / 8) * 3;
}  // namespace

__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N, int b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(b_mn) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One unit of work: an output tile of one item and a part of its k range, with the
// item's fields copied into registers (the kernel parameter lives in the constant
// bank; reading it through a reference inside loops that store to global memory
// makes every access a reload).
struct G32Unit {
    int i0, j0, k0, k1, kmax;
    int m, n, ldc, parts;
    int a_x0, a_y0, b_x0, b_y0;
    int64_t c_off;
};

// Unit u -> (item, row tile, column tile, k range); false for a tile the structure skips.
__device__ __forceinline__ bool g32_unit(const Tc32Params &p, int u, G32Unit &w) {
    int it = 0;
    while (it + 1 < p.nitems && u >= p.item[it + 1].unit0) ++it;
    const Tc32Item I = p.item[it];
    const int local = u - I.unit0;
    const int part = local % I.parts;
    const int tile = local / I.parts;
    const int tn = (I.n + G32_BN - 1) / G32_BN;
    w.i0 = (tile / tn) * G32_BM;
    w.j0 = (tile % tn) * G32_BN;
    int kb = 0, ke = I.k;
    if (p.a_upper) kb = (w.i0 / G32_BK) * G32_BK;
    if (p.b_upper) ke = min(ke, w.j0 + G32_BN);
    if (p.a_lower) ke = min(ke, w.i0 + G32_BM);
    if (p.b_lower) kb = max(kb, (w.j0 / G32_BK) * G32_BK);
    const int steps = ke > kb ? (ke - kb) / G32_BK : 0;
    w.k0 = kb + (int)((int64_t)steps * part / I.parts) * G32_BK;
    w.k1 = kb + (int)((int64_t)steps * (part + 1) / I.parts) * G32_BK;
    w.m = I.m; w.n = I.n; w.ldc = I.ldc; w.parts = I.parts; w.kmax = I.k;
    w.a_x0 = I.a_x0; w.a_y0 = I.a_y0; w.b_x0 = I.b_x0; w.b_y0 = I.b_y0;
    w.c_off = I.c_off;
    // every role decodes the same units, so a unit that fails is skipped by all three
    if (!GQ_IN_BOUNDS(p.status, it < p.nitems && w.i0 < w.m && w.j0 < w.n && w.k0 >= 0 &&
                                    w.k0 <= w.k1 && w.k1 <= w.kmax,
                      BS_TC32_TILE, u))
        return false;
    return !(p.upper_tiles && w.i0 > w.j0 + G32_BN - 1);
}

__global__ void __launch_bounds__(G32_THREADS, 1)
    k_gemm_tc32(const __grid_constant__ CUtensorMap ahi, const __grid_constant__ CUtensorMap alo,
                const __grid_constant__ CUtensorMap bhi, const __grid_constant__ CUtensorMap blo,
                const __grid_constant__ Tc32Params p) {
    if (failed(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + G32_STAGES * G32_STAGE);
    uint64_t *empty = full + G32_STAGES;
    uint64_t *tfull = empty + G32_STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *consumed = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G32_STAGES; ++s) {
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
    if (warp == 1) tc::tmem_alloc(tmem_slot, G32_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent (Tc32Params::pdl), the set-up above overlaps
    // the previous kernel's tail; nothing global is read or written before this wait,
    // which returns once that kernel has finished and its writes are visible (at once
    // for an ordinary launch).
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int u = blockIdx.x; u < p.units && !*abort; u += gridDim.x) {
                G32Unit w;
                if (!g32_unit(p, u, w)) continue;
                for (int k = w.k0; k < w.k1; k += G32_BK) {
                    // fp32 boxes: the innermost coordinate on a 16-byte boundary
                    if (!GQ_IN_BOUNDS(p.status, ((w.a_x0 + k) & 3) == 0 && ((w.b_x0 + k) & 3) == 0 &&
                                                    w.a_x0 + k >= 0 && w.b_x0 + k >= 0,
                                      BS_TC32_TMA, w.a_x0 + k)) {
                        *abort = 1;
                        break;
                    }
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort)) break;
                    tc::mbar_arrive_expect_tx(&full[stage], G32_STAGE);
                    uint8_t *st = smem + stage * G32_STAGE;
                    tc::tma_load_2d(st, &ahi, &full[stage], w.a_x0 + k, w.a_y0 + w.i0);
                    tc::tma_load_2d(st + G32_TILE, &alo, &full[stage], w.a_x0 + k, w.a_y0 + w.i0);
                    tc::tma_load_2d(st + 2 * G32_TILE, &bhi, &full[stage], w.b_x0 + k, w.b_y0 + w.j0);
                    tc::tma_load_2d(st + 3 * G32_TILE, &blo, &full[stage], w.b_x0 + k, w.b_y0 + w.j0);
                    ++issued;
                    if (++stage == G32_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (*abort) {
                for (int i = *reinterpret_cast<volatile int *>(consumed); i < issued; ++i) {
                    volatile int never = 0;
                    tc::mbar_wait(&full[i % G32_STAGES], (i / G32_STAGES) & 1, &never);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32_f32(G32_BM, G32_BN, 0);
            int stage = 0, acc = 0, n = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < p.units && !*abort; u += gridDim.x) {
                G32Unit w;
                if (!g32_unit(p, u, w)) continue;
                if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
                tc::fence_after_sync();
                const uint32_t d = tmem + acc * G32_BN;
                bool ok = true, first = true;
                for (int k = w.k0; k < w.k1; k += G32_BK) {
                    if (!tc::mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t s0 = tc::smem_u32(smem + stage * G32_STAGE);
#pragma unroll
                    for (int kk = 0; kk < G32_BK / 8; ++kk) {
                        const uint64_t ah = tc::desc_sw128(s0 + kk * 32, 16, 1024);
                        const uint64_t al = tc::desc_sw128(s0 + G32_TILE + kk * 32, 16, 1024);
                        const uint64_t bh = tc::desc_sw128(s0 + 2 * G32_TILE + kk * 32, 16, 1024);
                        const uint64_t bl = tc::desc_sw128(s0 + 3 * G32_TILE + kk * 32, 16, 1024);
                        mma_tf32(d, ah, bh, idesc, first ? 0u : 1u);
                        first = false;
                        mma_tf32(d, ah, bl, idesc, 1u);
                        mma_tf32(d, al, bh, idesc, 1u);
                    }
                    tc::mma_commit(&empty[stage]);
                    *reinterpret_cast<volatile int *>(consumed) = ++n;
                    if (++stage == G32_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc::mma_commit(&tfull[acc]);     // an empty k range leaves TMEM unread
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            tc::mma_commit(drain);
            volatile int never = 0;
            tc::mbar_wait(drain, 0, &never);
        }
    } else {
        const int quad = warp & 3;
        // a dependent launch may start its set-up now (it waits for this grid's end)
        asm volatile("griddepcontrol.launch_dependents;");
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            G32Unit w;
            if (!g32_unit(p, u, w)) continue;
            if (!tc::mbar_wait(&tfull[acc], acc_phase, abort)) break;
            tc::fence_after_sync();
            const bool empty_range = w.k1 <= w.k0;
            const float alpha = p.alpha;
            const bool mask = p.mask_strict_upper;
            const bool reduce = p.accumulate || w.parts > 1;
            float *cbase = p.C + w.c_off;
            const bool vec_c = (reinterpret_cast<uintptr_t>(p.C) & 15) == 0;
            // TMEM (thread = row): each thread writes its row's 32 columns of a chunk as
            // 16-byte stores or reductions when rows are 16-byte aligned
            const int row = w.i0 + quad * 32 + lane;
            const bool rvalid = row < w.m;
            float *crow = cbase + (int64_t)row * w.ldc;
            const bool v4 = ((w.ldc | (int)(w.c_off & 3)) & 3) == 0 && vec_c;
            float *const phi = reduce ? nullptr : p.pair_hi;
            float *const plo = p.pair_lo;
            const int64_t pld = p.pair_ld;
            const bool pv4 = phi && (pld & 3) == 0 &&
                             ((reinterpret_cast<uintptr_t>(phi) | reinterpret_cast<uintptr_t>(plo)) & 15) == 0;
#pragma unroll 1
            for (int c = 0; c < G32_BN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * G32_BN + c * 32 + ((uint32_t)(quad * 32) << 16), v);
                tc::tmem_ld_wait();
                const int col0 = w.j0 + c * 32;
                if (!rvalid || col0 >= w.n) continue;
                if (!GQ_IN_BOUNDS(p.status, p.c_extent == 0 || (w.c_off + (int64_t)row * w.ldc + col0 >= 0 &&
                                                                w.c_off + (int64_t)row * w.ldc + min(col0 + 32, w.n) <= p.c_extent),
                                  BS_TC32_C, w.c_off + (int64_t)row * w.ldc + col0))
                    continue;
                float x[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    x[q] = empty_range ? 0.f : alpha * __uint_as_float(v[q]);
                    if (mask && col0 + q <= row) x[q] = 0.f;
                }
                // no read-back: reductions (accumulate, or split inner range) and plain
                // stores (overwrite) are both fire-and-forget
                if (v4 && col0 + 32 <= w.n) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 f = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                        float4 *dst = reinterpret_cast<float4 *>(crow + col0 + 4 * q);
                        if (reduce) atomicAdd(dst, f);
                        else *dst = f;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        if (col0 + q >= w.n) break;
                        if (reduce) atomicAdd(crow + col0 + q, x[q]);
                        else crow[col0 + q] = x[q];
                    }
                }
                if (phi && GQ_IN_BOUNDS(p.status, p.pair_extent == 0 || ((int64_t)row * pld + min(col0 + 32, w.n) <= p.pair_extent),
                                        BS_TC32_PAIR, (int64_t)row * pld + col0)) {
                    // the stored values' tf32 pairs, as split_tf32 forms them
                    float *hrow = phi + (int64_t)row * pld + col0, *lrow = plo + (int64_t)row * pld + col0;
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        uint32_t b;
                        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(b) : "f"(x[q]));
                        v[q] = b;
                        x[q] -= __uint_as_float(b);
                    }
                    if (pv4 && col0 + 32 <= w.n) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            reinterpret_cast<float4 *>(hrow)[q] =
                                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                            reinterpret_cast<float4 *>(lrow)[q] =
                                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            if (col0 + q >= w.n) break;
                            hrow[q] = __uint_as_float(v[q]);
                            lrow[q] = x[q];
                        }
                    }
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
    }

    __syncwarp();   // each role warp reconverges before the block barrier
    tc::fence_before_sync();
    __syncthreads();
    if (*abort && threadIdx.x == 0) set_status(p.status, GPTQ_ERR_TIMEOUT);
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, G32_TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn tc32_encode_fn() {
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

bool tc32_available() { return tc32_encode_fn() != nullptr; }

// fp32 matrix [rows][ld] as boxes of box_cols x box_rows with the 128-byte swizzle.
gptq_status make_f32_map(CUtensorMap *m, const float *base, int64_t cols, int64_t rows, int64_t ld,
                         int box_cols, int box_rows) {
    EncodeTiledFn enc = tc32_encode_fn();
    if (!enc) return GPTQ_ERR_CUDA;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld * 4};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), gdim, gstride,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

// x -> (hi, lo): hi = tf32(x) (round to nearest), lo = x - hi. rows x cols (ld_in) into
// rows x cols (ld_out). One grid row per matrix row, batched over blockIdx.z.
__global__ void k_split_tf32(const float *__restrict__ in, int64_t ld_in, int cols,
                             float *__restrict__ hi, float *__restrict__ lo, int64_t ld_out,
                             int64_t batch_in, int64_t batch_out) {
    const int64_t r = blockIdx.y;
    in += blockIdx.z * batch_in + r * ld_in;
    hi += blockIdx.z * batch_out + r * ld_out;
    lo += blockIdx.z * batch_out + r * ld_out;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < cols; c += gridDim.x * blockDim.x) {
        const float x = in[c];
        uint32_t h;
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
        const float hf = __uint_as_float(h);
        hi[c] = hf;
        lo[c] = x - hf;
    }
}

// The same split, four columns per thread (16-byte loads and stores), the matrix
// flattened to rows x cols/4 units so that narrow column blocks still fill the grid;
// batched over blockIdx.y.
__global__ void k_split_tf32_v4(const float *__restrict__ in, int64_t ld_in, uint32_t c4,
                                uint32_t units, float *__restrict__ hi, float *__restrict__ lo,
                                int64_t ld_out, int64_t batch_in, int64_t batch_out) {
    in += blockIdx.y * batch_in;
    hi += blockIdx.y * batch_out;
    lo += blockIdx.y * batch_out;
    for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x) {
        const uint32_t r = u / c4, c = (u - r * c4) * 4;
        const float4 x = *reinterpret_cast<const float4 *>(in + r * ld_in + c);
        float4 h, l;
        uint32_t b;
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(b) : "f"(x.x));
        h.x = __uint_as_float(b);
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(b) : "f"(x.y));
        h.y = __uint_as_float(b);
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(b) : "f"(x.z));
        h.z = __uint_as_float(b);
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(b) : "f"(x.w));
        h.w = __uint_as_float(b);
        l = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
        *reinterpret_cast<float4 *>(hi + r * ld_out + c) = h;
        *reinterpret_cast<float4 *>(lo + r * ld_out + c) = l;
    }
}

gptq_status split_tf32(const float *in, int64_t ld_in, int rows, int cols, float *hi, float *lo,
                       int64_t ld_out, int batch, int64_t batch_in, int64_t batch_out,
                       cudaStream_t st) {
    if (rows <= 0 || cols <= 0) return GPTQ_OK;
    const int rec = prof_begin(GPTQ_PROF_SPLIT, st);
    const int64_t units = (int64_t)rows * (cols / 4);
    const bool vec = cols % 4 == 0 && ld_in % 4 == 0 && ld_out % 4 == 0 && batch_in % 4 == 0 &&
                     batch_out % 4 == 0 && aligned(in, 16) && aligned(hi, 16) && aligned(lo, 16) &&
                     units < (int64_t)1 << 31 && batch <= 65535;
    if (vec) {
        const int bx = (int)std::min<int64_t>((units + 255) / 256, 148 * 8);
        k_split_tf32_v4<<<dim3(bx, batch), 256, 0, st>>>(in, ld_in, (uint32_t)(cols / 4),
                                                         (uint32_t)units, hi, lo, ld_out, batch_in,
                                                         batch_out);
    } else {
        const int bx = (int)std::min<int64_t>(8, (cols + 255) / 256);
        k_split_tf32<<<dim3(bx, rows, batch), 256, 0, st>>>(in, ld_in, cols, hi, lo, ld_out,
                                                            batch_in, batch_out);
    }
    prof_end(rec, st);
    return launch_status();
}

// Transposing split: in rows x cols (ld_in) -> hi/lo cols x rows (ld_out), through
// 32 x 32 shared-memory tiles; batched over blockIdx.z.
__global__ void k_split_tf32_t(const float *__restrict__ in, int64_t ld_in, int rows, int cols,
                               float *__restrict__ hi, float *__restrict__ lo, int64_t ld_out,
                               int64_t batch_in, int64_t batch_out) {
    __shared__ float t[32][33];
    in += blockIdx.z * batch_in;
    hi += blockIdx.z * batch_out;
    lo += blockIdx.z * batch_out;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int r = r0 + y, c = c0 + threadIdx.x;
        t[y][threadIdx.x] = (r < rows && c < cols) ? in[(int64_t)r * ld_in + c] : 0.f;
    }
    __syncthreads();
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int c = c0 + y, r = r0 + threadIdx.x;      // output row c, column r
        if (c < cols && r < rows) {
            const float x = t[threadIdx.x][y];
            uint32_t h;
            asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
            const float hf = __uint_as_float(h);
            hi[(int64_t)c * ld_out + r] = hf;
            lo[(int64_t)c * ld_out + r] = x - hf;
        }
    }
}

gptq_status split_tf32_t(const float *in, int64_t ld_in, int rows, int cols, float *hi, float *lo,
                         int64_t ld_out, int batch, int64_t batch_in, int64_t batch_out,
                         cudaStream_t st) {
    if (rows <= 0 || cols <= 0) return GPTQ_OK;
    const int rec = prof_begin(GPTQ_PROF_SPLIT, st);
    k_split_tf32_t<<<dim3((cols + 31) / 32, (rows + 31) / 32, batch), dim3(32, 8), 0, st>>>(
        in, ld_in, rows, cols, hi, lo, ld_out, batch_in, batch_out);
    prof_end(rec, st);
    return launch_status();
}

int tc32_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Fill the unit table (tiles x parts per item, parts bounding the MMA chains) and
// launch. Items whose C needs zeroing when split (overwrite mode) are zeroed here.
gptq_status launch_gemm_tc32(const CUtensorMap maps[4], Tc32Params &p, cudaStream_t st) {
    if (p.nitems <= 0) return GPTQ_OK;
    int units = 0;
    const int max_steps_per_part = std::max(1, tc::MAX_MMA_CHAIN / G32_MMA_PER_KSTEP);
    for (int i = 0; i < p.nitems; ++i) {
        Tc32Item &I = p.item[i];
        const int tiles = ((I.m + G32_BM - 1) / G32_BM) * ((I.n + G32_BN - 1) / G32_BN);
        const int steps = (I.k + G32_BK - 1) / G32_BK;
        I.parts = std::max(1, (steps + max_steps_per_part - 1) / max_steps_per_part);
        I.unit0 = units;
        units += tiles * I.parts;
    }
    p.units = units;
    if (units == 0) return GPTQ_OK;
    if (p.pair_hi && (p.nitems != 1 || p.accumulate || p.item[0].parts != 1 || !p.pair_lo))
        return GPTQ_ERR_ARG;
    const int grid = std::min(units, p.max_grid > 0 ? std::min(p.max_grid, tc32_sms()) : tc32_sms());
    cudaFuncSetAttribute(k_gemm_tc32, cudaFuncAttributeMaxDynamicSharedMemorySize, G32_SMEM);
    const int rec = prof_begin(GPTQ_PROF_TC32, st);
    if (p.pdl) {
        // programmatic dependent launch: the kernel's set-up may overlap the previous
        // kernel on the stream; its griddepcontrol.wait orders every global access
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(G32_THREADS);
        cfg.dynamicSmemBytes = G32_SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaLaunchKernelEx(&cfg, k_gemm_tc32, maps[0], maps[1], maps[2], maps[3], p);
    } else {
        k_gemm_tc32<<<grid, G32_THREADS, G32_SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], p);
    }
    const gptq_status s = launch_status();
    prof_end(rec, st);
    return s;
}

}  // namespace gptq
