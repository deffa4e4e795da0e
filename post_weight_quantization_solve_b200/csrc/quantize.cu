// gptq_quantize_layer: per-channel scale, then the shared-order sweep with lazy
// blocks, optional GPTAQ row term, codes / reconstruction / loss outputs.
//
// [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": every output channel takes the
// input coordinates in the same order; inside a block of B coordinates
//   c = clamp(rint(w_j / s) + z, 0, 2^b - 1),  q = s (c - z),
//   E_j = (w_j - q) / U_jj,   W_k -= U_jk E_j  (k later in the block),
// and at the block end the far coordinates get W_far -= U[blk, far]^T E_blk.
// [ResComp] item 3: GPTAQ adds w_j^pre * P1[j, k] the same way.
//
// Two-level lazy scheme: blocks of B coordinates inside super-blocks of S = 512.
// After each block the rest of its super-block is updated ("near" update); after
// each super-block the coordinates beyond it ("far" update, inner length S). Both
// are tensor-core products (update_tc.cu); the blocking changes only the order of
// the work, and the far traffic drops by S / B.
//
// Layout on the device:
//   Wk        fp32 [N][K] working weights (dead coordinates zeroed)
//   Eh, El    bf16 [S][ldE] normalised errors of the super-block as hi + lo pairs,
//             row j - sb0, column grp * ldG + local channel (channel fastest, so the
//             sweep's stores coalesce; the update reads it as an MN-major operand)
//   Ph, Pl    bf16 [S][ldE] pre-rounding weights (GPTAQ), same layout
//   Uh, Ul    bf16 [g][K][ldU] U as hi + lo pairs;  Qh, Ql  the same for P1
// One CTA owns 128 channels of one group for a block; a thread owns a channel and
// keeps 32 of its block coordinates in registers at a time, the rest of the block
// in shared memory (coordinate-major so a warp's accesses hit distinct banks).
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "update_tc.cuh"

namespace gptq {

constexpr int SW_CH = 128;     // channels per CTA
constexpr int SW_MAXB = 128;   // largest block
constexpr int SW_ULD = SW_MAXB + 4;
constexpr int SW_WLD = SW_CH + 1;
constexpr int SW_CLD = SW_CH + 4;

__global__ void k_scale(const void *W, int wdtype, int N, int K, int bits,
                        const float *scales_in, float *scale, float *scales_out,
                        int32_t *status) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= N) return;
    float amax = 0.f;
    bool bad = false;
    for (int k = lane; k < K; k += 32) {
        const float v = wdtype == GPTQ_F32
                            ? static_cast<const float *>(W)[(int64_t)warp * K + k]
                            : __bfloat162float(
                                  static_cast<const __nv_bfloat16 *>(W)[(int64_t)warp * K + k]);
        bad |= !isfinite(v);
        amax = fmaxf(amax, fabsf(v));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
        float s;
        if (scales_in) {
            s = scales_in[warp];
            bad |= !(isfinite(s) && s > 0.f);
        } else {
            s = amax == 0.f ? 1.f : 2.f * amax / (float)((1 << bits) - 1);
        }
        if (bad) set_status(status, GPTQ_ERR_NONFINITE);
        scale[warp] = s;
        if (scales_out) scales_out[warp] = s;
    }
}

// One grid row (blockIdx.y) per output channel.
template <typename T>
__global__ void k_init_work(const T *W, float *Wk, int N, int K, int per_group,
                            const uint8_t *dead, float *loss_acc) {
    const int n = blockIdx.y;
    const int64_t row = (int64_t)n * K;
    const uint8_t *dg = dead ? dead + (int64_t)(n / per_group) * K : nullptr;
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x) {
        const bool d = dg && dg[k];
        Wk[row + k] = d ? 0.f : to_f32(W[row + k]);
        if (k == 0) loss_acc[n] = 0.f;
    }
}

template <bool GPTAQ>
__global__ void __launch_bounds__(SW_CH) k_sweep_block(
    float *__restrict__ Wk, int N, int per_group, int K, int i0, int bs,
    const float *__restrict__ U, const float *__restrict__ P1, const float *__restrict__ scale,
    int bits, uint8_t *__restrict__ codes, __nv_bfloat16 *__restrict__ Eh,
    __nv_bfloat16 *__restrict__ El, __nv_bfloat16 *__restrict__ Ph, __nv_bfloat16 *__restrict__ Pl,
    int ldE, int ldG, int erow0, float *__restrict__ loss_acc, const int32_t *status) {
    if (failed(status)) return;
    extern __shared__ __align__(16) unsigned char smem[];
    float *Us = reinterpret_cast<float *>(smem);                 // [SW_MAXB][SW_ULD]
    float *Ps = Us + SW_MAXB * SW_ULD;                           // GPTAQ only
    float *Wt = Ps + (GPTAQ ? SW_MAXB * SW_ULD : 0);             // [SW_MAXB][SW_WLD]
    uint8_t *Cs = reinterpret_cast<uint8_t *>(Wt + SW_MAXB * SW_WLD);  // [SW_MAXB][SW_CLD]

    const int grp = blockIdx.y;
    const int n0 = grp * per_group + blockIdx.x * SW_CH;
    const int nvalid = min(SW_CH, (grp + 1) * per_group - n0);
    const int tid = threadIdx.x;
    const int n = n0 + tid;
    const int64_t ecol = (int64_t)grp * ldG + blockIdx.x * SW_CH + tid;
    U += (int64_t)grp * K * K;

    // Stage U[blk, blk] (and P1[blk, blk]) with zero padding, and the W tile; loads
    // are unrolled so that many are in flight per thread.
#pragma unroll 8
    for (int it = 0; it < SW_MAXB; ++it) {
        const int r = it, c = tid;
        const bool in = r < bs && c < bs;
        Us[r * SW_ULD + c] = in ? U[(int64_t)(i0 + r) * K + i0 + c] : 0.f;
        if (GPTAQ) Ps[r * SW_ULD + c] = in ? P1[(int64_t)(i0 + r) * K + i0 + c] : 0.f;
    }
#pragma unroll 8
    for (int r = 0; r < SW_CH; ++r) {
        const bool in = r < nvalid && tid < bs;
        Wt[tid * SW_WLD + r] = in ? Wk[(int64_t)(n0 + r) * K + i0 + tid] : 0.f;
    }
    __syncthreads();
    // reciprocal pivots of the block (a multiply in the serial chain instead of a divide)
    float *rpiv = reinterpret_cast<float *>(Cs + SW_MAXB * SW_CLD);
    if (tid < bs) rpiv[tid] = 1.f / Us[tid * SW_ULD + tid];
    __syncthreads();

    const float s = tid < nvalid ? scale[n] : 1.f;
    const float rs = 1.f / s;
    const float zf = (float)(1 << (bits - 1));
    const float maxq = (float)((1 << bits) - 1);
    float lacc = 0.f;

    const int nsb = (bs + 31) / 32;
    for (int sb = 0; sb < nsb; ++sb) {
        const int jb = sb * 32;
        float w[32], e[32], wp[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) w[t] = Wt[(jb + t) * SW_WLD + tid];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int j = jb + t;
            e[t] = 0.f;
            wp[t] = 0.f;
            if (j < bs) {
                const float wj = w[t];
                const float c = fminf(fmaxf(rintf(wj * rs) + zf, 0.f), maxq);
                const float q = s * (c - zf);
                const float ej = (wj - q) * rpiv[j];
                e[t] = ej;
                wp[t] = wj;
                lacc = fmaf(ej, ej, lacc);
                Cs[j * SW_CLD + tid] = (uint8_t)c;
                if (tid < nvalid) {
                    const int64_t e = (int64_t)(erow0 + j) * ldE + ecol;
                    const __nv_bfloat16 eh = __float2bfloat16_rn(ej);
                    Eh[e] = eh;
                    El[e] = __float2bfloat16_rn(ej - __bfloat162float(eh));
                    if (GPTAQ) {
                        const __nv_bfloat16 ph = __float2bfloat16_rn(wj);
                        Ph[e] = ph;
                        Pl[e] = __float2bfloat16_rn(wj - __bfloat162float(ph));
                    }
                }
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    if (4 * q4 + 3 > t) {
                        const float4 u = *reinterpret_cast<const float4 *>(&Us[j * SW_ULD + jb + 4 * q4]);
                        const float uu[4] = {u.x, u.y, u.z, u.w};
                        float pp[4] = {0.f, 0.f, 0.f, 0.f};
                        if (GPTAQ) {
                            const float4 p4 = *reinterpret_cast<const float4 *>(&Ps[j * SW_ULD + jb + 4 * q4]);
                            pp[0] = p4.x; pp[1] = p4.y; pp[2] = p4.z; pp[3] = p4.w;
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int ui = 4 * q4 + r;
                            if (ui > t) {
                                w[ui] = fmaf(-ej, uu[r], w[ui]);
                                if (GPTAQ) w[ui] = fmaf(wj, pp[r], w[ui]);
                            }
                        }
                    }
                }
            }
        }
        // later coordinates of this block: 4 at a time
        for (int k = jb + 32; k < bs; k += 4) {
            float a0 = Wt[(k + 0) * SW_WLD + tid], a1 = Wt[(k + 1) * SW_WLD + tid];
            float a2 = Wt[(k + 2) * SW_WLD + tid], a3 = Wt[(k + 3) * SW_WLD + tid];
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const float4 u = *reinterpret_cast<const float4 *>(&Us[(jb + t) * SW_ULD + k]);
                a0 = fmaf(-e[t], u.x, a0); a1 = fmaf(-e[t], u.y, a1);
                a2 = fmaf(-e[t], u.z, a2); a3 = fmaf(-e[t], u.w, a3);
                if (GPTAQ) {
                    const float4 p4 = *reinterpret_cast<const float4 *>(&Ps[(jb + t) * SW_ULD + k]);
                    a0 = fmaf(wp[t], p4.x, a0); a1 = fmaf(wp[t], p4.y, a1);
                    a2 = fmaf(wp[t], p4.z, a2); a3 = fmaf(wp[t], p4.w, a3);
                }
            }
            Wt[(k + 0) * SW_WLD + tid] = a0; Wt[(k + 1) * SW_WLD + tid] = a1;
            Wt[(k + 2) * SW_WLD + tid] = a2; Wt[(k + 3) * SW_WLD + tid] = a3;
        }
    }
    if (tid < nvalid) loss_acc[n] += lacc;
    __syncthreads();
    for (int r = 0; r < nvalid; ++r)
        if (tid < bs) codes[(int64_t)(n0 + r) * K + i0 + tid] = Cs[tid * SW_CLD + r];
}

template <typename T>
__global__ void k_finalize(T *W, const uint8_t *codes, const float *scale, int N, int K,
                           int bits, int write_back, const float *loss_acc, float *loss) {
    const int n = blockIdx.y;
    const int64_t row = (int64_t)n * K;
    const float zf = (float)(1 << (bits - 1));
    const float s = scale[n];
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x) {
        if (write_back) W[row + k] = from_f32<T>(s * ((float)codes[row + k] - zf));
        if (loss && k == 0) loss[n] = 0.5f * loss_acc[n];
    }
}

constexpr int SUPER = 512;

struct QLayout {
    int ldU, ldG, ldE;
    explicit QLayout(int K, int N, int g) {
        ldU = (int)round_up((size_t)K, 8);
        ldG = (int)round_up((size_t)(N / g), 8);
        ldE = ldG * g;
    }
};

size_t quantize_workspace(int K, int N, int g, int blocksize) {
    (void)blocksize;
    const QLayout lay(K, N, g);
    Carver c(nullptr);
    c.take<float>((size_t)N * K);                           // Wk
    for (int i = 0; i < 2; ++i) c.take<__nv_bfloat16>((size_t)g * K * lay.ldU);   // Uh, Ul
    for (int i = 0; i < 2; ++i) c.take<__nv_bfloat16>((size_t)K * lay.ldU);       // Qh, Ql
    for (int i = 0; i < 4; ++i) c.take<__nv_bfloat16>((size_t)SUPER * lay.ldE);   // Eh El Ph Pl
    c.take<float>((size_t)N);                               // scale
    c.take<float>((size_t)N);                               // loss_acc
    return round_up(c.off, 256);
}

static size_t sweep_smem(bool gptaq) {
    return (size_t)SW_MAXB * SW_ULD * sizeof(float) * (gptaq ? 2 : 1) +
           (size_t)SW_MAXB * SW_WLD * sizeof(float) + (size_t)SW_MAXB * SW_CLD +
           SW_MAXB * sizeof(float);
}

gptq_status quantize_layer(void *W, int wdtype, int N, int K, const float *U, int groups, int bits,
                           int blocksize, const float *P1, const uint8_t *dead,
                           const float *scales_in, float *scales_out, uint8_t *codes, float *loss,
                           int write_back, void *ws, int32_t *status, cudaStream_t st) {
    if (!update_tc_available()) return GPTQ_ERR_CUDA;
    const QLayout lay(K, N, groups);
    Carver cv(ws);
    float *Wk = cv.take<float>((size_t)N * K);
    __nv_bfloat16 *Uh = cv.take<__nv_bfloat16>((size_t)groups * K * lay.ldU);
    __nv_bfloat16 *Ul = cv.take<__nv_bfloat16>((size_t)groups * K * lay.ldU);
    __nv_bfloat16 *Qh = cv.take<__nv_bfloat16>((size_t)K * lay.ldU);
    __nv_bfloat16 *Ql = cv.take<__nv_bfloat16>((size_t)K * lay.ldU);
    __nv_bfloat16 *Eh = cv.take<__nv_bfloat16>((size_t)SUPER * lay.ldE);
    __nv_bfloat16 *El = cv.take<__nv_bfloat16>((size_t)SUPER * lay.ldE);
    __nv_bfloat16 *Ph = cv.take<__nv_bfloat16>((size_t)SUPER * lay.ldE);
    __nv_bfloat16 *Pl = cv.take<__nv_bfloat16>((size_t)SUPER * lay.ldE);
    float *scale = cv.take<float>((size_t)N);
    float *loss_acc = cv.take<float>((size_t)N);
    const int per_group = N / groups;
    const int64_t KK = (int64_t)K * K;
    const bool gptaq = P1 != nullptr;
    const int rowgrid = std::min(8, (K + 255) / 256);

    k_scale<<<(N * 32 + 255) / 256, 256, 0, st>>>(W, wdtype, N, K, bits, scales_in, scale,
                                                   scales_out, status);
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    if (wdtype == GPTQ_F32)
        k_init_work<float><<<dim3(rowgrid, N), 256, 0, st>>>(static_cast<const float *>(W), Wk, N,
                                                            K, per_group, dead, loss_acc);
    else
        k_init_work<__nv_bfloat16><<<dim3(rowgrid, N), 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(W), Wk, N, K, per_group, dead, loss_acc);
    if ((s = launch_status()) != GPTQ_OK) return s;
    if ((s = split_bf16(U, K, K, K, Uh, Ul, lay.ldU, groups, KK, (int64_t)K * lay.ldU, st)) != GPTQ_OK)
        return s;
    if (gptaq && (s = split_bf16(P1, K, K, K, Qh, Ql, lay.ldU, 1, 0, 0, st)) != GPTQ_OK) return s;

    // tensor maps: A operands over the super-block buffers, B operands per group
    // [box rows 16 / 64][group]
    static thread_local UpdateMaps maps[2][8];
    if (groups > 8) return GPTQ_ERR_ARG;
    for (int bi = 0; bi < 2; ++bi) {
        const int box = bi == 0 ? 16 : 64;
        for (int gi = 0; gi < groups; ++gi) {
            UpdateMaps &m = maps[bi][gi];
            __nv_bfloat16 *a_src[4] = {Eh, El, Ph, Pl};
            for (int i = 0; i < 4; ++i)
                if ((s = make_bf16_map(&m.a[i], a_src[i], lay.ldE, SUPER, lay.ldE, box)) != GPTQ_OK)
                    return s;
            const __nv_bfloat16 *b_src[4] = {Uh + (int64_t)gi * K * lay.ldU,
                                             Ul + (int64_t)gi * K * lay.ldU, Qh, Ql};
            for (int i = 0; i < 4; ++i)
                if ((s = make_bf16_map(&m.b[i], b_src[i], K, K, lay.ldU, box)) != GPTQ_OK) return s;
        }
    }
    UpdateParams base{};
    base.ldc = K;
    base.M = per_group;
    base.vec4 = (K % 4 == 0);
    base.status = status;
    // -E (hi*hi + hi*lo + lo*hi) U, and for GPTAQ +W_pre (same splits) P1
    const int terms[6][3] = {{0, 0, 1}, {0, 1, 1}, {1, 0, 1}, {2, 2, 0}, {2, 3, 0}, {3, 2, 0}};
    base.nterms = gptaq ? 6 : 3;
    for (int t = 0; t < base.nterms; ++t) {
        base.a_id[t] = terms[t][0];
        base.b_id[t] = terms[t][1];
        base.neg[t] = terms[t][2];
    }

    const size_t smem = sweep_smem(gptaq);
    if (gptaq)
        cudaFuncSetAttribute(k_sweep_block<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else
        cudaFuncSetAttribute(k_sweep_block<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const dim3 grid((per_group + SW_CH - 1) / SW_CH, groups);
    for (int sb0 = 0; sb0 < K; sb0 += SUPER) {
        const int sb1 = min(K, sb0 + SUPER);
        for (int i0 = sb0; i0 < sb1; i0 += blocksize) {
            const int i1 = min(i0 + blocksize, sb1);
            const int bs = i1 - i0;
            if (gptaq)
                k_sweep_block<true><<<grid, SW_CH, smem, st>>>(
                    Wk, N, per_group, K, i0, bs, U, P1, scale, bits, codes, Eh, El, Ph, Pl,
                    lay.ldE, lay.ldG, i0 - sb0, loss_acc, status);
            else
                k_sweep_block<false><<<grid, SW_CH, smem, st>>>(
                    Wk, N, per_group, K, i0, bs, U, P1, scale, bits, codes, Eh, El, Ph, Pl,
                    lay.ldE, lay.ldG, i0 - sb0, loss_acc, status);
            if ((s = launch_status()) != GPTQ_OK) return s;
            if (i1 >= sb1) continue;
            for (int gi = 0; gi < groups; ++gi) {      // near: the rest of the super-block
                UpdateParams p = base;
                p.C = Wk + (int64_t)gi * per_group * K + i1;
                p.Ncols = sb1 - i1;
                p.L = bs;
                p.a_x0 = gi * lay.ldG;
                p.a_y0 = i0 - sb0;
                p.b_x0 = i1;
                p.b_y0 = i0;
                const int box = p.L % 64 == 0 ? 64 : 16;
                if ((s = launch_update_tc(maps[box == 64][gi], p, box, st)) != GPTQ_OK) return s;
            }
        }
        if (sb1 >= K) break;
        for (int gi = 0; gi < groups; ++gi) {          // far: everything after the super-block
            UpdateParams p = base;
            p.C = Wk + (int64_t)gi * per_group * K + sb1;
            p.Ncols = K - sb1;
            p.L = sb1 - sb0;
            p.a_x0 = gi * lay.ldG;
            p.a_y0 = 0;
            p.b_x0 = sb1;
            p.b_y0 = sb0;
            const int box = p.L % 64 == 0 ? 64 : 16;
            if ((s = launch_update_tc(maps[box == 64][gi], p, box, st)) != GPTQ_OK) return s;
        }
    }
    if (wdtype == GPTQ_F32)
        k_finalize<float><<<dim3(rowgrid, N), 256, 0, st>>>(static_cast<float *>(W), codes, scale,
                                                           N, K, bits, write_back, loss_acc, loss);
    else
        k_finalize<__nv_bfloat16><<<dim3(rowgrid, N), 256, 0, st>>>(
            static_cast<__nv_bfloat16 *>(W), codes, scale, N, K, bits, write_back, loss_acc, loss);
    return launch_status();
}

}  // namespace gptq
