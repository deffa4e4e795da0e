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
// Layout on the device:
//   Wk   fp32 [N][K] working weights (dead coordinates zeroed)
//   Eb   fp32 [B][N] normalised errors of the current block (channel fastest, so
//        the sweep's stores coalesce and the far update reads it as A^T)
//   Pb   fp32 [B][N] pre-rounding weights of the block (GPTAQ)
// One CTA owns 128 channels of one group for a block; a thread owns a channel and
// keeps 32 of its block coordinates in registers at a time, the rest of the block
// in shared memory (coordinate-major so a warp's accesses hit distinct banks).
#include "common.cuh"
#include "gemm_simt.cuh"

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

template <typename T>
__global__ void k_init_work(const T *W, float *Wk, int N, int K, int per_group,
                            const uint8_t *dead, float *loss_acc) {
    const int64_t total = (int64_t)N * K;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(i / K), k = (int)(i % K);
        const bool d = dead && dead[(int64_t)(n / per_group) * K + k];
        Wk[i] = d ? 0.f : to_f32(W[i]);
        if (k == 0) loss_acc[n] = 0.f;
    }
}

template <bool GPTAQ>
__global__ void __launch_bounds__(SW_CH) k_sweep_block(
    float *__restrict__ Wk, int N, int per_group, int K, int i0, int bs,
    const float *__restrict__ U, const float *__restrict__ P1, const float *__restrict__ scale,
    int bits, uint8_t *__restrict__ codes, float *__restrict__ Eb, float *__restrict__ Pb,
    float *__restrict__ loss_acc, const int32_t *status) {
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
    U += (int64_t)grp * K * K;

    // Stage U[blk, blk] (and P1[blk, blk]) with zero padding, and the W tile.
    for (int idx = tid; idx < SW_MAXB * SW_MAXB; idx += SW_CH) {
        const int r = idx / SW_MAXB, c = idx % SW_MAXB;
        const bool in = r < bs && c < bs;
        Us[r * SW_ULD + c] = in ? U[(int64_t)(i0 + r) * K + i0 + c] : 0.f;
        if (GPTAQ) Ps[r * SW_ULD + c] = in ? P1[(int64_t)(i0 + r) * K + i0 + c] : 0.f;
    }
    for (int r = 0; r < SW_CH; ++r) {
        const bool in = r < nvalid && tid < bs;
        Wt[tid * SW_WLD + r] = in ? Wk[(int64_t)(n0 + r) * K + i0 + tid] : 0.f;
    }
    __syncthreads();

    const float s = tid < nvalid ? scale[n] : 1.f;
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
                const float c = fminf(fmaxf(rintf(wj / s) + zf, 0.f), maxq);
                const float q = s * (c - zf);
                const float ej = (wj - q) / Us[j * SW_ULD + j];
                e[t] = ej;
                wp[t] = wj;
                lacc = fmaf(ej, ej, lacc);
                Cs[j * SW_CLD + tid] = (uint8_t)c;
                if (tid < nvalid) {
                    Eb[(int64_t)j * N + n] = ej;
                    if (GPTAQ) Pb[(int64_t)j * N + n] = wj;
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
    const int64_t total = (int64_t)N * K;
    const float zf = (float)(1 << (bits - 1));
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(i / K), k = (int)(i % K);
        if (write_back) W[i] = from_f32<T>(scale[n] * ((float)codes[i] - zf));
        if (loss && k == 0) loss[n] = 0.5f * loss_acc[n];
    }
}

size_t quantize_workspace(int K, int N, int g, int blocksize) {
    (void)g;
    Carver c(nullptr);
    c.take<float>((size_t)N * K);          // Wk
    c.take<float>((size_t)blocksize * N);  // Eb
    c.take<float>((size_t)blocksize * N);  // Pb
    c.take<float>((size_t)N);              // scale
    c.take<float>((size_t)N);              // loss_acc
    return round_up(c.off, 256);
}

static size_t sweep_smem(bool gptaq) {
    return (size_t)SW_MAXB * SW_ULD * sizeof(float) * (gptaq ? 2 : 1) +
           (size_t)SW_MAXB * SW_WLD * sizeof(float) + (size_t)SW_MAXB * SW_CLD;
}

gptq_status quantize_layer(void *W, int wdtype, int N, int K, const float *U, int groups, int bits,
                           int blocksize, const float *P1, const uint8_t *dead,
                           const float *scales_in, float *scales_out, uint8_t *codes, float *loss,
                           int write_back, void *ws, int32_t *status, cudaStream_t st) {
    Carver cv(ws);
    float *Wk = cv.take<float>((size_t)N * K);
    float *Eb = cv.take<float>((size_t)blocksize * N);
    float *Pb = cv.take<float>((size_t)blocksize * N);
    float *scale = cv.take<float>((size_t)N);
    float *loss_acc = cv.take<float>((size_t)N);
    const int per_group = N / groups;
    const int64_t KK = (int64_t)K * K;

    k_scale<<<(N * 32 + 255) / 256, 256, 0, st>>>(W, wdtype, N, K, bits, scales_in, scale,
                                                   scales_out, status);
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    if (wdtype == GPTQ_F32)
        k_init_work<float><<<1184, 256, 0, st>>>(static_cast<const float *>(W), Wk, N, K,
                                                 per_group, dead, loss_acc);
    else
        k_init_work<__nv_bfloat16><<<1184, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(W), Wk, N, K, per_group, dead, loss_acc);
    if ((s = launch_status()) != GPTQ_OK) return s;

    const bool gptaq = P1 != nullptr;
    const size_t smem = sweep_smem(gptaq);
    if (gptaq)
        cudaFuncSetAttribute(k_sweep_block<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else
        cudaFuncSetAttribute(k_sweep_block<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const dim3 grid((per_group + SW_CH - 1) / SW_CH, groups);
    for (int i0 = 0; i0 < K; i0 += blocksize) {
        const int bs = min(blocksize, K - i0);
        const int i1 = i0 + bs;
        if (gptaq)
            k_sweep_block<true><<<grid, SW_CH, smem, st>>>(Wk, N, per_group, K, i0, bs, U, P1, scale,
                                                          bits, codes, Eb, Pb, loss_acc, status);
        else
            k_sweep_block<false><<<grid, SW_CH, smem, st>>>(Wk, N, per_group, K, i0, bs, U, P1, scale,
                                                           bits, codes, Eb, Pb, loss_acc, status);
        if ((s = launch_status()) != GPTQ_OK) return s;
        if (i1 >= K) break;
        // W[:, i1:] -= E_blk U[blk, i1:]   per group: A(n, j) = Eb[j*N + n]
        GemmParams p = gemm_params(per_group, K - i1, bs, Eb, N, U + (int64_t)i0 * K + i1, K,
                                   Wk + i1, K, -1.f, 1, status);
        p.sA = per_group; p.sB = KK; p.sC = (int64_t)per_group * K;
        if ((s = gemm_simt<float, float, true, false>(p, groups, st)) != GPTQ_OK) return s;
        if (gptaq) {
            GemmParams q = gemm_params(N, K - i1, bs, Pb, N, P1 + (int64_t)i0 * K + i1, K,
                                       Wk + i1, K, 1.f, 1, status);
            if ((s = gemm_simt<float, float, true, false>(q, 1, st)) != GPTQ_OK) return s;
        }
    }
    if (wdtype == GPTQ_F32)
        k_finalize<float><<<1184, 256, 0, st>>>(static_cast<float *>(W), codes, scale, N, K, bits,
                                                write_back, loss_acc, loss);
    else
        k_finalize<__nv_bfloat16><<<1184, 256, 0, st>>>(static_cast<__nv_bfloat16 *>(W), codes,
                                                        scale, N, K, bits, write_back, loss_acc, loss);
    return launch_status();
}

}  // namespace gptq
