// gptq_quantize_layer: per-channel scale, then the shared-order sweep with lazy
// blocks, optional GPTAQ row term, codes / reconstruction / loss outputs.
//
// [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": every output channel takes the
// input coordinates in the same order; inside a block of B coordinates
//   c = clamp(rint(w_j / s) + z, 0, 2^b - 1),  q = s (c - z),
//   E_j = (w_j - q) / U_jj,   W_k -= U_jk E_j  (k later in the block),
// and at the block end the far coordinates get W_far -= U[blk, far]^T E_blk.
// [ResComp] item 3: GPTAQ adds w_j^pre * P1[j, k] the same way.
// [ResComp] items 1-3, compensation-aware error (CAE): the row term
// (w_j^(0) - w_j^pre) P2[j, k] with P2 = [((H + C) U^T) ⊙ M] U. Since U^T U = H_d^-1 and
// H_d differs from H only on the diagonal, the H part of P2 is I - diag(U)^-1 U, and
// the GPTQ step, the GPTAQ row and this row merge into one propagated error
// E'_j = (w_j^(0) - q) / U_jj and a P1 row scaled by w_j^(0): P2 is never formed, the
// sweep reads the starting weights w^(0) instead of the current ones for those two
// terms, and the lazy updates are unchanged.
//
// Two-level lazy scheme: blocks of B coordinates inside super-blocks of S = 512.
// After each block the rest of its super-block is updated ("near" update); after
// each super-block the coordinates beyond it ("far" update, inner length S). Both
// are tensor-core products (update_tc.cu); the blocking changes only the order of
// the work, and the far traffic drops by S / B. The tensor-core sweep (sweep_tc.cu)
// keeps the near updates in TMEM and runs the far updates by pairs of super-blocks
// (update_plan.h: inner length 2S after every second super-block).
//
// Layout on the device:
//   Wk        fp32 [N][K] working weights (dead coordinates zeroed)
//   Eh, El    bf16 normalised errors as hi + lo pairs. SIMT sweeps: [S][ldE], row
//             j - sb0, column grp * ldG + local channel (channel fastest, so their stores
//             coalesce; the update reads it as an MN-major operand). Tensor-core sweep:
//             [ldE][1024], a channel's row holding two super-blocks (columns 0 and S),
//             read by the update as a K-major operand.
//   Ph, Pl    pre-rounding weights (GPTAQ; with CAE the starting weights), same layouts
//   W0k       fp32 [N][K] starting weights w^(0) (CAE only)
//   Uh, Ul    bf16 [g][K][ldU] U as hi + lo pairs;  Qh, Ql  the same for P1
// The sweep keeps each channel's block coordinates in registers: one thread per
// channel for layers with many output channels (k_sweep_thread; two lanes per channel
// with CAE), four lanes per channel otherwise (k_sweep_lanes).
#include <cuda.h>

#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "sweep_tc.cuh"
#include "update_plan.h"
#include "update_tc.cuh"

namespace gptq {

constexpr int SW_MAXB = 128;   // largest block: four 32-coordinate sub-blocks

// Eight consecutive weights of a row as fp32 (one 16-byte load for bf16, two for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// One CTA per output channel n: the symmetric scale s_n = 2 max_k |W_nk| / (2^b - 1)
// from W as given (or the caller's scale), and the fp32 working row with dead
// coordinates zeroed, from one read of the row.
template <typename T>
__global__ void __launch_bounds__(256) k_scale_init(const T *__restrict__ W, float *__restrict__ Wk,
                                                    int K, int per_group, int bits,
                                                    const uint8_t *__restrict__ dead,
                                                    const float *__restrict__ scales_in,
                                                    float *__restrict__ scale, float *scales_out,
                                                    float *__restrict__ loss_acc, int vec,
                                                    int32_t *status, const int32_t *perm,
                                                    float *__restrict__ W0k) {
    const int n = blockIdx.x;
    const T *wr = W + (int64_t)n * K;
    float *kr = Wk + (int64_t)n * K;
    float *k0 = W0k ? W0k + (int64_t)n * K : nullptr;   // copy of the starting weights
    const uint8_t *dg = dead ? dead + (int64_t)(n / per_group) * K : nullptr;
    float amax = 0.f;
    bool bad = false;
    if (perm) {  // working copy in processing order: Wk[n][j] = W[n][perm[j]]
        for (int k = threadIdx.x; k < K; k += 256) {
            const float x = to_f32(wr[perm[k]]);
            bad |= !isfinite(x);
            amax = fmaxf(amax, fabsf(x));
            kr[k] = (dg && dg[k]) ? 0.f : x;
            if (k0) k0[k] = kr[k];
        }
    } else if (vec) {   // rows 16-byte aligned for both W and Wk, K % 8 == 0
        for (int k = threadIdx.x * 8; k < K; k += 256 * 8) {
            float x[8];
            load8(wr + k, x);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                bad |= !isfinite(x[i]);
                amax = fmaxf(amax, fabsf(x[i]));
                if (dg && dg[k + i]) x[i] = 0.f;
            }
            *reinterpret_cast<float4 *>(kr + k) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4 *>(kr + k + 4) = make_float4(x[4], x[5], x[6], x[7]);
            if (k0) {
                *reinterpret_cast<float4 *>(k0 + k) = make_float4(x[0], x[1], x[2], x[3]);
                *reinterpret_cast<float4 *>(k0 + k + 4) = make_float4(x[4], x[5], x[6], x[7]);
            }
        }
    } else {
        for (int k = threadIdx.x; k < K; k += 256) {
            const float x = to_f32(wr[k]);
            bad |= !isfinite(x);
            amax = fmaxf(amax, fabsf(x));
            kr[k] = (dg && dg[k]) ? 0.f : x;
            if (k0) k0[k] = kr[k];
        }
    }
    __shared__ float red[8];
    __shared__ int redb[8];
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const bool wbad = __any_sync(0xffffffffu, bad);
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5] = amax;
        redb[threadIdx.x >> 5] = wbad;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool b = false;
        for (int i = 0; i < 8; ++i) {
            amax = fmaxf(amax, red[i]);
            b |= redb[i] != 0;
        }
        float s;
        if (scales_in) {
            s = scales_in[n];
            b |= !(isfinite(s) && s > 0.f);
        } else {
            s = amax == 0.f ? 1.f : 2.f * amax / (float)((1 << bits) - 1);
        }
        if (b) set_status(status, GPTQ_ERR_NONFINITE);
        scale[n] = s;
        if (scales_out) scales_out[n] = s;
        loss_acc[n] = 0.f;
    }
}

// Input-dimension groups seen by the sweep: mode 0 per-channel scale, 1 re-estimated
// at group entry (written to gsc), 2 static (read from gsc); gsc is [N][ldg], gsel[j]
// the group of processing position j.
struct SweepGroups {
    int G;
    float *gsc;
    int ldg;
    const int32_t *gsel;
};

// 16-byte global -> shared copy that bypasses registers; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
// 4-byte global -> shared copy; src_bytes = 0 writes a zero.
__device__ __forceinline__ void cp_async4(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// In-block sweep, lane-group form (for layers with few output channels): one block
// [i0, i0 + bs) for 128 / LPC channels of one group.
// A warp serves 32 / LPC channels with LPC lanes each: lane LPC c + q of the warp holds,
// of channel c, the coordinates 32 b + CPL q + i (i < CPL = 32 / LPC) of every 32-wide
// sub-block b, so all of the block's coordinates stay in registers and every lane has
// work at every step. At step j = 32 p + t the lane holding coordinate j (slot
// q = t / CPL) rounds it and computes E_j; a shuffle inside the channel's lanes hands
// E_j to the others,
// and each lane applies it to its own coordinates (U's zero lower triangle makes the
// coordinates at or before j no-ops, so no lane masks). The sub-block in work is
// always w[0]: the register array shifts by one sub-block after each phase. No block
// barrier inside the sweep. U[blk, blk] (and P1) is staged once per CTA as its ten
// 32 x 32 blocks on or above the diagonal.
template <bool GPTAQ, int GMODE, bool CAE, int LPC>
__global__ void __launch_bounds__(128, (GPTAQ || LPC < 4) ? 2 : 4) k_sweep_lanes(
    float *__restrict__ Wk, int N, int per_group, int K, int i0, int bs,
    const float *__restrict__ U, const float *__restrict__ P1, const float *__restrict__ scale,
    int bits, uint8_t *__restrict__ codes, __nv_bfloat16 *__restrict__ Eh,
    __nv_bfloat16 *__restrict__ El, __nv_bfloat16 *__restrict__ Ph, __nv_bfloat16 *__restrict__ Pl,
    int ldE, int ldG, int erow0, float *__restrict__ loss_acc, int vec, const int32_t *status,
    const SweepGroups sg, const float *__restrict__ W0k) {
    constexpr int CPL = 32 / LPC, NCH = 128 / LPC, CLD = 132;   // CPL: a lane's coordinates per sub-block
    if (failed(status)) return;
    extern __shared__ __align__(16) unsigned char smem[];
    float *Us = reinterpret_cast<float *>(smem);                 // [10][32][32]
    float *Ps = Us + 10 * 1024;                                  // GPTAQ only
    uint8_t *Cs = reinterpret_cast<uint8_t *>(Ps + (GPTAQ ? 10 * 1024 : 0));  // [NCH][CLD]
    float *rpiv = reinterpret_cast<float *>(Cs + NCH * CLD);    // [SW_MAXB]
    float *sS = rpiv + SW_MAXB;                                  // static groups: [SW_MAXB][NCH]
    float *sR = sS + SW_MAXB * NCH;                              // and 1 / s

    const int grp = blockIdx.y;
    const int cta_ch0 = blockIdx.x * NCH;
    const int n0 = grp * per_group + cta_ch0;
    const int nvalid = min(NCH, per_group - cta_ch0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = lane & (LPC - 1);
    const int ch = warp * (32 / LPC) + lane / LPC;
    const bool valid = ch < nvalid;
    const int64_t n = (int64_t)n0 + ch;
    const int nsb = (bs + 31) / 32;
    const float *Ub = U + (int64_t)grp * K * K + (int64_t)i0 * K + i0;   // U[i0, i0]
    const float *Pb = GPTAQ ? P1 + (int64_t)i0 * K + i0 : nullptr;

    // the ten blocks (P, Q), P <= Q, of U[blk, blk]; zero outside [0, bs)
    for (int idx = tid; idx < 10 * 256; idx += 128) {
        const int blk = idx >> 8;
        const int P = blk < 4 ? 0 : blk < 7 ? 1 : blk < 9 ? 2 : 3;
        const int Q = P + blk - (P * 4 - P * (P - 1) / 2);
        if (Q >= nsb) continue;
        const int r = (idx >> 3) & 31, c4 = (idx & 7) * 4;
        const int row = 32 * P + r, col = 32 * Q + c4;
        float *du = Us + blk * 1024 + r * 32 + c4;
        float *dp = Ps + blk * 1024 + r * 32 + c4;
        if (vec & 1) {        // rows 16-byte aligned and bs % 4 == 0
            const bool in = row < bs && col < bs;
            const int64_t off = in ? (int64_t)row * K + col : 0;
            cp_async16(du, Ub + off, in ? 16 : 0);
            if (GPTAQ) cp_async16(dp, Pb + off, in ? 16 : 0);
        } else {
            for (int e = 0; e < 4; ++e) {
                const bool in = row < bs && col + e < bs;
                du[e] = in ? Ub[(int64_t)row * K + col + e] : 0.f;
                if (GPTAQ) dp[e] = in ? Pb[(int64_t)row * K + col + e] : 0.f;
            }
        }
    }
    if (tid < bs) rpiv[tid] = 1.f / __ldg(Ub + (int64_t)tid * K + tid);

    // a lane's CPL coordinates 32 p + CPL q + i of sub-block p of its channel
    auto fetch = [&](const float *base, int p, float (&d)[CPL]) {
        const int c0 = 32 * p + CPL * q;
        const float *src = base + n * K + i0 + c0;
        if (valid && (vec & 1) && c0 + CPL <= bs) {
#pragma unroll
            for (int v = 0; v < CPL / 4; ++v) {
                const float4 x = *reinterpret_cast<const float4 *>(src + 4 * v);
                d[4 * v] = x.x; d[4 * v + 1] = x.y; d[4 * v + 2] = x.z; d[4 * v + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < CPL; ++i) d[i] = (valid && c0 + i < bs) ? src[i] : 0.f;
        }
    };
    float w[4][CPL];
#pragma unroll
    for (int b = 0; b < 4; ++b) fetch(Wk, b, w[b]);
    // CAE: this lane's starting weights on the sub-block in work (w0c) and the next (w0n)
    float w0c[CPL], w0n[CPL];
    auto fetch_w0 = [&](int p, float (&d)[CPL]) { fetch(W0k, p, d); };
    if (CAE) fetch_w0(0, w0c);
    if (GMODE == 2) {
        for (int j = q; j < bs; j += LPC) {
            const float sj = valid ? sg.gsc[n * sg.ldg + sg.gsel[i0 + j]] : 1.f;
            sS[j * NCH + ch] = sj;
            sR[j * NCH + ch] = 1.f / sj;
        }
    }
    cp_async_wait_all();
    __syncthreads();

    float s = valid ? scale[n] : 1.f;
    float rs = 1.f / s;
    const float zf = (float)(1 << (bits - 1));
    const float cmin = -zf, cmax = (float)((1 << bits) - 1) - zf;
    const int gsrc = lane & ~(LPC - 1);
    float lacc = 0.f;
    uint8_t *crow = Cs + ch * CLD;
    const int64_t ecol = (int64_t)grp * ldG + cta_ch0 + ch;

#pragma unroll 1
    for (int p = 0; p < nsb; ++p) {
        const int bbase = p * 4 - p * (p - 1) / 2;       // block (p, p)
        int64_t eoff = (int64_t)(erow0 + 32 * p) * ldE + ecol;
        if (CAE && p + 1 < nsb) fetch_w0(p + 1, w0n);
        if (GMODE == 1 && (i0 + 32 * p) % sg.G == 0) {
            // entering a group: its scale from the channel's current weights
            float a = 0.f;
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (32 * b < sg.G)
#pragma unroll
                    for (int i = 0; i < CPL; ++i) a = fmaxf(a, fabsf(w[b][i]));
#pragma unroll
            for (int x = 1; x < LPC; x <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, x));
            s = a == 0.f ? 1.f : 2.f * a / (cmax - cmin);
            rs = 1.f / s;
            if (valid && q == 0) sg.gsc[n * sg.ldg + (i0 + 32 * p) / sg.G] = s;
        }
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int j = 32 * p + t;
            const int oq = t / CPL, oi = t % CPL;
            const bool live = j < bs;
            const float sj = GMODE == 2 ? sS[j * NCH + ch] : s;
            const float rsj = GMODE == 2 ? sR[j * NCH + ch] : rs;
            const float wj = w[0][oi];
            const float cf = fminf(fmaxf(rintf(wj * rsj), cmin), cmax);
            // ej: the rounding error of the value quantised (the loss); ep: the error
            // propagated, which CAE measures from the starting weight
            const float ej = live ? fmaf(-sj, cf, wj) * rpiv[j] : 0.f;
            const float w0j = CAE ? w0c[oi] : wj;
            const float ep = CAE ? (live ? fmaf(-sj, cf, w0j) * rpiv[j] : 0.f) : ej;
            const float e = __shfl_sync(0xffffffffu, ep, gsrc | oq);
            float v = 0.f;
            if (GPTAQ) v = __shfl_sync(0xffffffffu, live ? w0j : 0.f, gsrc | oq);
            if (q == oq && live) {
                lacc = fmaf(ej, ej, lacc);
                crow[j] = (uint8_t)(int)(cf + zf);
                if (valid) {
                    const __nv_bfloat16 eh = __float2bfloat16_rn(ep);
                    Eh[eoff] = eh;
                    El[eoff] = __float2bfloat16_rn(ep - __bfloat162float(eh));
                    if (GPTAQ) {
                        const __nv_bfloat16 ph = __float2bfloat16_rn(w0j);
                        Ph[eoff] = ph;
                        Pl[eoff] = __float2bfloat16_rn(w0j - __bfloat162float(ph));
                    }
                }
            }
            eoff += ldE;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (b > 0 && p + b >= nsb) break;
                const float *ur = Us + (bbase + b) * 1024 + t * 32 + CPL * q;
#pragma unroll
                for (int c = 0; c < CPL / 4; ++c) {
                    const float4 u = *reinterpret_cast<const float4 *>(ur + 4 * c);
                    w[b][4 * c] = fmaf(-e, u.x, w[b][4 * c]);
                    w[b][4 * c + 1] = fmaf(-e, u.y, w[b][4 * c + 1]);
                    w[b][4 * c + 2] = fmaf(-e, u.z, w[b][4 * c + 2]);
                    w[b][4 * c + 3] = fmaf(-e, u.w, w[b][4 * c + 3]);
                }
                if (GPTAQ) {
                    const float *pr = Ps + (bbase + b) * 1024 + t * 32 + CPL * q;
#pragma unroll
                    for (int c = 0; c < CPL / 4; ++c) {
                        const float4 u = *reinterpret_cast<const float4 *>(pr + 4 * c);
                        w[b][4 * c] = fmaf(v, u.x, w[b][4 * c]);
                        w[b][4 * c + 1] = fmaf(v, u.y, w[b][4 * c + 1]);
                        w[b][4 * c + 2] = fmaf(v, u.z, w[b][4 * c + 2]);
                        w[b][4 * c + 3] = fmaf(v, u.w, w[b][4 * c + 3]);
                    }
                }
            }
        }
        // the next sub-block becomes w[0]
#pragma unroll
        for (int b = 0; b < 3; ++b)
#pragma unroll
            for (int i = 0; i < CPL; ++i) w[b][i] = w[b + 1][i];
        if (CAE)
#pragma unroll
            for (int i = 0; i < CPL; ++i) w0c[i] = w0n[i];
    }
#pragma unroll
    for (int x = 1; x < LPC; x <<= 1) lacc += __shfl_xor_sync(0xffffffffu, lacc, x);
    if (q == 0 && valid) loss_acc[n] += lacc;
    __syncthreads();
    // codes: 16-byte chunks of each channel's block row
    const bool vecC = vec & 2;   // code rows 16-byte aligned
    for (int idx = tid; idx < NCH * (SW_MAXB / 16); idx += 128) {
        const int r = idx >> 3, c16 = (idx & 7) * 16;
        if (r >= nvalid || c16 >= bs) continue;
        uint8_t *dst = codes + ((int64_t)n0 + r) * K + i0 + c16;
        const uint32_t *srcw = reinterpret_cast<const uint32_t *>(Cs + r * CLD + c16);
        if (vecC && c16 + 16 <= bs) {
            *reinterpret_cast<uint4 *>(dst) = make_uint4(srcw[0], srcw[1], srcw[2], srcw[3]);
        } else {
            for (int e = 0; e < 16 && c16 + e < bs; ++e) dst[e] = Cs[r * CLD + c16 + e];
        }
    }
}

// In-block sweep, thread form (for layers with many output channels): one block
// [i0, i0 + bs) for SW_T channels of one group, one thread per channel with all of the block's coordinates in registers (as pairs).
// Phase p sweeps sub-block p (32 coordinates), always held in w[0]: step t rounds
// coordinate 32 p + t, forms E_j and applies it to the later coordinates of the
// sub-block (packed fp32 FMAs against a broadcast row of U); the phase's 32 errors then
// go to every later sub-block in one compact loop, and the register array shifts by
// one sub-block. U[blk, blk] (and P1)
// is staged once per CTA as its ten 32 x 32 blocks on or above the diagonal.
constexpr int SW_T = 64;

template <bool GPTAQ, int GMODE, bool CAE>
__global__ void __launch_bounds__(SW_T, 1) k_sweep_thread(
    float *__restrict__ Wk, int N, int per_group, int K, int i0, int bs,
    const float *__restrict__ U, const float *__restrict__ P1, const float *__restrict__ scale,
    int bits, uint8_t *__restrict__ codes, __nv_bfloat16 *__restrict__ Eh,
    __nv_bfloat16 *__restrict__ El, __nv_bfloat16 *__restrict__ Ph, __nv_bfloat16 *__restrict__ Pl,
    int ldE, int ldG, int erow0, float *__restrict__ loss_acc, int vec, const int32_t *status,
    const SweepGroups sg, const float *__restrict__ W0k) {
    if (failed(status)) return;
    extern __shared__ __align__(16) unsigned char smem[];
    float *Us = reinterpret_cast<float *>(smem);                 // [10][32][32]
    float *Ps = Us + 10 * 1024;                                  // GPTAQ only
    float *rpiv = Ps + (GPTAQ ? 10 * 1024 : 0);                  // [SW_MAXB]
    float *Es = rpiv + SW_MAXB;                                  // [32][SW_T] this phase's E
    float *Vs = Es + 32 * SW_T;                                  // GPTAQ: pre-rounding weights
    float *sS = Vs + (GPTAQ ? 32 * SW_T : 0);                    // static groups: [SW_MAXB][SW_T]
    float *sR = sS + SW_MAXB * SW_T;                             // and 1 / s
    float *W0s = sS + (GMODE == 2 ? 2 * SW_MAXB * SW_T : 0);     // CAE: [32][SW_T] w^(0)

    const int grp = blockIdx.y;
    const int cta_ch0 = blockIdx.x * SW_T;
    const int n0 = grp * per_group + cta_ch0;
    const int nvalid = min(SW_T, per_group - cta_ch0);
    const int tid = threadIdx.x;
    const bool valid = tid < nvalid;
    const int64_t n = (int64_t)n0 + tid;
    const int nsb = (bs + 31) / 32;
    const float *Ub = U + (int64_t)grp * K * K + (int64_t)i0 * K + i0;   // U[i0, i0]
    const float *Pb = GPTAQ ? P1 + (int64_t)i0 * K + i0 : nullptr;

    // the ten blocks (P, Q), P <= Q, of U[blk, blk]; zero outside [0, bs)
    for (int idx = tid; idx < 10 * 256; idx += SW_T) {
        const int blk = idx >> 8;
        const int P = blk < 4 ? 0 : blk < 7 ? 1 : blk < 9 ? 2 : 3;
        const int Q = P + blk - (P * 4 - P * (P - 1) / 2);
        if (Q >= nsb) continue;
        const int r = (idx >> 3) & 31, c4 = (idx & 7) * 4;
        const int row = 32 * P + r, col = 32 * Q + c4;
        float *du = Us + blk * 1024 + r * 32 + c4;
        float *dp = Ps + blk * 1024 + r * 32 + c4;
        if (vec & 1) {        // rows 16-byte aligned and bs % 4 == 0
            const bool in = row < bs && col < bs;
            const int64_t off = in ? (int64_t)row * K + col : 0;
            cp_async16(du, Ub + off, in ? 16 : 0);
            if (GPTAQ) cp_async16(dp, Pb + off, in ? 16 : 0);
        } else {
            for (int e = 0; e < 4; ++e) {
                const bool in = row < bs && col + e < bs;
                du[e] = in ? Ub[(int64_t)row * K + col + e] : 0.f;
                if (GPTAQ) dp[e] = in ? Pb[(int64_t)row * K + col + e] : 0.f;
            }
        }
    }
    for (int j = tid; j < bs; j += SW_T) rpiv[j] = 1.f / __ldg(Ub + (int64_t)j * K + j);
    // CAE: the channel's starting weights on sub-block p, into its own column of W0s
    // (each thread reads only its column, so no barrier guards the refill)
    auto fetch_w0 = [&](int p) {
        const float *src = W0k + n * K + i0 + 32 * p;
#pragma unroll 8
        for (int t = 0; t < 32; ++t) {
            const bool in = valid && 32 * p + t < bs;
            cp_async4(W0s + t * SW_T + tid, in ? src + t : W0k, in ? 4 : 0);
        }
    };
    if (CAE) fetch_w0(0);

    // the channel's block coordinates: sub-block b, pair i = coordinates (2 i, 2 i + 1)
    float2 w[4][16];
    {
        const float *src = Wk + n * K + i0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (valid && (vec & 1) && 32 * b + 32 <= bs) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 x = *reinterpret_cast<const float4 *>(src + 32 * b + 4 * i);
                    w[b][2 * i] = make_float2(x.x, x.y);
                    w[b][2 * i + 1] = make_float2(x.z, x.w);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = 32 * b + 2 * i;
                    w[b][i] = make_float2((valid && c < bs) ? src[c] : 0.f,
                                          (valid && c + 1 < bs) ? src[c + 1] : 0.f);
                }
            }
        }
    }
    if (GMODE == 2) {
        for (int j = 0; j < bs; ++j) {
            const float sj = valid ? sg.gsc[n * sg.ldg + sg.gsel[i0 + j]] : 1.f;
            sS[j * SW_T + tid] = sj;
            sR[j * SW_T + tid] = 1.f / sj;
        }
    }
    cp_async_wait_all();
    __syncthreads();

    float s = valid ? scale[n] : 1.f;
    float rs = 1.f / s;
    const float zf = (float)(1 << (bits - 1));
    const float cmin = -zf, cmax = (float)((1 << bits) - 1) - zf;
    float lacc = 0.f;
    const int64_t ecol = (int64_t)grp * ldG + cta_ch0 + tid;
    uint8_t *crow = codes + n * K + i0;
    const bool vcodes = valid && (vec & 2);

#pragma unroll 1
    for (int p = 0; p < nsb; ++p) {
        const int bbase = p * 4 - p * (p - 1) / 2;       // block (p, p)
        const int nblk = nsb - p;
        const float *Up = Us + bbase * 1024;
        const float *Pp = Ps + bbase * 1024;
        int64_t eoff = (int64_t)(erow0 + 32 * p) * ldE + ecol;
        uint32_t cw[4] = {0u, 0u, 0u, 0u};
        if (CAE && p > 0) cp_async_wait_all();   // this phase's W0s, fetched during the last
        if (GMODE == 1 && (i0 + 32 * p) % sg.G == 0) {
            // entering a group: its scale from the channel's current weights
            float a = 0.f;
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (32 * b < sg.G)
#pragma unroll
                    for (int i = 0; i < 16; ++i) a = fmaxf(a, fmaxf(fabsf(w[b][i].x), fabsf(w[b][i].y)));
            s = a == 0.f ? 1.f : 2.f * a / (cmax - cmin);
            rs = 1.f / s;
            if (valid) sg.gsc[n * sg.ldg + (i0 + 32 * p) / sg.G] = s;
        }
        // the 32 steps inside sub-block p; each step's error is kept for the later
        // sub-blocks, which take all 32 at once after the phase
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int j = 32 * p + t;
            const bool live = j < bs;
            const float sj = GMODE == 2 ? sS[j * SW_T + tid] : s;
            const float rsj = GMODE == 2 ? sR[j * SW_T + tid] : rs;
            const float wj = (t & 1) ? w[0][t >> 1].y : w[0][t >> 1].x;
            const float cf = fminf(fmaxf(rintf(wj * rsj), cmin), cmax);
            // ej: the rounding error of the value quantised (the loss); ep: the error
            // propagated, which CAE measures from the starting weight
            const float ej = live ? fmaf(-sj, cf, wj) * rpiv[j] : 0.f;
            const float w0j = CAE ? W0s[t * SW_T + tid] : wj;
            const float ep = CAE ? (live ? fmaf(-sj, cf, w0j) * rpiv[j] : 0.f) : ej;
            const float vj = (GPTAQ && live) ? w0j : 0.f;
            Es[t * SW_T + tid] = ep;
            if (GPTAQ) Vs[t * SW_T + tid] = vj;
            cw[(t >> 2) & 3] |= (uint32_t)(int)(cf + zf) << (8 * (t & 3));
            if (live) {
                lacc = fmaf(ej, ej, lacc);
                if (valid) {
                    const __nv_bfloat16 eh = __float2bfloat16_rn(ep);
                    Eh[eoff] = eh;
                    El[eoff] = __float2bfloat16_rn(ep - __bfloat162float(eh));
                    if (GPTAQ) {
                        const __nv_bfloat16 ph = __float2bfloat16_rn(vj);
                        Ph[eoff] = ph;
                        Pl[eoff] = __float2bfloat16_rn(vj - __bfloat162float(ph));
                    }
                }
            }
            eoff += ldE;
            const float2 ne = make_float2(-ep, -ep);
            const float2 vv = make_float2(vj, vj);
            // the rest of this sub-block: pairs from the one holding t + 1
#pragma unroll
            for (int i = (t + 1) / 2; i < 16; ++i) {
                const float2 u = *reinterpret_cast<const float2 *>(Up + t * 32 + 2 * i);
                w[0][i] = ffma2(ne, u, w[0][i]);
                if (GPTAQ) {
                    const float2 pp = *reinterpret_cast<const float2 *>(Pp + t * 32 + 2 * i);
                    w[0][i] = ffma2(vv, pp, w[0][i]);
                }
            }
            if ((t & 15) == 15) {
                // 16 codes of this channel
                const int c16 = 32 * p + (t & 16);
                if (valid && c16 < bs) {
                    if (vcodes && c16 + 16 <= bs) {
                        *reinterpret_cast<uint4 *>(crow + c16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                    } else {
                        for (int e = 0; e < 16 && c16 + e < bs; ++e)
                            crow[c16 + e] = (uint8_t)(cw[e >> 2] >> (8 * (e & 3)));
                    }
                }
                cw[0] = cw[1] = cw[2] = cw[3] = 0u;
            }
        }
        // the phase is done with W0s: fetch the next sub-block's while the later
        // sub-blocks are updated
        if (CAE && p + 1 < nsb) fetch_w0(p + 1);
        // later sub-blocks: w_b -= sum_t E_t U[32 p + t, sub-block b] (+ GPTAQ term)
        if (nblk > 1) {
#pragma unroll 2
            for (int t = 0; t < 32; ++t) {
                const float et = Es[t * SW_T + tid];
                const float2 ne = make_float2(-et, -et);
                float2 vv = make_float2(0.f, 0.f);
                if (GPTAQ) {
                    const float vt = Vs[t * SW_T + tid];
                    vv = make_float2(vt, vt);
                }
#pragma unroll
                for (int b = 1; b < 4; ++b) {
                    if (b >= nblk) break;
                    const float *ur = Up + b * 1024 + t * 32;
                    const float *pr = Pp + b * 1024 + t * 32;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 u = *reinterpret_cast<const float4 *>(ur + 4 * i);
                        w[b][2 * i] = ffma2(ne, make_float2(u.x, u.y), w[b][2 * i]);
                        w[b][2 * i + 1] = ffma2(ne, make_float2(u.z, u.w), w[b][2 * i + 1]);
                        if (GPTAQ) {
                            const float4 q = *reinterpret_cast<const float4 *>(pr + 4 * i);
                            w[b][2 * i] = ffma2(vv, make_float2(q.x, q.y), w[b][2 * i]);
                            w[b][2 * i + 1] = ffma2(vv, make_float2(q.z, q.w), w[b][2 * i + 1]);
                        }
                    }
                }
            }
        }
        // the next sub-block becomes w[0]
#pragma unroll
        for (int b = 0; b < 3; ++b)
#pragma unroll
            for (int i = 0; i < 16; ++i) w[b][i] = w[b + 1][i];
    }
    if (valid) loss_acc[n] += lacc;
}

// Static groups: s[n][g] from W as given on the original columns [gG, (g+1)G), one
// warp per (channel, group).
template <typename T>
__global__ void k_group_scales_static(const T *__restrict__ W, int N, int K, int G, int ng,
                                      int bits, float *__restrict__ gsc) {
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= (int64_t)N * ng) return;
    const int n = (int)(wid / ng), g = (int)(wid % ng);
    const T *wr = W + (int64_t)n * K;
    float a = 0.f;
    for (int k = g * G + lane; k < min(K, (g + 1) * G); k += 32) a = fmaxf(a, fabsf(to_f32(wr[k])));
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) gsc[(int64_t)n * ng + g] = a == 0.f ? 1.f : 2.f * a / (float)((1 << bits) - 1);
}

// gsel[j]: the group whose scale serves processing position j (re-estimated groups:
// j / G; static: the original group perm[j] / G); g_idx[original k] = that group.
__global__ void k_group_select(int K, int G, int static_groups, const int32_t *__restrict__ perm,
                               int32_t *__restrict__ gsel, int32_t *__restrict__ g_idx) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    const int k = perm ? perm[j] : j;
    const int g = static_groups ? k / G : j / G;
    gsel[j] = g;
    if (g_idx) g_idx[k] = g;
}

// One CTA per channel: codes from processing order to the original order, and the
// write-back s (c - z) with the group scale of each coordinate.
template <typename T>
__global__ void __launch_bounds__(256) k_finalize_grouped(
    T *__restrict__ W, const uint8_t *__restrict__ cp, uint8_t *__restrict__ codes,
    const int32_t *__restrict__ perm, const int32_t *__restrict__ gsel,
    const float *__restrict__ gsc, int ldg, const float *__restrict__ scale, int K, int bits,
    int write_back, const float *__restrict__ loss_acc, float *__restrict__ loss) {
    const int n = blockIdx.x;
    const float zf = (float)(1 << (bits - 1));
    if (loss && threadIdx.x == 0) loss[n] = 0.5f * loss_acc[n];
    const uint8_t *crow = cp + (int64_t)n * K;
    for (int j = threadIdx.x; j < K; j += 256) {
        const int k = perm ? perm[j] : j;
        const uint8_t c = crow[j];
        if (perm) codes[(int64_t)n * K + k] = c;
        if (write_back) {
            const float s = gsc ? gsc[(int64_t)n * ldg + gsel[j]] : scale[n];
            W[(int64_t)n * K + k] = from_f32<T>(s * ((float)c - zf));
        }
    }
}

// One CTA per channel: write-back s (c - z) in the weights' dtype and the loss.
template <typename T>
__global__ void __launch_bounds__(256) k_finalize(T *__restrict__ W, const uint8_t *__restrict__ codes,
                                                  const float *__restrict__ scale, int K, int bits,
                                                  int write_back, const float *__restrict__ loss_acc,
                                                  float *__restrict__ loss, int vec) {
    const int n = blockIdx.x;
    const float zf = (float)(1 << (bits - 1));
    const float s = scale[n];
    if (loss && threadIdx.x == 0) loss[n] = 0.5f * loss_acc[n];
    if (!write_back) return;
    T *wr = W + (int64_t)n * K;
    const uint8_t *cr = codes + (int64_t)n * K;
    if (vec) {   // W and code rows 16-byte aligned, K % 16 == 0
        for (int k = threadIdx.x * 16; k < K; k += 256 * 16) {
            const uint4 c = *reinterpret_cast<const uint4 *>(cr + k);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = s * ((float)((cw[i >> 2] >> (8 * (i & 3))) & 0xffu) - zf);
            if constexpr (sizeof(T) == 2) {
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
                    o[i] = *reinterpret_cast<const uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(wr + k) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(wr + k + 8) = make_uint4(o[4], o[5], o[6], o[7]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(wr) + k + 4 * i) =
                        make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            }
        }
    } else {
        for (int k = threadIdx.x; k < K; k += 256) wr[k] = from_f32<T>(s * ((float)cr[k] - zf));
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
    // Eh El Ph Pl: [SUPER][ldE] for the SIMT sweeps, [ldE][two super-blocks] for the
    // tensor-core sweep
    for (int i = 0; i < 4; ++i) c.take<__nv_bfloat16>((size_t)SWEEP_TC_ESTRIDE * lay.ldE);
    c.take<float>((size_t)N);                               // scale
    c.take<float>((size_t)N);                               // loss_acc
    c.take<float>((size_t)g * K);                           // 1 / U_jj (tensor-core sweep)
    return round_up(c.off, 256);
}

static size_t sweep_thread_smem(bool gptaq, int gmode, bool cae) {
    return sizeof(float) * ((10 * 1024 + 32 * SW_T) * (gptaq ? 2 : 1) + SW_MAXB +
                            (gmode == 2 ? 2 * SW_MAXB * SW_T : 0) + (cae ? 32 * SW_T : 0));
}
static size_t sweep_lanes_smem(bool gptaq, int gmode, int lpc) {
    const int nch = 128 / lpc;
    return sizeof(float) * (10 * 1024 * (gptaq ? 2 : 1) + SW_MAXB + (gmode == 2 ? 2 * SW_MAXB * nch : 0)) +
           (size_t)nch * 132;
}

typedef void (*SweepKernel)(float *, int, int, int, int, int, const float *, const float *,
                            const float *, int, uint8_t *, __nv_bfloat16 *, __nv_bfloat16 *,
                            __nv_bfloat16 *, __nv_bfloat16 *, int, int, int, float *, int,
                            const int32_t *, const SweepGroups, const float *);

// form 0: one thread per channel; 1: four lanes per channel; 2: two lanes per channel
#define GPTQ_SWEEP_MODES(K, A, C) {K<A, 0, C>, K<A, 1, C>, K<A, 2, C>}
#define GPTQ_LANES4(A, C, G) k_sweep_lanes<A, G, C, 4>
#define GPTQ_LANES2(A, C, G) k_sweep_lanes<A, G, C, 2>
#define GPTQ_LANE_MODES(L, A, C) {L(A, C, 0), L(A, C, 1), L(A, C, 2)}
static SweepKernel sweep_kernel(int form, bool gptaq, int gmode, bool cae) {
    static const SweepKernel tab[3][2][2][3] = {
        {{GPTQ_SWEEP_MODES(k_sweep_thread, false, false), GPTQ_SWEEP_MODES(k_sweep_thread, false, true)},
         {GPTQ_SWEEP_MODES(k_sweep_thread, true, false), GPTQ_SWEEP_MODES(k_sweep_thread, true, true)}},
        {{GPTQ_LANE_MODES(GPTQ_LANES4, false, false), GPTQ_LANE_MODES(GPTQ_LANES4, false, true)},
         {GPTQ_LANE_MODES(GPTQ_LANES4, true, false), GPTQ_LANE_MODES(GPTQ_LANES4, true, true)}},
        {{GPTQ_LANE_MODES(GPTQ_LANES2, false, false), GPTQ_LANE_MODES(GPTQ_LANES2, false, true)},
         {GPTQ_LANE_MODES(GPTQ_LANES2, true, false), GPTQ_LANE_MODES(GPTQ_LANES2, true, true)}}};
    return tab[form][gptaq][cae][gmode];
}
#undef GPTQ_SWEEP_MODES
#undef GPTQ_LANES4
#undef GPTQ_LANES2
#undef GPTQ_LANE_MODES

// Input-dimension groups and order of one quantisation (G == 0: per-channel scales,
// natural order).
struct QGroupOpts {
    int G = 0;
    int static_groups = 0;
    const int32_t *perm = nullptr;
    float *scales = nullptr;     // [N][ceil(K / G)] out, or NULL
    int32_t *g_idx = nullptr;    // [K] out, or NULL
};

size_t quantize_grouped_workspace(int K, int N, int blocksize) {
    Carver c(nullptr);
    c.off = quantize_workspace(K, N, 1, blocksize);
    c.take<float>((size_t)N * ((K + 31) / 32));   // group scales (smallest group: 32)
    c.take<uint8_t>((size_t)N * K);               // codes in processing order
    c.take<int32_t>((size_t)K);                   // group of each processing position
    return round_up(c.off, 256);
}

// The compensation-aware term keeps the starting weights, after the rest.
size_t quantize_cae_extra(int K, int N) { return round_up((size_t)N * K * sizeof(float), 256); }

static gptq_status quantize_impl(void *W, int wdtype, int N, int K, const float *U, int groups,
                                 int bits, int blocksize, const float *P1, const uint8_t *dead,
                                 const float *scales_in, float *scales_out, uint8_t *codes,
                                 float *loss, int write_back, void *ws, int32_t *status,
                                 cudaStream_t st, const QGroupOpts &go, int cae) {
    if (!update_tc_available()) return GPTQ_ERR_CUDA;
    const QLayout lay(K, N, groups);
    Carver cv(ws);
    float *Wk = cv.take<float>((size_t)N * K);
    __nv_bfloat16 *Uh = cv.take<__nv_bfloat16>((size_t)groups * K * lay.ldU);
    __nv_bfloat16 *Ul = cv.take<__nv_bfloat16>((size_t)groups * K * lay.ldU);
    __nv_bfloat16 *Qh = cv.take<__nv_bfloat16>((size_t)K * lay.ldU);
    __nv_bfloat16 *Ql = cv.take<__nv_bfloat16>((size_t)K * lay.ldU);
    __nv_bfloat16 *Eh = cv.take<__nv_bfloat16>((size_t)SWEEP_TC_ESTRIDE * lay.ldE);
    __nv_bfloat16 *El = cv.take<__nv_bfloat16>((size_t)SWEEP_TC_ESTRIDE * lay.ldE);
    __nv_bfloat16 *Ph = cv.take<__nv_bfloat16>((size_t)SWEEP_TC_ESTRIDE * lay.ldE);
    __nv_bfloat16 *Pl = cv.take<__nv_bfloat16>((size_t)SWEEP_TC_ESTRIDE * lay.ldE);
    float *scale = cv.take<float>((size_t)N);
    float *loss_acc = cv.take<float>((size_t)N);
    float *rp = cv.take<float>((size_t)groups * K);
    const bool grouped = go.G > 0 || go.perm != nullptr;
    const int G = go.G > 0 ? go.G : K;
    const int ng = (K + G - 1) / G;
    float *gsc = nullptr;
    uint8_t *cp = codes;
    int32_t *gsel = nullptr;
    if (grouped) {
        Carver gx(ws);
        gx.off = quantize_workspace(K, N, 1, blocksize);
        float *gws = gx.take<float>((size_t)N * ((K + 31) / 32));
        uint8_t *cws = gx.take<uint8_t>((size_t)N * K);
        gsel = gx.take<int32_t>((size_t)K);
        if (go.G > 0) gsc = go.scales ? go.scales : gws;
        if (go.perm) cp = cws;
    }
    float *W0k = nullptr;
    if (cae) {
        Carver cx(ws);
        cx.off = grouped ? quantize_grouped_workspace(K, N, blocksize)
                         : quantize_workspace(K, N, groups, blocksize);
        W0k = cx.take<float>((size_t)N * K);
    }
    const int gmode = go.G == 0 ? 0 : (go.static_groups ? 2 : 1);
    const int per_group = N / groups;
    const int64_t KK = (int64_t)K * K;
    const bool gptaq = P1 != nullptr;
    const int vin = (K % 8 == 0 && aligned(W, 16) && aligned(Wk, 16) && (!W0k || aligned(W0k, 16)))
                        ? 1 : 0;
    const int vfin = (K % 16 == 0 && aligned(W, 16) && aligned(codes, 16)) ? 1 : 0;
    if (wdtype == GPTQ_F32)
        k_scale_init<float><<<N, 256, 0, st>>>(static_cast<const float *>(W), Wk, K, per_group, bits,
                                              dead, scales_in, scale, scales_out, loss_acc, vin,
                                              status, go.perm, W0k);
    else
        k_scale_init<__nv_bfloat16><<<N, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(W), Wk, K,
                                                      per_group, bits, dead, scales_in, scale,
                                                      scales_out, loss_acc, vin, status, go.perm,
                                                      W0k);
    gptq_status s = launch_status();
    if (s != GPTQ_OK) return s;
    if (grouped) {
        k_group_select<<<(K + 255) / 256, 256, 0, st>>>(K, G, go.static_groups, go.perm, gsel,
                                                        go.g_idx);
        if ((s = launch_status()) != GPTQ_OK) return s;
        if (gmode == 2) {
            const int64_t warps = (int64_t)N * ng;
            const int blocks = (int)((warps * 32 + 255) / 256);
            if (wdtype == GPTQ_F32)
                k_group_scales_static<float><<<blocks, 256, 0, st>>>(
                    static_cast<const float *>(W), N, K, G, ng, bits, gsc);
            else
                k_group_scales_static<__nv_bfloat16><<<blocks, 256, 0, st>>>(
                    static_cast<const __nv_bfloat16 *>(W), N, K, G, ng, bits, gsc);
            if ((s = launch_status()) != GPTQ_OK) return s;
        }
    }
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
    base.ngroups = gptaq ? 2 : 1;
    base.neg[0] = 1;
    base.neg[1] = 0;

    // Per-channel scales take the tensor-core sweep (sweep_tc.cu: one launch per
    // super-block, the near updates accumulated in TMEM) whenever its TMA maps can be
    // built (K % 4 == 0). Otherwise, and for input groups: one thread per channel when
    // that still gives every SM two warps, two lanes per channel there instead for CAE
    // (its starting weights then stay in registers: 2.25 against 2.51 ms for a
    // 14336 x 4096 layer on B200, while the plain and GPTAQ sweeps time the same or
    // slower with two lanes); four lanes per channel for fewer channels.
    // GPTQ_SWEEP_FORM = 0, 1, 2 or 3 picks the form (comparisons and tests; 3 = tensor
    // core, used only where eligible).
    int form = (int64_t)N >= 2LL * 148 * 32 ? (cae ? 2 : 0) : 1;
    const bool tc_ok = gmode == 0 && sweep_tc_eligible(K, U, P1);
    if (tc_ok) form = 3;
    if (const char *f = getenv("GPTQ_SWEEP_FORM")) {
        const int fv = atoi(f);
        if (fv >= 0 && fv <= 2) form = fv;
        else if (fv == 3 && tc_ok) form = 3;
    }
    if (form == 3) {
        static thread_local SweepTcMaps stc_maps;
        SweepTcMaps *stc = &stc_maps;
        if ((s = sweep_tc_setup(stc, Wk, W0k, U, P1, Uh, Ul, Qh, Ql, lay.ldU, rp, N, K, groups,
                                st)) != GPTQ_OK)
            return s;
        const int S = sweep_tc_super(gptaq);
        // the far update reads the sweep's -E (and V) pairs as channel rows with two
        // super-blocks' coordinates contiguous ([ldE][2 x 512], 64 x 128 boxes) and adds
        static thread_local UpdateMaps kmaps[8];
        for (int gi = 0; gi < groups; ++gi) {
            kmaps[gi] = maps[1][gi];
            __nv_bfloat16 *a_src[4] = {Eh, El, Ph, Pl};
            for (int i = 0; i < 4; ++i)
                if ((s = make_bf16_map(&kmaps[gi].a[i], a_src[i], SWEEP_TC_ESTRIDE, lay.ldE,
                                       SWEEP_TC_ESTRIDE, 128)) != GPTQ_OK)
                    return s;
        }
        UpdateParams kbase = base;
        kbase.a_kmajor = 1;
        kbase.neg[0] = 0;
        // Far updates by pairs of super-blocks (update_plan.h): after an even super-block
        // only the next super-block's columns take its errors (the next sweep needs them);
        // after the odd one, everything after the pair takes both super-blocks' errors as
        // one product of inner length 2S, so the rest of W is read and written once per pair.
        const std::vector<FarUpdate> plan = far_update_plan(K, S);
        size_t next = 0;
        for (int idx = 0, sb0 = 0; sb0 < K; sb0 += S, ++idx) {
            const int sb1 = min(K, sb0 + S);
            if ((s = sweep_tc_launch(*stc, scale, bits, cp, Eh, El, Ph, Pl, lay.ldE, lay.ldG,
                                     loss_acc, status, N, per_group, K, groups, sb0, sb1 - sb0,
                                     sweep_error_column(idx, S), gptaq, cae != 0, st)) != GPTQ_OK)
                return s;
            for (; next < plan.size() && plan[next].after == idx; ++next) {
                const FarUpdate &u = plan[next];
                for (int gi = 0; gi < groups; ++gi) {
                    UpdateParams p = kbase;
                    p.C = Wk + (int64_t)gi * per_group * K + u.col0;
                    p.c_extent = (int64_t)N * K - (p.C - Wk);
                    p.Ncols = u.col1 - u.col0;
                    p.L = u.k1 - u.k0;
                    p.a_x0 = gi * lay.ldG;
                    p.a_y0 = 0;                   // E column of coordinate k0
                    p.b_x0 = u.col0;
                    p.b_y0 = u.k0;
                    if ((s = launch_update_tc(kmaps[gi], p, 64, st)) != GPTQ_OK) return s;
                }
            }
        }
    } else {
        const int cta = form == 0 ? SW_T : 128;
        const int per_cta = form == 0 ? SW_T : form == 1 ? 32 : 64;
        const dim3 grid((per_group + per_cta - 1) / per_cta, groups);
        SweepKernel kern = sweep_kernel(form, gptaq, gmode, cae != 0);
        const size_t smem = form == 0 ? sweep_thread_smem(gptaq, gmode, cae != 0)
                                      : sweep_lanes_smem(gptaq, gmode, form == 1 ? 4 : 2);
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return launch_status();
        const int vec = ((K % 4 == 0 && aligned(U, 16) && (!gptaq || aligned(P1, 16))) ? 1 : 0) |
                        ((K % 16 == 0 && aligned(cp, 16)) ? 2 : 0);
        SweepGroups sg{G, gsc, ng, gsel};
        for (int sb0 = 0; sb0 < K; sb0 += SUPER) {
            const int sb1 = min(K, sb0 + SUPER);
            for (int i0 = sb0; i0 < sb1; i0 += blocksize) {
                const int i1 = min(i0 + blocksize, sb1);
                const int bs = i1 - i0;
                const int rec = prof_begin(GPTQ_PROF_SWEEP, st);
                kern<<<grid, cta, smem, st>>>(Wk, N, per_group, K, i0, bs, U, P1, scale, bits, cp, Eh,
                                              El, Ph, Pl, lay.ldE, lay.ldG, i0 - sb0, loss_acc, vec,
                                              status, sg, W0k);
                s = launch_status();
                prof_end(rec, st);
                if (s != GPTQ_OK) return s;
                if (i1 >= sb1) continue;
                for (int gi = 0; gi < groups; ++gi) {      // near: the rest of the super-block
                    UpdateParams p = base;
                    p.C = Wk + (int64_t)gi * per_group * K + i1;
                    p.c_extent = (int64_t)N * K - (p.C - Wk);
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
                p.c_extent = (int64_t)N * K - (p.C - Wk);
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
    }
    if (grouped) {
        if (wdtype == GPTQ_F32)
            k_finalize_grouped<float><<<N, 256, 0, st>>>(static_cast<float *>(W), cp, codes, go.perm,
                                                         gsel, gsc, ng, scale, K, bits, write_back,
                                                         loss_acc, loss);
        else
            k_finalize_grouped<__nv_bfloat16><<<N, 256, 0, st>>>(
                static_cast<__nv_bfloat16 *>(W), cp, codes, go.perm, gsel, gsc, ng, scale, K, bits,
                write_back, loss_acc, loss);
        return launch_status();
    }
    if (wdtype == GPTQ_F32)
        k_finalize<float><<<N, 256, 0, st>>>(static_cast<float *>(W), codes, scale, K, bits,
                                             write_back, loss_acc, loss, vfin);
    else
        k_finalize<__nv_bfloat16><<<N, 256, 0, st>>>(static_cast<__nv_bfloat16 *>(W), codes, scale, K,
                                                     bits, write_back, loss_acc, loss, vfin);
    return launch_status();
}

gptq_status quantize_layer(void *W, int wdtype, int N, int K, const float *U, int groups, int bits,
                           int blocksize, const float *P1, int cae, const uint8_t *dead,
                           const float *scales_in, float *scales_out, uint8_t *codes, float *loss,
                           int write_back, void *ws, int32_t *status, cudaStream_t st) {
    return quantize_impl(W, wdtype, N, K, U, groups, bits, blocksize, P1, dead, scales_in,
                         scales_out, codes, loss, write_back, ws, status, st, QGroupOpts{}, cae);
}

gptq_status quantize_layer_grouped(void *W, int wdtype, int N, int K, const float *U, int bits,
                                   int blocksize, int groupsize, int static_groups,
                                   const int32_t *perm, const float *P1, int cae,
                                   const uint8_t *dead,
                                   float *scales_out, int32_t *g_idx, uint8_t *codes, float *loss,
                                   int write_back, void *ws, int32_t *status, cudaStream_t st) {
    QGroupOpts go;
    go.G = groupsize;
    go.static_groups = static_groups;
    go.perm = perm;
    go.scales = scales_out;
    go.g_idx = g_idx;
    // without groups the per-channel scales go straight to scales_out
    return quantize_impl(W, wdtype, N, K, U, 1, bits, blocksize, P1, dead, nullptr,
                         groupsize ? nullptr : scales_out, codes, loss, write_back, ws, status, st,
                         go, cae);
}

}  // namespace gptq
