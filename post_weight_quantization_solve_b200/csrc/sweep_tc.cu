// In-block sweep of one super-block with the near updates on the tensor cores.
//
// [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": all channels take the coordinates in
// one order; coordinate j is rounded, q = s (c - z), E_j = (w_j - q) / U_jj, and the
// later coordinates get W_k -= U_jk E_j. Lazy batching changes only the order of this
// work. Here one launch sweeps a super-block of S coordinates (S = 512, or 256 with
// the GPTAQ row term) for 128 output channels per CTA:
//   - a phase sweeps 32 coordinates: each thread owns one channel, rounds one
//     coordinate per step and applies E_j to the phase's later coordinates in fp32
//     (the dependent chain, as in the SIMT sweeps);
//   - the phase's errors then reach every later coordinate of the super-block as one
//     tensor-core product D[ch][k] += -E[ch][j] U[j][k] (+ V[ch][j] P1[j][k] for the
//     GPTAQ / compensation-aware rows), accumulated in TMEM: lane = channel, column =
//     coordinate inside the super-block. When a phase starts, its thread reads its own
//     lane's 32 columns (tcgen05.ld) and adds them to the weights staged from global
//     memory, which hold every earlier super-block's far update.
// The coordinates after the super-block are updated afterwards by the far update
// (update_tc.cu) from the -E (and V) pairs this kernel writes to global memory, one
// row per channel with the super-block's coordinates contiguous ([ldE][512]).
//
// Products are bf16 x3 splits (hi*hi + hi*lo + lo*hi) of fp32 operands, as in the far
// update. Operands: A = [-E | V] per channel row, K-major in a 128-byte swizzled tile
// written by the chain threads; B = rows of U (and P1) as bf16 pairs, MN-major 64-column
// chunks loaded by TMA. D starts at zero at phase 0 and is summed over the phases.
//
// Roles: warps 0-3 run the chain (thread = channel = TMEM lane); warp 4 issues the TMA
// loads (weights, U's diagonal block and 1 / U_jj one phase ahead into double-buffered
// slots; the B tile once the previous phase's products are done); warp 5 issues the
// MMAs, so that no chain warp waits for their issue. Every wait is bounded; a timeout
// sets the status word.
#include <cuda.h>

#include <algorithm>

#include "bounds.cuh"
#include "common.cuh"
#include "sweep_tc.cuh"
#include "tc_ptx.cuh"
#include "update_tc.cuh"

namespace gptq {

namespace {
constexpr int STC_CH = 128;                 // channels per CTA = TMEM lanes = MMA M
constexpr int STC_THREADS = 192;            // 4 chain warps, the producer warp, the MMA warp
constexpr uint32_t STC_TMEM_COLS = 512;
constexpr int A_TILE = 128 * 128;           // 128 rows x 128 bytes (64 bf16 of k)
constexpr int B_SPLIT = 32 * 1024;          // one split (hi or lo) of the B tile
constexpr int W_SLOT = 128 * 128;           // 128 rows x 32 fp32
constexpr int D_SLOT = 32 * 128;            // 32 x 32 fp32 diagonal block
constexpr int R_SLOT = 1024;                // 32 fp32 (1 / U_jj), 1 KB aligned slot
// row pitch of the E / V pairs in global memory: two super-blocks side by side, so that
// the far update can take the errors of two consecutive super-blocks as one product
constexpr int ESTRIDE = 1024;
constexpr int OFF_A = 0;                                  // [2 slots][hi, lo]
constexpr int OFF_B = OFF_A + 4 * A_TILE;                 // [hi, lo]
constexpr int OFF_W = OFF_B + 2 * B_SPLIT;                // [2 slots]
constexpr int OFF_W0 = OFF_W + 2 * W_SLOT;                // [2 slots] (CAE)
constexpr int OFF_UD = OFF_W0 + 2 * W_SLOT;               // [2 slots]
constexpr int OFF_PD = OFF_UD + 2 * D_SLOT;               // [2 slots] (GPTAQ)
constexpr int OFF_RP = OFF_PD + 2 * D_SLOT;               // [2 slots]
constexpr int OFF_BAR = OFF_RP + 2 * R_SLOT;
constexpr int STC_SMEM = OFF_BAR + 256 + 1024;            // + barriers, alignment slack
static_assert(STC_SMEM <= 227 * 1024, "one CTA's shared memory");
}  // namespace

struct SweepTcParams {
    const float *scale;
    uint8_t *codes;
    __nv_bfloat16 *Eh, *El, *Ph, *Pl;
    float *loss_acc;
    int32_t *status;
    int N, per_group, K, bits;
    int ldE, ldG;
    int sb0, S;             // super-block origin and length
    int eoff;               // column of this super-block's errors in the E / V rows
    int vcodes;             // code rows 16-byte aligned (K % 16 == 0)
};

template <bool GPTAQ, bool CAE>
__global__ void __launch_bounds__(STC_THREADS, 1)
    k_sweep_tc(const __grid_constant__ SweepTcMaps maps, const SweepTcParams p) {
    constexpr int KP = GPTAQ ? 64 : 32;     // inner length of one phase's product
    constexpr int CH_BYTES = KP * 128;      // one 64-column chunk of B
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *cfull = reinterpret_cast<uint64_t *>(smem + OFF_BAR);   // [2] chain inputs landed
    uint64_t *cfree = cfull + 2;                                      // [2] slot read by the chain
    uint64_t *bfull = cfree + 2;                                      // B tile landed
    uint64_t *abar = bfull + 1;          // every chain thread wrote its A row of the phase
    uint64_t *bar_next = abar + 1;       // products reaching the next phase's columns done
    uint64_t *bar_rest = bar_next + 1;   // all products of a phase done
    uint64_t *drain = bar_rest + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *skip = reinterpret_cast<volatile int *>(tmem_slot + 2);
    // one reading of the status word for the whole CTA, so that every thread agrees
    if (threadIdx.x == 0) *skip = failed(p.status) ? 1 : 0;
    __syncthreads();
    if (*skip) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = blockIdx.y;
    const int cta_ch0 = blockIdx.x * STC_CH;
    const int n0 = grp * p.per_group + cta_ch0;
    const int K = p.K, sb0 = p.sb0;
    const int nsub = (p.S + 31) / 32;
    const int nend = 32 * nsub;
    const int nmma = nsub - 1;           // phases whose errors reach later columns

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&cfull[s], 1);
            tc::mbar_init(&cfree[s], STC_CH);
        }
        tc::mbar_init(bfull, 1);
        tc::mbar_init(abar, STC_CH);
        tc::mbar_init(bar_next, 1);
        tc::mbar_init(bar_rest, 1);
        tc::mbar_init(drain, 1);
        *abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, STC_TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // set-up done: wait for the previous kernel on the stream (when launched as its
    // programmatic dependent; at once otherwise) before any global access, and let the
    // next kernel start its own set-up
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 4) {
        if (lane == 0) {
            // chain inputs of phase q into slot q & 1: weights (and starting weights),
            // U's diagonal block (and P1's), 1 / U_jj
            auto issue_chain = [&](int q) {
                const int s = q & 1;
                uint32_t bytes = W_SLOT + D_SLOT + 128;
                if (CAE) bytes += W_SLOT;
                if (GPTAQ) bytes += D_SLOT;
                const int x = sb0 + 32 * q;
                // fp32 boxes: the coordinate on a 16-byte boundary, inside W and U
                if (!GQ_IN_BOUNDS(p.status, x >= 0 && x < K && (x & 3) == 0 && n0 < p.N,
                                  BS_SWEEP_TMA, x)) {
                    *abort = 1;
                    return;
                }
                tc::mbar_arrive_expect_tx(&cfull[s], bytes);
                tc::tma_load_2d(smem + OFF_W + s * W_SLOT, &maps.w, &cfull[s], x, n0);
                if (CAE) tc::tma_load_2d(smem + OFF_W0 + s * W_SLOT, &maps.w0, &cfull[s], x, n0);
                tc::tma_load_2d(smem + OFF_UD + s * D_SLOT, &maps.ud, &cfull[s], x, grp * K + x);
                if (GPTAQ) tc::tma_load_2d(smem + OFF_PD + s * D_SLOT, &maps.pd, &cfull[s], x, x);
                tc::tma_load_2d(smem + OFF_RP + s * R_SLOT, &maps.rp, &cfull[s], x, grp);
            };
            // B tile of phase q: rows 32 q .. 32 q + 31 of U (and of P1) over the 64-column
            // chunks from round_down(32 (q + 1), 64) to the super-block's end
            auto issue_b = [&](int q) {
                const int xb = 64 * ((q + 1) / 2);
                const int nch = (nend - xb + 63) / 64;
                const int y = sb0 + 32 * q;
                // bf16 boxes: columns on 16-byte boundaries, from inside the super-block's
                // span of U; rows of U inside the factor
                if (!GQ_IN_BOUNDS(p.status, y >= 0 && y < K && ((sb0 + xb) & 7) == 0 &&
                                                sb0 + xb + 64 * (nch - 1) < K + 64,
                                  BS_SWEEP_TMA, (long long)y * K + sb0 + xb)) {
                    *abort = 1;
                    return;
                }
                tc::mbar_arrive_expect_tx(bfull, 2 * nch * CH_BYTES);
                for (int c = 0; c < nch; ++c) {
                    const int x = sb0 + xb + 64 * c;
                    uint8_t *dh = smem + OFF_B + c * CH_BYTES;
                    tc::tma_load_2d(dh, &maps.bh, bfull, x, grp * K + y);
                    tc::tma_load_2d(dh + B_SPLIT, &maps.bl, bfull, x, grp * K + y);
                    if (GPTAQ) {
                        tc::tma_load_2d(dh + 4096, &maps.qh, bfull, x, y);
                        tc::tma_load_2d(dh + B_SPLIT + 4096, &maps.ql, bfull, x, y);
                    }
                }
            };
            int nc = 0, nb = 0;
            issue_chain(nc++);
            if (nsub > 1) issue_chain(nc++);
            if (nmma > 0) issue_b(nb++);
            while (!*abort && (nc < nsub || nb < nmma)) {
                if (nc < nsub) {      // slot of phase nc - 2, free once that phase's chain is done
                    if (!tc::mbar_wait(&cfree[nc & 1], ((nc - 2) >> 1) & 1, abort)) break;
                    issue_chain(nc++);
                }
                if (nb < nmma) {      // B is free once the previous phase's products are done
                    if (!tc::mbar_wait(bar_rest, (nb - 1) & 1, abort)) break;
                    issue_b(nb++);
                }
            }
            if (*abort) {             // let the issued loads land before the CTA exits
                volatile int never = 0;
                for (int q = nc > 2 ? nc - 2 : 0; q < nc; ++q)
                    tc::mbar_wait(&cfull[q & 1], (q >> 1) & 1, &never);
                if (nb > 0) tc::mbar_wait(bfull, (nb - 1) & 1, &never);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // the products of phase q once every chain thread wrote its A row and B landed
            for (int q = 0; q < nmma; ++q) {
                if (!tc::mbar_wait(abar, q & 1, abort)) break;
                if (!tc::mbar_wait(bfull, q & 1, abort)) break;
                tc::fence_after_sync();
                const int xb = 64 * ((q + 1) / 2);
                const int nch = (nend - xb + 63) / 64;
                const uint32_t a0 = tc::smem_u32(smem + OFF_A + (q & 1) * 2 * A_TILE);
                const uint32_t b0 = tc::smem_u32(smem + OFF_B);
                // chunk groups: [0, 1) first (the next phase's columns), then <= 4 at a time
                for (int c0 = 0; c0 < nch;) {
                    const int cn = c0 == 0 ? 1 : min(4, nch - c0);
                    const uint32_t idesc = tc::idesc_bf16_f32(128, 64 * cn, 0, 1, 0);
                    const uint32_t d = tmem + xb + 64 * c0;
                    const uint32_t bb = b0 + c0 * CH_BYTES;
#pragma unroll
                    for (int kk = 0; kk < KP / 16; ++kk) {
                        const uint64_t ah = tc::desc_sw128(a0 + kk * 32, 16, 1024);
                        const uint64_t al = tc::desc_sw128(a0 + A_TILE + kk * 32, 16, 1024);
                        const uint64_t bh = tc::desc_sw128(bb + kk * 2048, CH_BYTES, 1024);
                        const uint64_t bl = tc::desc_sw128(bb + B_SPLIT + kk * 2048, CH_BYTES, 1024);
                        tc::mma_bf16(d, ah, bh, idesc, (q > 0 || kk > 0) ? 1u : 0u);
                        tc::mma_bf16(d, ah, bl, idesc, 1u);
                        tc::mma_bf16(d, al, bh, idesc, 1u);
                    }
                    if (c0 == 0) tc::mma_commit(bar_next);
                    c0 += cn;
                }
                tc::mma_commit(bar_rest);
            }
            tc::mma_commit(drain);      // every product is done before TMEM is released
            volatile int never = 0;
            tc::mbar_wait(drain, 0, &never);
        }
    } else {
        const int tid = threadIdx.x;                 // channel row 0..127
        const bool valid = cta_ch0 + tid < p.per_group;
        const int64_t n = (int64_t)n0 + tid;
        const float s = valid ? p.scale[n] : 1.f;
        const float rs = 1.f / s;
        const float zf = (float)(1 << (p.bits - 1));
        const float cmin = -zf, cmax = (float)((1 << p.bits) - 1) - zf;
        const int live_end = min(p.S, K - sb0);      // coordinates of this super-block
        const int64_t ecol = (int64_t)grp * p.ldG + cta_ch0 + tid;
        uint8_t *crow = p.codes + n * K + sb0;
        const bool vcodes = valid && p.vcodes;
        const uint32_t arow = (uint32_t)tid * 128;   // this row in the A tiles
        const int sw = tid & 7;
        float lacc = 0.f;

#pragma unroll 1
        for (int q = 0; q < nsub; ++q) {
            const int slot = q & 1;
            if (!tc::mbar_wait(&cfull[slot], (q >> 1) & 1, abort)) break;
            // this channel's 32 weights: row tid of the swizzled slot, chunk c at c ^ (tid & 7)
            float2 w[16];
            float w0[CAE ? 32 : 1];
            {
                const uint8_t *wr = smem + OFF_W + slot * W_SLOT + tid * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 x = *reinterpret_cast<const float4 *>(wr + ((c ^ sw) << 4));
                    w[2 * c] = make_float2(x.x, x.y);
                    w[2 * c + 1] = make_float2(x.z, x.w);
                }
                if (CAE) {
                    const uint8_t *wr0 = smem + OFF_W0 + slot * W_SLOT + tid * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 x = *reinterpret_cast<const float4 *>(wr0 + ((c ^ sw) << 4));
                        w0[4 * c] = x.x; w0[4 * c + 1] = x.y; w0[4 * c + 2] = x.z; w0[4 * c + 3] = x.w;
                    }
                }
            }
            if (q > 0) {      // the earlier phases' products for these 32 columns
                if (!tc::mbar_wait(bar_next, (q - 1) & 1, abort)) break;
                tc::fence_after_sync();
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem + 32 * q + ((uint32_t)(warp * 32) << 16), v);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    w[i].x += __uint_as_float(v[2 * i]);
                    w[i].y += __uint_as_float(v[2 * i + 1]);
                }
            }
            const uint8_t *ud = smem + OFF_UD + slot * D_SLOT;   // row t, chunk c at c ^ (t & 7)
            const uint8_t *pd = smem + OFF_PD + slot * D_SLOT;
            const float *rp = reinterpret_cast<const float *>(smem + OFF_RP + slot * R_SLOT);
            uint8_t *ahi = smem + OFF_A + slot * 2 * A_TILE + arow;
            uint8_t *alo = ahi + A_TILE;
            uint32_t cw[4] = {0u, 0u, 0u, 0u};
            float ebuf[8], vbuf[8];
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int j = 32 * q + t;                     // coordinate in the super-block
                const bool live = j < live_end;
                const float wj = (t & 1) ? w[t >> 1].y : w[t >> 1].x;
                const float cf = fminf(fmaxf(rintf(wj * rs), cmin), cmax);
                const float rpj = rp[t];
                // ej: the rounding error of the value quantised (the loss); ep: the error
                // propagated, which CAE measures from the starting weight
                const float ej = live ? fmaf(-s, cf, wj) * rpj : 0.f;
                const float ep = CAE ? (live ? fmaf(-s, cf, w0[t]) * rpj : 0.f) : ej;
                const float vj = GPTAQ ? (live ? (CAE ? w0[t] : wj) : 0.f) : 0.f;
                lacc = fmaf(ej, ej, lacc);
                cw[(t >> 2) & 3] |= (uint32_t)(int)(cf + zf) << (8 * (t & 3));
                ebuf[t & 7] = -ep;
                if (GPTAQ) vbuf[t & 7] = vj;
                // the rest of this phase's coordinates. The next one first, alone: its FMA
                // is the only update the next step's rounding waits for (with GPTAQ the row
                // term goes in before it, since it does not depend on this step's error).
                const uint8_t *urow = ud + t * 128;
                const uint8_t *prow = pd + t * 128;
                auto uval = [&](const uint8_t *row, int k) {
                    return *reinterpret_cast<const float *>(row + (((k >> 2) ^ (t & 7)) << 4) + ((k & 3) << 2));
                };
                if (t + 1 < 32) {
                    float &wn = ((t + 1) & 1) ? w[(t + 1) >> 1].y : w[(t + 1) >> 1].x;
                    if (GPTAQ) wn = fmaf(vj, uval(prow, t + 1), wn);
                    wn = fmaf(-ep, uval(urow, t + 1), wn);
                }
                if ((t & 1) && t + 2 < 32) {      // the other half of the next coordinate's pair
                    float &wn2 = w[(t + 2) >> 1].y;
                    if (GPTAQ) wn2 = fmaf(vj, uval(prow, t + 2), wn2);
                    wn2 = fmaf(-ep, uval(urow, t + 2), wn2);
                }
                {
                    const int p0 = (t & 1) ? (t >> 1) + 2 : (t >> 1) + 1;   // first whole pair
                    const float2 ne = make_float2(-ep, -ep);
                    const float2 vv = make_float2(vj, vj);
#pragma unroll
                    for (int c = p0 >> 1; c < 8; ++c) {
                        const int off = (c ^ (t & 7)) << 4;
                        const float4 u = *reinterpret_cast<const float4 *>(urow + off);
                        float4 pq;
                        if (GPTAQ) pq = *reinterpret_cast<const float4 *>(prow + off);
                        if (2 * c >= p0) {
                            if (GPTAQ) w[2 * c] = ffma2(vv, make_float2(pq.x, pq.y), w[2 * c]);
                            w[2 * c] = ffma2(ne, make_float2(u.x, u.y), w[2 * c]);
                        }
                        if (GPTAQ) w[2 * c + 1] = ffma2(vv, make_float2(pq.z, pq.w), w[2 * c + 1]);
                        w[2 * c + 1] = ffma2(ne, make_float2(u.z, u.w), w[2 * c + 1]);
                    }
                }
                if ((t & 7) == 7) {
                    // eight errors (and V values) as bf16 pairs: the A tiles (row tid,
                    // k chunk t / 8, and 4 + t / 8 for V) and the far update's E rows
                    const int c = t >> 3;
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __nv_bfloat162 hh = __floats2bfloat162_rn(ebuf[2 * i], ebuf[2 * i + 1]);
                        const float2 hf = __bfloat1622float2(hh);
                        const __nv_bfloat162 ll =
                            __floats2bfloat162_rn(ebuf[2 * i] - hf.x, ebuf[2 * i + 1] - hf.y);
                        h[i] = *reinterpret_cast<const uint32_t *>(&hh);
                        l[i] = *reinterpret_cast<const uint32_t *>(&ll);
                    }
                    *reinterpret_cast<uint4 *>(ahi + ((c ^ sw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4 *>(alo + ((c ^ sw) << 4)) = make_uint4(l[0], l[1], l[2], l[3]);
                    if (valid && GQ_IN_BOUNDS(p.status, ecol * ESTRIDE + p.eoff + 32 * q + 8 * c + 8 <= (int64_t)p.ldE * ESTRIDE,
                                              BS_SWEEP_OUT, ecol * ESTRIDE + p.eoff + 32 * q + 8 * c)) {
                        // the far update's copy: -E, this channel's row
                        const int64_t eo = ecol * ESTRIDE + p.eoff + 32 * q + 8 * c;
                        *reinterpret_cast<uint4 *>(p.Eh + eo) = make_uint4(h[0], h[1], h[2], h[3]);
                        *reinterpret_cast<uint4 *>(p.El + eo) = make_uint4(l[0], l[1], l[2], l[3]);
                    }
                    if (GPTAQ) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const __nv_bfloat162 hh = __floats2bfloat162_rn(vbuf[2 * i], vbuf[2 * i + 1]);
                            const float2 hf = __bfloat1622float2(hh);
                            const __nv_bfloat162 ll =
                                __floats2bfloat162_rn(vbuf[2 * i] - hf.x, vbuf[2 * i + 1] - hf.y);
                            h[i] = *reinterpret_cast<const uint32_t *>(&hh);
                            l[i] = *reinterpret_cast<const uint32_t *>(&ll);
                        }
                        *reinterpret_cast<uint4 *>(ahi + (((4 + c) ^ sw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
                        *reinterpret_cast<uint4 *>(alo + (((4 + c) ^ sw) << 4)) = make_uint4(l[0], l[1], l[2], l[3]);
                        if (valid && GQ_IN_BOUNDS(p.status, ecol * ESTRIDE + p.eoff + 32 * q + 8 * c + 8 <= (int64_t)p.ldE * ESTRIDE,
                                                  BS_SWEEP_OUT, ecol * ESTRIDE + p.eoff + 32 * q + 8 * c)) {
                            const int64_t eo = ecol * ESTRIDE + p.eoff + 32 * q + 8 * c;
                            *reinterpret_cast<uint4 *>(p.Ph + eo) = make_uint4(h[0], h[1], h[2], h[3]);
                            *reinterpret_cast<uint4 *>(p.Pl + eo) = make_uint4(l[0], l[1], l[2], l[3]);
                        }
                    }
                }
                if ((t & 15) == 15 && valid) {
                    const int c16 = 32 * q + (t & 16);        // 16 codes of this channel
                    if (c16 < live_end &&
                        GQ_IN_BOUNDS(p.status, n < p.N && sb0 + min(c16 + 16, live_end) <= K,
                                     BS_SWEEP_OUT, n * K + sb0 + c16)) {
                        if (vcodes && c16 + 16 <= live_end) {
                            *reinterpret_cast<uint4 *>(crow + c16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                        } else {
                            for (int e = 0; e < 16 && c16 + e < live_end; ++e)
                                crow[c16 + e] = (uint8_t)(cw[e >> 2] >> (8 * (e & 3)));
                        }
                    }
                    cw[0] = cw[1] = cw[2] = cw[3] = 0u;
                }
            }
            // the A tile is read by the tensor core (async proxy); the slot's inputs are done;
            // this thread's TMEM reads are ordered before the products that follow
            tc::fence_async_shared();
            tc::fence_before_sync();
            tc::mbar_arrive(&cfree[slot]);
            if (q < nmma) tc::mbar_arrive(abar);
        }
        if (valid) p.loss_acc[n] += lacc;
    }

    __syncwarp();
    tc::fence_before_sync();
    __syncthreads();
    if (*abort && threadIdx.x == 0) set_status(p.status, GPTQ_ERR_TIMEOUT);
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, STC_TMEM_COLS);
    }
}

// 1 / U_jj per group (the pivots the sweep multiplies by), [g][K].
__global__ void k_pivot_recip(const float *__restrict__ U, int K, float *__restrict__ rp) {
    const int g = blockIdx.y;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j < K) rp[(int64_t)g * K + j] = 1.f / U[(int64_t)g * K * K + (int64_t)j * K + j];
}

// ------------------------------------------------------------------------------ host side

typedef CUresult (*StcEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static StcEncodeFn stc_encode_fn() {
    static StcEncodeFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<StcEncodeFn>(ptr);
    }
    return fn;
}

// fp32 [rows][cols] (row pitch ld floats) in box_cols x box_rows boxes, 128-byte swizzle.
static gptq_status stc_f32_map(CUtensorMap *m, const float *base, int64_t cols, int64_t rows,
                               int64_t ld, int box_cols, int box_rows) {
    StcEncodeFn enc = stc_encode_fn();
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

// The tensor-core sweep serves plain per-channel quantisation (with or without the
// GPTAQ and compensation-aware rows); it needs 16-byte row pitches for its TMA maps.
bool sweep_tc_eligible(int K, const float *U, const float *P1) {
    return stc_encode_fn() != nullptr && K % 4 == 0 && aligned(U, 16) &&
           (!P1 || aligned(P1, 16));
}

int sweep_tc_super(bool gptaq) { return gptaq ? 256 : 512; }

// Maps and the pivot reciprocals of one quantisation (before the first super-block).
gptq_status sweep_tc_setup(SweepTcMaps *maps, float *Wk, const float *W0k, const float *U,
                           const float *P1, const __nv_bfloat16 *Uh, const __nv_bfloat16 *Ul,
                           const __nv_bfloat16 *Qh, const __nv_bfloat16 *Ql, int ldU, float *rp,
                           int N, int K, int g, cudaStream_t st) {
    gptq_status s;
    memset(maps, 0, sizeof(*maps));
    if ((s = stc_f32_map(&maps->w, Wk, K, N, K, 32, 128)) != GPTQ_OK) return s;
    maps->w0 = maps->w;
    if (W0k && (s = stc_f32_map(&maps->w0, W0k, K, N, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = stc_f32_map(&maps->ud, U, K, (int64_t)g * K, K, 32, 32)) != GPTQ_OK) return s;
    maps->pd = maps->ud;
    if (P1 && (s = stc_f32_map(&maps->pd, P1, K, K, K, 32, 32)) != GPTQ_OK) return s;
    if ((s = stc_f32_map(&maps->rp, rp, K, g, K, 32, 1)) != GPTQ_OK) return s;
    if ((s = make_bf16_map(&maps->bh, Uh, K, (int64_t)g * K, ldU, 32)) != GPTQ_OK) return s;
    if ((s = make_bf16_map(&maps->bl, Ul, K, (int64_t)g * K, ldU, 32)) != GPTQ_OK) return s;
    maps->qh = maps->bh;
    maps->ql = maps->bl;
    if (P1) {
        if ((s = make_bf16_map(&maps->qh, Qh, K, K, ldU, 32)) != GPTQ_OK) return s;
        if ((s = make_bf16_map(&maps->ql, Ql, K, K, ldU, 32)) != GPTQ_OK) return s;
    }
    k_pivot_recip<<<dim3((K + 255) / 256, g), 256, 0, st>>>(U, K, rp);
    return launch_status();
}

gptq_status sweep_tc_launch(const SweepTcMaps &maps, const float *scale, int bits, uint8_t *codes,
                            __nv_bfloat16 *Eh, __nv_bfloat16 *El, __nv_bfloat16 *Ph,
                            __nv_bfloat16 *Pl, int ldE, int ldG, float *loss_acc, int32_t *status,
                            int N, int per_group, int K, int groups, int sb0, int S, int eoff,
                            bool gptaq, bool cae, cudaStream_t st) {
    // the B tile holds at most 8 (plain) or 4 (GPTAQ, twice as deep) 64-column chunks
    if (S < 1 || S > sweep_tc_super(gptaq) || sb0 % 64 != 0 || sb0 + S > K) return GPTQ_ERR_ARG;
    if (eoff < 0 || eoff % 32 != 0 || eoff + 32 * ((S + 31) / 32) > ESTRIDE) return GPTQ_ERR_ARG;
    SweepTcParams p;
    p.scale = scale;
    p.codes = codes;
    p.Eh = Eh; p.El = El; p.Ph = Ph; p.Pl = Pl;
    p.loss_acc = loss_acc;
    p.status = status;
    p.N = N; p.per_group = per_group; p.K = K; p.bits = bits;
    p.ldE = ldE; p.ldG = ldG;
    p.sb0 = sb0; p.S = S;
    p.eoff = eoff;
    p.vcodes = (K % 16 == 0 && aligned(codes, 16)) ? 1 : 0;
    const dim3 grid((per_group + STC_CH - 1) / STC_CH, groups);
    typedef void (*Kern)(const SweepTcMaps, const SweepTcParams);
    const Kern kern = gptaq ? (cae ? k_sweep_tc<true, true> : k_sweep_tc<true, false>)
                            : (cae ? k_sweep_tc<false, true> : k_sweep_tc<false, false>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, STC_SMEM) !=
        cudaSuccess)
        return launch_status();
    const int rec = prof_begin(GPTQ_PROF_SWEEP, st);
    // a programmatic dependent of the previous kernel on the stream (the far update):
    // its set-up overlaps that kernel's end; griddepcontrol.wait orders its accesses
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(STC_THREADS);
    cfg.dynamicSmemBytes = STC_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, maps, p);
    const gptq_status s = launch_status();
    prof_end(rec, st);
    return s;
}

}  // namespace gptq
