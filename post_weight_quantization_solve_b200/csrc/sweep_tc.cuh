// Host interface of the tensor-core sweep (sweep_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace gptq {

// Tensor maps of one quantisation: the kernel's TMA sources.
struct SweepTcMaps {
    CUtensorMap w, w0;      // fp32 [N][K] working / starting weights, box 32 x 128
    CUtensorMap ud, pd;     // fp32 U [g K][K], P1 [K][K], box 32 x 32
    CUtensorMap rp;         // fp32 [g][K] 1 / U_jj, box 32 x 1
    CUtensorMap bh, bl;     // bf16 U pairs [g K][ldU], box 64 x 32
    CUtensorMap qh, ql;     // bf16 P1 pairs [K][ldU], box 64 x 32
};

// Per-channel quantisation whose row pitches suit the kernel's TMA maps (K % 4 == 0).
bool sweep_tc_eligible(int K, const float *U, const float *P1);
// Super-block length: 512, or 256 with the GPTAQ row term (its operands are twice as deep).
int sweep_tc_super(bool gptaq);
// Maps and 1 / U_jj (into rp, [g][K]) before the first super-block.
gptq_status sweep_tc_setup(SweepTcMaps *maps, float *Wk, const float *W0k, const float *U,
                           const float *P1, const __nv_bfloat16 *Uh, const __nv_bfloat16 *Ul,
                           const __nv_bfloat16 *Qh, const __nv_bfloat16 *Ql, int ldU, float *rp,
                           int N, int K, int g, cudaStream_t st);
// One super-block [sb0, sb0 + S) for every channel: codes, loss, and the E (and V) pairs
// of the super-block for the far update, at columns [eoff, eoff + S) of the channel rows.
gptq_status sweep_tc_launch(const SweepTcMaps &maps, const float *scale, int bits, uint8_t *codes,
                            __nv_bfloat16 *Eh, __nv_bfloat16 *El, __nv_bfloat16 *Ph,
                            __nv_bfloat16 *Pl, int ldE, int ldG, float *loss_acc, int32_t *status,
                            int N, int per_group, int K, int groups, int sb0, int S, int eoff,
                            bool gptaq, bool cae, cudaStream_t st);
// Row pitch of the E / V pair rows the sweep writes (elements): two super-blocks.
constexpr int SWEEP_TC_ESTRIDE = 1024;

}  // namespace gptq
