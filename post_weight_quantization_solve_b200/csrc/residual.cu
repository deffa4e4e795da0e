// gptaq_residual: P1 = [(C U^T) ⊙ M] U, M the strict upper mask.
//
// [ResComp] item 3 writes P1 = [(dX X^T L) ⊙ M_U] L^T with H^-1 = L L^T; in the
// K x N layout L = U^T, so P1 = [(C U^T) ⊙ M] U. With the strict mask, row q is
// C[q, F'] (H[F', F'])^-1 over the coordinates after q: the residual term of the
// OBC closed form ([GPTAQ] "基于最优脑压缩的闭式解") applied at q's step.
#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc32.cuh"

namespace gptq {

static bool residual_tc_eligible(int K) { return K % 32 == 0 && K >= 256; }

// T, plus on the tensor-core path two tf32 pair buffers (2 K^2 each), reused for
// (C, U) and then (T, U^T).
size_t residual_workspace(int K) {
    const size_t kk = (size_t)K * K;
    return round_up((residual_tc_eligible(K) ? 5 * kk : kk) * sizeof(float), 256);
}

// Tensor-core route (tf32x3, every operand K-major):
//   T  = C U^T, strict upper      A = rows of C, B^T = rows of U, upper tiles, masked
//   P1 = T U                      A = rows of T (upper), B^T = rows of U^T, U upper
static gptq_status residual_tc(float *P1, const float *C, const float *U, int K, float *ws,
                               cudaStream_t st) {
    const int64_t KK = (int64_t)K * K;
    float *T = ws, *Ah = T + KK, *Al = Ah + KK, *Bh = Al + KK, *Bl = Bh + KK;
    static thread_local Tc32Params p;
    CUtensorMap m[4];
    gptq_status s;
    if ((s = split_tf32(C, K, K, K, Ah, Al, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    if ((s = split_tf32(U, K, K, K, Bh, Bl, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[0], Ah, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[1], Al, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[2], Bh, K, K, K, 32, 128)) != GPTQ_OK) return s;
    if ((s = make_f32_map(&m[3], Bl, K, K, K, 32, 128)) != GPTQ_OK) return s;
    cudaMemsetAsync(T, 0, sizeof(float) * (size_t)KK, st);
    p = Tc32Params{};
    p.C = T; p.alpha = 1.f; p.accumulate = 1; p.upper_tiles = 1; p.mask_strict_upper = 1;
    p.c_extent = KK;
    p.nitems = 1;
    p.item[0].m = K; p.item[0].n = K; p.item[0].k = K;
    p.item[0].c_off = 0; p.item[0].ldc = K;
    if ((s = launch_gemm_tc32(m, p, st)) != GPTQ_OK) return s;
    if ((s = split_tf32(T, K, K, K, Ah, Al, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    if ((s = split_tf32_t(U, K, K, K, Bh, Bl, K, 1, 0, 0, st)) != GPTQ_OK) return s;
    cudaMemsetAsync(P1, 0, sizeof(float) * (size_t)KK, st);
    p = Tc32Params{};
    p.C = P1; p.alpha = 1.f; p.accumulate = 1; p.a_upper = 1; p.b_upper = 1;
    p.c_extent = KK;
    p.nitems = 1;
    p.item[0].m = K; p.item[0].n = K; p.item[0].k = K;
    p.item[0].c_off = 0; p.item[0].ldc = K;
    return launch_gemm_tc32(m, p, st);
}

gptq_status residual(float *P1, const float *C, const float *U, int K, void *ws,
                     cudaStream_t st) {
    if (residual_tc_eligible(K) && tc32_available())
        return residual_tc(P1, C, U, K, static_cast<float *>(ws), st);
    float *T = static_cast<float *>(ws);
    // T = C U^T, kept only where column > row (upper tiles, masked epilogue)
    GemmParams a = gemm_params(K, K, K, C, K, U, K, T, K, 1.f, 0, nullptr);
    a.upper_tiles = 1;
    a.mask_strict_upper = 1;
    gptq_status s = gemm_simt<float, float, false, true>(a, 1, st);
    if (s != GPTQ_OK) return s;
    // P1 = T U: T(q, t) = 0 for t <= q, U(t, k) = 0 for t > k
    GemmParams b = gemm_params(K, K, K, T, K, U, K, P1, K, 1.f, 0, nullptr);
    b.a_upper = 1;
    b.b_upper = 1;
    return gemm_simt<float, float, false, false>(b, 1, st);
}

}  // namespace gptq
