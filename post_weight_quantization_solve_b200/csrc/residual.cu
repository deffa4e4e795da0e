// gptaq_residual: P1 = [(C U^T) ⊙ M] U, M the strict upper mask.
//
// [ResComp] item 3 writes P1 = [(dX X^T L) ⊙ M_U] L^T with H^-1 = L L^T; in the
// K x N layout L = U^T, so P1 = [(C U^T) ⊙ M] U. With the strict mask, row q is
// C[q, F'] (H[F', F'])^-1 over the coordinates after q: the residual term of the
// OBC closed form ([GPTAQ] "基于最优脑压缩的闭式解") applied at q's step.
#include "common.cuh"
#include "gemm_simt.cuh"

namespace gptq {

size_t residual_workspace(int K) { return round_up((size_t)K * K * sizeof(float), 256); }

gptq_status residual(float *P1, const float *C, const float *U, int K, void *ws,
                     cudaStream_t st) {
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
