// Tensor-core (tcgen05) Gram path: not yet enabled; the SIMT path runs.
#include "common.cuh"

namespace gptq {
gptq_status gram_tc(float *H, int K, int g, const void *X, int64_t M, int64_t ldx, const float *w,
                    int64_t ldw, const void *X2, cudaStream_t st, bool *used) {
    (void)H; (void)K; (void)g; (void)X; (void)M; (void)ldx; (void)w; (void)ldw; (void)X2; (void)st;
    *used = false;
    return GPTQ_OK;
}
}  // namespace gptq
