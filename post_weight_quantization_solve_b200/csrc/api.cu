// C ABI entry points: argument checks, workspace sizing, dispatch. Every check
// here runs on the host before anything is enqueued.
#include <nvtx3/nvToolsExt.h>

#include <cmath>

#include <mutex>
#include <vector>

#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {
gptq_status gram_simt(float *H, int K, int g, const void *X, int xdtype, int64_t M, int64_t ldx,
                      const float *w, int64_t ldw, const int32_t *status, cudaStream_t st);
gptq_status cross_simt(float *C, int K, const void *Xfp, const void *Xq, int xdtype, int64_t M,
                       int64_t ldx, const int32_t *status, cudaStream_t st);
gptq_status gram_tc(float *H, int K, int g, const void *X, int64_t M, int64_t ldx,
                    const float *w, int64_t ldw, const void *X2, cudaStream_t st, int32_t *status,
                    bool *used);
gptq_status gram_x_tc(float *H, int K, int g, const void *X, const void *X2, int64_t M,
                      int64_t ldx, const float *w, int64_t ldw, int32_t *status, cudaStream_t st,
                      bool *used);
size_t prepare_workspace(int K, int g);
size_t prepare_workspace_compact(int K, int g);
gptq_status prepare(float *H, int K, int g, float percdamp, uint8_t *dead_out, void *ws,
                    size_t ws_bytes, int32_t *status, cudaStream_t st);
size_t residual_workspace(int K);
gptq_status residual(float *P1, const float *C, const float *U, int K, void *ws, cudaStream_t st);
size_t quantize_workspace(int K, int N, int g, int blocksize);
gptq_status quantize_layer(void *W, int wdtype, int N, int K, const float *U, int groups, int bits,
                           int blocksize, const float *P1, int cae, const uint8_t *dead,
                           const float *scales_in, float *scales_out, uint8_t *codes, float *loss,
                           int write_back, void *ws, int32_t *status, cudaStream_t st);
size_t quantize_grouped_workspace(int K, int N, int blocksize);
size_t quantize_cae_extra(int K, int N);
gptq_status quantize_layer_grouped(void *W, int wdtype, int N, int K, const float *U, int bits,
                                   int blocksize, int groupsize, int static_groups,
                                   const int32_t *perm, const float *P1, int cae,
                                   const uint8_t *dead,
                                   float *scales_out, int32_t *g_idx, uint8_t *codes, float *loss,
                                   int write_back, void *ws, int32_t *status, cudaStream_t st);
gptq_status act_order(const float *H, int K, int32_t *perm, cudaStream_t st);
gptq_status pack_codes(const uint8_t *codes, int N, int K, int64_t ldc, int bits, uint32_t *words,
                       int64_t ldw, cudaStream_t st);
gptq_status unpack_codes(const uint32_t *words, int N, int K, int64_t ldw, int bits,
                         uint8_t *codes, int64_t ldc, cudaStream_t st);
size_t first_order_workspace(int K, int N);
gptq_status first_order_shift(float *W, int N, int K, const float *U, const void *G, int gdtype,
                              float beta, double *gamma, void *ws, int32_t *status,
                              cudaStream_t st);
gptq_status permute_square(float *out, const float *H, int K, const int32_t *perm,
                           cudaStream_t st);
}  // namespace gptq

namespace gptq {
unsigned long long g_launches = 0;
}

using namespace gptq;

static bool valid_dtype(int d) { return d == GPTQ_BF16 || d == GPTQ_F32; }

// One NVTX range per entry point (a no-op unless a profiler collects NVTX).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
#define GPTQ_RANGE(name) NvtxRange gptq_nvtx_range_(name)

// One bounded wait on a barrier that nothing arrives on: after the wait budget the
// status word holds GPTQ_ERR_TIMEOUT and the kernel returns.
__global__ void k_selftest_timeout(int32_t *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, &abort_flag)) set_status(status, GPTQ_ERR_TIMEOUT);
}

#ifdef GPTQ_DEBUG_BOUNDS
// Readers of the translation units' check records, registered at load time.
static std::mutex &bounds_mu() {
    static std::mutex mu;
    return mu;
}
static std::vector<BoundsReader> &bounds_readers() {
    static std::vector<BoundsReader> v;
    return v;
}
void gptq::bounds_register(BoundsReader fn) {
    std::lock_guard<std::mutex> lock(bounds_mu());
    bounds_readers().push_back(fn);
}

// One check that always fails; no memory is accessed.
__global__ void k_bounds_selftest(int32_t *status, int never) {
    if (threadIdx.x == 0) (void)GQ_IN_BOUNDS(status, never != 0, BS_SELFTEST, -1);
}
#endif

static bool stream_ok(int xdtype, const void *X, int64_t ldx, int K) {
    if (ldx < K) return false;
    if (xdtype == GPTQ_BF16) return aligned(X, 16) && ldx % 8 == 0;
    return aligned(X, 4);
}

extern "C" {

gptq_status gptq_accumulate_hessian(float *H, int K, int g, const void *X, int xdtype, int64_t M,
                                    int64_t ldx, const float *w, int64_t ldw, int32_t *status,
                                    void *stream) {
    GPTQ_RANGE("gptq_accumulate_hessian");
    if (K < 1 || K > GPTQ_MAX_DIM || g < 1 || g > 65535 || M < 0 || !H || !valid_dtype(xdtype))
        return GPTQ_ERR_ARG;
    if (M > 0x7fffffff) return GPTQ_ERR_ARG;
    if (w == nullptr && g != 1) return GPTQ_ERR_ARG;
    if (w != nullptr && ldw < M) return GPTQ_ERR_ARG;
    if (M == 0) return GPTQ_OK;
    if (!X || !stream_ok(xdtype, X, ldx, K)) return GPTQ_ERR_ARG;
    if (xdtype == GPTQ_BF16 && K % 8 != 0) return GPTQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (xdtype == GPTQ_BF16) {
        bool used = false;
        gptq_status s = (w == nullptr)
                            ? gram_tc(H, K, g, X, M, ldx, w, ldw, nullptr, st, status, &used)
                            : gram_x_tc(H, K, g, X, nullptr, M, ldx, w, ldw, status, st, &used);
        if (used || s != GPTQ_OK) return s;
    }
    return gram_simt(H, K, g, X, xdtype, M, ldx, w, ldw, status, st);
}

gptq_status gptaq_accumulate_cross(float *C, int K, const void *X_fp, const void *X_q, int xdtype,
                                   int64_t M, int64_t ldx, int32_t *status, void *stream) {
    GPTQ_RANGE("gptaq_accumulate_cross");
    if (K < 1 || K > GPTQ_MAX_DIM || M < 0 || !C || !valid_dtype(xdtype)) return GPTQ_ERR_ARG;
    if (M > 0x7fffffff) return GPTQ_ERR_ARG;
    if (M == 0) return GPTQ_OK;
    if (!X_fp || !X_q || !stream_ok(xdtype, X_fp, ldx, K) || !stream_ok(xdtype, X_q, ldx, K))
        return GPTQ_ERR_ARG;
    if (xdtype == GPTQ_BF16 && K % 8 != 0) return GPTQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (xdtype == GPTQ_BF16) {
        bool used = false;
        gptq_status s = gram_x_tc(C, K, 1, X_fp, X_q, M, ldx, nullptr, 0, status, st, &used);
        if (used || s != GPTQ_OK) return s;
    }
    return cross_simt(C, K, X_fp, X_q, xdtype, M, ldx, status, st);
}

gptq_status gptq_prepare(float *H, int K, int g, float percdamp, uint8_t *dead_out, void *ws,
                         size_t ws_bytes, int32_t *status, void *stream) {
    GPTQ_RANGE("gptq_prepare");
    if (K < 1 || g < 1 || !H || !status || !(percdamp >= 0.f) || !aligned(H, 16))
        return GPTQ_ERR_ARG;
    if (K > GPTQ_MAX_DIM || g > 65535) return GPTQ_ERR_ARG;
    if (!ws || !aligned(ws, 256) || ws_bytes < prepare_workspace_compact(K, g))
        return GPTQ_ERR_WORKSPACE;
    return prepare(H, K, g, percdamp, dead_out, ws, ws_bytes, status,
                   static_cast<cudaStream_t>(stream));
}

gptq_status gptaq_residual(float *P1, const float *C, const float *U, int K, void *ws,
                           size_t ws_bytes, void *stream) {
    GPTQ_RANGE("gptaq_residual");
    if (K < 1 || K > GPTQ_MAX_DIM || !P1 || !C || !U) return GPTQ_ERR_ARG;
    if (!ws || !aligned(ws, 256) || ws_bytes < residual_workspace(K)) return GPTQ_ERR_WORKSPACE;
    return residual(P1, C, U, K, ws, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_quantize_layer(void *W, int wdtype, int N, int K, const float *U, int groups,
                                int bits, int blocksize, const float *P1, int cae,
                                const uint8_t *dead, const float *scales_in, float *scales_out,
                                uint8_t *codes, float *loss, int write_back, void *ws,
                                size_t ws_bytes, int32_t *status, void *stream) {
    GPTQ_RANGE("gptq_quantize_layer");
    if (N < 1 || K < 1 || groups < 1 || N % groups != 0 || !W || !U || !codes || !status)
        return GPTQ_ERR_ARG;
    if (N > GPTQ_MAX_DIM || K > GPTQ_MAX_DIM || groups > 8) return GPTQ_ERR_ARG;
    if (!valid_dtype(wdtype)) return GPTQ_ERR_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_ARG;
    if (blocksize != 16 && blocksize != 32 && blocksize != 64 && blocksize != 128)
        return GPTQ_ERR_ARG;
    if (P1 && groups != 1) return GPTQ_ERR_ARG;
    if (cae != 0 && cae != 1) return GPTQ_ERR_ARG;
    if (!aligned(U, 16) || (P1 && !aligned(P1, 16))) return GPTQ_ERR_ARG;
    if (!ws || !aligned(ws, 256) ||
        ws_bytes < quantize_workspace(K, N, groups, blocksize) + (cae ? quantize_cae_extra(K, N) : 0))
        return GPTQ_ERR_WORKSPACE;
    return quantize_layer(W, wdtype, N, K, U, groups, bits, blocksize, P1, cae, dead, scales_in,
                          scales_out, codes, loss, write_back, ws, status,
                          static_cast<cudaStream_t>(stream));
}

gptq_status gptq_act_order(const float *H, int K, int32_t *perm, void *stream) {
    GPTQ_RANGE("gptq_act_order");
    if (K < 1 || K > GPTQ_MAX_DIM || !H || !perm) return GPTQ_ERR_ARG;
    return act_order(H, K, perm, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_permute_hessian(float *out, const float *H, int K, const int32_t *perm,
                                 void *stream) {
    GPTQ_RANGE("gptq_permute_hessian");
    if (K < 1 || K > GPTQ_MAX_DIM || !out || !H || !perm || out == H) return GPTQ_ERR_ARG;
    return permute_square(out, H, K, perm, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_quantize_layer_grouped(void *W, int wdtype, int N, int K, const float *U,
                                        int bits, int blocksize, int groupsize, int static_groups,
                                        const int32_t *perm, const float *P1, int cae,
                                        const uint8_t *dead, float *scales_out,
                                        int32_t *g_idx_out, uint8_t *codes,
                                        float *loss, int write_back, void *ws, size_t ws_bytes,
                                        int32_t *status, void *stream) {
    GPTQ_RANGE("gptq_quantize_layer_grouped");
    if (N < 1 || K < 1 || !W || !U || !codes || !status) return GPTQ_ERR_ARG;
    if (N > GPTQ_MAX_DIM || K > GPTQ_MAX_DIM || !valid_dtype(wdtype)) return GPTQ_ERR_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_ARG;
    if (groupsize != 0 && groupsize != 32 && groupsize != 64 && groupsize != 128) return GPTQ_ERR_ARG;
    if (blocksize != 32 && blocksize != 64 && blocksize != 128) return GPTQ_ERR_ARG;
    if (groupsize && blocksize % groupsize != 0) return GPTQ_ERR_ARG;
    if (cae != 0 && cae != 1) return GPTQ_ERR_ARG;
    if (!aligned(U, 16) || (P1 && !aligned(P1, 16))) return GPTQ_ERR_ARG;
    if (!ws || !aligned(ws, 256) ||
        ws_bytes < quantize_grouped_workspace(K, N, blocksize) + (cae ? quantize_cae_extra(K, N) : 0))
        return GPTQ_ERR_WORKSPACE;
    return quantize_layer_grouped(W, wdtype, N, K, U, bits, blocksize, groupsize, static_groups,
                                  perm, P1, cae, dead, scales_out, g_idx_out, codes, loss, write_back,
                                  ws, status, static_cast<cudaStream_t>(stream));
}

static bool pack_args_ok(int N, int K, int bits, int64_t ldc, int64_t ldw) {
    if (N < 0 || K < 1 || N > GPTQ_MAX_DIM || K > GPTQ_MAX_DIM) return false;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return false;
    return ldc >= K && ldw >= ((int64_t)K * bits + 31) / 32;
}

gptq_status gptq_pack_codes(const uint8_t *codes, int N, int K, int64_t ld_codes, int bits,
                            uint32_t *words, int64_t ld_words, void *stream) {
    GPTQ_RANGE("gptq_pack_codes");
    if (!pack_args_ok(N, K, bits, ld_codes, ld_words)) return GPTQ_ERR_ARG;
    if (N > 0 && (!codes || !words)) return GPTQ_ERR_ARG;
    return pack_codes(codes, N, K, ld_codes, bits, words, ld_words,
                      static_cast<cudaStream_t>(stream));
}

gptq_status gptq_unpack_codes(const uint32_t *words, int N, int K, int64_t ld_words, int bits,
                              uint8_t *codes, int64_t ld_codes, void *stream) {
    GPTQ_RANGE("gptq_unpack_codes");
    if (!pack_args_ok(N, K, bits, ld_codes, ld_words)) return GPTQ_ERR_ARG;
    if (N > 0 && (!codes || !words)) return GPTQ_ERR_ARG;
    return unpack_codes(words, N, K, ld_words, bits, codes, ld_codes,
                        static_cast<cudaStream_t>(stream));
}

gptq_status gptq_first_order_shift(float *W, int N, int K, const float *U, const void *G,
                                  int gdtype, float beta, double *gamma, void *ws,
                                  size_t ws_bytes, int32_t *status, void *stream) {
    GPTQ_RANGE("gptq_first_order_shift");
    if (N < 1 || K < 1 || N > GPTQ_MAX_DIM || K > GPTQ_MAX_DIM) return GPTQ_ERR_ARG;
    if (!W || !U || !G || !status || !valid_dtype(gdtype)) return GPTQ_ERR_ARG;
    if (!(beta >= 0.f && beta <= 1.f)) return GPTQ_ERR_ARG;
    if (!ws || !aligned(ws, 256) || ws_bytes < first_order_workspace(K, N)) return GPTQ_ERR_WORKSPACE;
    return first_order_shift(W, N, K, U, G, gdtype, beta, gamma, ws, status,
                             static_cast<cudaStream_t>(stream));
}

float gptq_trust_region_beta(float alpha, double loss_gptq, double gamma) {
    // largest beta in [0, 1] with (beta - beta^2 / 2) gamma <= alpha loss_gptq
    if (!(gamma > 0.0)) return 1.f;
    const double x = (double)alpha * loss_gptq / gamma;
    if (!(x >= 0.0)) return 0.f;
    if (x >= 0.5) return 1.f;
    return (float)(1.0 - sqrt(1.0 - 2.0 * x));
}

gptq_status gptq_selftest_timeout(int32_t *status, void *stream) {
    if (!status) return GPTQ_ERR_ARG;
    k_selftest_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
    return launch_status();
}

size_t gptq_workspace_size(int op, int K, int N, int g, int blocksize) {
    if (K < 1 || g < 1) return 0;
    const bool cae = (op & GPTQ_WS_CAE) != 0;
    op &= ~GPTQ_WS_CAE;
    if (cae && op != GPTQ_OP_QUANTIZE && op != GPTQ_OP_QUANTIZE_GROUPED) return 0;
    if (cae && N < 1) return 0;
    const size_t extra = cae ? quantize_cae_extra(K, N) : 0;
    switch (op) {
        case GPTQ_OP_PREPARE: return prepare_workspace(K, g);
        case GPTQ_OP_RESIDUAL: return residual_workspace(K);
        case GPTQ_OP_QUANTIZE:
            if (N < 1 || blocksize < 1) return 0;
            return quantize_workspace(K, N, g, blocksize) + extra;
        case GPTQ_OP_QUANTIZE_GROUPED:
            if (N < 1 || blocksize < 1) return 0;
            return quantize_grouped_workspace(K, N, blocksize) + extra;
        case GPTQ_OP_FIRST_ORDER:
            if (N < 1) return 0;
            return first_order_workspace(K, N);
        default: return 0;
    }
}

unsigned long long gptq_kernel_launches(void) {
    return __atomic_load_n(&g_launches, __ATOMIC_RELAXED);
}

const char *gptq_status_string(int status) {
    switch (status) {
        case GPTQ_OK: return "ok";
        case GPTQ_ERR_ARG: return "invalid argument";
        case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
        case GPTQ_ERR_NONFINITE: return "non-finite value in an input or intermediate";
        case GPTQ_ERR_CUDA: return "CUDA launch or API error";
        case GPTQ_ERR_TIMEOUT: return "bounded device wait ran out";
        case GPTQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case GPTQ_ERR_BOUNDS: return "an index check failed (the access was skipped)";
        default: return "unknown status";
    }
}

gptq_status gptq_bounds_report(int *enabled, int *count, int *site, int64_t *index, int reset) {
    if (!enabled || !count || !site || !index) return GPTQ_ERR_ARG;
    *enabled = 0;
    *count = 0;
    *site = 0;
    *index = 0;
#ifdef GPTQ_DEBUG_BOUNDS
    *enabled = 1;
    if (cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return GPTQ_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(bounds_mu());
    for (BoundsReader fn : bounds_readers()) {
        BoundsRecord r{0, 0, 0};
        if (!fn(&r, reset != 0)) return GPTQ_ERR_CUDA;
        if (r.count > 0 && *count == 0) {
            *site = r.site;
            *index = r.index;
        }
        *count += r.count;
    }
#else
    (void)reset;
#endif
    return GPTQ_OK;
}

gptq_status gptq_bounds_selftest(int32_t *status, void *stream) {
    if (!status) return GPTQ_ERR_ARG;
#ifdef GPTQ_DEBUG_BOUNDS
    k_bounds_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, 0);
    return launch_status();
#else
    (void)stream;
    return GPTQ_ERR_ARG;
#endif
}

}  // extern "C"
