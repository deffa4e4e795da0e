// gptq_prepare_noalloc: gptq_prepare with its scratch in a fixed device array
// owned by the library instead of a caller workspace.
//
// For callers that cannot allocate device memory when they need the factor: for
// example code that runs inside a host application that owns every device
// allocation through its own pool and gives plug-ins no workspace, or a
// latency-critical path that must not take the device-wide synchronisation that
// cudaMalloc / cudaFree imply. This call allocates nothing: the scratch is the
// file-scope array below, which every GPU that loads the library holds until the
// process exits.
#include <mutex>

#include "common.cuh"

namespace gptq {

size_t prepare_workspace_compact(int K, int g);
gptq_status prepare(float *H, int K, int g, float percdamp, uint8_t *dead_out, void *ws,
                    size_t ws_bytes, int32_t *status, cudaStream_t st);

// 16 MiB + 64 KiB: enough for K <= 4096 with one Hessian (or K <= 2048 with g <= 4).
constexpr size_t NOALLOC_SCRATCH_BYTES = (16u << 20) + (64u << 10);

static __device__ __align__(256) unsigned char g_prepare_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
static void *g_scratch_ptr[NOALLOC_MAX_DEVICES];
static std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up once per
// device (the host-side name of the array is only a stand-in, not a device address).
static gptq_status scratch_for_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES)
        return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prepare_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return GPTQ_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GPTQ_OK;
}

}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_prepare_noalloc(float *H, int K, int g, float percdamp,
                                            uint8_t *dead_out, int32_t *status, void *stream) {
    if (K < 1 || g < 1 || !H || !status || !(percdamp >= 0.f) || !aligned(H, 16))
        return GPTQ_ERR_ARG;
    if (K > GPTQ_MAX_DIM) return GPTQ_ERR_ARG;
    if (prepare_workspace_compact(K, g) > NOALLOC_SCRATCH_BYTES) return GPTQ_ERR_ARG;
    void *ws = nullptr;
    gptq_status s = scratch_for_current_device(&ws);
    if (s != GPTQ_OK) return s;
    return prepare(H, K, g, percdamp, dead_out, ws, NOALLOC_SCRATCH_BYTES, status,
                   static_cast<cudaStream_t>(stream));
}
