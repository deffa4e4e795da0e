// Shared helpers of libgptq: status word, launch checks, small device utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gptq.h"

namespace gptq {

// Record the first numerical failure in the caller's status word.
__device__ __forceinline__ void set_status(int32_t *status, int code) {
    if (status) atomicCAS(reinterpret_cast<int *>(status), 0, code);
}

// Kernels of a chain skip their work once an earlier kernel failed.
__device__ __forceinline__ bool failed(const int32_t *status) {
    return status && *reinterpret_cast<const volatile int32_t *>(status) != 0;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Kernels enqueued by this process; every launch site is followed by exactly one
// launch_status() call, which counts it.
extern unsigned long long g_launches;

inline gptq_status launch_status() {
    __atomic_add_fetch(&g_launches, 1ull, __ATOMIC_RELAXED);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

// d = a * b + c on two fp32 lanes at once (sm_100 packed fp32 FMA, round to nearest).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)),
          "l"(*reinterpret_cast<const uint64_t *>(&c)));
    return *reinterpret_cast<const float2 *>(&d);
}

// Timing windows of gptq_profile_enable: events around a launch of one class on its
// stream (profile.cu). prof_begin returns -1 when nothing is recorded.
int prof_begin(int kind, cudaStream_t st);
void prof_end(int rec, cudaStream_t st);

inline bool aligned(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace carving: consecutive 256-byte aligned regions.
struct Carver {
    char *base;
    size_t off = 0;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <typename T>
    T *take(size_t count) {
        off = round_up(off, 256);
        T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
        off += count * sizeof(T);
        return p;
    }
};

}  // namespace gptq
