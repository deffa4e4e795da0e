// Index checks of the GPTQ_DEBUG_BOUNDS build (record and skip).
//
// Built with -DGPTQ_DEBUG_BOUNDS (python -m post_weight_quantization_solve_b200.build
// --debug-bounds, which writes libgptq_dbg.so), the kernels check their tile origins,
// TMA box coordinates and computed output offsets before using them. A failed check
// never faults or traps: it counts the failure in this translation unit's device
// record (the first failure's site and index kept), stores GPTQ_ERR_BOUNDS in the
// caller's status word, and the access is skipped (a skipped TMA load also raises the
// kernel's abort flag, so that its bounded waits end at once). gptq_bounds_report reads
// and clears the records of every translation unit. In the normal build every check
// is the constant true and compiles away.
#pragma once

#include "common.cuh"

namespace gptq {

// Check sites (the numbers gptq_bounds_report returns).
enum BoundsSite : int {
    BS_SELFTEST = 1,      // gptq_bounds_selftest: a check that always fails, no access
    BS_TC32_TILE = 2,     // tf32x3 GEMM: unit tile or inner range outside its item
    BS_TC32_TMA = 3,      // tf32x3 GEMM: TMA x coordinate not on a 16-byte boundary
    BS_TC32_C = 4,        // tf32x3 GEMM: epilogue element outside C's extent
    BS_TC32_PAIR = 5,     // tf32x3 GEMM: pair element outside the pair arrays' extent
    BS_GRAM_TMA = 6,      // Gram: token / feature box origin outside X or unaligned
    BS_GRAM_RED = 7,      // Gram: reduction box origin outside H or unaligned
    BS_SWEEP_TMA = 8,     // tensor-core sweep: box origin outside W / U / P1 or unaligned
    BS_SWEEP_OUT = 9,     // tensor-core sweep: code, error or weight offset outside its buffer
    BS_UPDATE_TMA = 10,   // lazy update: operand box origin unaligned or outside the product
    BS_UPDATE_C = 11,     // lazy update: output element outside W's extent
    BS_DIAG = 12,         // diagonal factor: block outside H
    BS_SITES = 13
};

struct BoundsRecord {
    int count;            // failed checks since the last reset
    int site;             // first failure's site (0: none)
    long long index;      // first failure's index (offset or coordinate)
};

#ifdef GPTQ_DEBUG_BOUNDS

// Host side: every translation unit registers a reader of its own record.
typedef bool (*BoundsReader)(BoundsRecord *out, bool reset);
void bounds_register(BoundsReader fn);

namespace {
__device__ BoundsRecord g_bounds_rec;     // this translation unit's record

__device__ __noinline__ bool bounds_fail(int32_t *status, int site, long long index) {
    if (atomicAdd(&g_bounds_rec.count, 1) == 0) {
        g_bounds_rec.site = site;
        g_bounds_rec.index = index;
    }
    set_status(status, GPTQ_ERR_BOUNDS);
    return false;
}

bool bounds_read_tu(BoundsRecord *out, bool reset) {
    if (cudaMemcpyFromSymbol(out, g_bounds_rec, sizeof(BoundsRecord)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (reset) {
        const BoundsRecord zero{0, 0, 0};
        if (cudaMemcpyToSymbol(g_bounds_rec, &zero, sizeof(BoundsRecord)) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
    }
    return true;
}

struct BoundsRegistrar {
    BoundsRegistrar() { bounds_register(&bounds_read_tu); }
};
const BoundsRegistrar g_bounds_registrar;
}  // namespace

#define GQ_IN_BOUNDS(status, cond, site, index) \
    ((cond) ? true : ::gptq::bounds_fail((status), (site), (long long)(index)))

#else

#define GQ_IN_BOUNDS(status, cond, site, index) true

#endif

}  // namespace gptq
