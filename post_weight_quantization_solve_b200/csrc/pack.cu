// gptq_pack_codes / gptq_unpack_codes: codes as low-bit words and back.
//
// [GPTQ blog] "落在格点上与真正存成低位权重是两步": codes on the grid become storage
// only once they are packed into wider integer containers. Layout (the pages fix
// none): per output channel, code k occupies bits [b k, b k + b) of a little-endian
// bit stream, and stream bit t is bit t mod 32 of 32-bit word t / 32. Thirty-two
// codes therefore fill exactly b words, so one thread takes 32 codes of a row and
// writes (or reads) its b words: no word is shared between threads, nothing is
// read twice, and a warp moves 1 KB of codes and 128 b bytes of words, both
// contiguous. Pure data movement, bound by HBM.
#include "common.cuh"

namespace gptq {

template <int B>
__global__ void __launch_bounds__(256) k_pack(const uint8_t *__restrict__ codes, int N, int K,
                                              int64_t ldc, uint32_t *__restrict__ words,
                                              int64_t ldw, int vec) {
    const int per_row = (K + 31) / 32;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)N * per_row) return;
    const int64_t n = gid / per_row;
    const int t = (int)(gid % per_row);
    const uint8_t *src = codes + n * ldc + 32 * t;
    const int nk = min(32, K - 32 * t);
    uint32_t c4[8];   // the 32 codes, four to a register (code i in byte i % 4 of c4[i / 4])
    if (vec && nk == 32) {
        const uint4 a = *reinterpret_cast<const uint4 *>(src);
        const uint4 b = *reinterpret_cast<const uint4 *>(src + 16);
        c4[0] = a.x; c4[1] = a.y; c4[2] = a.z; c4[3] = a.w;
        c4[4] = b.x; c4[5] = b.y; c4[6] = b.z; c4[7] = b.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) c4[i] = 0u;
        for (int i = 0; i < nk; ++i) c4[i >> 2] |= (uint32_t)src[i] << (8 * (i & 3));
    }
    uint32_t w[B];
#pragma unroll
    for (int j = 0; j < B; ++j) w[j] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const uint32_t v = (c4[i >> 2] >> (8 * (i & 3))) & ((1u << B) - 1u);
        const int bit = i * B;
        w[bit >> 5] |= v << (bit & 31);
        if ((bit & 31) + B > 32) w[(bit >> 5) + 1] |= v >> (32 - (bit & 31));
    }
    const int nw = (int)(((int64_t)K * B + 31) / 32);
    uint32_t *dst = words + n * ldw + (int64_t)B * t;
#pragma unroll
    for (int j = 0; j < B; ++j)
        if (B * t + j < nw) dst[j] = w[j];
}

template <int B>
__global__ void __launch_bounds__(256) k_unpack(const uint32_t *__restrict__ words, int N, int K,
                                                int64_t ldw, uint8_t *__restrict__ codes,
                                                int64_t ldc, int vec) {
    const int per_row = (K + 31) / 32;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)N * per_row) return;
    const int64_t n = gid / per_row;
    const int t = (int)(gid % per_row);
    const int nk = min(32, K - 32 * t);
    const int nw = (int)(((int64_t)K * B + 31) / 32);
    const uint32_t *src = words + n * ldw + (int64_t)B * t;
    uint32_t w[B];
#pragma unroll
    for (int j = 0; j < B; ++j) w[j] = (B * t + j < nw) ? src[j] : 0u;
    uint32_t c4[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) c4[i] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int bit = i * B;
        uint32_t v = w[bit >> 5] >> (bit & 31);
        if ((bit & 31) + B > 32) v |= w[(bit >> 5) + 1] << (32 - (bit & 31));
        c4[i >> 2] |= (v & ((1u << B) - 1u)) << (8 * (i & 3));
    }
    uint8_t *dst = codes + n * ldc + 32 * t;
    if (vec && nk == 32) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(c4[0], c4[1], c4[2], c4[3]);
        *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(c4[4], c4[5], c4[6], c4[7]);
    } else {
        for (int i = 0; i < nk; ++i) dst[i] = (uint8_t)(c4[i >> 2] >> (8 * (i & 3)));
    }
}

gptq_status pack_codes(const uint8_t *codes, int N, int K, int64_t ldc, int bits, uint32_t *words,
                       int64_t ldw, cudaStream_t st) {
    if (N == 0) return GPTQ_OK;
    const int64_t threads = (int64_t)N * ((K + 31) / 32);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    const int vec = (ldc % 16 == 0 && aligned(codes, 16)) ? 1 : 0;
    switch (bits) {
        case 2: k_pack<2><<<blocks, 256, 0, st>>>(codes, N, K, ldc, words, ldw, vec); break;
        case 3: k_pack<3><<<blocks, 256, 0, st>>>(codes, N, K, ldc, words, ldw, vec); break;
        case 4: k_pack<4><<<blocks, 256, 0, st>>>(codes, N, K, ldc, words, ldw, vec); break;
        default: k_pack<8><<<blocks, 256, 0, st>>>(codes, N, K, ldc, words, ldw, vec); break;
    }
    return launch_status();
}

gptq_status unpack_codes(const uint32_t *words, int N, int K, int64_t ldw, int bits,
                         uint8_t *codes, int64_t ldc, cudaStream_t st) {
    if (N == 0) return GPTQ_OK;
    const int64_t threads = (int64_t)N * ((K + 31) / 32);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    const int vec = (ldc % 16 == 0 && aligned(codes, 16)) ? 1 : 0;
    switch (bits) {
        case 2: k_unpack<2><<<blocks, 256, 0, st>>>(words, N, K, ldw, codes, ldc, vec); break;
        case 3: k_unpack<3><<<blocks, 256, 0, st>>>(words, N, K, ldw, codes, ldc, vec); break;
        case 4: k_unpack<4><<<blocks, 256, 0, st>>>(words, N, K, ldw, codes, ldc, vec); break;
        default: k_unpack<8><<<blocks, 256, 0, st>>>(words, N, K, ldw, codes, ldc, vec); break;
    }
    return launch_status();
}

}  // namespace gptq
