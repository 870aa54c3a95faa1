// Packing a frozen scaffold into sign bits.
//
// "Density Field State Space Models" (gist.science technical summary), §2.B:
// after training the scaffold weights are frozen at their rounded values;
// §2.C and §3: they are stored and streamed at 1 bit per weight. Mapping used
// here: value >= 0 (including -0.0) -> +1 -> bit 1, value < 0 -> bit 0; column j
// of a row is bit (j % 8) of byte j / 8.
//
// One thread produces 16 packed bytes (128 source values) and writes them with
// one 128-bit store; d_in % 128 == 0 keeps every row a whole number of those.
#include "dfssm_internal.cuh"

namespace dfssm {

template <typename T>
__device__ __forceinline__ uint32_t nonneg_bit(T v);

template <>
__device__ __forceinline__ uint32_t nonneg_bit<int8_t>(int8_t v) { return v >= 0 ? 1u : 0u; }

template <>
__device__ __forceinline__ uint32_t nonneg_bit<float>(float v) {
    // -0.0 counts as >= 0; the sign-bit test alone would send it to -1
    return (v < 0.0f) ? 0u : 1u;
}

template <typename T>
__global__ void __launch_bounds__(256) pack_sign_kernel(const T* __restrict__ src, int64_t n_chunks,
                                                        uint4* __restrict__ packed) {
    int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= n_chunks) return;
    const T* s = src + c * 128;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 32; ++b) word |= nonneg_bit<T>(s[q * 32 + b]) << b;
        w[q] = word;
    }
    packed[c] = make_uint4(w[0], w[1], w[2], w[3]);
}

cudaError_t launch_pack_sign(const void* src, int src_dtype, int d_out, int d_in, uint8_t* packed,
                             cudaStream_t s) {
    int64_t n_chunks = (int64_t)d_out * (d_in / 128);
    int64_t blocks = (n_chunks + 255) / 256;
    if (src_dtype == DFSSM_I8)
        pack_sign_kernel<int8_t><<<(unsigned)blocks, 256, 0, s>>>((const int8_t*)src, n_chunks, (uint4*)packed);
    else
        pack_sign_kernel<float><<<(unsigned)blocks, 256, 0, s>>>((const float*)src, n_chunks, (uint4*)packed);
    return cudaGetLastError();
}

}  // namespace dfssm
