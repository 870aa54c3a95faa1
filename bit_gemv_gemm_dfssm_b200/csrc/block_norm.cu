// The frame of a Mamba-2 block around the layer: the residual add and the RMS norm in
// front of each in_proj (and in front of the LM head), one kernel for m tokens.
//
// "Density Field State Space Models" (gist.science technical summary), §2.B and §3: the
// model is Mamba-2 1.3B (48 layers, d_model 2048) with its in_proj and out_proj replaced
// by the 1-bit scaffold + int8 LoRA linear and its tied embedding / LM head in int8. The
// block frame is Mamba-2's: an fp32 residual stream r; r += the previous block's out_proj
// output; the next in_proj reads out = r / sqrt(mean(r^2) + eps) * w.
//
// One CTA of 256 threads per token. Thread i owns the 8 columns [8 i, 8 i + 8) of each
// 2048-column pass: 16-byte loads of r, of the delta and of w; r_new = r + delta (one fp32
// addition) is stored back and kept in shared memory; the thread sums r_new^2 over its
// columns in order (fmaf), the warp by a shuffle tree, the warps in order. The factor is
// 1 / sqrt(sum / d + eps) with correctly rounded square root and division, and out =
// (r_new * factor) * w, rounded once to bf16 (nearest even) or kept in fp32. Every order is
// fixed, so results repeat bit for bit. The kernel reads and writes a few KB per token: it
// is bound by its launch and one pass of latency, not by bandwidth.
#include <cmath>
#include <cstdint>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"

namespace dfssm {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxD = 8192;

struct NormArgs {
    const float* w;
    const float* rin;
    const void* delta;
    float* rout;
    void* out;
    int d;
    float eps;
    int delta_bf16;   // 1: delta is bf16, 0: fp32 (ignored when delta is NULL)
    int out_bf16;     // 1: out is bf16, 0: fp32
};

__device__ __forceinline__ void load8(const float* p, float v[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8(float* p, const float v[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

__global__ void __launch_bounds__(kThreads) add_rmsnorm_kernel(const NormArgs a) {
    extern __shared__ float r_s[];           // r_new of this token (d floats)
    __shared__ float red[kThreads / 32];
    __shared__ float factor_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t base = (int64_t)blockIdx.x * a.d;
    float ss = 0.0f;
    for (int c = 8 * tid; c < a.d; c += 8 * kThreads) {
        float v[8];
        load8(a.rin + base + c, v);
        if (a.delta) {
            if (a.delta_bf16) {
                const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.delta) + base + c);
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[2 * k] = __fadd_rn(v[2 * k], bf16_lo(w4[k]));
                    v[2 * k + 1] = __fadd_rn(v[2 * k + 1], bf16_hi(w4[k]));
                }
            } else {
                float dv[8];
                load8(static_cast<const float*>(a.delta) + base + c, dv);
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = __fadd_rn(v[k], dv[k]);
            }
        }
        store8(a.rout + base + c, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            r_s[c + k] = v[k];
            ss = __fmaf_rn(v[k], v[k], ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        float tot = red[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) tot = __fadd_rn(tot, red[w]);
        factor_s = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)a.d), a.eps)));
    }
    __syncthreads();
    const float f = factor_s;
    for (int c = 8 * tid; c < a.d; c += 8 * kThreads) {
        float w[8], o[8];
        load8(a.w + c, w);
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = __fmul_rn(__fmul_rn(r_s[c + k], f), w[k]);
        if (a.out_bf16) {
            uint32_t p[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                p[k] = (uint32_t)f32_to_bf16_bits(o[2 * k]) | ((uint32_t)f32_to_bf16_bits(o[2 * k + 1]) << 16);
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + base + c) = make_uint4(p[0], p[1], p[2], p[3]);
        } else {
            store8(static_cast<float*>(a.out) + base + c, o);
        }
    }
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace dfssm

using namespace dfssm;

extern "C" dfssm_status dfssm_add_rmsnorm(const float* norm_w, int32_t d, float eps, const float* resid_in,
                                          const void* delta, int32_t delta_dtype, int32_t m, float* resid_out,
                                          void* out, int32_t out_dtype, void* stream) {
    if (d < 8 || d > kMaxD || d % 8 != 0 || m < 1 || m > 65536) return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (!norm_w || !resid_in || !resid_out || !out || !al16(norm_w) || !al16(resid_in) || !al16(resid_out) ||
        !al16(out) || !al16(delta))
        return DFSSM_ERR_INVALID_ARG;
    if (!std::isfinite(eps) || eps < 0.0f) return DFSSM_ERR_INVALID_ARG;
    if ((delta && delta_dtype != DFSSM_BF16 && delta_dtype != DFSSM_F32) ||
        (out_dtype != DFSSM_BF16 && out_dtype != DFSSM_F32))
        return DFSSM_ERR_INVALID_ARG;
    NormArgs a{norm_w, resid_in, delta, resid_out, out, d, eps, delta_dtype == DFSSM_BF16 ? 1 : 0,
               out_dtype == DFSSM_BF16 ? 1 : 0};
    add_rmsnorm_kernel<<<m, kThreads, (size_t)d * sizeof(float), static_cast<cudaStream_t>(stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? DFSSM_OK : DFSSM_ERR_CUDA;
}
