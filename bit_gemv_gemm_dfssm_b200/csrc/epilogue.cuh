// Dequantisation epilogue shared by the decode and prefill kernels, so both give
// bit-identical outputs. Per (token t, output row o):
//
//   dot = sum_{k even} W_A[o,k] u[t,k]  +  sum_{k odd} W_A[o,k] u[t,k]
//         (each half an fmaf chain in ascending k, then one fp32 add)
//   y   = s_x[t] * fmaf(alpha[o], acc, s_A[o] * dot)
//
// with u = s_B * h in fp32 ("Density Field State Space Models", gist.science
// technical summary, §2.B: the int8 LoRA correction W_A (W_B x) with per-row
// scales). Conversions avoid the XU pipe: an int32 below 2^22 in magnitude is
// turned into fp32 exactly with the 1.5 * 2^23 bias trick, and fp32 -> bf16
// rounds to nearest-even with integer operations.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace dfssm {

// exact for |v| < 2^22 (acc is bounded by 127 * 8192 < 2^20)
__device__ __forceinline__ float small_int_to_float(int v) {
    return __fsub_rn(__int_as_float(v + 0x4B400000), 12582912.0f);
}

// ---- the activation quantiser (IEEE fp32, round to nearest) --------------------------
// inv = 127 / amax and s_x = amax / 127 as correctly rounded divisions; q = clamp(rint(x * inv))
__device__ __forceinline__ int quant1(float x, float inv, bool zero) {
    const int q = zero ? 0 : __float2int_rn(__fmul_rn(x, inv));
    return max(-127, min(127, q));
}
__device__ __forceinline__ float quant_inv(float amax) { return amax == 0.0f ? 0.0f : __fdiv_rn(127.0f, amax); }
__device__ __forceinline__ float quant_sx(float amax) { return amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f); }
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 4 bf16 (8 bytes) -> 4 int8 packed little-endian
__device__ __forceinline__ uint32_t quant4(uint2 raw, float inv, bool zero, int& sum) {
    const int q0 = quant1(bf16_lo(raw.x), inv, zero);
    const int q1 = quant1(bf16_hi(raw.x), inv, zero);
    const int q2 = quant1(bf16_lo(raw.y), inv, zero);
    const int q3 = quant1(bf16_hi(raw.y), inv, zero);
    sum += q0 + q1 + q2 + q3;
    return (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) | ((uint32_t)(q2 & 0xFF) << 16) |
           ((uint32_t)(q3 & 0xFF) << 24);
}

// running max of |x| over 8 bf16 values, as fp32 bit patterns: for |x| the unsigned order is
// the numeric order, and a NaN (bits above Inf) wins, so a non-finite row is still seen
__device__ __forceinline__ uint32_t absmax8_bits(uint4 v, uint32_t m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = max(m, (w[i] << 16) & 0x7FFFFFFFu);
        m = max(m, w[i] & 0x7FFF0000u);
    }
    return m;
}

// round-to-nearest-even fp32 -> bf16 bits (NaN kept quiet)
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    const uint32_t u = __float_as_uint(f);
    const uint32_t rounded = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
    const uint32_t quiet_nan = (u >> 16) | 0x40u;
    return (uint16_t)(((u & 0x7FFFFFFFu) > 0x7F800000u) ? quiet_nan : rounded);   // a select, not a branch
}

// W_A row as 16 floats (exact: int8)
struct WaRow {
    float w[16];
};

__device__ __forceinline__ WaRow wa_row_from_int4(int4 v) {
    WaRow r;
    const uint32_t q[4] = {(uint32_t)v.x, (uint32_t)v.y, (uint32_t)v.z, (uint32_t)v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int b = 0; b < 4; ++b) r.w[4 * i + b] = small_int_to_float((int)(int8_t)(q[i] >> (8 * b)));
    }
    return r;
}

// two fp32 FMAs in one instruction (sm_100): d.x = fma(a.x, b.x, c.x), d.y = fma(a.y, b.y, c.y),
// each rounded exactly like a scalar fmaf
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// two fp32 products / sums in one instruction each, rounded like the scalar __fmul_rn / __fadd_rn
// (use fadd2 only where no product feeds it: a product followed by an add may be fused)
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// (lo, hi) -> bf16x2, round to nearest even (low half = lo)
__device__ __forceinline__ uint32_t bf16x2_of(float2 v) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// u: 16 floats, 16-byte aligned (shared or global)
__device__ __forceinline__ float lora_dot(const WaRow& wa, const float* __restrict__ u) {
    const float4 u0 = *reinterpret_cast<const float4*>(u);
    const float4 u1 = *reinterpret_cast<const float4*>(u + 4);
    const float4 u2 = *reinterpret_cast<const float4*>(u + 8);
    const float4 u3 = *reinterpret_cast<const float4*>(u + 12);
    const float uu[16] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w,
                          u2.x, u2.y, u2.z, u2.w, u3.x, u3.y, u3.z, u3.w};
    // .x: chain over even k, .y: chain over odd k
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < 16; k += 2)
        acc = ffma2(make_float2(wa.w[k], wa.w[k + 1]), make_float2(uu[k], uu[k + 1]), acc);
    return __fadd_rn(acc.x, acc.y);
}

// two int8 (low byte = lower k) -> two bf16 (exact: |v| <= 128), low half = lower k
__device__ __forceinline__ uint32_t int8_pair_to_bf16x2(uint32_t w) {
    const uint32_t b0 = __float_as_uint(small_int_to_float((int)(int8_t)(w & 0xFFu))) >> 16;
    const uint32_t b1 = __float_as_uint(small_int_to_float((int)(int8_t)((w >> 8) & 0xFFu))) & 0xFFFF0000u;
    return b0 | b1;
}

// (a, b) as bf16 pairs hi = bf16(x) and lo = bf16(x - hi), low half = a: hi + lo is x to
// within 2^-18 |x| (x - hi is exact in fp32)
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    const float ha = __uint_as_float(hi << 16), hb = __uint_as_float(hi & 0xFFFF0000u);
    const __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(a, ha), __fsub_rn(b, hb));
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ float dequant(float sx, float alpha, float sa, int acc, float dot) {
    return __fmul_rn(sx, __fmaf_rn(alpha, small_int_to_float(acc), __fmul_rn(sa, dot)));
}

}  // namespace dfssm
