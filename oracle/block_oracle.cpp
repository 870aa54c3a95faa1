// CPU oracle for the frame of a Mamba-2 block around the layer: the residual add and the
// RMS norm in front of each in_proj (and in front of the LM head).
//
// TEST INFRASTRUCTURE ONLY (like dfssm_oracle.cpp, built into the same library): only the
// tests, the smoke check and the benchmark's CPU-baseline leg load it; it shares no code
// with the CUDA path.
//
// "Density Field State Space Models" (gist.science technical summary), §2.B and §3: the
// model is Mamba-2 1.3B (48 layers, d_model 2048) with its in_proj and out_proj replaced by
// the 1-bit scaffold + int8 LoRA linear, and the tied embedding / LM head in int8. The pages
// say nothing more about the block; the frame is Mamba-2's published one, restated here for
// m tokens of width d:
//
//   residual stream  r_new = r + delta          delta: the previous block's out_proj output
//                                               (absent in front of the first block)
//   RMS norm         out = r_new / sqrt(mean(r_new^2) + eps) * w
//
// The residual stream is kept in fp32 (Mamba-2 keeps it in fp32), so r_new is the one fp32
// rounding of r + delta, as the next block sees it; the norm is taken in float64 from that
// stored value.
#include <cmath>
#include <cstdint>
#include <cstring>

namespace {

float bf16_to_f32(uint16_t b) {
    const uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

}  // namespace

extern "C" {

// resid_in, resid_out: m x d fp32 (resid_out may equal resid_in); delta: m x d, bf16 bits when
// delta_bf16 != 0, else fp32, or NULL; w: d fp32; out: m x d float64; r_out: m float64 (the
// factor 1/sqrt(mean(r_new^2) + eps), may be NULL).
void dfssm_oracle_add_rmsnorm(int d, double eps, int m, const float* resid_in, const void* delta, int delta_bf16,
                              const float* w, float* resid_out, double* out, double* r_out) {
    for (int t = 0; t < m; ++t) {
        const float* ri = resid_in + (int64_t)t * d;
        float* ro = resid_out + (int64_t)t * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) {
            float v = ri[j];
            if (delta) {
                const int64_t k = (int64_t)t * d + j;
                const float dv = delta_bf16 ? bf16_to_f32(static_cast<const uint16_t*>(delta)[k])
                                            : static_cast<const float*>(delta)[k];
                v = v + dv;   // one IEEE single-precision addition
            }
            ro[j] = v;
            ss += (double)v * (double)v;
        }
        const double r = 1.0 / std::sqrt(ss / (double)d + eps);
        if (r_out) r_out[t] = r;
        for (int j = 0; j < d; ++j) out[(int64_t)t * d + j] = (double)ro[j] * r * (double)w[j];
    }
}

}  // extern "C"
