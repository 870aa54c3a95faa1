// CPU oracle for one decode step of the Mamba-2 state operations between a
// layer's in_proj and out_proj: the conv shift register and the SSM recurrence.
//
// TEST INFRASTRUCTURE ONLY (like dfssm_oracle.cpp, built into the same library):
// only the tests, the smoke check and the benchmark's CPU-baseline leg load it;
// it shares no code with the CUDA path.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C,
// state operations: custom kernels handle the state shift register (the causal
// convolution) and the SSM recurrence (a warp-level reduction). The pages name
// these steps only; what they compute is the Mamba-2 decode step, restated here
// from that published design for one token of one layer (all arithmetic in
// float64 from the exact bf16 / fp32 inputs):
//
//   in_proj output  [ z (d_inner) | xBC (conv_dim) | dt_raw (nheads) ],
//                   conv_dim = d_inner + 2 d_state (one group of B and C)
//   shift register  window[c] = (state[c][1], ..., state[c][d_conv-1], xBC[c]);
//                   the new state is that window (stored back in bf16: exact)
//   convolution     xc[c] = silu(conv_b[c] + sum_k conv_w[c][k] window[c][k])
//   split           x = xc[0, d_inner), B = xc[d_inner, +d_state), C = the rest
//   step size       dt_h = softplus(dt_raw_h + dt_bias_h), A_h = -exp(a_log_h),
//                   dA_h = exp(dt_h A_h)
//   recurrence      S[h][p][n] = S[h][p][n] dA_h + dt_h x[h P + p] B[n]   (P = headdim)
//   readout         y[h P + p] = sum_n S[h][p][n] C[n] + D_h x[h P + p]
//   gate and norm   g = y silu(z);  out = g / sqrt(mean(g^2) + eps) * norm_w
//
// silu(v) = v / (1 + e^-v); softplus(v) = log(1 + e^v), and v itself above 20.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

double bf16_to_f64(uint16_t b) {
    const uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return (double)f;
}

double silu(double v) { return v / (1.0 + std::exp(-v)); }
double softplus(double v) { return v > 20.0 ? v : std::log1p(std::exp(v)); }

}  // namespace

extern "C" {

// m tokens of one layer. conv_state (m x conv_dim x d_conv bf16 bits) is updated in place;
// ssm_in (m x nheads x headdim x d_state fp32) is read and ssm_out (same shape, float64)
// written. out: m x d_inner (float64). The optional outputs (NULL to skip) give the
// intermediates the tests' error bounds need: xc (m x conv_dim), dt and dA (m x nheads),
// y before the gate (m x d_inner), and the norm factor 1/sqrt(mean(g^2) + eps) (m).
void dfssm_oracle_ssm_step(int d_inner, int headdim, int d_state, int d_conv, double eps, int m,
                           const uint16_t* zxbcdt, uint16_t* conv_state, const float* ssm_in, double* ssm_out,
                           const float* conv_w, const float* conv_b, const float* dt_bias, const float* a_log,
                           const float* d_skip, const float* norm_w, double* out, double* xc_out, double* dt_out,
                           double* da_out, double* y_out, double* r_out) {
    const int nheads = d_inner / headdim;
    const int conv_dim = d_inner + 2 * d_state;
    const int row = 2 * d_inner + 2 * d_state + nheads;
    std::vector<double> xc(conv_dim), y(d_inner), g(d_inner);
    for (int t = 0; t < m; ++t) {
        const uint16_t* zr = zxbcdt + (int64_t)t * row;
        // shift register and convolution
        for (int c = 0; c < conv_dim; ++c) {
            uint16_t* st = conv_state + ((int64_t)t * conv_dim + c) * d_conv;
            for (int k = 0; k + 1 < d_conv; ++k) st[k] = st[k + 1];
            st[d_conv - 1] = zr[d_inner + c];
            double pre = (double)conv_b[c];
            for (int k = 0; k < d_conv; ++k) pre += (double)conv_w[(int64_t)c * d_conv + k] * bf16_to_f64(st[k]);
            xc[c] = silu(pre);
            if (xc_out) xc_out[(int64_t)t * conv_dim + c] = xc[c];
        }
        const double* x = xc.data();
        const double* B = xc.data() + d_inner;
        const double* C = xc.data() + d_inner + d_state;
        // recurrence and readout, head by head
        for (int h = 0; h < nheads; ++h) {
            const double dt = softplus(bf16_to_f64(zr[d_inner + conv_dim + h]) + (double)dt_bias[h]);
            const double A = -std::exp((double)a_log[h]);
            const double dA = std::exp(dt * A);
            if (dt_out) dt_out[(int64_t)t * nheads + h] = dt;
            if (da_out) da_out[(int64_t)t * nheads + h] = dA;
            for (int p = 0; p < headdim; ++p) {
                const int ch = h * headdim + p;
                const int64_t base = (((int64_t)t * nheads + h) * headdim + p) * d_state;
                double acc = 0.0;
                for (int n = 0; n < d_state; ++n) {
                    const double s = (double)ssm_in[base + n] * dA + dt * x[ch] * B[n];
                    ssm_out[base + n] = s;
                    acc += s * C[n];
                }
                y[ch] = acc + (double)d_skip[h] * x[ch];
                if (y_out) y_out[(int64_t)t * d_inner + ch] = y[ch];
            }
        }
        // gate, then RMS normalisation over the whole d_inner (one group)
        double ss = 0.0;
        for (int c = 0; c < d_inner; ++c) {
            g[c] = y[c] * silu(bf16_to_f64(zr[c]));
            ss += g[c] * g[c];
        }
        const double r = 1.0 / std::sqrt(ss / (double)d_inner + eps);
        if (r_out) r_out[t] = r;
        for (int c = 0; c < d_inner; ++c) out[(int64_t)t * d_inner + c] = g[c] * r * (double)norm_w[c];
    }
}

}  // extern "C"
