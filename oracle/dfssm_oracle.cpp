// CPU oracle for the DF-SSM 1-bit scaffold + int8 LoRA linear, and for the int8
// embedding table / LM head (at the end of this file).
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously correct
// statement of what the layer computes. Only the tests, the smoke check and the
// benchmark's CPU-baseline leg may load it; the library never does. It shares
// no code, header, table or helper with the CUDA path.
//
// What the layer computes (per token t, output row o):
//
//   y[t,o] = s_x[t] * ( alpha[o] * acc[t,o]
//                       + s_A[o] * sum_k W_A[o,k] * (s_B[k] * h[t,k]) )
//   acc[t,o] = sum_j w[o,j] * q[t,j]        w = +-1 scaffold weight (int32 sum)
//   h[t,k]   = sum_j W_B[k,j] * q[t,j]      rank-16 LoRA down-projection (int32)
//   q, s_x   = per-token symmetric absmax int8 quantisation of x
//
// Sources: "Density Field State Space Models" (gist.science technical summary):
//   §2.B  frozen 1-bit scaffold, int8 LoRA W_A (d_out x r), W_B (r x d_in), r = 16,
//         on every in_proj and out_proj; int8 LoRA with per-channel/row scales;
//   §2.C  packed 1-bit scaffold weights expanded to int8 and multiplied by an
//         int8 x int8 -> int32 matmul (so activations are int8 as well);
//   §3    scaffold stored at 1 bit per weight (56 % of the 278 MB model).
// The pages leave open the bit order, the sign mapping, the per-row scale alpha,
// the quantiser and where s_x applies. This oracle takes these readings:
//   - bit = 1 -> +1, bit = 0 -> -1; row-major rows of d_in/8 bytes; column j of
//     a row is bit (j mod 8) of byte j/8 (least significant bit first);
//   - alpha is one fp32 scale per output row;
//   - q: amax = max_j |x_j| in fp32; amax == 0 gives q = 0 and s_x = 0; else
//     inv = 127/amax (fp32 division, round to nearest), q_j = clamp(rint(x_j*inv),
//     -127, 127) with rint = round half to even, s_x = amax/127 (fp32 division);
//   - s_x multiplies both terms; s_B * h is not re-quantised (kept in float).
// The dequantisation runs in float64 with every fp32 parameter widened exactly.
//
// Parity pins (tests/test_oracle_pins.py): brute-force dense f64 matmul of the
// unpacked +-1 matrix, closed-form constructed cases, the invariants all-ones
// row -> acc = sum(q), one bit flip -> acc changes by exactly +-2 q_j, zero LoRA
// -> scaffold term alone, quantiser ties / symmetry / power-of-two scaling, and
// hand-computed golden fixtures in tests/golden/.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---- bf16 <-> float ------------------------------------------------------------

// bf16 is the top 16 bits of an IEEE-754 binary32; widening is exact.
static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// Round a double to the nearest bf16 (8 significant bits), ties to even.
// Used only to state the expected bf16 output of the layer.
uint16_t dfssm_oracle_f64_to_bf16(double v) {
    if (std::isnan(v)) return 0x7FC0;
    if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
    if (std::isinf(v)) return v > 0 ? 0x7F80 : 0xFF80;
    int e = 0;
    double f = std::frexp(std::fabs(v), &e);      // |v| = f * 2^e, 0.5 <= f < 1
    double s;
    if (e - 1 < -126) {
        // below the normal range: bf16 subnormals have a fixed quantum of 2^-133
        s = std::nearbyint(std::ldexp(std::fabs(v), 133));
        double r = std::ldexp(s, -133);
        float rf = (float)r;
        uint32_t u; std::memcpy(&u, &rf, 4);
        u >>= 16;
        return (uint16_t)(u | (v < 0 ? 0x8000u : 0u));
    }
    s = std::nearbyint(std::ldexp(f, 8));         // significand in [128, 256]
    double r = std::ldexp(s, e - 8);
    if (r > 0x1.FEp127) return v > 0 ? 0x7F80 : 0xFF80;  // beyond the largest finite bf16
    float rf = (float)r;                          // exact: 8 significant bits
    uint32_t u;
    std::memcpy(&u, &rf, 4);
    u >>= 16;
    return (uint16_t)(u | (v < 0 ? 0x8000u : 0u));
}

void dfssm_oracle_f64_to_bf16_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = dfssm_oracle_f64_to_bf16(v[i]);
}

// ---- packed sign matrix ---------------------------------------------------------

// One weight: bit (j mod 8) of byte (o, j/8); 1 -> +1, 0 -> -1.
static int sign_at(const uint8_t* packed, int d_in, int o, int j) {
    const uint8_t byte = packed[(int64_t)o * (d_in / 8) + j / 8];
    return ((byte >> (j % 8)) & 1) ? +1 : -1;
}

// Unpack the d_out x d_in scaffold into +-1 int8 (row-major).
void dfssm_oracle_unpack_sign(const uint8_t* packed, int d_out, int d_in, int8_t* w) {
    for (int o = 0; o < d_out; ++o)
        for (int j = 0; j < d_in; ++j)
            w[(int64_t)o * d_in + j] = (int8_t)sign_at(packed, d_in, o, j);
}

// Pack a frozen scaffold: value >= 0 (including -0.0) -> +1 -> bit 1; value < 0 -> bit 0.
// Returns 0, or 1 if a NaN is met (then `packed` is left partly written).
int dfssm_oracle_pack_sign_f32(const float* src, int d_out, int d_in, uint8_t* packed) {
    for (int o = 0; o < d_out; ++o) {
        for (int b = 0; b < d_in / 8; ++b) {
            uint8_t byte = 0;
            for (int i = 0; i < 8; ++i) {
                float v = src[(int64_t)o * d_in + 8 * b + i];
                if (std::isnan(v)) return 1;
                if (!(v < 0.0f)) byte |= (uint8_t)(1u << i);
            }
            packed[(int64_t)o * (d_in / 8) + b] = byte;
        }
    }
    return 0;
}

int dfssm_oracle_pack_sign_i8(const int8_t* src, int d_out, int d_in, uint8_t* packed) {
    for (int o = 0; o < d_out; ++o) {
        for (int b = 0; b < d_in / 8; ++b) {
            uint8_t byte = 0;
            for (int i = 0; i < 8; ++i)
                if (src[(int64_t)o * d_in + 8 * b + i] >= 0) byte |= (uint8_t)(1u << i);
            packed[(int64_t)o * (d_in / 8) + b] = byte;
        }
    }
    return 0;
}

// ---- activation quantiser (fp32, exactly as stated) ------------------------------

static void quantize_token(const uint16_t* x, int d_in, int8_t* q, float* sx) {
    float amax = 0.0f;
    for (int j = 0; j < d_in; ++j) {
        float a = std::fabs(bf16_to_float(x[j]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        for (int j = 0; j < d_in; ++j) q[j] = 0;
        *sx = 0.0f;
        return;
    }
    volatile float inv = 127.0f / amax;            // one fp32 division, RN
    for (int j = 0; j < d_in; ++j) {
        volatile float v = bf16_to_float(x[j]) * inv;   // one fp32 product, RN
        float r = std::nearbyintf(v);                   // ties to even
        // amax below 127 / FLT_MAX makes inv = +inf: a zero entry gives 0 * inf = NaN, taken as 0
        // (x = 0 quantises to 0); a nonzero entry gives +-inf, clamped to +-127 below
        if (std::isnan(r)) r = 0.0f;
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[j] = (int8_t)r;
    }
    volatile float s = amax / 127.0f;
    *sx = s;
}

void dfssm_oracle_quantize(const uint16_t* x, int m, int d_in, int8_t* q, float* sx) {
    for (int t = 0; t < m; ++t)
        quantize_token(x + (int64_t)t * d_in, d_in, q + (int64_t)t * d_in, sx + t);
}

// ---- the linear -------------------------------------------------------------------

// y for one (t, o) from the int32 sums, in float64.
static double dequant(float sx, float alpha, float sa, const int8_t* wa_row, const float* sb,
                      const int32_t* h_t, int rank, int32_t acc) {
    double lora = 0.0;
    for (int k = 0; k < rank; ++k)
        lora += (double)wa_row[k] * ((double)sb[k] * (double)h_t[k]);
    return (double)sx * ((double)alpha * (double)acc + (double)sa * lora);
}

// Full layer for m tokens. Any of q_out, sx_out, acc_out, h_out may be NULL.
// threads <= 0 uses the OpenMP default; 1 runs single-threaded.
// The layer from the unpacked +-1 matrix w (d_out x d_in int8): everything after the unpack.
void dfssm_oracle_linear_unpacked(const uint16_t* x, int m, int d_in, int d_out, int rank,
                                  const int8_t* w, const float* alpha, const int8_t* wa,
                                  const float* sa, const int8_t* wb, const float* sb,
                                  int8_t* q_out, float* sx_out, int32_t* acc_out, int32_t* h_out,
                                  double* y, int threads);

void dfssm_oracle_linear(const uint16_t* x, int m, int d_in, int d_out, int rank,
                         const uint8_t* sign, const float* alpha, const int8_t* wa,
                         const float* sa, const int8_t* wb, const float* sb,
                         int8_t* q_out, float* sx_out, int32_t* acc_out, int32_t* h_out,
                         double* y, int threads) {
    std::vector<int8_t> w((size_t)d_out * d_in);
    dfssm_oracle_unpack_sign(sign, d_out, d_in, w.data());
    dfssm_oracle_linear_unpacked(x, m, d_in, d_out, rank, w.data(), alpha, wa, sa, wb, sb, q_out, sx_out, acc_out,
                                 h_out, y, threads);
}

void dfssm_oracle_linear_unpacked(const uint16_t* x, int m, int d_in, int d_out, int rank,
                                  const int8_t* w_pm1, const float* alpha, const int8_t* wa,
                                  const float* sa, const int8_t* wb, const float* sb,
                                  int8_t* q_out, float* sx_out, int32_t* acc_out, int32_t* h_out,
                                  double* y, int threads) {
    const int8_t* w = w_pm1;
    std::vector<int8_t> q((size_t)m * d_in);
    std::vector<float> sx((size_t)m);
    dfssm_oracle_quantize(x, m, d_in, q.data(), sx.data());

    std::vector<int32_t> h((size_t)m * rank);
    for (int t = 0; t < m; ++t)
        for (int k = 0; k < rank; ++k) {
            int32_t s = 0;
            for (int j = 0; j < d_in; ++j)
                s += (int32_t)wb[(int64_t)k * d_in + j] * (int32_t)q[(int64_t)t * d_in + j];
            h[(size_t)t * rank + k] = s;
        }

#ifdef _OPENMP
    int nt = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel for collapse(2) schedule(static) num_threads(nt)
#endif
    for (int t = 0; t < m; ++t) {
        for (int o = 0; o < d_out; ++o) {
            int32_t acc = 0;
            const int8_t* wr = w + (int64_t)o * d_in;
            const int8_t* qt = q.data() + (int64_t)t * d_in;
            for (int j = 0; j < d_in; ++j) acc += (int32_t)wr[j] * (int32_t)qt[j];
            if (acc_out) acc_out[(int64_t)t * d_out + o] = acc;
            y[(int64_t)t * d_out + o] = dequant(sx[t], alpha[o], sa[o], wa + (int64_t)o * rank, sb,
                                                h.data() + (size_t)t * rank, rank, acc);
        }
    }
    if (q_out) std::memcpy(q_out, q.data(), q.size());
    if (sx_out) std::memcpy(sx_out, sx.data(), sx.size() * sizeof(float));
    if (h_out) std::memcpy(h_out, h.data(), h.size() * sizeof(int32_t));
}

// Selected outputs only: y and acc at the n pairs (t_idx[i], o_idx[i]), computed one
// by one straight from the packed rows (for full-size workloads). Same arithmetic.
void dfssm_oracle_linear_sampled(const uint16_t* x, int m, int d_in, int d_out, int rank,
                                 const uint8_t* sign, const float* alpha, const int8_t* wa,
                                 const float* sa, const int8_t* wb, const float* sb,
                                 const int32_t* t_idx, const int32_t* o_idx, int64_t n,
                                 int32_t* acc_out, double* y) {
    (void)m; (void)d_out;
    std::vector<int8_t> q((size_t)d_in);
    std::vector<int32_t> h((size_t)rank);
    int cur_t = -1;
    float sx = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        int t = t_idx[i], o = o_idx[i];
        if (t != cur_t) {
            quantize_token(x + (int64_t)t * d_in, d_in, q.data(), &sx);
            for (int k = 0; k < rank; ++k) {
                int32_t s = 0;
                for (int j = 0; j < d_in; ++j) s += (int32_t)wb[(int64_t)k * d_in + j] * (int32_t)q[j];
                h[k] = s;
            }
            cur_t = t;
        }
        int32_t acc = 0;
        for (int j = 0; j < d_in; ++j) acc += sign_at(sign, d_in, o, j) * (int32_t)q[j];
        if (acc_out) acc_out[i] = acc;
        y[i] = dequant(sx, alpha[o], sa[o], wa + (int64_t)o * rank, sb, h.data(), rank, acc);
    }
}

// Bytes of one linear as stored: 1 bit per scaffold weight, int8 LoRA factors,
// fp32 alpha / s_A per output row and s_B per LoRA row.
void dfssm_oracle_weight_bytes(int d_in, int d_out, int rank, int64_t* sign_bytes,
                               int64_t* lora_bytes, int64_t* scale_bytes) {
    *sign_bytes = (int64_t)d_out * d_in / 8;
    *lora_bytes = (int64_t)d_out * rank + (int64_t)rank * d_in;
    *scale_bytes = 4 * ((int64_t)d_out * 2 + rank);
}

// ---- int8 embedding table and LM head ------------------------------------------------
// "Density Field State Space Models" (gist.science technical summary), §2.B: the embedding
// and the LM head are quantised to int8 with per-channel/row scales; §3: they are 37 % of
// the 278 MB model. One table E (vocab x d int8, row-major) with one fp32 scale per row
// serves both (Mamba ties the two). Readings taken here:
//   - a looked-up row is the fp32 product s_E[id] * E[id, j], rounded once (the exact
//     product in float64, then to fp32);
//   - the head reads the activations through the layer's own quantiser (q, s_x of the
//     final hidden state, as for every linear) and sums E[v, j] * q[t, j] in int32;
//     logits[t, v] = s_x[t] * s_E[v] * sum, in float64.

// Returns the number of ids outside [0, vocab); their rows are zeros.
int dfssm_oracle_embed(const int8_t* table, const float* scale, int vocab, int d, const int32_t* ids, int m,
                       float* out) {
    int bad = 0;
    for (int t = 0; t < m; ++t) {
        const int32_t id = ids[t];
        float* o = out + (int64_t)t * d;
        if (id < 0 || id >= vocab) {
            ++bad;
            for (int j = 0; j < d; ++j) o[j] = 0.0f;
            continue;
        }
        for (int j = 0; j < d; ++j)
            o[j] = (float)((double)scale[id] * (double)table[(int64_t)id * d + j]);   // exact, then one rounding
    }
    return bad;
}

// logits (float64, m x vocab) and, if acc_out is not NULL, the int32 sums.
void dfssm_oracle_lm_head(const int8_t* table, const float* scale, int vocab, int d, const uint16_t* h, int m,
                          int32_t* acc_out, double* logits, int threads) {
    std::vector<int8_t> q((size_t)m * d);
    std::vector<float> sx((size_t)m);
    dfssm_oracle_quantize(h, m, d, q.data(), sx.data());
#ifdef _OPENMP
    int nt = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel for collapse(2) schedule(static) num_threads(nt)
#endif
    for (int t = 0; t < m; ++t) {
        for (int v = 0; v < vocab; ++v) {
            int32_t acc = 0;
            const int8_t* er = table + (int64_t)v * d;
            const int8_t* qt = q.data() + (int64_t)t * d;
            for (int j = 0; j < d; ++j) acc += (int32_t)er[j] * (int32_t)qt[j];
            if (acc_out) acc_out[(int64_t)t * vocab + v] = acc;
            logits[(int64_t)t * vocab + v] = (double)sx[t] * (double)scale[v] * (double)acc;
        }
    }
}

// The same at the n pairs (t_idx[i], v_idx[i]) only (for full-size tables).
void dfssm_oracle_lm_head_sampled(const int8_t* table, const float* scale, int vocab, int d, const uint16_t* h,
                                  int m, const int32_t* t_idx, const int32_t* v_idx, int64_t n, int32_t* acc_out,
                                  double* logits) {
    (void)vocab; (void)m;
    std::vector<int8_t> q((size_t)d);
    float sx = 0.0f;
    int cur_t = -1;
    for (int64_t i = 0; i < n; ++i) {
        const int t = t_idx[i], v = v_idx[i];
        if (t != cur_t) {
            quantize_token(h + (int64_t)t * d, d, q.data(), &sx);
            cur_t = t;
        }
        int32_t acc = 0;
        for (int j = 0; j < d; ++j) acc += (int32_t)table[(int64_t)v * d + j] * (int32_t)q[j];
        if (acc_out) acc_out[i] = acc;
        logits[i] = (double)sx * (double)scale[v] * (double)acc;
    }
}

}  // extern "C"
