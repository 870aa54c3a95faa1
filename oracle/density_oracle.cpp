// CPU oracle for the state density field: the compression cycle that the pages apply to the
// SSM state at chunk boundaries.
//
// TEST INFRASTRUCTURE ONLY (like dfssm_oracle.cpp, built into the same library): only the
// tests, the smoke check and the benchmark's CPU-baseline leg load it; it shares no code
// with the CUDA path.
//
// "Density Field State Space Models" (gist.science technical summary), §2.D, state density
// field representation: a K x K binary field is kept per state element, with K^2 about
// 4 d_state; the cycle is normalisation, sigma-delta injection (error feedback),
// binarisation, and a popcount readout that recovers continuous values, applied at chunk
// boundaries. The section says no more; the steps below take the plainest reading of it:
//
//   state element  one row S[h][p][0..d_state) of the SSM state (d_state values), so a
//                  field of K^2 ~ 4 d_state bits holds about four bits per value
//   normalisation  scale = max_n |s_n| over the row (kept in fp32); v_n = s_n / scale in
//                  [-1, 1], and the target density of ones u_n = (v_n + 1) / 2 in [0, 1]
//                  (a zero row takes v = 0)
//   cells          the K^2 cells in row-major order; value n owns cells
//                  [floor(n K^2 / d_state), floor((n + 1) K^2 / d_state))
//   sigma-delta    one first-order modulator over all cells of the row in order, its error
//                  carried from cell to cell and from one value's cells to the next:
//                  acc = u_n + e;  bit = (acc >= 1/2);  e = acc - bit
//   readout        the value of n is scale (2 popcount_n - len_n) / len_n
//
// The modulator runs in fp32 (v by one division, u = 0.5 v + 0.5, acc by one addition; e is
// then exact), so that a kernel doing the same fp32 steps takes the same bit decisions; the
// readout is in float64. Bits are packed LSB-first: cell c is bit c % 8 of byte c / 8 of the
// row's ceil(K^2 / 8) bytes.
#include <cmath>
#include <cstdint>
#include <cstring>

extern "C" {

// rows x d_state fp32 state in; per row the fp32 scale and the packed field out.
void dfssm_oracle_density_encode(int rows, int d_state, int K, const float* state, float* scale, uint8_t* bits) {
    const int cells = K * K;
    const int row_bytes = (cells + 7) / 8;
    for (int r = 0; r < rows; ++r) {
        const float* s = state + (int64_t)r * d_state;
        float amax = 0.0f;
        for (int n = 0; n < d_state; ++n) amax = std::fmax(amax, std::fabs(s[n]));
        scale[r] = amax;
        uint8_t* b = bits + (int64_t)r * row_bytes;
        std::memset(b, 0, row_bytes);
        float e = 0.0f;
        for (int n = 0; n < d_state; ++n) {
            const float v = amax == 0.0f ? 0.0f : s[n] / amax;
            const float u = 0.5f * v + 0.5f;
            const int c0 = (int)((int64_t)n * cells / d_state), c1 = (int)((int64_t)(n + 1) * cells / d_state);
            for (int c = c0; c < c1; ++c) {
                const float acc = u + e;
                const int bit = acc >= 0.5f ? 1 : 0;
                e = acc - (float)bit;
                if (bit) b[c >> 3] |= (uint8_t)(1u << (c & 7));
            }
        }
    }
}

// The popcount readout: rows x d_state float64 values from the scales and fields.
void dfssm_oracle_density_decode(int rows, int d_state, int K, const float* scale, const uint8_t* bits,
                                 double* state_out) {
    const int cells = K * K;
    const int row_bytes = (cells + 7) / 8;
    for (int r = 0; r < rows; ++r) {
        const uint8_t* b = bits + (int64_t)r * row_bytes;
        for (int n = 0; n < d_state; ++n) {
            const int c0 = (int)((int64_t)n * cells / d_state), c1 = (int)((int64_t)(n + 1) * cells / d_state);
            int pop = 0;
            for (int c = c0; c < c1; ++c) pop += (b[c >> 3] >> (c & 7)) & 1;
            const int len = c1 - c0;
            state_out[(int64_t)r * d_state + n] = (double)scale[r] * (double)(2 * pop - len) / (double)len;
        }
    }
}

}  // extern "C"
