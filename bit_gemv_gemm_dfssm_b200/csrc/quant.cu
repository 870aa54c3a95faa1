// Per-token activation quantisation and the fused LoRA down-projection.
//
// The scaffold matmul runs on int8 activations ("Density Field State Space
// Models", gist.science technical summary, §2.C: packed bits expanded to int8
// for an int8 x int8 -> int32 matmul), and the rank-16 int8 LoRA
// (§2.B: W_B in R^{r x d_in}, r = 16, int8 with per-row scales) reads the
// same int8 activations. For each token t of each linear this kernel computes
//   amax   = max_j |x[t,j]|                       (fp32, exact)
//   q[t,j] = clamp(rint(x[t,j] * (127/amax)), +-127), s_x = amax/127 (IEEE fp32,
//            round-to-nearest; amax == 0 gives q = 0, s_x = 0)
//   sumq   = sum_j q[t,j]                          (int32)
//   h[t,k] = sum_j W_B[k,j] q[t,j]                 (int32, dp4a)
//   u[t,k] = s_B[k] * h[t,k]                       (fp32)
// and stores q in the permuted int8 layout the scaffold kernels read, plus
// s_x, sumq and u. One block owns one linear and a group of tokens; W_B is
// staged in shared memory once per block.
#include "dfssm_internal.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxChunks = kMaxDIn / 8 / kThreads;   // 8-column chunks per thread (<= 4)

struct QuantSmem {
    float red_f[kWarps];
    int red_i[kWarps];
    int red_h[kWarps][kRank];
};

__global__ void __launch_bounds__(kThreads) quant_kernel(
    const dfssm_stack_entry* __restrict__ entries, const dfssm_stack_entry single,
    const DevDesc* __restrict__ descs, int m, int tok_per_block,
    int8_t* __restrict__ q_ws, TokStats* __restrict__ st_ws, uint32_t* __restrict__ err) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // let the dependent scaffold kernel start streaming weights right away;
    // it waits for this grid's results before reading them
    ptx::pdl_launch_dependents();
    const int lin = blockIdx.y;
    const dfssm_stack_entry& e = entry_at(entries, single, lin);
    const DevDesc d = descs[lin];
    if (entries && e.desc_index != lin) {
        if (threadIdx.x == 0) atomicOr(err, DFSSM_DEVERR_ENTRY_DESC);
        return;
    }
    if (!entry_ptrs_ok(e)) {
        if (threadIdx.x == 0) atomicOr(err, DFSSM_DEVERR_ENTRY_PTR);
        return;
    }
    const int d_in = d.d_in;
    const int n_chunk = d_in / 8;                 // 8-column chunks per row
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    int8_t* wb_s = reinterpret_cast<int8_t*>(smem_raw);             // 16 x d_in
    int8_t* qrow = wb_s + kRank * d_in;                              // d_in
    QuantSmem& red = *reinterpret_cast<QuantSmem*>(qrow + d_in);

    // stage W_B
    {
        const uint4* src = reinterpret_cast<const uint4*>(e.w.wb);
        uint4* dst = reinterpret_cast<uint4*>(wb_s);
        for (int i = tid; i < kRank * d_in / 16; i += kThreads) dst[i] = src[i];
    }
    float sb[kRank];
#pragma unroll
    for (int k = 0; k < kRank; ++k) sb[k] = e.w.sb[k];
    __syncthreads();

    const int t0 = blockIdx.x * tok_per_block;
    const int t1 = min(m, t0 + tok_per_block);
    const uint16_t* xbase = reinterpret_cast<const uint16_t*>(e.x);

    for (int t = t0; t < t1; ++t) {
        // ---- load x and find amax
        float xv[kMaxChunks][8];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < kMaxChunks; ++c) {
            int ch = tid + c * kThreads;
            if (ch < n_chunk) {
                uint4 raw = *reinterpret_cast<const uint4*>(xbase + (int64_t)t * d_in + ch * 8);
                uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xv[c][2 * i] = bf16_bits_to_float(wv[i] & 0xFFFFu);
                    xv[c][2 * i + 1] = bf16_bits_to_float(wv[i] >> 16);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(xv[c][i]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) red.red_f[warp] = amax;
        __syncthreads();
        amax = red.red_f[0];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) amax = fmaxf(amax, red.red_f[w]);
        // NaN compares false in fmaxf chains, so check finiteness of the inputs' max explicitly
        if (!isfinite(amax) && tid == 0) atomicOr(err, DFSSM_DEVERR_NONFINITE);

        const bool zero = (amax == 0.0f);
        const float inv = zero ? 0.0f : __fdiv_rn(127.0f, amax);
        const float sx = zero ? 0.0f : __fdiv_rn(amax, 127.0f);

        // ---- quantise, sum, LoRA down-projection
        int sumq = 0;
        int hp[kRank];
#pragma unroll
        for (int k = 0; k < kRank; ++k) hp[k] = 0;
#pragma unroll
        for (int c = 0; c < kMaxChunks; ++c) {
            int ch = tid + c * kThreads;
            if (ch < n_chunk) {
                uint32_t qw[2] = {0u, 0u};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    int qi = zero ? 0 : __float2int_rn(__fmul_rn(xv[c][i], inv));
                    qi = max(-127, min(127, qi));
                    sumq += qi;
                    qw[i >> 2] |= (uint32_t)(qi & 0xFF) << (8 * (i & 3));
                }
                *reinterpret_cast<uint2*>(qrow + ch * 8) = make_uint2(qw[0], qw[1]);
                if (e.dbg.q)
                    *reinterpret_cast<uint2*>(e.dbg.q + (int64_t)t * d_in + ch * 8) = make_uint2(qw[0], qw[1]);
#pragma unroll
                for (int k = 0; k < kRank; ++k) {
                    uint2 wbk = *reinterpret_cast<const uint2*>(wb_s + k * d_in + ch * 8);
                    hp[k] = __dp4a((int)qw[0], (int)wbk.x, hp[k]);
                    hp[k] = __dp4a((int)qw[1], (int)wbk.y, hp[k]);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sumq += __shfl_xor_sync(0xffffffffu, sumq, o);
#pragma unroll
        for (int k = 0; k < kRank; ++k) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) hp[k] += __shfl_xor_sync(0xffffffffu, hp[k], o);
        }
        if (lane == 0) {
            red.red_i[warp] = sumq;
#pragma unroll
            for (int k = 0; k < kRank; ++k) red.red_h[warp][k] = hp[k];
        }
        __syncthreads();   // qrow complete, partial sums visible

        // ---- per-token scalars
        TokStats* st = st_ws + d.st_off + t;
        if (tid < kRank) {
            int h = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) h += red.red_h[w][tid];
            st->u[tid] = __fmul_rn(sb[tid], (float)h);
            if (e.dbg.h) e.dbg.h[(int64_t)t * kRank + tid] = h;
        }
        if (tid == kRank) {
            int s = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) s += red.red_i[w];
            st->sx = sx;
            st->sumq = s;
            if (e.dbg.sx) e.dbg.sx[t] = sx;
        }

        // ---- permuted int8 row: position 32g + 4p + i <- column 32g + 8i + p
        int8_t* qdst = q_ws + d.q_off + (int64_t)t * d_in;
        for (int s16 = tid; s16 < d_in / 16; s16 += kThreads) {
            const int g = s16 >> 1, half = s16 & 1;
            uint32_t outw[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {           // output word r: p = 4*half + r, i = 0..3
                const int p = 4 * half + r;
                uint32_t wv = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    wv |= (uint32_t)(uint8_t)qrow[32 * g + 8 * i + p] << (8 * i);
                outw[r] = wv;
            }
            *reinterpret_cast<uint4*>(qdst + 16 * s16) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
        __syncthreads();   // qrow / red reused by the next token
    }
}

}  // namespace

cudaError_t launch_quant(const LaunchCtx& c) {
    int tpb = c.m >= 256 ? 32 : (c.m >= 64 ? 8 : (c.m >= 16 ? 2 : 1));
    dim3 grid((c.m + tpb - 1) / tpb, c.n);
    size_t smem = (size_t)(kRank + 1) * c.max_d_in + sizeof(QuantSmem);
    quant_kernel<<<grid, kThreads, smem, c.stream>>>(c.entries, c.single, c.desc, c.m, tpb,
                                                     c.q_ws, c.st_ws, c.err);
    return cudaGetLastError();
}

void set_quant_attr(int max_dyn_smem) {
    cudaFuncSetAttribute(quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn_smem);
}

}  // namespace dfssm
