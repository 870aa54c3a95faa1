// One decode step of the Mamba-2 state operations between a layer's in_proj and
// out_proj, for n independent layers in one call: the conv shift register and the
// SSM recurrence.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C,
// state operations: custom kernels handle the state shift register (the causal
// convolution) and the SSM recurrence (a warp-level reduction). The arithmetic is
// the Mamba-2 decode step (one group of B and C, 64-channel heads, d_state 128,
// 4 taps). Two kernels:
//
//   ssm_step_kernel, one CTA of 8 warps per (head, token, layer):
//   1. the head's 64 x channels and the 256 B and C channels of the convolution:
//      window = (state[c][1..3], xBC[c]), xc[c] = silu(conv_b[c] + sum_k conv_w[c][k]
//      window[k]) (fp32 fmaf chain in k order); the window is written back as the new
//      shift register of the head's own x channels (bf16, exact); dt = softplus(dt_raw +
//      dt_bias) (v itself above 20), dA = exp(-exp(a_log) dt);
//   2. the recurrence: lane i owns columns [4 i, 4 i + 4) of the head's state rows, warp
//      w rows w, w + 8, ..., so one warp instruction loads or stores a whole 512-byte row;
//      S = fmaf(S, dA, dt x_p B[n]), and y of the row is the warp-level reduction of the
//      lanes' sums of S C[n] (shuffle tree); y += D x_p, g = y silu(z_p), and the head's
//      sum of g^2 (per warp over its rows, then in warp order);
//   ssm_norm_kernel, 1024 channels per CTA, after every head has read the B and C
//   registers: the first CTA of a (token, layer) shifts them, and each applies the RMS
//   norm to its channels: r = 1 / sqrt(mean(g^2) + eps) from
//   the heads' sums (lane i adds heads i, i + 32, ..., then a shuffle tree),
//   out = g r norm_w (bf16 round-to-nearest-even or fp32).
// (One kernel with a last-CTA ticket for the norm measured slower: the fence before the
// ticket holds every CTA until its 32 KB of state stores are visible.)
//
// The state stream (2 MB of fp32 per layer and token, read and written) bounds the
// step. Every order of summation is fixed, so results repeat bit for bit.
#include <cstdint>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"

namespace dfssm {

namespace {

constexpr int kHeadDim = 64;
constexpr int kDState = 128;
constexpr int kDConv = 4;
constexpr int kThreads = 256;              // 8 warps, 8 state rows each
constexpr int kMaxDInner = 16384;
constexpr int kNormCols = 1024;            // channels per CTA of the norm kernel

struct SsmShape {
    int d_inner, nheads, conv_dim, row, m, n_layers;
    float eps;
    int out_dtype;
};

// workspace pieces (byte offsets, 256-aligned): error word, g, per-head sum of g^2
struct SsmWs {
    uint32_t* err;
    float* g;
    float* ssq;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

__host__ __device__ inline size_t ws_layout(const SsmShape& s, size_t* off_g, size_t* off_ssq) {
    const size_t lt = (size_t)s.n_layers * s.m;
    size_t o = 256;                                          // error word
    *off_g = o;
    o = align256(o + lt * s.d_inner * sizeof(float));
    *off_ssq = o;
    o = align256(o + lt * s.nheads * sizeof(float));
    return o;
}

__device__ __forceinline__ bool layer_ok(const dfssm_ssm_layer& L) {
    return L.zxbcdt != nullptr && ptr_ok(L.conv_state) && ptr_ok(L.ssm_state) && ptr_ok(L.conv_w) &&
           ptr_ok(L.conv_b) && ptr_ok(L.dt_bias) && ptr_ok(L.a_log) && ptr_ok(L.d_skip) && ptr_ok(L.norm_w) &&
           ptr_ok(L.out) && (reinterpret_cast<uintptr_t>(L.zxbcdt) & 1u) == 0;
}

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ float silu_f(float v) { return __fdiv_rn(v, __fadd_rn(1.0f, expf(-v))); }

// The shift register of channel c of token t: its window (old state[1..3], the new input) as
// packed bf16, and the convolution output silu(conv_b + sum_k conv_w window[k]).
struct ConvOut {
    float xc;
    uint2 window;
};
__device__ __forceinline__ ConvOut conv_channel(const dfssm_ssm_layer& L, const SsmShape& s, const uint16_t* zr,
                                                int t, int c) {
    const uint2 old = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(L.conv_state) +
                                                      ((int64_t)t * s.conv_dim + c) * kDConv);
    const uint16_t win[kDConv] = {(uint16_t)(old.x >> 16), (uint16_t)(old.y & 0xFFFFu), (uint16_t)(old.y >> 16),
                                  zr[s.d_inner + c]};
    const float4 w = *reinterpret_cast<const float4*>(L.conv_w + (int64_t)c * kDConv);
    const float wk[kDConv] = {w.x, w.y, w.z, w.w};
    float pre = L.conv_b[c];
#pragma unroll
    for (int k = 0; k < kDConv; ++k) pre = __fmaf_rn(wk[k], bf16f(win[k]), pre);
    return ConvOut{silu_f(pre), make_uint2((uint32_t)win[0] | ((uint32_t)win[1] << 16),
                                           (uint32_t)win[2] | ((uint32_t)win[3] << 16))};
}

__device__ __forceinline__ uint2* state_slot(const dfssm_ssm_layer& L, const SsmShape& s, int t, int c) {
    return reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(L.conv_state) + ((int64_t)t * s.conv_dim + c) * kDConv);
}

__global__ void __launch_bounds__(kThreads, 4) ssm_step_kernel(const dfssm_ssm_layer* __restrict__ layers,
                                                            const SsmShape s, SsmWs ws) {
    constexpr int kWarps = kThreads / 32;
    constexpr int kRows = kHeadDim / kWarps;        // state rows per warp
    __shared__ __align__(16) float xs[kHeadDim];
    __shared__ __align__(16) float bc[2 * kDState];  // B then C
    __shared__ float red[kWarps];
    __shared__ float2 dta_s;
    const int h = blockIdx.x, t = blockIdx.y, l = blockIdx.z;
    const dfssm_ssm_layer L = layers[l];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (!layer_ok(L)) {
        if (h == 0 && t == 0 && tid == 0) atomicOr(ws.err, DFSSM_DEVERR_ENTRY_PTR);
        return;
    }
    const uint16_t* zr = reinterpret_cast<const uint16_t*>(L.zxbcdt) + (int64_t)t * s.row;
    const int64_t lt = (int64_t)l * s.m + t;
    // the head's state rows warp + kWarps r (r < kRows), loaded first: their latency overlaps the
    // convolution below
    float4* S = reinterpret_cast<float4*>(L.ssm_state + ((int64_t)t * s.nheads + h) * kHeadDim * kDState) + lane;
    float4 sv[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) sv[r] = S[(warp + kWarps * r) * (kDState / 4)];

    // ---- 1. convolution of the B and C channels (read only here) and of the head's x channels
    {
        bc[tid] = conv_channel(L, s, zr, t, s.d_inner + tid).xc;
        if (tid < kHeadDim) {
            const int c = h * kHeadDim + tid;
            const ConvOut co = conv_channel(L, s, zr, t, c);
            xs[tid] = co.xc;
            *state_slot(L, s, t, c) = co.window;     // only this CTA reads the head's x registers
        }
        if (tid == kThreads - 1) {
            const float v = __fadd_rn(bf16f(zr[s.d_inner + s.conv_dim + h]), L.dt_bias[h]);
            const float dt = v > 20.0f ? v : log1pf(expf(v));
            const float A = -expf(L.a_log[h]);
            dta_s = make_float2(dt, expf(__fmul_rn(dt, A)));
        }
    }
    __syncthreads();

    // ---- 2. the recurrence and the readout
    const float2 dta = dta_s;
    const float4 b = reinterpret_cast<const float4*>(bc)[lane];
    const float4 c = reinterpret_cast<const float4*>(bc + kDState)[lane];
    float g2 = 0.0f;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int p = warp + kWarps * r, ch = h * kHeadDim + p;
        const float xp = xs[p];
        const float dtx = __fmul_rn(dta.x, xp);
        float4 v = sv[r];
        v.x = __fmaf_rn(v.x, dta.y, __fmul_rn(dtx, b.x));
        v.y = __fmaf_rn(v.y, dta.y, __fmul_rn(dtx, b.y));
        v.z = __fmaf_rn(v.z, dta.y, __fmul_rn(dtx, b.z));
        v.w = __fmaf_rn(v.w, dta.y, __fmul_rn(dtx, b.w));
        S[p * (kDState / 4)] = v;
        float acc = __fmaf_rn(v.x, c.x, __fmaf_rn(v.y, c.y, __fmaf_rn(v.z, c.z, __fmul_rn(v.w, c.w))));
        // y of row p: the warp-level reduction over the 32 lanes' column groups
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
        const float y = __fmaf_rn(L.d_skip[h], xp, acc);
        const float g = __fmul_rn(y, silu_f(bf16f(zr[ch])));
        if (lane == 0) ws.g[lt * s.d_inner + ch] = g;
        g2 = __fmaf_rn(g, g, g2);                   // every lane holds the same g
    }
    if (lane == 0) red[warp] = g2;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum = __fadd_rn(sum, red[w]);
        ws.ssq[lt * s.nheads + h] = sum;
    }
}

__global__ void __launch_bounds__(kThreads) ssm_norm_kernel(const dfssm_ssm_layer* __restrict__ layers,
                                                            const SsmShape s, SsmWs ws) {
    __shared__ float r_s;
    const int t = blockIdx.y, l = blockIdx.z, tid = threadIdx.x;
    const dfssm_ssm_layer L = layers[l];
    if (!layer_ok(L)) return;                        // reported by the step kernel
    const uint16_t* zr = reinterpret_cast<const uint16_t*>(L.zxbcdt) + (int64_t)t * s.row;
    const int64_t lt = (int64_t)l * s.m + t;
    if (blockIdx.x == 0) {
        const int cch = s.d_inner + tid;             // every head has read these registers
        *state_slot(L, s, t, cch) = conv_channel(L, s, zr, t, cch).window;
    }
    if (tid < 32) {
        float sum = 0.0f;
        for (int hh = tid; hh < s.nheads; hh += 32) sum = __fadd_rn(sum, ws.ssq[lt * s.nheads + hh]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
        if (tid == 0) r_s = __frsqrt_rn(__fadd_rn(__fdiv_rn(sum, (float)s.d_inner), s.eps));
    }
    __syncthreads();
    const float r = r_s;
    // this CTA's kNormCols channels, kNormCols / kThreads per thread, loads first
    constexpr int kPer = kNormCols / kThreads;
    const int c0 = blockIdx.x * kNormCols + tid;
    float gv[kPer], wv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int cc = c0 + i * kThreads;
        gv[i] = cc < s.d_inner ? ws.g[lt * s.d_inner + cc] : 0.0f;
        wv[i] = cc < s.d_inner ? L.norm_w[cc] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int cc = c0 + i * kThreads;
        if (cc >= s.d_inner) break;
        const float o = __fmul_rn(__fmul_rn(gv[i], r), wv[i]);
        const int64_t idx = (int64_t)t * s.d_inner + cc;
        if (s.out_dtype == DFSSM_BF16) reinterpret_cast<uint16_t*>(L.out)[idx] = f32_to_bf16_bits(o);
        else reinterpret_cast<float*>(L.out)[idx] = o;
    }
}

dfssm_status shape_of(const dfssm_ssm_dims* d, int32_t n_layers, int32_t m, SsmShape* s) {
    if (!d) return DFSSM_ERR_INVALID_ARG;
    if (d->headdim != kHeadDim || d->d_state != kDState || d->d_conv != kDConv) return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (d->d_inner < kHeadDim || d->d_inner > kMaxDInner || d->d_inner % kHeadDim != 0)
        return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (!(d->eps >= 0.0f) || d->eps > 1.0f) return DFSSM_ERR_INVALID_ARG;
    if (d->out_dtype != DFSSM_BF16 && d->out_dtype != DFSSM_F32) return DFSSM_ERR_INVALID_ARG;
    if (n_layers < 1 || n_layers > 65535 || m < 1 || m > 65535) return DFSSM_ERR_INVALID_ARG;
    s->d_inner = d->d_inner;
    s->nheads = d->d_inner / kHeadDim;
    s->conv_dim = d->d_inner + 2 * kDState;
    s->row = 2 * d->d_inner + 2 * kDState + s->nheads;
    s->m = m;
    s->n_layers = n_layers;
    s->eps = d->eps;
    s->out_dtype = d->out_dtype;
    return DFSSM_OK;
}

}  // namespace

}  // namespace dfssm

using namespace dfssm;

extern "C" dfssm_status dfssm_ssm_workspace_bytes(const dfssm_ssm_dims* dims, int32_t n_layers, int32_t m,
                                                  size_t* bytes) {
    SsmShape s;
    const dfssm_status st = shape_of(dims, n_layers, m, &s);
    if (st != DFSSM_OK) return st;
    if (!bytes) return DFSSM_ERR_INVALID_ARG;
    size_t a, b;
    *bytes = ws_layout(s, &a, &b);
    return DFSSM_OK;
}

extern "C" dfssm_status dfssm_ssm_step(const dfssm_ssm_dims* dims, const dfssm_ssm_layer* layers_dev,
                                       int32_t n_layers, int32_t m, void* workspace, size_t workspace_bytes,
                                       void* stream) {
    SsmShape s;
    const dfssm_status st = shape_of(dims, n_layers, m, &s);
    if (st != DFSSM_OK) return st;
    if (!layers_dev || (reinterpret_cast<uintptr_t>(layers_dev) & 7u)) return DFSSM_ERR_INVALID_ARG;
    size_t o_g, o_ssq;
    const size_t need = ws_layout(s, &o_g, &o_ssq);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return DFSSM_ERR_INVALID_ARG;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    SsmWs ws{reinterpret_cast<uint32_t*>(w), reinterpret_cast<float*>(w + o_g), reinterpret_cast<float*>(w + o_ssq)};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    ssm_step_kernel<<<dim3(s.nheads, m, n_layers), kThreads, 0, cs>>>(layers_dev, s, ws);
    ssm_norm_kernel<<<dim3((s.d_inner + kNormCols - 1) / kNormCols, m, n_layers), kThreads, 0, cs>>>(layers_dev, s,
                                                                                                        ws);
    return cudaGetLastError() == cudaSuccess ? DFSSM_OK : DFSSM_ERR_CUDA;
}

extern "C" dfssm_status dfssm_ssm_read_error(void* workspace, uint32_t* bits, void* stream) {
    if (!workspace || !bits || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DFSSM_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(bits, workspace, 4, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess || cudaMemsetAsync(workspace, 0, 4, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess)
        return DFSSM_ERR_CUDA;
    return *bits ? DFSSM_ERR_DEVICE_CHECK : DFSSM_OK;
}
