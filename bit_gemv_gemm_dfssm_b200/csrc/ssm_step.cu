// One decode step of the Mamba-2 state operations between a layer's in_proj and
// out_proj, for n independent layers in one call: the conv shift register and the
// SSM recurrence.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C,
// state operations: custom kernels handle the state shift register (the causal
// convolution) and the SSM recurrence (a warp-level reduction). The arithmetic is
// the Mamba-2 decode step (one group of B and C, 64-channel heads, d_state 128,
// 4 taps):
//
//   ssm_conv_kernel   per channel c: window = (state[c][1..3], xBC[c]) is written
//                     back as the new shift register (bf16, exact), and
//                     xc[c] = silu(conv_b[c] + sum_k conv_w[c][k] window[k]) (fp32 fmaf
//                     chain in k order); per head h: dt = softplus(dt_raw + dt_bias)
//                     (v itself above 20), dA = exp(-exp(a_log) dt)
//   ssm_scan_kernel   per (head, token, layer), 256 threads: thread (p, q) owns state row
//                     p of the head and columns [32 q, 32 q + 32): it streams them with
//                     16-byte loads and stores, S = fmaf(S, dA, dt x_p B[n]), sums
//                     S C[n] for its columns, and the four threads of a row add their
//                     sums with warp shuffles; y = sum + D x_p, g = y silu(z_p), and
//                     the head's sum of g^2 (warp shuffles, then in warp order)
//   ssm_norm_kernel   per token: r = 1 / sqrt(mean(g^2) + eps) from the heads' sums in
//                     head order, out = g r norm_w (bf16 round-to-nearest-even or fp32)
//
// The state stream (2 MB of fp32 per layer and token, read and written) bounds the
// step; the conv and norm kernels move a few tens of KB per layer. Every order of
// summation is fixed, so results repeat bit for bit.
#include <cstdint>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"

namespace dfssm {

namespace {

constexpr int kHeadDim = 64;
constexpr int kDState = 128;
constexpr int kDConv = 4;
constexpr int kConvThreads = 256;
constexpr int kScanThreads = 256;          // 64 rows x 4 column quarters
constexpr int kNormThreads = 256;
constexpr int kMaxDInner = 16384;

struct SsmShape {
    int d_inner, nheads, conv_dim, row, m, n_layers;
    float eps;
    int out_dtype;
};

// workspace pieces (byte offsets, 256-aligned): error word, xc, (dt, dA), g, per-head sum of g^2
struct SsmWs {
    uint32_t* err;
    float* xc;
    float2* dta;
    float* g;
    float* ssq;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

__host__ __device__ inline size_t ws_layout(const SsmShape& s, size_t* off_xc, size_t* off_dta, size_t* off_g,
                                            size_t* off_ssq) {
    const size_t lt = (size_t)s.n_layers * s.m;
    size_t o = 256;                                          // error word
    *off_xc = o;
    o = align256(o + lt * s.conv_dim * sizeof(float));
    *off_dta = o;
    o = align256(o + lt * s.nheads * sizeof(float2));
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

__global__ void __launch_bounds__(kConvThreads) ssm_conv_kernel(const dfssm_ssm_layer* __restrict__ layers,
                                                                const SsmShape s, SsmWs ws) {
    const int l = blockIdx.z, t = blockIdx.y;
    const dfssm_ssm_layer L = layers[l];
    if (!layer_ok(L)) {
        if (blockIdx.x == 0 && t == 0 && threadIdx.x == 0) atomicOr(ws.err, DFSSM_DEVERR_ENTRY_PTR);
        return;
    }
    const uint16_t* zr = reinterpret_cast<const uint16_t*>(L.zxbcdt) + (int64_t)t * s.row;
    const int64_t lt = (int64_t)l * s.m + t;
    const int c = blockIdx.x * kConvThreads + threadIdx.x;
    if (c < s.conv_dim) {
        uint2* stp = reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(L.conv_state) +
                                              ((int64_t)t * s.conv_dim + c) * kDConv);
        const uint2 old = *stp;
        const uint16_t nv = zr[s.d_inner + c];
        // window = (state[1], state[2], state[3], new)
        const uint16_t win[kDConv] = {(uint16_t)(old.x >> 16), (uint16_t)(old.y & 0xFFFFu), (uint16_t)(old.y >> 16),
                                      nv};
        const float4 w = *reinterpret_cast<const float4*>(L.conv_w + (int64_t)c * kDConv);
        const float wk[kDConv] = {w.x, w.y, w.z, w.w};
        float pre = L.conv_b[c];
#pragma unroll
        for (int k = 0; k < kDConv; ++k) pre = __fmaf_rn(wk[k], bf16f(win[k]), pre);
        ws.xc[lt * s.conv_dim + c] = silu_f(pre);
        *stp = make_uint2((uint32_t)win[0] | ((uint32_t)win[1] << 16), (uint32_t)win[2] | ((uint32_t)win[3] << 16));
    }
    if (blockIdx.x == 0 && threadIdx.x < s.nheads) {
        const int h = threadIdx.x;
        const float v = __fadd_rn(bf16f(zr[s.d_inner + s.conv_dim + h]), L.dt_bias[h]);
        const float dt = v > 20.0f ? v : log1pf(expf(v));
        const float A = -expf(L.a_log[h]);
        ws.dta[lt * s.nheads + h] = make_float2(dt, expf(__fmul_rn(dt, A)));
    }
}

__global__ void __launch_bounds__(kScanThreads) ssm_scan_kernel(const dfssm_ssm_layer* __restrict__ layers,
                                                                const SsmShape s, SsmWs ws) {
    __shared__ float red[kScanThreads / 32];
    const int h = blockIdx.x, t = blockIdx.y, l = blockIdx.z;
    const dfssm_ssm_layer L = layers[l];
    if (!layer_ok(L)) return;                       // reported by the conv kernel
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p = tid >> 2, q = tid & 3;
    const int64_t lt = (int64_t)l * s.m + t;
    const float* xc = ws.xc + lt * s.conv_dim;
    const int ch = h * kHeadDim + p;
    const float2 dta = ws.dta[lt * s.nheads + h];
    const float dtx = __fmul_rn(dta.x, xc[ch]);
    const float4* Bv = reinterpret_cast<const float4*>(xc + s.d_inner + 32 * q);
    const float4* Cv = reinterpret_cast<const float4*>(xc + s.d_inner + kDState + 32 * q);
    float4* S = reinterpret_cast<float4*>(L.ssm_state + (((int64_t)t * s.nheads + h) * kHeadDim + p) * kDState + 32 * q);
    float4 sv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sv[i] = S[i];
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 b = Bv[i], c = Cv[i];
        float4 v = sv[i];
        v.x = __fmaf_rn(v.x, dta.y, __fmul_rn(dtx, b.x));
        v.y = __fmaf_rn(v.y, dta.y, __fmul_rn(dtx, b.y));
        v.z = __fmaf_rn(v.z, dta.y, __fmul_rn(dtx, b.z));
        v.w = __fmaf_rn(v.w, dta.y, __fmul_rn(dtx, b.w));
        acc = __fmaf_rn(v.x, c.x, acc);
        acc = __fmaf_rn(v.y, c.y, acc);
        acc = __fmaf_rn(v.z, c.z, acc);
        acc = __fmaf_rn(v.w, c.w, acc);
        sv[i] = v;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) S[i] = sv[i];
    // the four column quarters of row p are lanes 4 (p % 8) .. + 3 of this warp
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 1));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 2));
    const float y = __fmaf_rn(L.d_skip[h], xc[ch], acc);
    const uint16_t* zr = reinterpret_cast<const uint16_t*>(L.zxbcdt) + (int64_t)t * s.row;
    const float g = __fmul_rn(y, silu_f(bf16f(zr[ch])));
    if (q == 0) ws.g[lt * s.d_inner + ch] = g;
    float g2 = q == 0 ? __fmul_rn(g, g) : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) g2 = __fadd_rn(g2, __shfl_xor_sync(0xffffffffu, g2, o));
    if (lane == 0) red[warp] = g2;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < kScanThreads / 32; ++w) sum = __fadd_rn(sum, red[w]);
        ws.ssq[lt * s.nheads + h] = sum;
    }
}

__global__ void __launch_bounds__(kNormThreads) ssm_norm_kernel(const dfssm_ssm_layer* __restrict__ layers,
                                                                const SsmShape s, SsmWs ws) {
    __shared__ float r_s;
    const int t = blockIdx.y, l = blockIdx.z;
    const dfssm_ssm_layer L = layers[l];
    if (!layer_ok(L)) return;
    const int64_t lt = (int64_t)l * s.m + t;
    if (threadIdx.x == 0) {
        float sum = 0.0f;
        for (int h = 0; h < s.nheads; ++h) sum = __fadd_rn(sum, ws.ssq[lt * s.nheads + h]);
        r_s = __frsqrt_rn(__fadd_rn(__fdiv_rn(sum, (float)s.d_inner), s.eps));
    }
    __syncthreads();
    const float r = r_s;
    for (int c = blockIdx.x * kNormThreads + threadIdx.x; c < s.d_inner; c += gridDim.x * kNormThreads) {
        const float o = __fmul_rn(__fmul_rn(ws.g[lt * s.d_inner + c], r), L.norm_w[c]);
        const int64_t idx = (int64_t)t * s.d_inner + c;
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
    size_t a, b, c, d;
    *bytes = ws_layout(s, &a, &b, &c, &d);
    return DFSSM_OK;
}

extern "C" dfssm_status dfssm_ssm_step(const dfssm_ssm_dims* dims, const dfssm_ssm_layer* layers_dev,
                                       int32_t n_layers, int32_t m, void* workspace, size_t workspace_bytes,
                                       void* stream) {
    SsmShape s;
    const dfssm_status st = shape_of(dims, n_layers, m, &s);
    if (st != DFSSM_OK) return st;
    if (!layers_dev || (reinterpret_cast<uintptr_t>(layers_dev) & 7u)) return DFSSM_ERR_INVALID_ARG;
    size_t o_xc, o_dta, o_g, o_ssq;
    const size_t need = ws_layout(s, &o_xc, &o_dta, &o_g, &o_ssq);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return DFSSM_ERR_INVALID_ARG;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    SsmWs ws{reinterpret_cast<uint32_t*>(w), reinterpret_cast<float*>(w + o_xc), reinterpret_cast<float2*>(w + o_dta),
             reinterpret_cast<float*>(w + o_g), reinterpret_cast<float*>(w + o_ssq)};
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    ssm_conv_kernel<<<dim3((s.conv_dim + kConvThreads - 1) / kConvThreads, m, n_layers), kConvThreads, 0, cs>>>(
        layers_dev, s, ws);
    ssm_scan_kernel<<<dim3(s.nheads, m, n_layers), kScanThreads, 0, cs>>>(layers_dev, s, ws);
    ssm_norm_kernel<<<dim3((s.d_inner + 4 * kNormThreads - 1) / (4 * kNormThreads), m, n_layers), kNormThreads, 0,
                      cs>>>(layers_dev, s, ws);
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
