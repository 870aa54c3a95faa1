// The int8 embedding table and LM head with one fp32 scale per row.
//
// "Density Field State Space Models" (gist.science technical summary), §2.B: the
// embedding and the LM head are quantised to int8 with per-channel/row scales;
// §3: they are 37 % of the 278 MB model, so a decode step streams them like the
// scaffold. One table E (vocab x d int8, row-major) with one fp32 scale per row
// serves both.
//
//  * embed_kernel: out[t, j] = s[id_t] * E[id_t, j], one fp32 product (exact
//    operands, one rounding), then bf16 round-to-nearest-even if asked. An id
//    outside [0, vocab) gives a row of zeros and sets DFSSM_DEVERR_TOKEN_ID.
//  * lm_head_kernel (1 <= m <= 16 tokens): logits[t, v] = s_x[t] * (s[v] * acc)
//    with acc = sum_j E[v, j] q[t, j] in int32, q and s_x from the layer's
//    per-token quantiser (epilogue.cuh, the same fp32 arithmetic as the linears).
//    Persistent CTAs; each quantises h into shared memory once (h is at most
//    16 x 8192 bf16, read from L2), then every warp takes rows in turn: the
//    lanes stream a row with 16-byte loads that skip L1 (the table is read once),
//    multiply by the shared q with dp4a, and the warp sums with redux.sync. The
//    kernel is bound by the table's HBM stream (about 103 MB for Mamba-2 1.3B).
#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kEmbedThreads = 256;
constexpr int kHeadThreads = 512;
constexpr int kHeadWarps = kHeadThreads / 32;
constexpr int kHeadMaxTok = 16;
constexpr int kRowsPerIter = 2;       // rows a warp has in flight
constexpr int kPieces = 4;            // 16-byte pieces per lane and row in flight (2 KB rows: all of them)

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// ---------------------------------------------------------------- embedding rows
// Block (t, piece): 8 columns per thread.
__global__ void __launch_bounds__(kEmbedThreads) embed_kernel(const int8_t* __restrict__ table,
                                                              const float* __restrict__ scale, int vocab, int d,
                                                              const int32_t* __restrict__ ids, void* out,
                                                              int out_dtype, uint32_t* err) {
    const int t = blockIdx.y;
    const int id = ids[t];
    const int j8 = blockIdx.x * kEmbedThreads + threadIdx.x;     // 8-column chunk
    if (8 * j8 >= d) return;
    const bool ok = id >= 0 && id < vocab;
    if (!ok && err && j8 == 0) atomicOr(err, DFSSM_DEVERR_TOKEN_ID);
    float v[8];
    if (ok) {
        const uint2 e = *reinterpret_cast<const uint2*>(table + (int64_t)id * d + 8 * j8);
        const float s = scale[id];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = i < 4 ? e.x : e.y;
            v[i] = __fmul_rn(s, small_int_to_float((int)(int8_t)(w >> (8 * (i & 3)))));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
    const int64_t o = (int64_t)t * d + 8 * j8;
    if (out_dtype == DFSSM_BF16) {
        uint4 pk;
        pk.x = bf16x2_of(make_float2(v[0], v[1]));
        pk.y = bf16x2_of(make_float2(v[2], v[3]));
        pk.z = bf16x2_of(make_float2(v[4], v[5]));
        pk.w = bf16x2_of(make_float2(v[6], v[7]));
        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + o) = pk;
    } else {
        float4* f = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o);
        f[0] = make_float4(v[0], v[1], v[2], v[3]);
        f[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// ---------------------------------------------------------------- LM head
struct HeadShared {
    float sx[kHeadMaxTok];
    uint32_t amax[kHeadMaxTok];
};

template <int MT>   // tokens rounded up: 1, 4 or 16 (loop bounds known at compile time)
__global__ void __launch_bounds__(kHeadThreads, 1) lm_head_kernel(const int8_t* __restrict__ table,
                                                                  const float* __restrict__ scale, int vocab, int d,
                                                                  const uint16_t* __restrict__ h, int m,
                                                                  void* logits, int out_dtype, int32_t* acc_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    HeadShared& hs = *reinterpret_cast<HeadShared*>(smem);
    int8_t* q = reinterpret_cast<int8_t*>(smem + ((sizeof(HeadShared) + 127) & ~(size_t)127));   // [m][d]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- the tokens' int8 activations (same arithmetic as the linears' quantiser)
    for (int t = warp; t < m; t += kHeadWarps) {
        const uint4* p = reinterpret_cast<const uint4*>(h + (int64_t)t * d);
        uint32_t am = 0u;
        for (int i = lane; i < (d >> 3); i += 32) {
            const uint4 v = p[i];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                am = max(am, (w[k] << 16) & 0x7FFFFFFFu);
                am = max(am, w[k] & 0x7FFF0000u);
            }
        }
        am = __reduce_max_sync(0xffffffffu, am);
        if (lane == 0) hs.amax[t] = am;
    }
    __syncthreads();
    for (int i = tid; i < m * (d >> 2); i += kHeadThreads) {
        const int t = i / (d >> 2), j4 = i - t * (d >> 2);
        const float am = __uint_as_float(hs.amax[t]);
        const float inv = quant_inv(am);
        const bool zero = am == 0.0f;
        const uint2 raw = *reinterpret_cast<const uint2*>(h + (int64_t)t * d + 4 * j4);
        const int q0 = quant1(bf16_lo(raw.x), inv, zero), q1 = quant1(bf16_hi(raw.x), inv, zero);
        const int q2 = quant1(bf16_lo(raw.y), inv, zero), q3 = quant1(bf16_hi(raw.y), inv, zero);
        reinterpret_cast<uint32_t*>(q + t * d)[j4] = (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) |
                                                      ((uint32_t)(q2 & 0xFF) << 16) | ((uint32_t)(q3 & 0xFF) << 24);
    }
    if (tid < m) hs.sx[tid] = quant_sx(__uint_as_float(hs.amax[tid]));
    __syncthreads();

    // ---- rows: warp w of CTA b takes rows (b * warps + w) + k * (grid * warps), two at a time
    const int nw = gridDim.x * kHeadWarps;
    const int n16 = d >> 4;                         // 16-byte pieces per row
    for (int v0 = blockIdx.x * kHeadWarps + warp; v0 < vocab; v0 += kRowsPerIter * nw) {
        int acc[kRowsPerIter][MT];
#pragma unroll
        for (int r = 0; r < kRowsPerIter; ++r)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[r][t] = 0;
        // kPieces 16-byte pieces of each of the rows in flight per lane before any arithmetic
        for (int p0 = 0; p0 < n16; p0 += 32 * kPieces) {
            uint4 e[kRowsPerIter][kPieces];
#pragma unroll
            for (int r = 0; r < kRowsPerIter; ++r)
#pragma unroll
                for (int k = 0; k < kPieces; ++k) {
                    const int p = p0 + 32 * k + lane, v = v0 + r * nw;
                    e[r][k] = (p < n16 && v < vocab) ? ld_stream16(table + (int64_t)v * d + 16 * p)
                                                     : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t >= m) break;
#pragma unroll
                for (int k = 0; k < kPieces; ++k) {
                    const int p = p0 + 32 * k + lane;
                    if (p < n16) {
                        const uint4 qq = *reinterpret_cast<const uint4*>(q + t * d + 16 * p);
#pragma unroll
                        for (int r = 0; r < kRowsPerIter; ++r) {
                            int s = acc[r][t];
                            s = __dp4a((int)e[r][k].x, (int)qq.x, s);
                            s = __dp4a((int)e[r][k].y, (int)qq.y, s);
                            s = __dp4a((int)e[r][k].z, (int)qq.z, s);
                            s = __dp4a((int)e[r][k].w, (int)qq.w, s);
                            acc[r][t] = s;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRowsPerIter; ++r) {
            const int v = v0 + r * nw;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t >= m) break;
                const int a = __reduce_add_sync(0xffffffffu, acc[r][t]);
                if (lane == t && v < vocab) {
                    const float y = __fmul_rn(hs.sx[t], __fmul_rn(scale[v], (float)a));
                    const int64_t idx = (int64_t)t * vocab + v;
                    if (out_dtype == DFSSM_BF16)
                        reinterpret_cast<uint16_t*>(logits)[idx] = f32_to_bf16_bits(y);
                    else
                        reinterpret_cast<float*>(logits)[idx] = y;
                    if (acc_out) acc_out[idx] = a;
                }
            }
        }
    }
}

template <int MT>
cudaError_t launch_head(const Int8TableArgs& a, int sm_count, cudaStream_t s) {
    const size_t smem = ((sizeof(HeadShared) + 127) & ~(size_t)127) + (size_t)a.m * a.d;
    lm_head_kernel<MT><<<sm_count, kHeadThreads, smem, s>>>(a.table, a.scale, a.vocab, a.d,
                                                             reinterpret_cast<const uint16_t*>(a.in), a.m, a.out,
                                                             a.out_dtype, a.acc);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_embed(const Int8TableArgs& a, cudaStream_t s) {
    dim3 grid((a.d / 8 + kEmbedThreads - 1) / kEmbedThreads, a.m);
    embed_kernel<<<grid, kEmbedThreads, 0, s>>>(a.table, a.scale, a.vocab, a.d, a.ids, a.out, a.out_dtype, a.err);
    return cudaGetLastError();
}

cudaError_t launch_lm_head(const Int8TableArgs& a, int sm_count, cudaStream_t s) {
    if (a.m <= 1) return launch_head<1>(a, sm_count, s);
    if (a.m <= 4) return launch_head<4>(a, sm_count, s);
    return launch_head<16>(a, sm_count, s);
}

cudaError_t set_int8_table_attr(int optin) {
    cudaError_t e = allow_dyn_smem(lm_head_kernel<1>, optin);
    if (e == cudaSuccess) e = allow_dyn_smem(lm_head_kernel<4>, optin);
    if (e == cudaSuccess) e = allow_dyn_smem(lm_head_kernel<16>, optin);
    return e;
}

}  // namespace dfssm
