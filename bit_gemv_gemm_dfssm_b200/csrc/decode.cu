// Decode path (1 <= m <= 16 tokens): the scaffold contraction streamed from HBM
// with the LoRA up-projection and both dequantisation epilogues fused.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C:
// the 1-bit scaffold weights are expanded on the fly to int8 and fed to int8
// tensor cores, which cuts weight traffic 8x against int8 weights; at batch 1
// the layer is bound by that weight stream. Here the bits never leave
// registers as bytes in memory:
//
//  * A CTA owns 64 output rows of one linear. Its rows are brought into shared
//    memory by the TMA bulk-copy engine (one cp.async.bulk per row, padded row
//    stride so the fragment reads below are bank-conflict free), completion
//    tracked by one mbarrier. No multicast.
//  * Expansion: for a 32-bit word of sign bits w and bit position p,
//    w & (0x01010101 << p) is four bytes that are each 0 or 2^p: the bits of
//    columns 8i + p (i = 0..3) scaled by 2^p. One LOP3 expands four weights.
//  * These bytes are the u8 A operand of the legacy warp MMA
//    m16n8k32 (u8 x s8 -> s32); the int8 activations, stored in the matching
//    permuted column order (byte 4p + i of a 32-column group = column 8i + p),
//    are the s8 B operand, with the tokens as the N = 8 columns.
//  * One accumulator set per bit position p, so each sums 2^p * S_p exactly;
//    S1 = sum_p D_p / 2^p = sum_{bit = 1} q, and acc = 2 * S1 - sum_j q
//    (a +-1 weight is 2b - 1).
//  * Epilogue per (token t, row o), in fp32 in this fixed order:
//      dot = sum_{k=0..15} W_A[o,k] * u[t,k]   (fmaf, k ascending)
//      y   = s_x[t] * fmaf(alpha[o], acc, s_A[o] * dot)
//    the same order as the prefill path, so the two paths agree bit for bit.
//
// The kernel is launched with programmatic dependent launch: it issues its
// weight copies first and only then waits for the quantisation kernel that
// produces q, s_x, sum q and u.
#include "dfssm_internal.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kRowsPerCta = 64;
constexpr int kWarps = 4;
constexpr int kRowPad = 32;      // bytes added to each staged sign row
constexpr int kTokPad = 64;      // bytes added to each staged q row

struct DecodeArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* desc;   // desc[0] is the first linear of this launch
    int n;
    int m;
    const int8_t* q_ws;
    const TokStats* st_ws;
    uint32_t* err;
};

__device__ __forceinline__ int find_linear(const DevDesc* desc, int n, int blk) {
    // largest l with desc[l].blk_begin - desc[0].blk_begin <= blk
    const int base = desc[0].blk_begin;
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (desc[mid].blk_begin - base <= blk) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int NT>
__global__ void __launch_bounds__(kWarps * 32) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
    TokStats* st_s = reinterpret_cast<TokStats*>(smem + 16);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;

    const int lin = find_linear(a.desc, a.n, blockIdx.x);
    const DevDesc d = a.desc[lin];
    const dfssm_stack_entry& e = entry_at(a.entries, a.single, lin);
    const int m = a.m;
    const int d_in = d.d_in;
    const int rb = d_in >> 3;                      // sign bytes per row
    const int wstride = rb + kRowPad;
    const int qstride = d_in + kTokPad;
    const int row0 = (blockIdx.x - (d.blk_begin - a.desc[0].blk_begin)) * kRowsPerCta;
    const int nrows = min(kRowsPerCta, d.d_out - row0);

    if (!entry_ptrs_ok(e)) return;     // flagged by the quantisation kernel

    uint8_t* q_s = smem + 16 + ((m * (int)sizeof(TokStats) + 127) & ~127);
    uint8_t* w_s = q_s + ((m * qstride + 127) & ~127);

    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();

    // ---- 1. weight rows: bulk copies, issued before waiting on the producer kernel
    if (warp == 0) {
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar, (uint32_t)(nrows * rb));
        __syncwarp();
        const uint8_t* src = e.w.sign + (int64_t)row0 * rb;
        for (int r = lane; r < nrows; r += 32)
            ptx::bulk_g2s(w_s + r * wstride, src + (int64_t)r * rb, (uint32_t)rb, bar);
    }

    // epilogue parameters of this thread's two rows (independent of the producer)
    const int oA = row0 + warp * 16 + g, oB = oA + 8;
    float alphaA = 0.f, alphaB = 0.f, saA = 0.f, saB = 0.f;
    int4 waA = make_int4(0, 0, 0, 0), waB = make_int4(0, 0, 0, 0);
    if (oA < d.d_out) {
        alphaA = e.w.alpha[oA]; saA = e.w.sa[oA];
        waA = *reinterpret_cast<const int4*>(e.w.wa + (int64_t)oA * kRank);
    }
    if (oB < d.d_out) {
        alphaB = e.w.alpha[oB]; saB = e.w.sa[oB];
        waB = *reinterpret_cast<const int4*>(e.w.wa + (int64_t)oB * kRank);
    }

    // ---- 2. wait for q / stats, stage them
    ptx::pdl_wait();
    {
        const uint4* src = reinterpret_cast<const uint4*>(a.st_ws + d.st_off);
        uint4* dst = reinterpret_cast<uint4*>(st_s);
        for (int i = tid; i < m * (int)(sizeof(TokStats) / 16); i += kWarps * 32) dst[i] = src[i];
        // q rows, chunk (G, c', k) of a 64-byte block stored at slot (k + c') & 3
        const int chunks = d_in >> 4;
        for (int i = tid; i < m * chunks; i += kWarps * 32) {
            const int t = i / chunks, s = i - t * chunks;
            const int G = s >> 4, cc = (s >> 2) & 3, k = s & 3;
            const uint4 v = *reinterpret_cast<const uint4*>(a.q_ws + d.q_off + (int64_t)t * d_in + 16 * s);
            *reinterpret_cast<uint4*>(q_s + t * qstride + 256 * G + 64 * cc + 16 * ((k + cc) & 3)) = v;
        }
    }
    __syncthreads();
    if (a.entries != nullptr && e.desc_index != lin) {
        if (tid == 0) atomicOr(a.err, DFSSM_DEVERR_ENTRY_DESC);
    }

    // ---- 3. wait for the weight rows
    if (!ptx::mbar_wait(bar, 0)) {
        if (lane == 0) atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
        ptx::mbar_wait(bar, 0);   // second bounded wait for the copies still in flight
        return;
    }

    // ---- 4. main loop: 16 rows per warp, all of d_in
    int D[NT][8][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int p = 0; p < 8; ++p)
#pragma unroll
            for (int r = 0; r < 4; ++r) D[nt][p][r] = 0;

    const uint8_t* wrA = w_s + (warp * 16 + g) * wstride + 8 * c;
    const uint8_t* wrB = wrA + 8 * wstride;
    // groups of 256 columns; when d_in % 256 == 128 the last group is half full and
    // only lanes with c < 2 (words 0..3 of the group) carry data
    const int ngroups = (d_in + 255) >> 8;
    const bool warp_active = warp * 16 < nrows;
    if (warp_active) {
        for (int G = 0; G < ngroups; ++G) {
            const bool lane_has = (256 * G + 64 * c) < d_in;
            const uint2 wa2 = lane_has ? *reinterpret_cast<const uint2*>(wrA + 32 * G) : make_uint2(0u, 0u);
            const uint2 wb2 = lane_has ? *reinterpret_cast<const uint2*>(wrB + 32 * G) : make_uint2(0u, 0u);
            uint32_t b[NT][4][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tk = nt * 8 + g;
                if (tk < m && lane_has) {
                    const uint8_t* qb = q_s + tk * qstride + 256 * G + 64 * c;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint4 v = *reinterpret_cast<const uint4*>(qb + 16 * ((k + c) & 3));
                        b[nt][k][0] = v.x; b[nt][k][1] = v.y; b[nt][k][2] = v.z; b[nt][k][3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int j = 0; j < 4; ++j) b[nt][k][j] = 0u;
                }
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint32_t msk = 0x01010101u << p;
                const uint32_t a0 = wa2.x & msk, a1 = wb2.x & msk, a2 = wa2.y & msk, a3 = wb2.y & msk;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // chunk 0/1: b0 for p 0..3 / 4..7; chunk 2/3: b1 for p 0..3 / 4..7
                    const uint32_t b0 = b[nt][p >> 2][p & 3];
                    const uint32_t b1 = b[nt][2 + (p >> 2)][p & 3];
                    ptx::mma_u8s8(D[nt][p], a0, a1, a2, a3, b0, b1);
                }
            }
        }
    }

    // ---- 5. epilogue
    if (!warp_active) return;
    const int8_t* waAb = reinterpret_cast<const int8_t*>(&waA);
    const int8_t* waBb = reinterpret_cast<const int8_t*>(&waB);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            // d0: (row g, token 2c), d1: (row g, token 2c+1), d2/d3: row g + 8
            int T = 0;
#pragma unroll
            for (int p = 0; p < 8; ++p) T += D[nt][p][r] << (7 - p);
            const int s1 = T >> 7;
            const int t = nt * 8 + 2 * c + (r & 1);
            const int o = (r < 2) ? oA : oB;
            if (t >= m || o >= d.d_out) continue;
            const TokStats& st = st_s[t];
            const int acc = 2 * s1 - st.sumq;
            const int8_t* wa = (r < 2) ? waAb : waBb;
            float dot = 0.0f;
#pragma unroll
            for (int k = 0; k < kRank; ++k) dot = __fmaf_rn((float)wa[k], st.u[k], dot);
            const float alpha = (r < 2) ? alphaA : alphaB;
            const float sa = (r < 2) ? saA : saB;
            const float y = __fmul_rn(st.sx, __fmaf_rn(alpha, (float)acc, __fmul_rn(sa, dot)));
            const int64_t idx = (int64_t)t * d.d_out + o;
            if (d.y_dtype == DFSSM_BF16)
                reinterpret_cast<__nv_bfloat16*>(e.y)[idx] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float*>(e.y)[idx] = y;
            if (e.dbg.acc) e.dbg.acc[idx] = acc;
        }
    }
}

template <int NT>
cudaError_t launch_nt(const LaunchCtx& c, int blocks) {
    DecodeArgs a{c.entries, c.single, c.desc, c.n, c.m, c.q_ws, c.st_ws, c.err};
    const int rb_max = c.max_d_in / 8;
    size_t smem = 16 + ((c.m * sizeof(TokStats) + 127) & ~(size_t)127) +
                  ((size_t)(c.m * (c.max_d_in + kTokPad) + 127) & ~(size_t)127) +
                  (size_t)kRowsPerCta * (rb_max + kRowPad);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<NT>, a);
}

}  // namespace

int decode_blocks(const DevDesc* host_desc, int n) {
    int total = 0;
    for (int i = 0; i < n; ++i) total += (host_desc[i].d_out + kRowsPerCta - 1) / kRowsPerCta;
    return total;
}

cudaError_t launch_decode(const LaunchCtx& c) {
    const int blocks = decode_blocks(c.host_desc, c.n);
    if (c.m <= 8) return launch_nt<1>(c, blocks);
    return launch_nt<2>(c, blocks);
}

void set_decode_attr(int max_dyn_smem) {
    cudaFuncSetAttribute(decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn_smem);
    cudaFuncSetAttribute(decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn_smem);
}

}  // namespace dfssm
