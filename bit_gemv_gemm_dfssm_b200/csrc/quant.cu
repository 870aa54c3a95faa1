// Per-token activation quantisation and the fused LoRA down-projection for the
// decode path (1 <= m <= 16 tokens; many tokens go to quant_rows.cu). One token
// takes the slice kernel at the end of this file.
//
// The scaffold matmul runs on int8 activations ("Density Field State Space
// Models", gist.science technical summary, §2.C: packed bits expanded to int8
// for an int8 x int8 -> int32 matmul), and the rank-16 int8 LoRA
// (§2.B: W_B in R^{r x d_in}, r = 16, int8 with per-row scales) reads the
// same int8 activations. For each token t of each linear:
//   amax   = max_j |x[t,j]|                       (fp32, exact)
//   q[t,j] = clamp(rint(x[t,j] * (127/amax)), +-127), s_x = amax/127 (IEEE fp32,
//            round-to-nearest; amax == 0 gives q = 0, s_x = 0)
//   h[t,k] = sum_j W_B[k,j] q[t,j]                 (int32, warp MMA s8 x s8)
// The decode kernel quantises x again into its own shared memory (same
// arithmetic, same bytes) and computes s_x and sum q itself, so this kernel only
// supplies h, as partial sums.
//
// The 128-column pieces of a linear are split over S blocks so that W_B (the
// only large read) streams through many SMs. Every block finds the full-row amax
// itself (x is a few KB per token), quantises its own columns straight into
// warp-MMA A fragments and writes its partial h; the decode kernel adds the S
// partials in split order (exact integer sums) and scales them by s_B. The W_B
// fragments of each warp's first k-blocks are loaded before the amax pass, so
// their latency hides behind the activation reads.
#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTok = 16;              // tokens per round
constexpr int kQsPad = 16;            // bytes of padding per shared q row

struct QuantRed {
    unsigned int amax[kTok];     // fp32 bits of max |x| (order-preserving as unsigned; NaN above Inf)
    int sumq[kWarps][kTok];
    int h[kWarps][kTok][kRank];
    float inv[kTok];
    float sx[kTok];
};

__device__ __forceinline__ void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct QuantArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* descs;
    int m;                  // tokens, 1..16
    int splits;             // blocks per linear along d_in
    int* part;              // [linear][split][16 tokens][kPartInts] partial h (the decode kernel adds them)
    uint32_t* err;
};

// W_B fragments of up to kWbAhead k-blocks per warp are loaded before the activation pass
constexpr int kWbAhead = 4;

__global__ void __launch_bounds__(kThreads) quant_kernel(const __grid_constant__ QuantArgs qa) {
    const dfssm_stack_entry* entries = qa.entries;
    const DevDesc* descs = qa.descs;
    const int m = qa.m;
    uint32_t* err = qa.err;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // let the dependent scaffold kernel start streaming weights right away;
    // it waits for this grid's results before reading them
    ptx::pdl_launch_dependents();
    const int lin = blockIdx.y;
    const dfssm_stack_entry& e = entry_at(entries, qa.single, lin);
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
    const int nquad = d_in >> 7;                  // 128-column pieces (4 k-blocks of 32 columns)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;

    QuantRed& red = *reinterpret_cast<QuantRed*>(smem_raw);
    // [m][qs_row]: rows padded by 16 bytes so the 8 token rows of an MMA fragment hit 8 bank groups
    const int qs_row = d_in + kQsPad;
    int8_t* q_s = reinterpret_cast<int8_t*>(smem_raw + ((sizeof(QuantRed) + 127) & ~(size_t)127));

    const uint16_t* xg = reinterpret_cast<const uint16_t*>(e.x);
    const uint8_t* wb = reinterpret_cast<const uint8_t*>(e.w.wb);

    // this block's 128-column pieces of the linear
    const int split = blockIdx.x;
    const int pc_lo = split * nquad / qa.splits, pc_hi = (split + 1) * nquad / qa.splits;
    const int kb_lo = 4 * pc_lo, kb_hi = 4 * pc_hi;
    const int nt = m;

    // B fragments (W_B rows g and g + 8) of this warp's first k-blocks: in flight during pass 1
    uint32_t wbf[kWbAhead][4];
#pragma unroll
    for (int j = 0; j < kWbAhead; ++j) {
        const int kb = kb_lo + warp + kWarps * j;
        const int col = 32 * kb;
        if (kb < kb_hi) {
            wbf[j][0] = __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)g * d_in + col + 4 * c));
            wbf[j][1] = __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)g * d_in + col + 16 + 4 * c));
            wbf[j][2] = __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)(g + 8) * d_in + col + 4 * c));
            wbf[j][3] = __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)(g + 8) * d_in + col + 16 + 4 * c));
        } else {
            wbf[j][0] = wbf[j][1] = wbf[j][2] = wbf[j][3] = 0u;
        }
    }

    // ---- pass 1: amax of each token's row, one warp per token, lanes across the row
    for (int tk = warp; tk < nt; tk += kWarps) {
        const uint4* p = reinterpret_cast<const uint4*>(xg + (int64_t)tk * d_in);
        uint32_t am = 0u;
#pragma unroll 8
        for (int i = lane; i < (d_in >> 3); i += 32) am = absmax8_bits(p[i], am);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
        if (lane == 0) red.amax[tk] = am;
    }
    if (tid >= nt && tid < kTok) red.amax[tid] = 0u;    // tokens past m: q = 0
    __syncthreads();
    if (tid < kTok) {
        const float am = __uint_as_float(red.amax[tid]);
        if (tid < nt && !isfinite(am)) atomicOr(err, DFSSM_DEVERR_NONFINITE);
        red.inv[tid] = quant_inv(am);
        red.sx[tid] = quant_sx(am);
    }
    __syncthreads();

    // ---- pass 2: quantise into A fragments, h += q * W_B^T, q -> shared tile (debug export)
    const float invA = red.inv[g], invB = red.inv[g + 8];
    const bool zA = invA == 0.0f, zB = invB == 0.0f;
    const bool hasA = g < nt, hasB = g + 8 < nt;
    const uint16_t* xA = xg + (int64_t)g * d_in + 4 * c;
    const uint16_t* xB = xg + (int64_t)(g + 8) * d_in + 4 * c;
    int D0[4] = {0, 0, 0, 0}, D1[4] = {0, 0, 0, 0};
    auto kblock = [&](int kb, uint32_t b00, uint32_t b01, uint32_t b10, uint32_t b11) {
        const int col = 32 * kb;
        const uint2 zero2 = make_uint2(0u, 0u);
        const uint2 xa0 = hasA ? *reinterpret_cast<const uint2*>(xA + col) : zero2;
        const uint2 xa1 = hasA ? *reinterpret_cast<const uint2*>(xA + col + 16) : zero2;
        const uint2 xb0 = hasB ? *reinterpret_cast<const uint2*>(xB + col) : zero2;
        const uint2 xb1 = hasB ? *reinterpret_cast<const uint2*>(xB + col + 16) : zero2;
        int unused = 0;
        const uint32_t a0 = quant4(xa0, invA, zA, unused);
        const uint32_t a2 = quant4(xa1, invA, zA, unused);
        const uint32_t a1 = quant4(xb0, invB, zB, unused);
        const uint32_t a3 = quant4(xb1, invB, zB, unused);
        mma_s8s8(D0, a0, a1, a2, a3, b00, b01);
        mma_s8s8(D1, a0, a1, a2, a3, b10, b11);
        if (hasA) {
            *reinterpret_cast<uint32_t*>(q_s + g * qs_row + col + 4 * c) = a0;
            *reinterpret_cast<uint32_t*>(q_s + g * qs_row + col + 16 + 4 * c) = a2;
        }
        if (hasB) {
            *reinterpret_cast<uint32_t*>(q_s + (g + 8) * qs_row + col + 4 * c) = a1;
            *reinterpret_cast<uint32_t*>(q_s + (g + 8) * qs_row + col + 16 + 4 * c) = a3;
        }
    };
#pragma unroll
    for (int j = 0; j < kWbAhead; ++j) {
        const int kb = kb_lo + warp + kWarps * j;
        if (kb < kb_hi) kblock(kb, wbf[j][0], wbf[j][1], wbf[j][2], wbf[j][3]);
    }
    for (int kb = kb_lo + warp + kWarps * kWbAhead; kb < kb_hi; kb += kWarps) {
        const int col = 32 * kb;
        kblock(kb, __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)g * d_in + col + 4 * c)),
               __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)g * d_in + col + 16 + 4 * c)),
               __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)(g + 8) * d_in + col + 4 * c)),
               __ldg(reinterpret_cast<const uint32_t*>(wb + (int64_t)(g + 8) * d_in + col + 16 + 4 * c)));
    }
    // D fragment: (token g, lora 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1); D1 for lora + 8
    red.h[warp][g][2 * c] = D0[0];
    red.h[warp][g][2 * c + 1] = D0[1];
    red.h[warp][g + 8][2 * c] = D0[2];
    red.h[warp][g + 8][2 * c + 1] = D0[3];
    red.h[warp][g][8 + 2 * c] = D1[0];
    red.h[warp][g][8 + 2 * c + 1] = D1[1];
    red.h[warp][g + 8][8 + 2 * c] = D1[2];
    red.h[warp][g + 8][8 + 2 * c + 1] = D1[3];
    __syncthreads();

    // ---- this split's partial h: thread (token tid / 16, lora row tid % 16). The decode kernel
    // adds the splits' partials in split order and scales by s_B (exact integer sums).
    {
        const int tk = tid >> 4, k = tid & 15;
        if (tk < nt) {
            int h = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) h += red.h[w][tk][k];
            qa.part[part_index(lin, qa.splits, split, tk, k)] = h;
            if (split == 0 && k == 0 && e.dbg.sx) e.dbg.sx[tk] = red.sx[tk];
        }
    }

    // ---- debug export of q (natural order), this block's columns
    if (e.dbg.q) {
        const int npc = pc_hi - pc_lo;
        for (int i = tid; i < nt * npc; i += kThreads) {
            const int tk = i / npc, pc = pc_lo + (i - tk * npc);
            const uint4* sq = reinterpret_cast<const uint4*>(q_s + tk * qs_row + 128 * pc);
            uint4* dq = reinterpret_cast<uint4*>(e.dbg.q + (int64_t)tk * d_in + 128 * pc);
#pragma unroll
            for (int u = 0; u < 8; ++u) dq[u] = sq[u];
        }
    }
}

// ---- one token: LoRA down-projection slices beside the decode kernel ------------------
// Item (linear, slice) covers columns [2048 s, 2048 (s + 1)) of that linear. A CTA of two
// warps brings the slice of W_B into shared memory with bulk copies (kWbRows rows per pass)
// while it finds the token's amax over the whole row, then quantises its columns (the same
// fp32 arithmetic as above) and takes h over the slice with dp4a, summed across the CTA with
// warp reductions. The CTA is kept small (64 threads, 32 registers, ~33 KB of shared memory)
// so that it fits beside three decode CTAs on an SM: the decode kernel starts streaming
// weights at once and waits for h only before its first epilogue.
#ifndef DFSSM_SLICE_THREADS
#define DFSSM_SLICE_THREADS 64
#endif
constexpr int kSliceThreads = DFSSM_SLICE_THREADS;
constexpr int kSliceHead = 256;      // shared bytes before the W_B slice
#ifndef DFSSM_SLICE_WB_ROWS
#define DFSSM_SLICE_WB_ROWS 16
#endif
constexpr int kWbRows = DFSSM_SLICE_WB_ROWS;                    // W_B rows per shared-memory pass
constexpr int kSliceChunks = kLoraSliceCols / 8 / kSliceThreads;  // 8-column chunks per thread
#ifndef DFSSM_SLICE_REGS
#define DFSSM_SLICE_REGS 32
#endif
constexpr int kSliceRegs = DFSSM_SLICE_REGS;     // register cap per thread
static_assert(kSliceThreads % 32 == 0 && kLoraSliceCols % (8 * kSliceThreads) == 0, "slice chunks per thread");
static_assert(kRank % kWbRows == 0, "W_B passes");

struct SliceArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* descs;
    int n_items;
    int* part;
    uint32_t* err;
    uint32_t item[kMaxSliceItems];   // linear << 8 | slice
};

struct SliceShared {
    uint64_t bar;
    unsigned int amax[kSliceThreads / 32];
    int h[kSliceThreads / 32][kRank];
};
static_assert(sizeof(SliceShared) <= kSliceHead, "slice kernel shared header");

__global__ void __launch_bounds__(kSliceThreads, 65536 / (kSliceThreads * kSliceRegs)) lora_slice_kernel(const __grid_constant__ SliceArgs sa) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SliceShared& sh = *reinterpret_cast<SliceShared*>(smem_raw);
    int8_t* wb_s = reinterpret_cast<int8_t*>(smem_raw + kSliceHead);     // [16][kLoraSliceCols]
    // the decode kernel may start streaming weights now; it waits for this grid before its epilogues
    ptx::pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        ptx::mbar_init(&sh.bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    uint32_t phase = 0;
    for (int it = blockIdx.x; it < sa.n_items; it += gridDim.x) {
        const int lin = (int)(sa.item[it] >> 8), sl = (int)(sa.item[it] & 0xFFu);
        const dfssm_stack_entry& e = entry_at(sa.entries, sa.single, lin);
        const bool desc_ok = !(sa.entries && e.desc_index != lin), ptrs_ok = entry_ptrs_ok(e);
        if (!desc_ok || !ptrs_ok) {
            if (tid == 0 && sl == 0) atomicOr(sa.err, desc_ok ? DFSSM_DEVERR_ENTRY_PTR : DFSSM_DEVERR_ENTRY_DESC);
            continue;
        }
        const int d_in = sa.descs[lin].d_in;
        const int c0 = sl * kLoraSliceCols, ncols = min(kLoraSliceCols, d_in - c0);
        const int8_t* wb = e.w.wb + c0;
        __syncthreads();                           // the previous item is done with wb_s and sh
        if (tid == 0) {
            ptx::mbar_arrive_expect_tx(&sh.bar, (uint32_t)(kWbRows * ncols));
            for (int k = 0; k < kWbRows; ++k)
                ptx::bulk_g2s(wb_s + k * kLoraSliceCols, wb + (int64_t)k * d_in, (uint32_t)ncols, &sh.bar);
        }
        // amax of the whole row, as fp32 bit patterns (a NaN wins)
        const uint16_t* x = reinterpret_cast<const uint16_t*>(e.x);
        uint32_t am = 0u;
        for (int ch = tid; ch < (d_in >> 3); ch += kSliceThreads)
            am = absmax8_bits(__ldg(reinterpret_cast<const uint4*>(x) + ch), am);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
        if (lane == 0) sh.amax[warp] = am;
        __syncthreads();
        am = sh.amax[0];
#pragma unroll
        for (int w = 1; w < kSliceThreads / 32; ++w) am = max(am, sh.amax[w]);
        const float amax = __uint_as_float(am);
        const float inv = quant_inv(amax);
        const bool zero = inv == 0.0f;
        if (tid == 0 && sl == 0) {
            if (!isfinite(amax)) atomicOr(sa.err, DFSSM_DEVERR_NONFINITE);
            if (e.dbg.sx) e.dbg.sx[0] = quant_sx(amax);
        }
        // this thread's 8-column chunks j = tid + kSliceThreads i of the slice, quantised
        uint32_t qv[kSliceChunks][2];
#pragma unroll
        for (int i = 0; i < kSliceChunks; ++i) {
            const int j = tid + kSliceThreads * i;
            qv[i][0] = qv[i][1] = 0u;
            if (j < (ncols >> 3)) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + c0) + j);
                int unused = 0;
                qv[i][0] = quant4(make_uint2(v.x, v.y), inv, zero, unused);
                qv[i][1] = quant4(make_uint2(v.z, v.w), inv, zero, unused);
                if (e.dbg.q) *reinterpret_cast<uint2*>(e.dbg.q + c0 + 8 * j) = make_uint2(qv[i][0], qv[i][1]);
            }
        }
        // h += q . W_B, kWbRows LoRA rows per pass through the shared buffer, each pass summed
        // across the warp (redux.sync) into sh.h
#pragma unroll
        for (int k0 = 0; k0 < kRank; k0 += kWbRows) {
            if (k0 > 0) {
                __syncthreads();                   // every thread is done with the previous rows
                if (tid == 0) {
                    ptx::mbar_arrive_expect_tx(&sh.bar, (uint32_t)(kWbRows * ncols));
                    for (int k = 0; k < kWbRows; ++k)
                        ptx::bulk_g2s(wb_s + k * kLoraSliceCols, wb + (int64_t)(k0 + k) * d_in, (uint32_t)ncols,
                                      &sh.bar);
                }
            }
            // a wait that gave up stops the CTA: it reports the error, lets the copies in flight
            // into its shared memory land (bounded) and issues nothing more
            const bool got = ptx::mbar_wait(&sh.bar, phase);
            if (__syncthreads_or(!got)) {
                if (tid == 0) {
                    atomicOr(sa.err, DFSSM_DEVERR_TIMEOUT);
                    ptx::mbar_wait(&sh.bar, phase);
                }
                return;
            }
            phase ^= 1u;
            int h[kWbRows];
#pragma unroll
            for (int k = 0; k < kWbRows; ++k) h[k] = 0;
#pragma unroll
            for (int i = 0; i < kSliceChunks; ++i) {
                const int j = tid + kSliceThreads * i;
#pragma unroll
                for (int k = 0; k < kWbRows; ++k) {
                    const uint2 w = *reinterpret_cast<const uint2*>(wb_s + k * kLoraSliceCols + 8 * j);
                    h[k] = __dp4a((int)qv[i][0], (int)w.x, h[k]);
                    h[k] = __dp4a((int)qv[i][1], (int)w.y, h[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < kWbRows; ++k) {
                const int v = __reduce_add_sync(0xffffffffu, h[k]);
                if (lane == k) sh.h[warp][k0 + k] = v;
            }
        }
        __syncthreads();
        if (tid < kRank) {
            int hs = 0;
#pragma unroll
            for (int w = 0; w < kSliceThreads / 32; ++w) hs += sh.h[w][tid];
            sa.part[part_index(lin, kLoraMaxSlices, sl, 0, tid)] = hs;
        }
    }
}

}  // namespace

cudaError_t launch_quant_rows(const LaunchCtx& c);

// d_in splits of the quantisation kernel for m <= 16 tokens: enough blocks to cover the SMs
// twice, at least two 128-column pieces (8 k-blocks, one per warp) per split. The decode kernel
// uses the same count to add the partials.
int quant_splits(const LaunchCtx& c) {
    int min_pc = 1 << 30;
    for (int i = 0; i < c.n; ++i) min_pc = min(min_pc, c.host_desc[i].d_in / 128);
    int splits = (2 * c.sm_count + c.n - 1) / c.n;
    return max(1, min(splits, min(kMaxSplits, min_pc / 2)));
}

cudaError_t launch_quant_rows(const LaunchCtx& c);

cudaError_t launch_quant(const LaunchCtx& c) {
    if (c.m > kDecodeMaxTokens) return launch_quant_rows(c);
    if (use_lora_slices(c)) {
        SliceArgs sa{c.entries, c.single, c.desc, 0, c.part, c.err, {}};
        for (int i = 0; i < c.n; ++i)
            for (int s = 0; s < lora_slices(c.host_desc[i].d_in); ++s) sa.item[sa.n_items++] = ((uint32_t)i << 8) | (uint32_t)s;
        const int grid = lora_slice_grid(c);
        const size_t smem = kSliceHead + (size_t)kWbRows * kLoraSliceCols;
        lora_slice_kernel<<<grid, kSliceThreads, smem, c.stream>>>(sa);
        return cudaGetLastError();
    }
    const int splits = quant_splits(c);
    dim3 grid(splits, c.n);
    // the shared q tile holds the call's m <= 16 tokens
    const size_t smem = ((sizeof(QuantRed) + 127) & ~(size_t)127) + (size_t)c.m * (c.max_d_in + kQsPad);
    QuantArgs qa{c.entries, c.single, c.desc, c.m, splits, c.part, c.err};
    quant_kernel<<<grid, kThreads, smem, c.stream>>>(qa);
    return cudaGetLastError();
}

cudaError_t set_quant_attr(int optin) {
    cudaError_t e = allow_dyn_smem(quant_kernel, optin);
    if (e == cudaSuccess) e = allow_dyn_smem(lora_slice_kernel, optin);
    // shared memory carved out like the decode kernel's, so both can share an SM
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(lora_slice_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    return e;
}

}  // namespace dfssm
