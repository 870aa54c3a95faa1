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
//   h[t,k] = sum_j W_B[k,j] q[t,j]                 (int32, warp MMA s8 x s8)
//   u[t,k] = s_B[k] * h[t,k]                       (fp32)
// and, for the prefill (m > 16), stores q in the plane-major int8 rows its
// tensor-core kernel reads, plus s_x, sumq and u.
//
// A block owns one linear and up to kTokPerBlock = 16 tokens (one MMA tile;
// many small blocks keep enough loads in flight). The 8 warps split the 32-column k-blocks of d_in
// between them: pass 1 finds each token's amax, pass 2 quantises x straight
// into MMA A fragments (16 tokens x 32 columns), runs h += q * W_B^T on the
// warp MMA (m16n8k32, two n-tiles for the 16 LoRA rows) and writes q to a
// shared tile. From there each thread takes 128 columns of a token and stores
// them as eight 16-byte plane pieces (two 4x4 byte transposes with PRMT per
// 32-column group).
//
// Few tokens (m <= 16, one round): the 128-column pieces of a linear are split
// over S blocks so that W_B (the only large read) streams through many SMs. Every
// split block finds the full-row amax itself, handles its own columns, and
// writes partial h and sum q; the last split block to finish (atomic ticket)
// adds the partials in split order, writes the per-token scalars and resets
// the ticket for the next call.
#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTok = 16;              // tokens per round
constexpr int kQsPad = 16;            // bytes of padding per shared q row
constexpr int kTokPerBlock = 16;      // one round per block: more blocks in flight hide the loads

struct QuantRed {
    unsigned int amax[kTok];     // fp32 bits of max |x| (order-preserving as unsigned; NaN above Inf)
    int sumq[kWarps][kTok];
    int h[kWarps][kTok][kRank];
    float inv[kTok];
    float sx[kTok];
};

// 4 bf16 (8 bytes) -> 4 int8 packed little-endian
__device__ __forceinline__ uint32_t quant4(uint2 raw, float inv, bool zero, int& sum) {
    const int q0 = quant1(bf16_bits_to_float(raw.x & 0xFFFFu), inv, zero);
    const int q1 = quant1(bf16_bits_to_float(raw.x >> 16), inv, zero);
    const int q2 = quant1(bf16_bits_to_float(raw.y & 0xFFFFu), inv, zero);
    const int q3 = quant1(bf16_bits_to_float(raw.y >> 16), inv, zero);
    sum += q0 + q1 + q2 + q3;
    return (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) | ((uint32_t)(q2 & 0xFF) << 16) |
           ((uint32_t)(q3 & 0xFF) << 24);
}

// running max of |x| over 8 bf16 values, as fp32 bit patterns: for |x| the unsigned order is
// the numeric order, and a NaN (bits above Inf) wins, so a non-finite row is still seen
__device__ __forceinline__ uint32_t absmax8_bits(uint4 v, uint32_t m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = max(m, (w[i] << 16) & 0x7FFFFFFFu);
        m = max(m, w[i] & 0x7FFF0000u);
    }
    return m;
}

__device__ __forceinline__ void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) { return __byte_perm(a, b, sel); }

// word r of the result = byte r of a, b, c, d (4x4 byte transpose)
__device__ __forceinline__ uint4 transpose4x4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    const uint32_t t0 = prmt(a, b, 0x5140), t1 = prmt(a, b, 0x7362);
    const uint32_t t2 = prmt(c, d, 0x5140), t3 = prmt(c, d, 0x7362);
    return make_uint4(prmt(t0, t2, 0x5410), prmt(t0, t2, 0x7632), prmt(t1, t3, 0x5410), prmt(t1, t3, 0x7632));
}

struct QuantArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* descs;
    int m;
    int splits;             // blocks per linear along d_in (1 when m > 16)
    int8_t* q_ws;
    TokStats* st_ws;
    int* part;              // [linear][split][16 tokens][kPartInts] partial h and sum q (splits > 1)
    unsigned int* tickets;  // one per linear, zero between calls
    uint32_t* err;
};

constexpr int kPartInts = 20;   // 16 h + sum q, padded

__global__ void __launch_bounds__(kThreads) quant_kernel(const __grid_constant__ QuantArgs qa) {
    const dfssm_stack_entry* entries = qa.entries;
    const DevDesc* descs = qa.descs;
    const int m = qa.m;
    int8_t* __restrict__ q_ws = qa.q_ws;
    TokStats* __restrict__ st_ws = qa.st_ws;
    uint32_t* err = qa.err;
    extern __shared__ __align__(16) uint8_t smem_raw[];
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
    // [kTok][qs_row]: rows padded by 16 bytes so the 8 token rows of an MMA fragment hit 8 bank groups
    const int qs_row = d_in + kQsPad;
    int8_t* q_s = reinterpret_cast<int8_t*>(smem_raw + ((sizeof(QuantRed) + 127) & ~(size_t)127));

    const uint16_t* xg = reinterpret_cast<const uint16_t*>(e.x);
    const uint8_t* wb = reinterpret_cast<const uint8_t*>(e.w.wb);

    // split along d_in (few tokens) or along tokens (many tokens)
    const int split = qa.splits > 1 ? (int)blockIdx.x : 0;
    const int pc_lo = split * nquad / qa.splits, pc_hi = (split + 1) * nquad / qa.splits;
    const int kb_lo = 4 * pc_lo, kb_hi = 4 * pc_hi;
    const int tb0 = qa.splits > 1 ? 0 : blockIdx.x * kTokPerBlock;
    const int tb1 = min(m, tb0 + kTokPerBlock);
    for (int t0 = tb0; t0 < tb1; t0 += kTok) {
        const int nt = min(kTok, tb1 - t0);

        // ---- pass 1: amax of each token's row, one warp per token, lanes across the row
        for (int tk = warp; tk < nt; tk += kWarps) {
            const uint4* p = reinterpret_cast<const uint4*>(xg + (int64_t)(t0 + tk) * d_in);
            uint32_t am = 0u;
#pragma unroll 8
            for (int i = lane; i < (d_in >> 3); i += 32) am = absmax8_bits(p[i], am);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (lane == 0) red.amax[tk] = am;
        }
        if (tid >= nt && tid < kTok) red.amax[tid] = 0u;    // tokens past the round: q = 0
        __syncthreads();
        if (tid < kTok) {
            const float am = __uint_as_float(red.amax[tid]);
            if (tid < nt && !isfinite(am)) atomicOr(err, DFSSM_DEVERR_NONFINITE);
            red.inv[tid] = quant_inv(am);
            red.sx[tid] = quant_sx(am);
        }
        __syncthreads();

        // ---- pass 2: quantise into A fragments, h += q * W_B^T, q -> shared tile
        const float invA = red.inv[g], invB = red.inv[g + 8];
        const bool zA = invA == 0.0f, zB = invB == 0.0f;
        const bool hasA = g < nt, hasB = g + 8 < nt;
        const uint16_t* xA = xg + (int64_t)(t0 + g) * d_in + 4 * c;
        const uint16_t* xB = xg + (int64_t)(t0 + g + 8) * d_in + 4 * c;
        int D0[4] = {0, 0, 0, 0}, D1[4] = {0, 0, 0, 0};
        int sA = 0, sB = 0;
#pragma unroll 4
        for (int kb = kb_lo + warp; kb < kb_hi; kb += kWarps) {
            const int col = 32 * kb;
            const uint2 zero2 = make_uint2(0u, 0u);
            const uint2 xa0 = hasA ? *reinterpret_cast<const uint2*>(xA + col) : zero2;
            const uint2 xa1 = hasA ? *reinterpret_cast<const uint2*>(xA + col + 16) : zero2;
            const uint2 xb0 = hasB ? *reinterpret_cast<const uint2*>(xB + col) : zero2;
            const uint2 xb1 = hasB ? *reinterpret_cast<const uint2*>(xB + col + 16) : zero2;
            const uint32_t a0 = quant4(xa0, invA, zA, sA);
            const uint32_t a2 = quant4(xa1, invA, zA, sA);
            const uint32_t a1 = quant4(xb0, invB, zB, sB);
            const uint32_t a3 = quant4(xb1, invB, zB, sB);
            // B fragments: W_B rows g (n-tile 0) and g + 8 (n-tile 1), k = 4c.. and 16 + 4c..
            const uint32_t b00 = *reinterpret_cast<const uint32_t*>(wb + (int64_t)g * d_in + col + 4 * c);
            const uint32_t b01 = *reinterpret_cast<const uint32_t*>(wb + (int64_t)g * d_in + col + 16 + 4 * c);
            const uint32_t b10 = *reinterpret_cast<const uint32_t*>(wb + (int64_t)(g + 8) * d_in + col + 4 * c);
            const uint32_t b11 = *reinterpret_cast<const uint32_t*>(wb + (int64_t)(g + 8) * d_in + col + 16 + 4 * c);
            mma_s8s8(D0, a0, a1, a2, a3, b00, b01);
            mma_s8s8(D1, a0, a1, a2, a3, b10, b11);
            // the shared tile holds the round's nt tokens only
            if (hasA) {
                *reinterpret_cast<uint32_t*>(q_s + g * qs_row + col + 4 * c) = a0;
                *reinterpret_cast<uint32_t*>(q_s + g * qs_row + col + 16 + 4 * c) = a2;
            }
            if (hasB) {
                *reinterpret_cast<uint32_t*>(q_s + (g + 8) * qs_row + col + 4 * c) = a1;
                *reinterpret_cast<uint32_t*>(q_s + (g + 8) * qs_row + col + 16 + 4 * c) = a3;
            }
        }
        // quad reduction of the token sums
        sA += __shfl_xor_sync(0xffffffffu, sA, 1);
        sA += __shfl_xor_sync(0xffffffffu, sA, 2);
        sB += __shfl_xor_sync(0xffffffffu, sB, 1);
        sB += __shfl_xor_sync(0xffffffffu, sB, 2);
        if (c == 0) {
            red.sumq[warp][g] = sA;
            red.sumq[warp][g + 8] = sB;
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

        // ---- per-token scalars: thread (token tid / 16, lora row tid % 16)
        {
            const int tk = tid >> 4, k = tid & 15;
            int h = 0, sq = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) h += red.h[w][tk][k];
            if (k == 0) {
#pragma unroll
                for (int w = 0; w < kWarps; ++w) sq += red.sumq[w][tk];
            }
            bool final_block = true;
            if (qa.splits > 1) {
                int* mine = qa.part + ((int64_t)lin * qa.splits + split) * kTok * kPartInts + tk * kPartInts;
                mine[k] = h;
                if (k == 0) mine[16] = sq;
                // the block's partials are ordered before its ticket by the barrier and one
                // device-scope fence (cumulative over what the barrier made visible to thread 0)
                __syncthreads();
                __shared__ unsigned int ticket;
                if (tid == 0) {
                    __threadfence();
                    ticket = atomicAdd(qa.tickets + lin, 1u);
                }
                __syncthreads();
                final_block = ticket == (unsigned int)(qa.splits - 1);
                if (final_block) {
                    __threadfence();
                    h = 0;
                    sq = 0;
                    for (int sp = 0; sp < qa.splits; ++sp) {
                        const int* pp = qa.part + ((int64_t)lin * qa.splits + sp) * kTok * kPartInts + tk * kPartInts;
                        h += __ldcg(pp + k);
                        if (k == 0) sq += __ldcg(pp + 16);
                    }
                    if (tid == 0) qa.tickets[lin] = 0u;
                }
            }
            if (final_block && tk < nt) {
                TokStats* st = st_ws + d.st_off + t0 + tk;
                st->u[k] = __fmul_rn(e.w.sb[k], (float)h);
                if (e.dbg.h) e.dbg.h[(int64_t)(t0 + tk) * kRank + k] = h;
                if (k == 0) {
                    st->sx = red.sx[tk];
                    st->sumq = sq;
                    if (e.dbg.sx) e.dbg.sx[t0 + tk] = red.sx[tk];
                }
            }
        }

        // ---- q out: token tk, 128-column piece pc = half hc of segment sg. For each 32-column
        // group c4 of the piece, words W0..W7 of the natural bytes give plane p's four bytes
        // (columns 32c + 8i + p, i = 0..3) as byte p % 4 of W[p / 4], W[2 + p / 4], W[4 + p / 4],
        // W[6 + p / 4]; the four groups' words of plane p form one 16-byte piece.
        const int npc = pc_hi - pc_lo;
        // the decode kernel (m <= 16) quantises into its own shared memory; only the prefill reads rows
        const bool rows = m > kDecodeMaxTokens;
        for (int i = tid; i < nt * npc; i += kThreads) {
            const int tk = i / npc, pc = pc_lo + (i - tk * npc);
            const int sg = pc >> 1, hc = pc & 1, t = t0 + tk;
            const uint32_t* src = reinterpret_cast<const uint32_t*>(q_s + tk * qs_row + 128 * pc);
            if (rows) {
                uint32_t P[8][4];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t* W = src + 8 * c4;
                    const uint4 lo = transpose4x4(W[0], W[2], W[4], W[6]);   // planes 0..3
                    const uint4 hi = transpose4x4(W[1], W[3], W[5], W[7]);   // planes 4..7
                    P[0][c4] = lo.x; P[1][c4] = lo.y; P[2][c4] = lo.z; P[3][c4] = lo.w;
                    P[4][c4] = hi.x; P[5][c4] = hi.y; P[6][c4] = hi.z; P[7][c4] = hi.w;
                }
                // plane p of segment sg, K half hc: 16 bytes at 256 sg + 32 p + 16 hc of the token row
                int8_t* base = q_ws + d.q_off + (int64_t)t * d.qrow + 256 * sg + 16 * hc;
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    *reinterpret_cast<uint4*>(base + 32 * p) = make_uint4(P[p][0], P[p][1], P[p][2], P[p][3]);
            }
            if (e.dbg.q) {
                const uint4* sq = reinterpret_cast<const uint4*>(src);
                uint4* dq = reinterpret_cast<uint4*>(e.dbg.q + (int64_t)t * d_in + 128 * pc);
#pragma unroll
                for (int u = 0; u < 8; ++u) dq[u] = sq[u];
            }
        }
        __syncthreads();   // q_s and red are reused by the next round
    }
}

}  // namespace

cudaError_t launch_quant_rows(const LaunchCtx& c);

cudaError_t launch_quant(const LaunchCtx& c) {
    if (c.m > kDecodeMaxTokens) return launch_quant_rows(c);
    int splits = 1;
    if (c.m <= kTok) {
        // enough blocks to cover the SMs twice, at least two 128-column pieces (8 k-blocks,
        // one per warp) per split
        int min_pc = 1 << 30;
        for (int i = 0; i < c.n; ++i) min_pc = min(min_pc, c.host_desc[i].d_in / 128);
        splits = (2 * c.sm_count + c.n - 1) / c.n;
        splits = max(1, min(splits, min(kMaxSplits, min_pc / 2)));
    }
    dim3 grid(splits > 1 ? splits : (c.m + kTokPerBlock - 1) / kTokPerBlock, c.n);
    const size_t smem = ((sizeof(QuantRed) + 127) & ~(size_t)127) + (size_t)kTok * (c.max_d_in + kQsPad);
    QuantArgs qa{c.entries, c.single, c.desc, c.m, splits, c.q_ws, c.st_ws, c.part, c.tickets, c.err};
    quant_kernel<<<grid, kThreads, smem, c.stream>>>(qa);
    return cudaGetLastError();
}

cudaError_t set_quant_attr(int optin) { return allow_dyn_smem(quant_kernel, optin); }

}  // namespace dfssm
