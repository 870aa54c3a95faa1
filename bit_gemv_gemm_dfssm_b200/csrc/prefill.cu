// Prefill path (many tokens): the scaffold contraction as a dense int8 GEMM on
// the 5th-generation tensor cores (tcgen05, accumulators in TMEM), with the
// LoRA up-projection and both dequantisation epilogues fused.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C:
// packed 1-bit scaffold weights are expanded on the fly to int8 and multiplied
// on INT8 tensor cores. With many tokens the contraction is a dense GEMM
// (2 * d_in ops per token per output row), so here the expansion happens in
// registers and tensor memory, once per 128-row x 128-column weight block, and
// the block is reused by 192 tokens:
//
//   D[o, t] = sum_k b[o, k] * q[t, k]    (b = sign bit as 0/1, int32 in TMEM)
//   acc     = 2 * D - sum_k q[t, k]       (a +-1 weight is 2b - 1)
//
// Persistent kernel, one CTA per SM, 16 warps with fixed roles:
//   warp 0      TMA producer: 192-token x 128-byte tiles of the int8
//               activations (permuted column order, 128B swizzle), no multicast
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma.kind::i8 with A in TMEM,
//               M=128 rows, N=192 tokens, K=32 per instruction, 4 per 128-column
//               block
//   warps 4-7   bit expansion: each thread owns one weight row of the tile (its
//               TMEM lane), loads the 32 sign bytes of a 256-column segment and
//               stores, per 128-byte k-block (four bit planes of that segment, the
//               activation order of dfssm_internal.cuh), 128 0/1 bytes into the
//               k-block's TMEM stage with one tcgen05.st (no shared-memory traffic
//               for the weights: shared memory carries only the activation tiles)
//   warps 8-15  epilogue over its 32 TMEM lanes (= output rows) and half of the
//               192 token columns, 16 tokens at a time: tcgen05.ld in the
//               16x256b shape, which is the register layout of an mma.sync
//               m16n8 accumulator, acc = 2D - sum q; the LoRA up-projection
//               W_A u as bf16 warp MMAs in that same layout (W_A exact in bf16,
//               u split into bf16 hi + lo, fp32 accumulation); dequantisation
//               and stores. The per-token scalars and the hi/lo u of each
//               16-token chunk are staged in a warp-private, double-buffered
//               smem slice
// 4-stage ring (activation tiles in shared memory, expanded weights in TMEM,
// mbarriers), two TMEM accumulator buffers of 192 columns so the epilogue of one
// tile overlaps the main loop of the next (2 x 192 + 4 x 32 = 512 columns).
// Every mbarrier wait is bounded; a timeout sets the plan's error word.
#include <cuda.h>

#include <type_traits>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int BM = 128;            // output rows per tile (MMA M, TMEM lanes)
constexpr int BN = 192;            // tokens per tile (MMA N, TMEM columns)
constexpr int BK = 128;            // k (bytes) per TMA box (the 128-byte swizzle span)
constexpr int SEG = kSegCols;      // k (bytes) per pipeline stage: one 256-column segment, 8 MMAs
constexpr int A_STAGES = 2;        // expanded-weight stages (TMEM)
constexpr int B_STAGES = 3;        // activation stages (shared memory)
constexpr int B_HALF = BN * BK;    // 24 KB: one TMA box, K bytes 128 h .. of the segment
constexpr int B_STAGE = 2 * B_HALF;
// TMEM: two accumulator buffers of BN columns, then the A stages, SEG / 4 columns each
// (4 int8 per 32-bit column, one weight row per lane)
constexpr uint32_t A_COL0 = 2 * BN;
constexpr uint32_t A_COLS = SEG / 4;
constexpr int NUM_THREADS = 16 * 32;
constexpr int EPI_WARPS = 8;                         // warps 8..15
constexpr int EPI_THREADS = EPI_WARPS * 32;
// staged per 16-token chunk: s_x[16], sum q[16], then u as bf16 pairs (k = 2j, 2j + 1), hi and lo,
// in rows of 12 words so the B-fragment loads of a warp hit distinct banks
constexpr int U_ROW = 12;                                 // words per token row (8 used)
constexpr int STAT_CHUNK = 128 + 2 * 16 * U_ROW * 4;      // 1664 B
constexpr int STAT_BYTES = EPI_WARPS * 2 * STAT_CHUNK;  // double-buffered, one pair per epilogue warp
// descriptor and stack entry of the first kLinCache linears, copied to shared memory at the
// start: every role looks up each tile's linear, and chains of dependent global loads there
// would stall the pipeline at every tile boundary
constexpr int kLinCache = 256;
struct LinCache {
    DevDesc d;
    dfssm_stack_entry e;
};
constexpr int LIN_CACHE_BYTES = kLinCache * (int)sizeof(LinCache);
constexpr int SMEM_BYTES = B_STAGES * B_STAGE + STAT_BYTES + 256 + LIN_CACHE_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
static_assert(A_COL0 + A_STAGES * A_COLS <= TMEM_COLS, "TMEM budget");
static_assert(B_HALF % 1024 == 0, "SWIZZLE_128B atoms");

struct PrefillArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* desc;          // desc[0] is the first linear of this launch
    const CUtensorMap* tmaps;     // tmaps[l] maps linear l's q rows (same indexing as desc)
    int n;
    int m;
    int n_tiles;
    const TokStats* st_ws;
    uint32_t* err;
};

// K-major, 128-byte swizzle shared-memory matrix descriptor: 8-row x 128-byte
// atoms stacked every 1024 bytes (SBO), leading offset 1 (unused for this
// layout), descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::i8 instruction descriptor: D s32, A s8, B s8, both K-major, N = BN, M = BM.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct TileCoord {
    int lin, row0, tok0;
};

__device__ __forceinline__ const DevDesc& lin_desc(const PrefillArgs& a, const LinCache* lc, int l) {
    return l < kLinCache ? lc[l].d : a.desc[l];
}
__device__ __forceinline__ const dfssm_stack_entry& lin_entry(const PrefillArgs& a, const LinCache* lc, int l) {
    return l < kLinCache ? lc[l].e : entry_at(a.entries, a.single, l);
}

__device__ __forceinline__ TileCoord tile_coord(const PrefillArgs& a, const LinCache* lc, int n_tt, int tile) {
    const int rt = tile / n_tt;                 // global 128-row tile index
    const int tt = tile - rt * n_tt;
    const int base = lin_desc(a, lc, 0).rt_begin;
    int lo = 0, hi = a.n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (lin_desc(a, lc, mid).rt_begin - base <= rt) lo = mid; else hi = mid - 1;
    }
    TileCoord c;
    c.lin = lo;
    c.row0 = (rt - (lin_desc(a, lc, lo).rt_begin - base)) * BM;
    c.tok0 = tt * BN;
    return c;
}

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }


// Spin on a phase with the non-blocking probe (no suspend, so the waiter reacts as soon as the
// phase completes); bounded by time like ptx::mbar_wait. Used where the hand-off latency is on
// the critical path: the expansion warps refilling a TMEM stage the MMAs just released.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(ptx::smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_spin(uint64_t* bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (!mbar_test(bar, parity)) {
        if (ptx::globaltimer() - t0 > 1000000000ull) return false;
    }
    return true;
}
__device__ __forceinline__ uint64_t globaltimer_elapsed(uint64_t t0) { return ptx::globaltimer() - t0; }

// Wait for two mbarrier phases at once: the two probes go out back to back, so their latencies
// overlap. Bounded like ptx::mbar_wait; false on timeout.
__device__ __forceinline__ bool mbar_wait2(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1) {
    bool r0 = ptx::mbar_try_wait(b0, p0), r1 = ptx::mbar_try_wait(b1, p1);
    if (r0 && r1) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (!(r0 && r1)) {
        if (!r0) r0 = ptx::mbar_try_wait(b0, p0);
        if (!r1) r1 = ptx::mbar_try_wait(b1, p1);
        if (globaltimer_elapsed(t0) > 1000000000ull) return false;
    }
    return true;
}

__global__ void __launch_bounds__(NUM_THREADS, 1) prefill_kernel(const __grid_constant__ PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (SWIZZLE_128B atoms), offset from the __shared__ array so the
    // compiler keeps shared-memory addressing
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sB = smem;
    uint8_t* sStat = sB + B_STAGES * B_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sStat + STAT_BYTES);
    LinCache* lc = reinterpret_cast<LinCache*>(sStat + STAT_BYTES + 256);
    uint64_t* full_a = bars;                         // [A_STAGES], 128 arrivals (TMEM stores done)
    uint64_t* empty_a = full_a + A_STAGES;           // [A_STAGES], MMA commit
    uint64_t* full_b = empty_a + A_STAGES;           // [B_STAGES], TMA transaction bytes
    uint64_t* empty_b = full_b + B_STAGES;           // [B_STAGES], MMA commit
    uint64_t* acc_full = empty_b + B_STAGES;         // [2], MMA commit
    uint64_t* acc_empty = acc_full + 2;              // [2], EPI_THREADS epilogue arrivals
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tt = (a.m + BN - 1) / BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < A_STAGES; ++s) {
            ptx::mbar_init(&full_a[s], 128);
            ptx::mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < B_STAGES; ++s) {
            ptx::mbar_init(&full_b[s], 1);
            ptx::mbar_init(&empty_b[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&acc_full[b], 1);
            ptx::mbar_init(&acc_empty[b], EPI_THREADS);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    for (int l = threadIdx.x; l < a.n && l < kLinCache; l += NUM_THREADS) {
        lc[l].d = a.desc[l];
        lc[l].e = entry_at(a.entries, a.single, l);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (activations)
        if (lane == 0) {
            ptx::pdl_wait();
            int it = 0;
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x) {
                const TileCoord tc = tile_coord(a, lc, n_tt, tile);
                const CUtensorMap* tm = a.tmaps + tc.lin;
                const int nseg = lin_desc(a, lc, tc.lin).qrow / SEG;
                for (int sg = 0; sg < nseg; ++sg, ++it) {
                    const int s = it % B_STAGES;
                    const uint32_t ph = (uint32_t)(it / B_STAGES) & 1u;
                    if (!ptx::mbar_wait(&empty_b[s], ph ^ 1u)) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; break; }
                    ptx::mbar_arrive_expect_tx(&full_b[s], B_STAGE);
                    ptx::tma_load_2d(sB + s * B_STAGE, tm, sg * SEG, tc.tok0, &full_b[s]);
                    ptx::tma_load_2d(sB + s * B_STAGE + B_HALF, tm, sg * SEG + BK, tc.tok0, &full_b[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int ita = 0, itb = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x, ++tcount) {
                const TileCoord tc = tile_coord(a, lc, n_tt, tile);
                const int nseg = lin_desc(a, lc, tc.lin).qrow / SEG;
                const int buf = tcount & 1;
                const uint32_t acc_ph = (uint32_t)(tcount >> 1) & 1u;
                if (!ptx::mbar_wait(&acc_empty[buf], acc_ph ^ 1u)) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
                bool ok = true;
                for (int sg = 0; sg < nseg; ++sg, ++ita, ++itb) {
                    const int sa = ita % A_STAGES, sb = itb % B_STAGES;
                    if (!mbar_wait2(&full_a[sa], (uint32_t)(ita / A_STAGES) & 1u, &full_b[sb],
                                    (uint32_t)(itb / B_STAGES) & 1u)) {
                        set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; ok = false; break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_tmem = tmem_base + A_COL0 + (uint32_t)sa * A_COLS;
                    // segment half h = B box h; +32 bytes along K: +8 TMEM columns for A, +2 in the
                    // 16-byte address field for B
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t bdesc = sw128_desc(ptx::smem_u32(sB + sb * B_STAGE + h * B_HALF));
#pragma unroll
                        for (int kk = 0; kk < BK / 32; ++kk)
                            ptx::mma_i8_ts(d_tmem, a_tmem + 32 * h + 8 * kk, bdesc + 2 * kk, kIdesc, (sg | h | kk) != 0);
                    }
                    ptx::mma_commit(&empty_a[sa]);
                    ptx::mma_commit(&empty_b[sb]);
                }
                if (!ok) break;
                ptx::mma_commit(&acc_full[buf]);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ bit expansion (one weight row per thread)
        // The sign bytes of this thread's row are loaded two segments ahead, across tile
        // boundaries too: the first segments of the next tile are in flight while the last ones
        // of this tile are expanded.
        const int r = threadIdx.x - 128;
        struct RowSrc {
            const uint8_t* src;
            int nseg, rb;
            bool valid;
        };
        auto row_src = [&](int tile) {
            RowSrc rs{nullptr, 0, 0, false};
            if (tile < a.n_tiles) {
                const TileCoord tc = tile_coord(a, lc, n_tt, tile);
                const DevDesc& d = lin_desc(a, lc, tc.lin);
                const dfssm_stack_entry& e = lin_entry(a, lc, tc.lin);
                rs.nseg = d.qrow / kSegCols;
                rs.rb = d.d_in >> 3;
                const int o = tc.row0 + r;
                rs.valid = o < d.d_out && entry_ptrs_ok(e);
                rs.src = e.w.sign + (int64_t)(rs.valid ? o : 0) * rs.rb;
            }
            return rs;
        };
        // segment sg of a row: words 0..3 and 4..7 (the second half is absent in a final half segment)
        auto load_seg = [&](const RowSrc& rs, int sg, uint4& lo, uint4& hi) {
            lo = make_uint4(0, 0, 0, 0);
            hi = make_uint4(0, 0, 0, 0);
            if (rs.valid && sg < rs.nseg) {
                lo = __ldg(reinterpret_cast<const uint4*>(rs.src + 32 * sg));
                if (32 * sg + 16 < rs.rb) hi = __ldg(reinterpret_cast<const uint4*>(rs.src + 32 * sg + 16));
            }
        };
        // this row is TMEM lane r (the warp's lane quarter 32 (warp - 4) .. + 31)
        const uint32_t a_lane = tmem_base + ((uint32_t)(32 * (warp - 4)) << 16) + A_COL0;
        int it = 0;
        RowSrc cur = row_src(blockIdx.x), nxt = row_src(blockIdx.x + gridDim.x);
        uint4 c_lo, c_hi, n_lo, n_hi;          // the next two segments of the stream
        int have = 0;                          // how many of them belong to `cur` and are loaded
        for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x) {
            if (have < 1) load_seg(cur, 0, c_lo, c_hi);
            if (have < 2) load_seg(cur, 1, n_lo, n_hi);
            bool ok = true;
            for (int sg = 0; sg < cur.nseg && ok; ++sg, ++it) {
                const uint32_t w[8] = {c_lo.x, c_lo.y, c_lo.z, c_lo.w, c_hi.x, c_hi.y, c_hi.z, c_hi.w};
                c_lo = n_lo;
                c_hi = n_hi;
                // the segment two ahead: this tile's, else the next tile's first ones
                const int k = sg + 2;
                if (k < cur.nseg) load_seg(cur, k, n_lo, n_hi);
                else load_seg(nxt, k - cur.nseg, n_lo, n_hi);
                // segment sg: K byte 32 p + 4 c + i is plane p (0/1 bytes), i.e. TMEM column 8 p + c of
                // the stage holds (w[c] >> p) & 0x01010101. Expanded before waiting for the stage, so
                // that only the two 32-column stores follow the wait
                uint32_t e[2][32];
#pragma unroll
                for (int p = 0; p < 8; ++p)
#pragma unroll
                    for (int c = 0; c < 8; ++c) e[p >> 2][8 * (p & 3) + c] = (w[c] >> p) & 0x01010101u;
                const int s = it % A_STAGES;
                // one lane polls, the warp follows
                bool got = true;
                if ((threadIdx.x & 31) == 0) got = mbar_spin(&empty_a[s], ((uint32_t)(it / A_STAGES) & 1u) ^ 1u);
                got = __shfl_sync(0xffffffffu, got, 0);
                __syncwarp();
                if (!got) { if ((threadIdx.x & 31) == 0) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; } ok = false; break; }
                ptx::tc_fence_after();                 // the MMAs that read this stage have completed
                ptx::tmem_st_32x32b_x32(a_lane + (uint32_t)s * A_COLS, e[0]);
                ptx::tmem_st_32x32b_x32(a_lane + (uint32_t)s * A_COLS + 32u, e[1]);
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&full_a[s]);
            }
            if (!ok) break;
            // the last two look-ahead loads of this tile fetched the next tile's segments 0 and 1
            // (a one-segment tile reached only its segment 1: start over)
            have = cur.nseg >= 2 ? min(2, nxt.nseg) : 0;
            cur = nxt;
            nxt = row_src(tile + 2 * gridDim.x);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------ epilogue
        // warp 8 + 4h + q4 handles TMEM lanes 32 q4 .. (output rows) and token columns
        // [128h, 128h + 128); lane (g, c) = (lane / 4, lane % 4) holds, in mma-fragment order,
        // rows 32 q4 + 16 rt + g + 8 hh (rt, hh = 0, 1) and tokens 8 tt + 2c + e (tt, e = 0, 1)
        ptx::pdl_wait();
        const int q4 = warp & 3;
        const int half = (warp - 8) >> 2;
        const int g = lane >> 2, cq = lane & 3;
        uint8_t* stat_buf = sStat + (warp - 8) * 2 * STAT_CHUNK;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x, ++tcount) {
            const TileCoord tc = tile_coord(a, lc, n_tt, tile);
            const DevDesc d = lin_desc(a, lc, tc.lin);
            const dfssm_stack_entry& e = lin_entry(a, lc, tc.lin);
            const bool lin_ok = entry_ptrs_ok(e);
            // entry fields in registers: the stores below must not force reloads
            void* const y_ptr = e.y;
            int32_t* const dbg_acc = e.dbg.acc;
            const bool y_bf16 = d.y_dtype == DFSSM_BF16;
            const int d_out = d.d_out;
            // this thread's 4 rows: alpha, s_A, and the W_A rows as bf16 A fragments
            int orow[2][2];
            bool rok[2][2];
            float alpha[2][2], sa[2][2];
            uint32_t afr[2][4];
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                uint32_t wlo[2], whi[2];     // k = 2c, 2c+1 and 2c+8, 2c+9 of rows g, g + 8 (int8 pairs)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int o = tc.row0 + 32 * q4 + 16 * rt + g + 8 * hh;
                    orow[rt][hh] = o;
                    rok[rt][hh] = lin_ok && o < d_out;
                    alpha[rt][hh] = 0.f;
                    sa[rt][hh] = 0.f;
                    wlo[hh] = whi[hh] = 0u;
                    if (rok[rt][hh]) {
                        alpha[rt][hh] = e.w.alpha[o];
                        sa[rt][hh] = e.w.sa[o];
                        const uint16_t* wrow = reinterpret_cast<const uint16_t*>(e.w.wa + (int64_t)o * kRank);
                        wlo[hh] = wrow[cq];
                        whi[hh] = wrow[4 + cq];
                    }
                }
                afr[rt][0] = int8_pair_to_bf16x2(wlo[0]);
                afr[rt][1] = int8_pair_to_bf16x2(wlo[1]);
                afr[rt][2] = int8_pair_to_bf16x2(whi[0]);
                afr[rt][3] = int8_pair_to_bf16x2(whi[1]);
            }
            float2 alpha2[2][2], sa2[2][2];
#pragma unroll
            for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    alpha2[rt][hh] = make_float2(alpha[rt][hh], alpha[rt][hh]);
                    sa2[rt][hh] = make_float2(sa[rt][hh], sa[rt][hh]);
                }
            uint16_t* const yb = reinterpret_cast<uint16_t*>(y_ptr);
            float* const yf = reinterpret_cast<float*>(y_ptr);
            // this warp's 32 rows as 16-byte row pieces per token: bf16, no debug export, all 32 rows
            // inside d_out and d_out a multiple of 8 (16-byte aligned token rows)
            const int orow_base = tc.row0 + 32 * q4;
            const bool vec_store = lin_ok && y_bf16 && dbg_acc == nullptr && (d_out & 7) == 0 &&
                                   orow_base + 32 <= d_out;
            // per-token scalars and u of chunk ch (tokens tok_base + 16 ch ..): lane l takes token
            // l / 2 and u[8 (l % 2) ..]; s_x and sum q from the even lanes
            const int tok_base = tc.tok0 + half * (BN / 2);
            const TokStats* st_src = a.st_ws + d.st_off;
            const int tl = lane >> 1, kh = lane & 1;
            struct Staged {
                float4 u0, u1;
                float sx;
                int sumq;
            };
            auto load_chunk = [&](int ch, Staged& sg) {
                const int tok = tok_base + 16 * ch + tl;
                sg.u0 = sg.u1 = make_float4(0.f, 0.f, 0.f, 0.f);
                sg.sx = 0.f;
                sg.sumq = 0;
                if (tok < a.m) {
                    const TokStats* st = st_src + tok;
                    sg.u0 = *reinterpret_cast<const float4*>(st->u + 8 * kh);
                    sg.u1 = *reinterpret_cast<const float4*>(st->u + 8 * kh + 4);
                    sg.sx = st->sx;
                    sg.sumq = st->sumq;
                }
            };
            auto store_chunk = [&](int buf_i, const Staged& sg) {
                uint8_t* base = stat_buf + buf_i * STAT_CHUNK;
                uint32_t h[4], l[4];
                split_bf16x2(sg.u0.x, sg.u0.y, h[0], l[0]);
                split_bf16x2(sg.u0.z, sg.u0.w, h[1], l[1]);
                split_bf16x2(sg.u1.x, sg.u1.y, h[2], l[2]);
                split_bf16x2(sg.u1.z, sg.u1.w, h[3], l[3]);
                uint32_t* uhi = reinterpret_cast<uint32_t*>(base + 128);
                uint32_t* ulo = uhi + 16 * U_ROW;
                *reinterpret_cast<uint4*>(uhi + tl * U_ROW + 4 * kh) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(ulo + tl * U_ROW + 4 * kh) = make_uint4(l[0], l[1], l[2], l[3]);
                if (kh == 0) {
                    reinterpret_cast<float*>(base)[tl] = sg.sx;
                    reinterpret_cast<int*>(base + 64)[tl] = sg.sumq;
                }
            };
            Staged sg;
            load_chunk(0, sg);
            store_chunk(0, sg);

            const int buf = tcount & 1;
            const uint32_t acc_ph = (uint32_t)(tcount >> 1) & 1u;
            bool got = true;
            if (lane == 0) got = ptx::mbar_wait(&acc_full[buf], acc_ph);
            got = __shfl_sync(0xffffffffu, got, 0);
            __syncwarp();
            if (!got) {
                if (lane == 0) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; }
                break;
            }
            ptx::tc_fence_after();
            const uint32_t tcol = tmem_base + (uint32_t)(buf * BN + half * (BN / 2));
            constexpr int NCH = BN / 2 / 16;
            for (int ch = 0; ch < NCH; ++ch) {
                __syncwarp();
                const int t0c = tok_base + 16 * ch;
                const bool more = ch + 1 < NCH && t0c + 16 < a.m;
                if (more) load_chunk(ch + 1, sg);
                uint32_t v[2][8];
#pragma unroll
                for (int rt = 0; rt < 2; ++rt)
                    ptx::tmem_ld_16x256b_x2(tcol + ((uint32_t)(32 * q4 + 16 * rt) << 16) + (uint32_t)(16 * ch), v[rt]);
                ptx::tmem_ld_wait();
                if (t0c < a.m) {
                    const uint8_t* base = stat_buf + (ch & 1) * STAT_CHUNK;
                    const uint32_t* uhi = reinterpret_cast<const uint32_t*>(base + 128);
                    const uint32_t* ulo = uhi + 16 * U_ROW;
                    // W_A u for the 32 rows x 16 tokens of the chunk: hi then lo, fp32 accumulation
                    float lora[2][2][4];
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const int tk = 8 * tt + g;
                        const uint32_t bh0 = uhi[tk * U_ROW + cq], bh1 = uhi[tk * U_ROW + 4 + cq];
                        const uint32_t bl0 = ulo[tk * U_ROW + cq], bl1 = ulo[tk * U_ROW + 4 + cq];
#pragma unroll
                        for (int rt = 0; rt < 2; ++rt) {
                            float* dd = lora[rt][tt];
                            dd[0] = dd[1] = dd[2] = dd[3] = 0.f;
                            ptx::mma_bf16_16816(lora[rt][tt], afr[rt][0], afr[rt][1], afr[rt][2], afr[rt][3], bh0, bh1);
                            ptx::mma_bf16_16816(lora[rt][tt], afr[rt][0], afr[rt][1], afr[rt][2], afr[rt][3], bl0, bl1);
                        }
                    }
                    // y for rows (rt, hh) and the token pair (2 cq, 2 cq + 1) of n-tile tt, in packed fp32
                    // pairs: acc = 2 D - sum q as fp32 (the 1.5 * 2^23 bias, exact below 2^22), then
                    // y = s_x (alpha acc + s_A (W_A u)) with the same roundings as the scalar form
                    const float* sx_s = reinterpret_cast<const float*>(base);
                    const int* sq_s = reinterpret_cast<const int*>(base + 64);
                    float2 sx2[2];
                    int kq[2][2];                              // 0x4B400000 - sum q per token
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const int tj = 8 * tt + 2 * cq;
                        sx2[tt] = make_float2(sx_s[tj], sx_s[tj + 1]);
                        kq[tt][0] = 0x4B400000 - sq_s[tj];
                        kq[tt][1] = 0x4B400000 - sq_s[tj + 1];
                    }
                    float2 y2[2][2][2];                        // [rt][hh][tt]
#pragma unroll
                    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                            for (int tt = 0; tt < 2; ++tt) {
                                const int i0 = 4 * tt + 2 * hh;
                                const float2 accf = fadd2(
                                    make_float2(__int_as_float(2 * (int)v[rt][i0] + kq[tt][0]),
                                                __int_as_float(2 * (int)v[rt][i0 + 1] + kq[tt][1])),
                                    make_float2(-12582912.0f, -12582912.0f));
                                const float2 l2 = make_float2(lora[rt][tt][2 * hh], lora[rt][tt][2 * hh + 1]);
                                y2[rt][hh][tt] = fmul2(sx2[tt], ffma2(alpha2[rt][hh], accf, fmul2(sa2[rt][hh], l2)));
                            }
                    __syncwarp();                              // every lane is done with this chunk's staged values
                    if (vec_store) {
                        // bf16 pairs in the mma C layout -> stmatrix.trans into the chunk's (now free) staging
                        // buffer as [16 tokens][32 rows], 16-byte pieces swizzled by (token / 2) % 4; then each
                        // lane stores two 16-byte row pieces of one token
                        const uint32_t stg = ptx::smem_u32(base);
#pragma unroll
                        for (int tt = 0; tt < 2; ++tt) {
                            const int r = lane & 7, mi = lane >> 3;      // this lane addresses row r of matrix mi
                            const uint32_t addr = stg + (uint32_t)((8 * tt + r) * 64 + 16 * (mi ^ ((r >> 1) & 3)));
                            ptx::stmatrix_x4_trans(addr, bf16x2_of(y2[0][0][tt]), bf16x2_of(y2[0][1][tt]),
                                                   bf16x2_of(y2[1][0][tt]), bf16x2_of(y2[1][1][tt]));
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int j = (lane >> 2) + 8 * i, c = lane & 3;
                            const uint4 piece = ptx::lds128(stg + (uint32_t)(j * 64 + 16 * (c ^ ((j >> 1) & 3))));
                            if (t0c + j < a.m)
                                *reinterpret_cast<uint4*>(yb + (int64_t)(t0c + j) * d_out + orow_base + 8 * c) = piece;
                        }
                    } else {
                        // element (rt, hh, tt, ee): row orow[rt][hh], token t0c + 8 tt + 2 cq + ee, with the
                        // validity of row and token as store predicates
                        auto elements = [&](auto store_y, auto dbg_tag) {
                            constexpr bool kDbg = decltype(dbg_tag)::value;
#pragma unroll
                            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                                for (int ee = 0; ee < 2; ++ee) {
                                    const int t = t0c + 8 * tt + 2 * cq + ee;
                                    const bool tok_ok = t < a.m;
#pragma unroll
                                    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                                        for (int hh = 0; hh < 2; ++hh) {
                                            const float y = ee ? y2[rt][hh][tt].y : y2[rt][hh][tt].x;
                                            const bool ok = tok_ok && rok[rt][hh];
                                            const int64_t idx = (int64_t)t * d_out + orow[rt][hh];
                                            store_y(ok, idx, y);
                                            if constexpr (kDbg) {
                                                const int acc = 2 * (int)v[rt][4 * tt + 2 * hh + ee] -
                                                                (0x4B400000 - kq[tt][ee]);
                                                if (ok) dbg_acc[idx] = acc;
                                            }
                                        }
                                }
                        };
                        auto st_bf16 = [&](bool ok, int64_t idx, float y) {
                            const uint16_t b = f32_to_bf16_bits(y);
                            if (ok) yb[idx] = b;
                        };
                        auto st_f32 = [&](bool ok, int64_t idx, float y) {
                            if (ok) yf[idx] = y;
                        };
                        using kNo = std::integral_constant<bool, false>;
                        using kYes = std::integral_constant<bool, true>;
                        if (dbg_acc == nullptr) {
                            if (y_bf16) elements(st_bf16, kNo{}); else elements(st_f32, kNo{});
                        } else {
                            if (y_bf16) elements(st_bf16, kYes{}); else elements(st_f32, kYes{});
                        }
                    }
                }
                __syncwarp();
                if (more) store_chunk((ch + 1) & 1, sg);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&acc_empty[buf]);
        }
    }

    // ------------------------------------------------ teardown
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace

cudaError_t launch_prefill(const LaunchCtx& c) {
    int row_tiles = 0;
    for (int i = 0; i < c.n; ++i) row_tiles += (c.host_desc[i].d_out + BM - 1) / BM;
    const int n_tt = (c.m + BN - 1) / BN;
    PrefillArgs a{c.entries, c.single, c.desc, reinterpret_cast<const CUtensorMap*>(c.tmaps), c.n, c.m,
                  row_tiles * n_tt, c.st_ws, c.err};
    const int grid = c.sm_count < a.n_tiles ? c.sm_count : a.n_tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel, a);
}

cudaError_t set_prefill_attr(int optin) {
    return cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                optin < SMEM_BYTES ? optin : SMEM_BYTES);
}

int prefill_box_tokens() { return BN; }
int prefill_box_bytes() { return BK; }

}  // namespace dfssm
