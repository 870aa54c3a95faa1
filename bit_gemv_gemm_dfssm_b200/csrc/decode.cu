// Decode path (1 <= m <= 16 tokens): the scaffold contraction streamed from HBM
// on the tcgen05 tensor cores, with the LoRA up-projection and both
// dequantisation epilogues fused.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C:
// the 1-bit scaffold weights are expanded on the fly to int8 and fed to int8
// tensor cores, which cuts weight traffic 8x against int8 weights; at batch 1
// the layer is bound by that weight stream. The expansion is the only work
// left on the SM's integer pipes here:
//
//  * Bit planes. For a 32-bit word w of sign bits (columns 32c .. 32c+31 of a
//    256-column segment) and a bit position p, w & (0x01010101 << p) is four
//    bytes, each 0 or 2^p: the bits of columns 32c + 8i + p (i = 0..3), scaled
//    by 2^p. One LOP3 expands four weights. The eight words of a segment give,
//    for each p, 32 bytes: the K = 32 operand of one int8 MMA.
//  * A operand in tensor memory. Each expander thread owns one of the 128 rows
//    of a tile (= one TMEM lane) and writes its 64 expanded words with
//    tcgen05.st; the MMA reads A from TMEM, so the 8x larger expanded operand
//    never passes through shared memory. Planes 0-3 are taken as
//    (w >> p) & 0x01010101 (bytes 0 or 1), planes 4-7 as (w >> p) & 0x10101010
//    (bytes 0 or 16), so two int32 accumulators per tile suffice:
//    D_lo = sum_{p<4} S_p and D_hi = 16 * sum_{p>=4} S_p, exactly.
//  * B operand: the int8 activations of up to 16 tokens (MMA N = 16) in the
//    same plane-major order (K position 32p + 4c + i <-> column 32c + 8i + p),
//    copied once per linear into shared memory as 8-row x 16-byte core
//    matrices (the quantisation kernel writes them in that layout).
//  * S1 = D_lo + D_hi / 16 = sum_{bit = 1} q, and acc = 2 * S1 - sum_j q (a +-1
//    weight is 2b - 1).
//
// Persistent kernel, one CTA per SM, 16 warps with fixed roles:
//   warp 0       TMA producer of sign tiles (128 rows x 128 bytes, 128B swizzle,
//                no multicast) through a per-linear tensor map whose global
//                address it sets on the device (tensormap.replace); 4 stages
//   warp 1       TMEM owner; bulk copy of each linear's activation image
//   warps 4-11   two expander warpgroups taking alternate 256-column segments
//                of a tile; a group writes a segment into one of its three TMEM
//                slots and hands it over at a named barrier
//   warps 2, 3   one MMA issuer per group: after the barrier it issues the
//                segment's 8 MMAs (tcgen05.mma.kind::i8, A in TMEM) into the
//                group's own pair of accumulators. Two issue streams, each a
//                single thread (so each accumulator is written in issue order),
//                and a hardware barrier instead of an mbarrier round trip per
//                segment
//   warps 12-15  epilogue: add the groups' accumulators, LoRA up-projection,
//                dequantisation (epilogue.cuh), coalesced stores
// Work: the 128-row tiles of all linears of the call, split into contiguous
// ranges holding equal shares of the sign bytes. Every mbarrier wait is
// bounded; a timeout sets the error word, later waits return at once, and the
// CTA runs to its end without blocking.
#include <cuda.h>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int BM = 128;                    // rows per tile: MMA M, TMEM lanes
constexpr int NTOK = 16;                   // MMA N: token columns (columns >= m are dropped)
constexpr int STAGE_ROW_BYTES = 128;       // sign bytes per row per TMA stage (4 segments)
constexpr int SIGN_STAGE = BM * STAGE_ROW_BYTES;   // 16 KB
constexpr int NS = 4;                      // sign ring stages
constexpr int NGRP = 2;                    // expander / issuer warpgroups
constexpr int NSLOT = 3;                   // TMEM A slots per group
constexpr uint32_t A_COLS = 64;            // TMEM columns per A slot: 8 planes x 8 words
constexpr uint32_t D_COLS = 2 * NTOK;      // accumulators of one group and buffer: lo, hi (16 tokens each)
constexpr uint32_t A_COL0 = NGRP * 2 * D_COLS;   // A slots after [group][buffer] accumulators
constexpr uint32_t TMEM_COLS = 512;
static_assert(A_COL0 + NGRP * NSLOT * A_COLS <= TMEM_COLS, "TMEM budget");
constexpr int THREADS = 512;
constexpr int EPI_WARP0 = 12;
constexpr int STAT_FLOATS = NTOK * (2 + kRank);   // per-token s_x, sum q, u[16] of one linear
constexpr int kMapSlots = 4;               // per-CTA ring of device-edited sign tensor maps

// kind::i8 instruction descriptor: D s32, A u8 (bytes 0 or 2^p), B s8, both K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(NTOK >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct DecodeArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* desc;           // desc[0] is the first linear of this launch
    const CUtensorMap* sign_tmpl;  // per linear: its sign map with a placeholder address
    CUtensorMap* map_slots;        // kMapSlots per CTA
    const int8_t* q_ws;
    const TokStats* st_ws;
    uint32_t* err;
    int n;
    int m;
    int total_tiles;
    int img_bytes;                 // bytes of one activation-image buffer (16 x qrow of the widest linear)
    int img_bufs;                  // 1 or 2
    int64_t total_bytes;           // sign bytes of the n linears
};

// Shared-memory B descriptor, K-major, no swizzle: core matrices of 8 rows x 16 bytes,
// the two 16-byte K halves 128 bytes apart (leading offset), groups of 8 token rows
// 256 bytes apart (stride offset), descriptor version 1.
__device__ __forceinline__ uint64_t img_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(256 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

// The linear a tile belongs to, with the fields every role needs.
struct Cursor {
    int lin, t_in, ntiles, nseg, nstage, d_out;
    __device__ void load(const DecodeArgs& a, int l) {
        const DevDesc& d = a.desc[l];
        lin = l;
        d_out = d.d_out;
        ntiles = (d.d_out + BM - 1) / BM;
        nseg = d.qrow >> 8;
        nstage = (d.d_in / 8 + STAGE_ROW_BYTES - 1) / STAGE_ROW_BYTES;
    }
    // position on flattened tile T, which lies in linear l or a later one
    __device__ void start(const DecodeArgs& a, int l, int T) {
        load(a, l);
        t_in = T - (a.desc[l].rt_begin - a.desc[0].rt_begin);
        while (t_in >= ntiles && lin + 1 < a.n) {
            t_in -= ntiles;
            load(a, lin + 1);
        }
    }
    // next tile; true when it belongs to another linear
    __device__ bool advance(const DecodeArgs& a) {
        if (++t_in < ntiles) return false;
        t_in = 0;
        if (lin + 1 < a.n) load(a, lin + 1);
        return true;
    }
};

// First flattened tile of linear l whose first sign byte is at or after byte `pos`
// of the call (the first tile of linear l + 1 if there is none).
__device__ int tile_at(const DecodeArgs& a, int l, int64_t pos) {
    const DevDesc& d = a.desc[l];
    const int64_t tb = (int64_t)BM * (d.d_in / 8);
    const int64_t t = (pos - (d.byte_begin - a.desc[0].byte_begin) + tb - 1) / tb;
    const int nt = (d.d_out + BM - 1) / BM;
    return d.rt_begin - a.desc[0].rt_begin + (int)(t < nt ? t : nt);
}

// lane 0 waits, the warp follows. Returns false on timeout, or at once once
// `abort` is set; the caller then sets `abort` (and the error word) and keeps
// walking its loop without waiting, so no partner is left blocked.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int lane, volatile uint32_t* abort) {
    bool ok = true;
    if (lane == 0) ok = !*abort && ptx::mbar_wait(bar, parity);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok;
}
__device__ __forceinline__ bool thread_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort) {
    return !*abort && ptx::mbar_wait(bar, parity);
}
__device__ __forceinline__ void fail(uint32_t* err, volatile uint32_t* abort) {
    set_err(err, DFSSM_DEVERR_TIMEOUT);
    *abort = 1;
}

template <int NT>
__global__ void __launch_bounds__(THREADS, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, offset from the __shared__ array so addressing stays in shared space
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = smem;                                       // NS sign stages
    uint8_t* img = ring + NS * SIGN_STAGE;                      // img_bufs activation images
    float* stats = reinterpret_cast<float*>(img + a.img_bufs * a.img_bytes);   // [4 epilogue warps][STAT_FLOATS]
    uint8_t* map_s = reinterpret_cast<uint8_t*>(stats + 4 * STAT_FLOATS);        // 128 bytes, 128-aligned
    uint64_t* bars = reinterpret_cast<uint64_t*>(map_s + 128);
    uint64_t* sign_full = bars;                      // [NS] TMA bytes
    uint64_t* sign_empty = bars + NS;                // [NS] 8 expander warps
    uint64_t* a_empty = bars + 2 * NS;               // [NGRP][NSLOT] MMA commit
    uint64_t* d_full = a_empty + NGRP * NSLOT;       // [2] one arrival per group
    uint64_t* d_empty = d_full + 2;                  // [2] 4 epilogue warps
    uint64_t* q_full = d_empty + 2;                  // [2] bulk-copy bytes
    uint64_t* q_empty = q_full + 2;                  // [2] one arrival per group
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + 2);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* loc = reinterpret_cast<int*>(tmem_slot + 2);   // linears holding this CTA's first and end byte

    // This CTA's byte range [lo, hi) of the call's sign bytes; every thread tests a few
    // linears at once, so locating it costs one round of loads instead of a search.
    const int64_t lo = a.total_bytes * blockIdx.x / gridDim.x;
    const int64_t hi = a.total_bytes * (blockIdx.x + 1) / gridDim.x;
    {
        const int64_t b0 = a.desc[0].byte_begin;
        for (int i = threadIdx.x; i < a.n; i += THREADS) {
            const int64_t b = a.desc[i].byte_begin - b0;
            const int64_t bn = i + 1 < a.n ? a.desc[i + 1].byte_begin - b0 : INT64_MAX;
            if (b <= lo && lo < bn) loc[0] = i;     // exactly one linear matches each position
            if (b <= hi && hi < bn) loc[1] = i;
        }
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&sign_full[s], 1);
            ptx::mbar_init(&sign_empty[s], NGRP * 4);
        }
        for (int s = 0; s < NGRP * NSLOT; ++s) ptx::mbar_init(&a_empty[s], 1);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&d_full[b], NGRP);
            ptx::mbar_init(&d_empty[b], 4);
            ptx::mbar_init(&q_full[b], 1);
            ptx::mbar_init(&q_empty[b], NGRP);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int lin0 = loc[0];
    const int t_lo = tile_at(a, lin0, lo);
    const int t_hi = blockIdx.x + 1 == gridDim.x ? a.total_tiles : tile_at(a, loc[1], hi);
    const uint32_t nb = (uint32_t)a.img_bufs;

    if (warp == 0) {
        // ------------------------------------------------ sign producer (whole warp: the map copy is warp-wide)
        Cursor cur;
        if (t_lo < t_hi) cur.start(a, lin0, t_lo);
        uint32_t S = 0;
        int map_i = 0, prev_lin = -1;
        const CUtensorMap* gmap = nullptr;
        bool lin_ok = false;
        for (int T = t_lo; T < t_hi && !*abort_flag; ++T) {
            const int row0 = cur.t_in * BM;
            const bool new_lin = cur.lin != prev_lin;
            prev_lin = cur.lin;
            for (int k = 0; k < cur.nstage; ++k, ++S) {
                const int s = (int)(S % NS);
                if (!warp_wait(&sign_empty[s], ((S / NS) & 1u) ^ 1u, lane, abort_flag)) {
                    if (lane == 0) fail(a.err, abort_flag);
                    break;
                }
                if (k == 0 && new_lin) {
                    // Stage S - NS has been consumed, so every load issued before it has
                    // completed; the slot edited here was last used at least NS stages ago.
                    const dfssm_stack_entry& e = entry_at(a.entries, a.single, cur.lin);
                    lin_ok = entry_ptrs_ok(e);
                    if (lin_ok) {
                        CUtensorMap* slot = a.map_slots + (size_t)blockIdx.x * kMapSlots + map_i;
                        map_i = (map_i + 1) % kMapSlots;
                        if (lane < 8)
                            reinterpret_cast<uint4*>(map_s)[lane] =
                                reinterpret_cast<const uint4*>(a.sign_tmpl + cur.lin)[lane];
                        __syncwarp();
                        if (lane == 0) ptx::tensormap_replace_addr(map_s, e.w.sign);
                        __syncwarp();
                        ptx::tensormap_copy_release(slot, map_s);
                        if (lane == 0) ptx::tensormap_acquire(slot);
                        __syncwarp();
                        gmap = slot;
                    }
                }
                if (lane == 0) {
                    if (lin_ok) {
                        ptx::mbar_arrive_expect_tx(&sign_full[s], SIGN_STAGE);
                        ptx::tma_load_2d(ring + s * SIGN_STAGE, gmap, k * STAGE_ROW_BYTES, row0, &sign_full[s]);
                    } else {
                        ptx::mbar_arrive(&sign_full[s]);    // an entry with bad pointers: nothing is read
                    }
                }
                __syncwarp();
            }
            cur.advance(a);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ activation images (from the quantisation kernel)
        if (lane == 0) {
            Cursor cur;
            if (t_lo < t_hi) cur.start(a, lin0, t_lo);
            uint32_t qv = 0;
            int prev_lin = -1;
            bool waited = false;
            for (int T = t_lo; T < t_hi && !*abort_flag; ++T) {
                if (cur.lin != prev_lin) {
                    prev_lin = cur.lin;
                    const uint32_t qb = qv % nb;
                    if (!thread_wait(&q_empty[qb], ((qv / nb) & 1u) ^ 1u, abort_flag)) {
                        fail(a.err, abort_flag);
                        break;
                    }
                    ++qv;
                    if (!waited) { ptx::pdl_wait(); waited = true; }
                    const dfssm_stack_entry& e = entry_at(a.entries, a.single, cur.lin);
                    if (entry_ptrs_ok(e)) {
                        const DevDesc& d = a.desc[cur.lin];
                        const uint32_t bytes = (uint32_t)(NTOK * d.qrow);
                        ptx::mbar_arrive_expect_tx(&q_full[qb], bytes);
                        const uint8_t* src = reinterpret_cast<const uint8_t*>(a.q_ws) + d.dq_off;
                        uint8_t* dst = img + qb * a.img_bytes;
                        for (uint32_t off = 0; off < bytes; off += 32768u)
                            ptx::bulk_g2s(dst + off, src + off, min(32768u, bytes - off), &q_full[qb]);
                    } else {
                        ptx::mbar_arrive(&q_full[qb]);
                    }
                }
                cur.advance(a);
            }
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------ MMA issuer of group g (one thread, so the
        // group's MMAs into its accumulators are issued in order by one thread)
        const int g = warp - 2;
        uint64_t* my_empty = a_empty + g * NSLOT;
        const uint64_t desc0 = img_desc(ptx::smem_u32(img));
        Cursor cur;
        if (t_lo < t_hi) cur.start(a, lin0, t_lo);
        uint32_t L = 0, tc = 0, qv = 0, qb = 0;
        int prev_lin = -1;
        // No early exit: the issuer meets its expander group at a named barrier every segment.
        for (int T = t_lo; T < t_hi; ++T, ++tc) {
            const bool new_lin = cur.lin != prev_lin;
            if (new_lin) {
                qb = qv % nb;
                ++qv;
                prev_lin = cur.lin;
            }
            const bool last_tile = cur.t_in + 1 == cur.ntiles || T + 1 == t_hi;
            const uint32_t buf = tc & 1u;
            const uint32_t d_lo = tmem_base + (uint32_t)(2 * g + (int)buf) * D_COLS;
            const uint64_t bdesc = desc0 + (uint64_t)((qb * (uint32_t)a.img_bytes) >> 4);
            for (int j = g; j < cur.nseg; j += NGRP, ++L) {
                const uint32_t slot = L % NSLOT;
                ptx::named_barrier(1 + g, 160);          // the group has written segment j into the slot
                ptx::tc_fence_after();
                if (ptx::elect_one()) {
                    const bool first = j == g, last = j + NGRP >= cur.nseg;
                    bool ok = true;
                    if (first) {
                        if (new_lin) ok = thread_wait(&q_full[qb], ((qv - 1) / nb) & 1u, abort_flag);
                        ok = ok && thread_wait(&d_empty[buf], ((tc >> 1) & 1u) ^ 1u, abort_flag);
                        if (!ok) fail(a.err, abort_flag);
                        ptx::tc_fence_after();
                    }
                    if (!*abort_flag) {
                        const uint32_t a_tmem = tmem_base + A_COL0 + (uint32_t)(g * NSLOT + (int)slot) * A_COLS;
                        const uint64_t bj = bdesc + (uint64_t)(256 * j);
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            ptx::mma_i8_ts(d_lo, a_tmem + 8 * p, bj + 32 * p, kIdesc, !first || p > 0);
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            ptx::mma_i8_ts(d_lo + NTOK, a_tmem + 32 + 8 * p, bj + 32 * (4 + p), kIdesc,
                                           !first || p > 0);
                    }
                    // each commit arrives once this thread's earlier MMAs have completed
                    ptx::mma_commit(&my_empty[slot]);
                    if (last) {
                        ptx::mma_commit(&d_full[buf]);
                        if (last_tile) ptx::mma_commit(&q_empty[qb]);
                    }
                }
                __syncwarp();
            }
            if (cur.nseg <= g && lane == 0) {
                // no segment of this tile for the group: its arrivals, without MMAs
                ptx::mbar_arrive(&d_full[buf]);
                if (last_tile) ptx::mbar_arrive(&q_empty[qb]);
            }
            __syncwarp();
            cur.advance(a);
        }
    } else if (warp >= 4 && warp < EPI_WARP0) {
        // ------------------------------------------------ bit-plane expansion into TMEM
        const int g = (warp - 4) >> 2;                    // segments j with j % 2 == g
        const int q4 = warp & 3;                          // TMEM lanes 32 q4 .. 32 q4 + 31
        const int r = q4 * 32 + lane;                     // tile row of this thread
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const uint32_t xr = (uint32_t)(r & 7);
        const uint32_t row_off = (uint32_t)r * STAGE_ROW_BYTES;
        uint64_t* my_empty = a_empty + g * NSLOT;
        Cursor cur;
        if (t_lo < t_hi) cur.start(a, lin0, t_lo);
        uint32_t S = 0, L = 0;
        // No early exit: the group meets its issuer at a named barrier every segment.
        for (int T = t_lo; T < t_hi; ++T) {
            for (int k = 0; k < cur.nstage; ++k, ++S) {
                const int s = (int)(S % NS);
                if (!warp_wait(&sign_full[s], (S / NS) & 1u, lane, abort_flag) && lane == 0) fail(a.err, abort_flag);
                const uint8_t* stage = ring + s * SIGN_STAGE + row_off;
                const int jn = min(4, cur.nseg - 4 * k);
                for (int jj = g; jj < jn; jj += NGRP, ++L) {
                    const uint32_t slot = L % NSLOT;
                    // the segment's 32 sign bytes: 16-byte chunks 2 jj, 2 jj + 1 of this row (128B swizzle)
                    const uint4 lo = *reinterpret_cast<const uint4*>(stage + (((2u * jj) ^ xr) << 4));
                    const uint4 hi = *reinterpret_cast<const uint4*>(stage + (((2u * jj + 1u) ^ xr) << 4));
                    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    if (!warp_wait(&my_empty[slot], ((L / NSLOT) & 1u) ^ 1u, lane, abort_flag) && lane == 0)
                        fail(a.err, abort_flag);
                    ptx::tc_fence_after();
                    const uint32_t taddr = tmem_base + lane_addr + A_COL0 + (uint32_t)(g * NSLOT + (int)slot) * A_COLS;
                    {
                        // columns 8 p + c: plane p (0..3) of word c as bytes 0 / 1
                        uint32_t e[32];
#pragma unroll
                        for (int p = 0; p < 4; ++p)
#pragma unroll
                            for (int c = 0; c < 8; ++c) e[8 * p + c] = (w[c] >> p) & 0x01010101u;
                        ptx::tmem_st_32x32b_x32(taddr, e);
                    }
                    {
                        // columns 32 + 8 p + c: plane p + 4 of word c as bytes 0 / 16
                        uint32_t e[32];
#pragma unroll
                        for (int p = 0; p < 4; ++p)
#pragma unroll
                            for (int c = 0; c < 8; ++c) e[8 * p + c] = (w[c] >> p) & 0x10101010u;
                        ptx::tmem_st_32x32b_x32(taddr + 32, e);
                    }
                    ptx::tmem_st_wait();
                    ptx::tc_fence_before();
                    ptx::named_barrier(1 + g, 160);       // hand the segment to the group's issuer
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sign_empty[s]);
            }
            cur.advance(a);
        }
    } else if (warp >= EPI_WARP0) {
        // ------------------------------------------------ epilogue (one output row per thread)
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const int m = a.m;
        // this warp's copy of the current linear's per-token scalars
        float* st_sx = stats + q4 * STAT_FLOATS;
        int* st_sumq = reinterpret_cast<int*>(st_sx + NTOK);
        float* st_u = st_sx + 2 * NTOK;
        // Pointers of a linear are read once per linear, and the next tile's row parameters
        // are loaded while the current tile is being computed.
        struct EpiLin {
            const float* alpha;
            const float* sa;
            const int8_t* wa;
            void* y;
            int32_t* acc;
            int d_out;
            bool bf16, ok;
        };
        auto load_lin = [&](int l) {
            const dfssm_stack_entry& e = entry_at(a.entries, a.single, l);
            EpiLin L;
            L.ok = entry_ptrs_ok(e);
            L.alpha = e.w.alpha;
            L.sa = e.w.sa;
            L.wa = e.w.wa;
            L.y = e.y;
            L.acc = e.dbg.acc;
            L.d_out = a.desc[l].d_out;
            L.bf16 = a.desc[l].y_dtype == DFSSM_BF16;
            return L;
        };
        struct RowP {
            float alpha, sa;
            int4 wa;
        };
        auto load_row = [&](const EpiLin& L, int o) {
            RowP p{0.f, 0.f, make_int4(0, 0, 0, 0)};
            if (L.ok && o < L.d_out) {
                p.alpha = L.alpha[o];
                p.sa = L.sa[o];
                p.wa = *reinterpret_cast<const int4*>(L.wa + (int64_t)o * kRank);
            }
            return p;
        };
        Cursor cur;
        EpiLin lin{};
        RowP row{0.f, 0.f, make_int4(0, 0, 0, 0)};
        if (t_lo < t_hi) {
            cur.start(a, lin0, t_lo);
            lin = load_lin(cur.lin);
            row = load_row(lin, cur.t_in * BM + r);
        }
        uint32_t tc = 0;
        int prev_lin = -1;
        bool waited = false;
        for (int T = t_lo; T < t_hi && !*abort_flag; ++T, ++tc) {
            if (cur.lin != prev_lin) {
                if (!waited) { ptx::pdl_wait(); waited = true; }
                prev_lin = cur.lin;
                __syncwarp();
                const TokStats* st = a.st_ws + a.desc[cur.lin].st_off;
                for (int i = lane; i < m * 18; i += 32) {
                    const int t = i / 18, f = i - 18 * t;
                    if (f == 0) st_sx[t] = st[t].sx;
                    else if (f == 1) st_sumq[t] = st[t].sumq;
                    else st_u[t * kRank + f - 2] = st[t].u[f - 2];
                }
                __syncwarp();
            }
            const EpiLin L = lin;
            const RowP rp = row;
            const int o = cur.t_in * BM + r;
            const int nseg = cur.nseg;
            // prefetch the next tile's row parameters (and its linear's pointers)
            if (T + 1 < t_hi) {
                if (cur.advance(a)) lin = load_lin(cur.lin);
                row = load_row(lin, cur.t_in * BM + r);
            }
            const uint32_t buf = tc & 1u;
            if (!warp_wait(&d_full[buf], (tc >> 1) & 1u, lane, abort_flag)) {
                if (lane == 0) fail(a.err, abort_flag);
                break;
            }
            ptx::tc_fence_after();
            // S1 = sum over groups of D_lo + D_hi / 16
            int s_lo[NT], s_hi[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j) s_lo[j] = s_hi[j] = 0;
            const int ngrp = nseg < NGRP ? nseg : NGRP;
            for (int g = 0; g < ngrp; ++g) {
                uint32_t vl[NT], vh[NT];
                const uint32_t col = tmem_base + lane_addr + (uint32_t)(2 * g + (int)buf) * D_COLS;
                ptx::tmem_ld_32x32b<NT>(col, vl);
                ptx::tmem_ld_32x32b<NT>(col + NTOK, vh);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    s_lo[j] += (int)vl[j];
                    s_hi[j] += (int)vh[j];
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&d_empty[buf]);
            if (L.ok && o < L.d_out) {
                const WaRow wa = wa_row_from_int4(rp.wa);
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j >= m) break;
                    const int acc = 2 * (s_lo[j] + (s_hi[j] >> 4)) - st_sumq[j];
                    const float y = dequant(st_sx[j], rp.alpha, rp.sa, acc, lora_dot(wa, st_u + j * kRank));
                    const int64_t idx = (int64_t)j * L.d_out + o;
                    if (L.bf16) reinterpret_cast<uint16_t*>(L.y)[idx] = f32_to_bf16_bits(y);
                    else reinterpret_cast<float*>(L.y)[idx] = y;
                    if (L.acc) L.acc[idx] = acc;
                }
            }
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

size_t smem_bytes(int img_bytes, int img_bufs) {
    return 1024 + (size_t)NS * SIGN_STAGE + (size_t)img_bufs * img_bytes + sizeof(float) * 4 * STAT_FLOATS + 128 +
           8 * (2 * NS + NGRP * NSLOT + 8) + 32;
}

template <int NT>
cudaError_t launch_nt(const LaunchCtx& c, const DecodeArgs& a, size_t smem, int grid) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<NT>, a);
}

template <int NT>
cudaError_t set_attr_nt(int optin) {
    return allow_dyn_smem(decode_kernel<NT>, optin);
}

int g_optin = 0;

}  // namespace

int decode_map_slots() { return kMapSlots; }
int decode_tile_rows() { return BM; }
int decode_stage_bytes() { return STAGE_ROW_BYTES; }

cudaError_t launch_decode(const LaunchCtx& c) {
    int64_t total_bytes = 0;
    int tiles = 0, max_qrow = 0;
    for (int i = 0; i < c.n; ++i) {
        total_bytes += (int64_t)c.host_desc[i].d_out * (c.host_desc[i].d_in / 8);
        tiles += (c.host_desc[i].d_out + BM - 1) / BM;
        max_qrow = max(max_qrow, c.host_desc[i].qrow);
    }
    const int img_bytes = NTOK * max_qrow;
    const int bufs = smem_bytes(img_bytes, 2) <= (size_t)g_optin ? 2 : 1;
    const size_t smem = smem_bytes(img_bytes, bufs);
    if (smem > (size_t)g_optin) return cudaErrorInvalidConfiguration;
    int grid = c.sm_count < tiles ? c.sm_count : tiles;
    if (grid > c.map_slot_ctas) grid = c.map_slot_ctas;
    DecodeArgs a{c.entries, c.single, c.desc, reinterpret_cast<const CUtensorMap*>(c.sign_tmpl),
                 reinterpret_cast<CUtensorMap*>(c.map_slots), c.q_ws, c.st_ws, c.err, c.n, c.m, tiles, img_bytes,
                 bufs, total_bytes};
    if (c.m <= 1) return launch_nt<1>(c, a, smem, grid);
    if (c.m <= 2) return launch_nt<2>(c, a, smem, grid);
    if (c.m <= 4) return launch_nt<4>(c, a, smem, grid);
    if (c.m <= 8) return launch_nt<8>(c, a, smem, grid);
    return launch_nt<16>(c, a, smem, grid);
}

cudaError_t set_decode_attr(int optin) {
    cudaError_t e = set_attr_nt<1>(optin);
    if (e == cudaSuccess) e = set_attr_nt<2>(optin);
    if (e == cudaSuccess) e = set_attr_nt<4>(optin);
    if (e == cudaSuccess) e = set_attr_nt<8>(optin);
    if (e == cudaSuccess) e = set_attr_nt<16>(optin);
    if (e == cudaSuccess) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, decode_kernel<16>);
        if (e == cudaSuccess) g_optin = optin - (int)fa.sharedSizeBytes;
    }
    return e;
}

}  // namespace dfssm
