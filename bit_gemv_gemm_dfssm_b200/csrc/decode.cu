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
//    of a tile (= one TMEM lane) and writes its 64 expanded words (8 planes x
//    8 words) with tcgen05.st; the MMA reads A from TMEM, so the 8x larger
//    expanded operand never passes through shared memory.
//  * B operand: the int8 activations of up to 16 tokens (MMA N = 16) in the
//    same plane-major order (K position 32p + 4c + i <-> column 32c + 8i + p),
//    copied once per linear into shared memory as 8-row x 16-byte core
//    matrices (the quantisation kernel writes them in that layout).
//  * One accumulator per bit plane: D_p = 2^p * S_p exactly (int32 in TMEM),
//    S1 = sum_p D_p / 2^p = sum_{bit = 1} q, and acc = 2 * S1 - sum_j q
//    (a +-1 weight is 2b - 1).
//
// Persistent kernel, one CTA per SM, 16 warps with fixed roles:
//   warp 0       TMA producer of sign tiles (128 rows x 128 bytes, 128B swizzle,
//                no multicast) through a per-linear tensor map whose global
//                address it sets on the device (tensormap.replace); 4 stages
//   warp 1       TMEM owner and MMA issuer (tcgen05.mma.kind::i8, A in TMEM)
//   warp 2       bulk copy of each linear's activation image into shared memory
//   warps 4-11   two expander warpgroups taking alternate 256-column segments
//   warps 12-15  epilogue: combine the plane accumulators, LoRA up-projection,
//                dequantisation (epilogue.cuh), coalesced stores
// Work: the 128-row tiles of all linears of the call, split into contiguous
// ranges holding equal shares of the sign bytes. Every mbarrier wait is
// bounded; a timeout sets the error word and the CTA winds down.
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
constexpr int NA = 4;                      // TMEM A slots (2 per expander warpgroup)
constexpr uint32_t A_COLS = 64;            // TMEM columns per A slot: 8 planes x 8 words
constexpr uint32_t D_COLS = 8 * NTOK;      // one accumulator buffer: 8 planes x 16 tokens
constexpr uint32_t A_COL0 = 2 * D_COLS;    // A slots after the two accumulator buffers
constexpr uint32_t TMEM_COLS = 512;
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
    // position on flattened tile T
    __device__ void start(const DecodeArgs& a, int T) {
        const int base = a.desc[0].rt_begin;
        int lo = 0, hi = a.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.desc[mid].rt_begin - base <= T) lo = mid; else hi = mid - 1;
        }
        load(a, lo);
        t_in = T - (a.desc[lo].rt_begin - base);
    }
    // next tile; true when it belongs to another linear
    __device__ bool advance(const DecodeArgs& a) {
        if (++t_in < ntiles) return false;
        t_in = 0;
        if (lin + 1 < a.n) load(a, lin + 1);
        return true;
    }
};

// First flattened tile whose first sign byte is at or after byte `lo` of the call.
__device__ int first_tile(const DecodeArgs& a, int64_t lo) {
    const int64_t b0 = a.desc[0].byte_begin;
    const int r0 = a.desc[0].rt_begin;
    int l = 0, h = a.n - 1;
    while (l < h) {
        const int mid = (l + h + 1) >> 1;
        if (a.desc[mid].byte_begin - b0 <= lo) l = mid; else h = mid - 1;
    }
    const DevDesc& d = a.desc[l];
    const int64_t tb = (int64_t)BM * (d.d_in / 8);
    const int64_t t = (lo - (d.byte_begin - b0) + tb - 1) / tb;
    const int nt = (d.d_out + BM - 1) / BM;
    if (t >= nt) return l + 1 < a.n ? a.desc[l + 1].rt_begin - r0 : a.total_tiles;
    return d.rt_begin - r0 + (int)t;
}

// lane 0 waits, the warp follows; false on timeout
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int lane) {
    bool ok = true;
    if (lane == 0) ok = ptx::mbar_wait(bar, parity);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok;
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
    uint64_t* sign_full = bars;              // [NS] TMA bytes
    uint64_t* sign_empty = bars + NS;        // [NS] 8 expander warps
    uint64_t* a_full = bars + 2 * NS;        // [NA] 4 warps of one expander group
    uint64_t* a_empty = a_full + NA;         // [NA] MMA commit
    uint64_t* d_full = a_empty + NA;         // [2] MMA commit
    uint64_t* d_empty = d_full + 2;          // [2] 4 epilogue warps
    uint64_t* q_full = d_empty + 2;          // [2] bulk-copy bytes
    uint64_t* q_empty = q_full + 2;          // [2] MMA commit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + 2);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&sign_full[s], 1);
            ptx::mbar_init(&sign_empty[s], 8);
        }
        for (int s = 0; s < NA; ++s) {
            ptx::mbar_init(&a_full[s], 4);
            ptx::mbar_init(&a_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&d_full[b], 1);
            ptx::mbar_init(&d_empty[b], 4);
            ptx::mbar_init(&q_full[b], 1);
            ptx::mbar_init(&q_empty[b], 1);
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

    const int t_lo = first_tile(a, a.total_bytes * blockIdx.x / gridDim.x);
    const int t_hi = blockIdx.x + 1 == gridDim.x ? a.total_tiles
                                                 : first_tile(a, a.total_bytes * (blockIdx.x + 1) / gridDim.x);

    if (warp == 0) {
        // ------------------------------------------------ sign producer (whole warp: the map copy is warp-wide)
        Cursor cur;
        if (t_lo < t_hi) cur.start(a, t_lo);
        uint32_t S = 0;
        int map_i = 0, prev_lin = -1;
        const CUtensorMap* gmap = nullptr;
        bool lin_ok = false, ok = true;
        for (int T = t_lo; T < t_hi && ok && !*abort_flag; ++T) {
            const int row0 = cur.t_in * BM;
            const bool new_lin = cur.lin != prev_lin;
            prev_lin = cur.lin;
            for (int k = 0; k < cur.nstage; ++k, ++S) {
                const int s = (int)(S % NS);
                if (!warp_wait(&sign_empty[s], ((S / NS) & 1u) ^ 1u, lane)) { ok = false; break; }
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
        if (!ok && lane == 0) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            Cursor cur;
            if (t_lo < t_hi) cur.start(a, t_lo);
            uint32_t G = 0, tc = 0, qv = 0, qb = 0;
            const uint32_t nb = (uint32_t)a.img_bufs;
            int prev_lin = -1;
            bool ok = true;
            for (int T = t_lo; T < t_hi && ok && !*abort_flag; ++T, ++tc) {
                if (cur.lin != prev_lin) {
                    qb = qv % nb;
                    if (!ptx::mbar_wait(&q_full[qb], (qv / nb) & 1u)) { ok = false; break; }
                    ++qv;
                    prev_lin = cur.lin;
                }
                const uint32_t buf = tc & 1u;
                if (!ptx::mbar_wait(&d_empty[buf], ((tc >> 1) & 1u) ^ 1u)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * D_COLS;
                const uint32_t img_s = ptx::smem_u32(img + qb * a.img_bytes);
                for (int j = 0; j < cur.nseg; ++j, ++G) {
                    const uint32_t slot = G % NA;
                    if (!ptx::mbar_wait(&a_full[slot], (G / NA) & 1u)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t a_tmem = tmem_base + A_COL0 + slot * A_COLS;
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        ptx::mma_i8_ts(d_tmem + p * NTOK, a_tmem + 8 * p, img_desc(img_s + (8 * j + p) * 512), kIdesc,
                                       j > 0);
                    ptx::mma_commit(&a_empty[slot]);
                }
                if (!ok) break;
                ptx::mma_commit(&d_full[buf]);
                if (cur.advance(a) || T + 1 == t_hi) ptx::mma_commit(&q_empty[qb]);
            }
            if (!ok) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; }
        }
    } else if (warp == 2) {
        // ------------------------------------------------ activation images (from the quantisation kernel)
        if (lane == 0) {
            Cursor cur;
            if (t_lo < t_hi) cur.start(a, t_lo);
            uint32_t qv = 0;
            const uint32_t nb = (uint32_t)a.img_bufs;
            int prev_lin = -1;
            bool waited = false;
            for (int T = t_lo; T < t_hi && !*abort_flag; ++T) {
                if (cur.lin != prev_lin) {
                    prev_lin = cur.lin;
                    const uint32_t qb = qv % nb;
                    if (!ptx::mbar_wait(&q_empty[qb], ((qv / nb) & 1u) ^ 1u)) {
                        set_err(a.err, DFSSM_DEVERR_TIMEOUT);
                        *abort_flag = 1;
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
    } else if (warp >= 4 && warp < EPI_WARP0) {
        // ------------------------------------------------ bit-plane expansion into TMEM
        const uint32_t grp = (uint32_t)(warp - 4) >> 2;   // segments with (G & 1) == grp
        const int q4 = warp & 3;                          // TMEM lanes 32 q4 .. 32 q4 + 31
        const int r = q4 * 32 + lane;                     // tile row of this thread
        const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
        const uint32_t xr = (uint32_t)(r & 7);
        const uint32_t row_off = (uint32_t)r * STAGE_ROW_BYTES;
        Cursor cur;
        if (t_lo < t_hi) cur.start(a, t_lo);
        uint32_t S = 0, G = 0;
        bool ok = true;
        for (int T = t_lo; T < t_hi && ok && !*abort_flag; ++T) {
            for (int k = 0; k < cur.nstage && ok; ++k, ++S) {
                const int s = (int)(S % NS);
                if (!warp_wait(&sign_full[s], (S / NS) & 1u, lane)) { ok = false; break; }
                const uint8_t* stage = ring + s * SIGN_STAGE + row_off;
                const int jn = min(4, cur.nseg - 4 * k);
                for (int jj = 0; jj < jn; ++jj) {
                    const uint32_t Gj = G + 4 * k + jj;
                    if ((Gj & 1u) != grp) continue;
                    const uint32_t slot = Gj % NA;
                    // the segment's 32 sign bytes: 16-byte chunks 2 jj, 2 jj + 1 of this row (128B swizzle)
                    const uint4 lo = *reinterpret_cast<const uint4*>(stage + (((2u * jj) ^ xr) << 4));
                    const uint4 hi = *reinterpret_cast<const uint4*>(stage + (((2u * jj + 1u) ^ xr) << 4));
                    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    if (!warp_wait(&a_empty[slot], ((Gj / NA) & 1u) ^ 1u, lane)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t taddr = tmem_base + lane_addr + A_COL0 + slot * A_COLS;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        // column 8 p + c of the slot = plane p of word c
                        uint32_t e[32];
#pragma unroll
                        for (int pp = 0; pp < 4; ++pp)
#pragma unroll
                            for (int c = 0; c < 8; ++c) e[8 * pp + c] = w[c] & (0x01010101u << (4 * half + pp));
                        ptx::tmem_st_32x32b_x32(taddr + 32 * half, e);
                    }
                    ptx::tmem_st_wait();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&a_full[slot]);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sign_empty[s]);
            }
            G += cur.nseg;
            cur.advance(a);
        }
        if (!ok && lane == 0) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; }
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
        Cursor cur;
        if (t_lo < t_hi) cur.start(a, t_lo);
        uint32_t tc = 0;
        int prev_lin = -1;
        bool waited = false, lin_ok = false;
        for (int T = t_lo; T < t_hi && !*abort_flag; ++T, ++tc) {
            const dfssm_stack_entry& e = entry_at(a.entries, a.single, cur.lin);
            if (cur.lin != prev_lin) {
                if (!waited) { ptx::pdl_wait(); waited = true; }
                prev_lin = cur.lin;
                lin_ok = entry_ptrs_ok(e);
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
            const int o = cur.t_in * BM + r;
            const bool valid = lin_ok && o < cur.d_out;
            void* const y_ptr = e.y;
            int32_t* const dbg_acc = e.dbg.acc;
            const bool y_bf16 = a.desc[cur.lin].y_dtype == DFSSM_BF16;
            const int d_out = cur.d_out;
            float alpha = 0.f, sa = 0.f;
            int4 wa4 = make_int4(0, 0, 0, 0);
            if (valid) {
                alpha = e.w.alpha[o];
                sa = e.w.sa[o];
                wa4 = *reinterpret_cast<const int4*>(e.w.wa + (int64_t)o * kRank);
            }
            const uint32_t buf = tc & 1u;
            if (!warp_wait(&d_full[buf], (tc >> 1) & 1u, lane)) {
                if (lane == 0) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; }
                break;
            }
            ptx::tc_fence_after();
            // T = sum_p D_p * 2^(7 - p) = 128 * S1
            int Tt[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j) Tt[j] = 0;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                uint32_t v[NT];
                ptx::tmem_ld_32x32b<NT>(tmem_base + lane_addr + buf * D_COLS + p * NTOK, v);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < NT; ++j) Tt[j] += (int)v[j] * (1 << (7 - p));
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&d_empty[buf]);
            if (valid) {
                const WaRow wa = wa_row_from_int4(wa4);
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j >= m) break;
                    const int acc = 2 * (Tt[j] >> 7) - st_sumq[j];
                    const float y = dequant(st_sx[j], alpha, sa, acc, lora_dot(wa, st_u + j * kRank));
                    const int64_t idx = (int64_t)j * d_out + o;
                    if (y_bf16) reinterpret_cast<uint16_t*>(y_ptr)[idx] = f32_to_bf16_bits(y);
                    else reinterpret_cast<float*>(y_ptr)[idx] = y;
                    if (dbg_acc) dbg_acc[idx] = acc;
                }
            }
            cur.advance(a);
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
           8 * (2 * NS + 2 * NA + 8) + 16;
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
