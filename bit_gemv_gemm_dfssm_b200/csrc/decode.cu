// Decode path (1 <= m <= 16 tokens): the scaffold contraction streamed from HBM
// with the LoRA up-projection and both dequantisation epilogues fused.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C:
// the 1-bit scaffold weights are expanded on the fly to int8 and fed to int8
// tensor cores, which cuts weight traffic 8x against int8 weights; at batch 1
// the layer is bound by that weight stream. Here the bits never exist as int8
// bytes in memory:
//
//  * Work: blocks of R = 16 * RT * W output rows (W warps, RT 16-row tiles per
//    warp): up to 8 tokens 4 warps x 2 tiles (128 rows, three CTAs per SM);
//    9 to 16 tokens 12 warps x 1 tile (192 rows, one CTA per SM, so the 16
//    tokens' activations are held once per SM), flattened over all linears of
//    the call. Each CTA is persistent and
//    owns a contiguous range of blocks holding an equal share of the work units
//    (per k-chunk, per block epilogue and for entering a linear; dfssm_internal.cuh):
//    CTA durations follow these units, not bytes (a partial last block costs
//    as many iterations as a full one, and entering a linear costs a quantisation).
//  * Streaming: a block is consumed in k-chunks of 1024 columns (128 bytes per
//    row), each one TMA load (cp.async.bulk.tensor, no multicast) of an
//    R x 128-byte box into a ring of kStages shared-memory slots, issued by one
//    thread; the 128-byte swizzle puts 16-byte piece j of slot row r at
//    j ^ (r & 7), so the ldmatrix reads of 8 rows hit 8 different bank groups,
//    and rows past d_out or bytes past the row end arrive as zeros. The last
//    k-chunk of a block also brings its alpha, s_A and W_A (16-byte cp.async).
//    A slot's mbarrier completes when the TMA bytes and every thread's
//    cp.async have landed (cp.async.mbarrier.arrive), so a chunk costs the
//    computing threads no copy instructions and one CTA barrier. The tensor
//    map of a single linear is encoded on the host and passed with the launch;
//    for a stack (pointers in device memory) warp 0 copies the linear's
//    template map into shared memory, sets its global address
//    (tensormap.replace) and publishes it to one of the CTA's map slots.
//  * Activations: when a CTA reaches a new linear it quantises that linear's
//    x itself (same fp32 arithmetic as the quantisation kernel, so the same
//    bits) into shared memory, while its weight chunks are already in flight.
//    Only the LoRA vector u = s_B * h comes from the quantisation kernel (for
//    one token the slice kernel, which shares the SMs with this one), and the
//    CTA waits for that kernel (programmatic dependent launch) just before its
//    first epilogue.
//  * Expansion: for a 32-bit word of sign bits w and bit position p,
//    w & (0x01010101 << p) is four bytes, each 0 or 2^p: the bits of columns
//    8i + p (i = 0..3) scaled by 2^p. One LOP3 expands four weights.
//  * These bytes are the u8 A operand of the warp MMA m16n8k32 (u8 x s8 -> s32),
//    loaded with ldmatrix.x4 straight from the staged bits; the int8
//    activations in the matching permuted column order (byte 4p + i of a
//    32-column group = column 8i + p) are the s8 B operand, tokens = N. In
//    shared memory each 256-column group of a token row is laid out so that
//    thread c of a quad reads its 16 B-fragment words with four 16-byte loads
//    as (b0, b1) register pairs, one pair per bit position p.
//  * One accumulator set per p, so set p sums 2^p * S_p exactly;
//    S1 = sum_p D_p / 2^p = sum_{bit = 1} q, and acc = 2 * S1 - sum_j q
//    (a +-1 weight is 2b - 1).
//  * Epilogue (epilogue.cuh): lane i of a warp takes output row i, gathers its
//    sums with warp shuffles, and applies the LoRA up-projection and the
//    dequantisation in the same fp32 order as the prefill path.
#include <algorithm>
#include <cstring>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kMaxWarps = 12;      // warps per CTA: 4 (up to 8 tokens) or 12 (9 to 16 tokens)
#ifndef DFSSM_DECODE_CHUNK_BYTES
#define DFSSM_DECODE_CHUNK_BYTES 128
#endif
#ifndef DFSSM_DECODE_STAGES
#define DFSSM_DECODE_STAGES 2
#endif
constexpr int kChunkBytes = DFSSM_DECODE_CHUNK_BYTES;   // sign bytes per row per k-chunk (8 columns per byte)
constexpr int kGroups = kChunkBytes / 32;                // 256-column groups per chunk
constexpr int kTokPad = 64;        // q row stride = round_up(d_in, 256) + 64 (= 64 mod 128: conflict-free B reads)

// every 256-column group of a staged q row takes 256 bytes, even a half-filled last one
__host__ __device__ __forceinline__ int q_stride(int d_in) { return ((d_in + 255) & ~255) + kTokPad; }
constexpr int kStages = DFSSM_DECODE_STAGES;
constexpr int kMaxTok = 16;

constexpr int kStartTable = 600;   // CTAs whose start the host supplies (keeps the arguments under 4 KB)
constexpr int kMapSlots = 4;       // device-edited maps per CTA; >= kStages, so a slot's old loads are done
constexpr int kMaxCtasPerSm = 8;   // map slots are allocated for this many CTAs per SM
static_assert(kMapSlots >= kStages, "map slot reuse");

struct DecodeArgs {
    CUtensorMap single_map;  // sign map of `single` (one linear), encoded on the host
    const CUtensorMap* tmpl; // stack: per linear, its sign map with a placeholder address
    CUtensorMap* map_slots;  // stack: kMapSlots per CTA
    uint64_t wait_limit_ns;
    int stall_test;          // test hook: CTA 0 waits on a barrier nothing arrives on
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* desc;     // desc[0] is the first linear of this launch
    int n;
    int m;
    const int* part;         // partial h of the quantisation kernel, per split
    int splits;
    int slices;              // 1: one token, partial h per kLoraSliceCols-column slice (lora_slice_kernel)
    int64_t total_units;     // decode work units of the n linears (dfssm_internal.cuh)
    int ri;                  // which work_begin: 0 for 128-row blocks, 1 for 192-row blocks
    int slot_bytes;          // bytes of one ring slot
    int q_region;            // bytes of the staged-q region
    // the grid's contiguous work ranges, found on the host: range r runs from start[r] (linear
    // << 16 | block) up to start[r + 1], so a CTA needs no search through the descriptors before
    // its first loads; CTA i runs range perm[i]. has_start = 0 when the grid is larger than the
    // table (CTA i then finds range i itself).
    int has_start;
    uint32_t* err;           // the plan's device error word
    uint32_t start[kStartTable];
    uint16_t perm[kStartTable];
};
static_assert(sizeof(DecodeArgs) <= 4096, "decode kernel arguments");

// Fields of one linear, cached in registers while a cursor is on it.
// (kStartTable is defined before DecodeArgs.)
struct Lin {
    int d_in, d_out, rb, nchunks, nblocks, y_dtype;
    int bunits;              // work units of one block
    int64_t work_rel;        // first work unit relative to desc[0]
    const uint8_t* sign;
    const float* alpha;
    const float* sa;
    const int8_t* wa;
    const float* sb;
    const uint16_t* x;
    void* y;
    int32_t* dbg_acc;
    int32_t* dbg_h;
    bool ok;                 // entry pointers valid
};

template <int R>
__device__ __forceinline__ void load_lin(const DecodeArgs& a, int l, Lin& L) {
    const DevDesc& d = a.desc[l];
    const dfssm_stack_entry& e = entry_at(a.entries, a.single, l);
    L.d_in = d.d_in;
    L.d_out = d.d_out;
    L.rb = d.d_in >> 3;
    L.nchunks = (d.d_in / 8 + kChunkBytes - 1) / kChunkBytes;
    L.bunits = decode_block_units(d.d_in);
    L.nblocks = (d.d_out + R - 1) / R;
    L.y_dtype = d.y_dtype;
    L.work_rel = d.work_begin[a.ri] - a.desc[0].work_begin[a.ri];
    L.sign = e.w.sign;
    L.alpha = e.w.alpha;
    L.sa = e.w.sa;
    L.wa = e.w.wa;
    L.sb = e.w.sb;
    L.x = reinterpret_cast<const uint16_t*>(e.x);
    L.y = e.y;
    L.dbg_acc = e.dbg.acc;
    L.dbg_h = e.dbg.h;
    L.ok = entry_ptrs_ok(e);
}

struct Cursor {
    int l, b, kc;   // linear, block within the linear, k-chunk within the block
};

template <int R>
struct Walk {
    Cursor c;
    Lin L;
    // with the host's start table a CTA runs up to the next CTA's first block (`end`, packed as
    // linear << 16 | block); otherwise up to its last work unit `hi`
    __device__ __forceinline__ bool valid(const DecodeArgs& a, int64_t hi, uint32_t end) const {
        if (a.has_start) return (((uint32_t)c.l << 16) | (uint32_t)c.b) < end;
        return c.l < a.n && L.work_rel + kDecodeLinStart + (int64_t)c.b * L.bunits < hi;
    }
    __device__ __forceinline__ void advance(const DecodeArgs& a) {
        if (++c.kc >= L.nchunks) {
            c.kc = 0;
            if (++c.b >= L.nblocks) {
                c.b = 0;
                if (++c.l < a.n) load_lin<R>(a, c.l, L);
            }
        }
    }
    // start at (linear l, block b), as found by the host
    __device__ void start_at(const DecodeArgs& a, int l, int b) {
        c = Cursor{l, b, 0};
        if (c.l < a.n) load_lin<R>(a, c.l, L);
    }
    // first block whose first work unit is at or after `lo` (a linear's blocks follow its
    // kDecodeLinStart entry units)
    __device__ void start(const DecodeArgs& a, int64_t lo) {
        const int64_t base = a.desc[0].work_begin[a.ri];
        int lo_l = 0, hi_l = a.n - 1;
        while (lo_l < hi_l) {
            const int mid = (lo_l + hi_l + 1) >> 1;
            if (a.desc[mid].work_begin[a.ri] - base <= lo) lo_l = mid; else hi_l = mid - 1;
        }
        c = Cursor{lo_l, 0, 0};
        load_lin<R>(a, c.l, L);
        const int64_t rel = lo - L.work_rel - kDecodeLinStart;
        c.b = rel <= 0 ? 0 : (int)((rel + L.bunits - 1) / L.bunits);
        if (c.b >= L.nblocks) {
            c.b = 0;
            if (++c.l < a.n) load_lin<R>(a, c.l, L);
        }
    }
};

// Control block in shared memory.
struct DecCtl {
    alignas(128) uint8_t map_s[128];   // tensor map being edited (stack calls)
    uint64_t full[kStages];            // slot filled: TMA bytes + every thread's cp.async
    uint64_t never;                    // test hook: nothing arrives on it
};

// Fill a ring slot with k-chunk kc of block b: R rows x 128 sign bytes by one TMA load (thread 0),
// plus alpha, s_A and W_A of the block (cp.async, all threads) when kc is its last chunk. Every
// thread then arrives on the slot's barrier once its own copies have landed.
template <int R, int W>
__device__ __forceinline__ void issue_step(const Cursor& c, const Lin& L, uint32_t slot_s, const CUtensorMap* map,
                                           uint64_t* full) {
    constexpr int kThreads = W * 32;
    const int row0 = c.b * R;
    if (L.ok) {
        if (threadIdx.x == 0) {
            ptx::mbar_arrive_expect_tx(full, (uint32_t)(R * kChunkBytes));
            ptx::tma_load_2d_s(slot_s, map, kChunkBytes * c.kc, row0, full);
        }
        if (c.kc == L.nchunks - 1) {
            const int nrows = min(R, L.d_out - row0);
            const uint32_t par = slot_s + R * kChunkBytes;
            const int n4 = (nrows + 3) >> 2;
            for (int i = threadIdx.x; i < n4; i += kThreads) {
                const uint32_t bytes = (uint32_t)min(16, 4 * (nrows - 4 * i));
                ptx::cp_async16_zfill_s(par + 16 * i, L.alpha + row0 + 4 * i, bytes);
                ptx::cp_async16_zfill_s(par + 4 * R + 16 * i, L.sa + row0 + 4 * i, bytes);
            }
            for (int r = threadIdx.x; r < nrows; r += kThreads)
                ptx::cp_async16_s(par + 8 * R + 16 * r, L.wa + (int64_t)(row0 + r) * kRank);
        }
    } else if (threadIdx.x == 0) {
        ptx::mbar_arrive(full);        // bad entry (flagged by the quantisation kernel): nothing is read
    }
    ptx::cp_async_mbar_arrive_noinc(full);
}

// The sign map for linear l: the launch's own map (one linear), or this CTA's next map slot
// with the linear's template and its sign address (all 32 lanes of warp 0 call this).
__device__ __forceinline__ const CUtensorMap* linear_map(const DecodeArgs& a, const Lin& L, int l, int& nmap,
                                                        DecCtl& dc) {
    if (a.entries == nullptr || !L.ok) return &a.single_map;
    const int lane = threadIdx.x & 31;
    CUtensorMap* ms = a.map_slots + (size_t)blockIdx.x * kMapSlots + (nmap++ % kMapSlots);
    if (lane < 8) reinterpret_cast<uint4*>(dc.map_s)[lane] = reinterpret_cast<const uint4*>(a.tmpl + l)[lane];
    __syncwarp();
    if (lane == 0) ptx::tensormap_replace_addr(dc.map_s, L.sign);
    __syncwarp();
    ptx::tensormap_copy_release(ms, dc.map_s);
    if (lane == 0) ptx::tensormap_acquire(ms);
    __syncwarp();
    return ms;
}

// Shared-memory position of q for column 32 gg + 8 i + p of a token row (gg: 32-column
// group, i = 0..3, p = bit position). The 256-column group G = gg / 8 occupies 256
// bytes; thread c = gg % 4 of an MMA quad owns 64 of them, holding for each p the
// word of group gg (w = 0, B fragment b0) next to the word of group gg + 4 (w = 1,
// b1). Logical 16-byte chunk k = p / 2 of that block is stored at (k + c) mod 4, so
// the 8 lanes of a quarter-warp hit 8 different bank groups (with a token stride of
// 64 mod 128).
__device__ __forceinline__ int q_pos(int gg, int i, int p) {
    const int G = gg >> 3, c = gg & 3, w = (gg >> 2) & 1;
    return 256 * G + 64 * c + 16 * (((p >> 1) + c) & 3) + 8 * (p & 1) + 4 * w + i;
}

struct TokShared {
    float sx[kMaxTok];
    int sumq[kMaxTok];
    uint32_t amax_u[kMaxTok];          // max |x| per token as fp32 bit patterns
    float u[kMaxTok][kRank];
};

// Quantise the m x d_in activations of linear L into the permuted int8 layout
// (token stride d_in + kTokPad), with per-token s_x and sum q. Same arithmetic
// as the quantisation kernel (epilogue.cuh), so the same bytes. Both passes run over
// the (token, 8-column chunk) pairs of the whole m x d_in block, kQuantLoads 16-byte loads
// in flight per thread whatever m is; a thread's per-token max and sum go to shared memory
// (atomics) when its pairs move on to the next token.
constexpr int kQuantLoads = 4;
template <int W>
__device__ void quantise_into_smem(const Lin& L, int m, uint8_t* q_s, TokShared& ts) {
    constexpr int kThreads = W * 32;
    const int tid = threadIdx.x;
    const int n8 = L.d_in >> 3;                      // 8-column chunks per row
    const int total = m * n8;
    const int qstride = q_stride(L.d_in);
    const uint4* xv = reinterpret_cast<const uint4*>(L.x);    // pair k = t n8 + ch is xv[k]
    if (tid < m) {
        ts.amax_u[tid] = 0u;
        ts.sumq[tid] = 0;
    }
    __syncthreads();
    {
        uint32_t am = 0u;
        int tcur = -1;
        for (int k0 = tid; k0 < total; k0 += kQuantLoads * kThreads) {
            uint4 v[kQuantLoads];
#pragma unroll
            for (int j = 0; j < kQuantLoads; ++j) {
                const int k = k0 + j * kThreads;
                v[j] = k < total ? xv[k] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < kQuantLoads; ++j) {
                const int k = k0 + j * kThreads;
                if (k >= total) break;
                const int t = k / n8;
                if (t != tcur) {
                    if (tcur >= 0) atomicMax(&ts.amax_u[tcur], am);
                    am = 0u;
                    tcur = t;
                }
                am = absmax8_bits(v[j], am);
            }
        }
        if (tcur >= 0) atomicMax(&ts.amax_u[tcur], am);
    }
    __syncthreads();
    {
        int sum = 0, tcur = -1;
        float inv = 0.0f;
        bool zero = true;
        for (int k0 = tid; k0 < total; k0 += kQuantLoads * kThreads) {
            uint4 v[kQuantLoads];
#pragma unroll
            for (int j = 0; j < kQuantLoads; ++j) {
                const int k = k0 + j * kThreads;
                v[j] = k < total ? xv[k] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < kQuantLoads; ++j) {
                const int k = k0 + j * kThreads;
                if (k >= total) break;
                const int t = k / n8, ch = k - t * n8;
                if (t != tcur) {
                    if (tcur >= 0) atomicAdd(&ts.sumq[tcur], sum);
                    sum = 0;
                    tcur = t;
                    const float am = __uint_as_float(ts.amax_u[t]);
                    inv = quant_inv(am);
                    zero = am == 0.0f;
                }
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                // columns 8 ch + p (p = 0..7) of 32-column group gg = ch / 4 (i = ch % 4)
                uint8_t* row = q_s + t * qstride;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int q0 = quant1(bf16_lo(w[i]), inv, zero), q1 = quant1(bf16_hi(w[i]), inv, zero);
                    sum += q0 + q1;
                    row[q_pos(ch >> 2, ch & 3, 2 * i)] = (uint8_t)q0;
                    row[q_pos(ch >> 2, ch & 3, 2 * i + 1)] = (uint8_t)q1;
                }
            }
        }
        if (tcur >= 0) atomicAdd(&ts.sumq[tcur], sum);
    }
    if (tid < m) ts.sx[tid] = quant_sx(__uint_as_float(ts.amax_u[tid]));
    // (the caller synchronises before sumq and sx are read)
}

template <int RT, int NT, int W>
__global__ void __launch_bounds__(W * 32) decode_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int kThreads = W * 32;
    constexpr int R = 16 * RT * W;
    extern __shared__ __align__(1024) uint8_t smem[];
    // 1024-byte aligned ring first (the 128-byte swizzle of the TMA boxes repeats every 1 KB)
    uint8_t* ring = smem + ((1024u - (ptx::smem_u32(smem) & 1023u)) & 1023u);
    uint8_t* q_s = ring + kStages * a.slot_bytes;
    TokShared& ts = *reinterpret_cast<TokShared*>(q_s + a.q_region);
    DecCtl& dc = *reinterpret_cast<DecCtl*>(q_s + a.q_region + ((sizeof(TokShared) + 127) & ~(size_t)127));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int m = a.m;
    const uint64_t lim = a.wait_limit_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) ptx::mbar_init(&dc.full[s], 1 + kThreads);
        ptx::mbar_init(&dc.never, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (a.stall_test && blockIdx.x == 0) {
        // test hook: a wait that nothing ends; every thread gives up after the limit, the CTA
        // reports DFSSM_DEVERR_TIMEOUT and stops before issuing anything
        const bool ok = ptx::mbar_wait(&dc.never, 0u, lim);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
            return;
        }
    }

    const int64_t lo = a.total_units * blockIdx.x / gridDim.x;
    const int64_t hi = a.total_units * (blockIdx.x + 1) / gridDim.x;
    const int range = a.has_start ? (int)a.perm[blockIdx.x] : (int)blockIdx.x;
    const uint32_t end = a.has_start && range + 1 < (int)gridDim.x ? a.start[range + 1] : ((uint32_t)a.n << 16);
    Walk<R> cw, lw;
    if (a.has_start) cw.start_at(a, (int)(a.start[range] >> 16), (int)(a.start[range] & 0xFFFFu));
    else cw.start(a, lo);
    lw = cw;
    // the first linear's activations into L2 ahead of the weight stream (quantised below)
    if (cw.valid(a, hi, end) && cw.L.ok) {
        const char* xp = reinterpret_cast<const char*>(cw.L.x);
        const int xbytes = m * cw.L.d_in * 2;
        for (int off = 16 * tid; off < xbytes; off += 16 * kThreads)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(xp + off));
    }

    // ---- prologue: kStages - 1 slots in flight (warp 0 keeps the sign map of the look-ahead
    // cursor's linear; thread 0 issues the TMA loads)
    const CUtensorMap* map = &a.single_map;
    int map_lin = -1, nmap = 0;
    auto issue = [&](int slot) {
        if (warp == 0 && lw.c.l != map_lin) {
            map = linear_map(a, lw.L, lw.c.l, nmap, dc);
            map_lin = lw.c.l;
        }
        issue_step<R, W>(lw.c, lw.L, ptx::smem_u32(ring + slot * a.slot_bytes), map, &dc.full[slot]);
        lw.advance(a);
    };
    int issued = 0;
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (lw.valid(a, hi, end)) {
            issue(s);
            ++issued;
        }
    }
    bool failed = false;

    int D[RT][NT][8][4];
    int q_lin = -1, u_lin = -1;
    // ldmatrix lane role: matrix (lane / 8) = (row half, 16-byte half of the 32-byte group)
    const int lm_row = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int lm_hi = lane >> 4;
    const int wrow0 = warp * 16 * RT;             // first row of this warp in a block
    const int q_off = (int)(q_s - smem);          // staged q, as an offset into the shared array

    for (int it = 0; cw.valid(a, hi, end); ++it) {
        const Lin& L = cw.L;
        if (cw.c.l != q_lin) {
            // a new linear: quantise its activations (its weights are already streaming)
            if (L.ok) quantise_into_smem<W>(L, m, q_s, ts);
            q_lin = cw.c.l;
            __syncthreads();
        }
        if (lw.valid(a, hi, end)) {
            issue((it + kStages - 1) % kStages);
            ++issued;
        }
        // this chunk's slot: TMA bytes and every thread's cp.async landed
        if (!ptx::mbar_wait(&dc.full[it % kStages], (uint32_t)((it / kStages) & 1), lim)) failed = true;
        const bool last_chunk = cw.c.kc == L.nchunks - 1;
        if (last_chunk && u_lin != cw.c.l) {
            // the LoRA vector u = s_B * h of this linear: h is the sum, in split order, of the
            // quantisation kernel's partials (exact integers)
            ptx::pdl_wait();
            for (int i = tid; i < m * kRank; i += kThreads) {
                const int t = i >> 4, k = i & 15;
                const int nsp = a.slices ? lora_slices(L.d_in) : a.splits;
                const int stride = a.slices ? kLoraMaxSlices : a.splits;
                int h = 0;
                for (int sp = 0; sp < nsp; ++sp) h += __ldcg(a.part + part_index(cw.c.l, stride, sp, t, k));
                ts.u[t][k] = __fmul_rn(L.sb[k], (float)h);
                if (L.dbg_h) L.dbg_h[(int64_t)t * kRank + k] = h;
            }
            u_lin = cw.c.l;
            __syncthreads();
        }

        const uint8_t* slot = ring + (it % kStages) * a.slot_bytes;
        const int row0 = cw.c.b * R;
        const int nrows = min(R, L.d_out - row0);
        const bool active = wrow0 < nrows && L.ok;
        if (cw.c.kc == 0) {
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int p = 0; p < 8; ++p)
#pragma unroll
                        for (int r = 0; r < 4; ++r) D[rt][nt][p][r] = 0;
        }
        if (active) {
            const int qstride = q_stride(L.d_in);
            const int cb = min(kChunkBytes, L.rb - kChunkBytes * cw.c.kc);
            const uint32_t slot_s = ptx::smem_u32(slot);
            // ldmatrix row addresses: the TMA's 128-byte swizzle puts row r's 16-byte piece j at
            // j ^ (r & 7); rows of a tile start at multiples of 16, so the XOR depends on the lane only
            const int sw = lm_row & 7;
            uint32_t a_addr[RT][kGroups];
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                for (int G = 0; G < kGroups; ++G)
                    a_addr[rt][G] = slot_s + (wrow0 + 16 * rt + lm_row) * kChunkBytes + 16 * ((2 * G + lm_hi) ^ sw);
            // B rows: tokens nt * 8 + g; lanes past m read token 0 (their MMA columns are never stored)
            // (32-bit offsets into the shared array, so the loads need no 64-bit address math)
            int qk[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tk = nt * 8 + g;
                const int qrow = q_off + (tk < m ? tk : 0) * qstride + 256 * (kGroups * cw.c.kc) + 64 * c;
#pragma unroll
                for (int k = 0; k < 4; ++k) qk[nt][k] = qrow + 16 * ((k + c) & 3);
            }
            auto group = [&](int G, bool half) {
                uint32_t A[RT][4];
#pragma unroll
                for (int rt = 0; rt < RT; ++rt) {
                    ptx::ldmatrix_x4(a_addr[rt][G], A[rt][0], A[rt][1], A[rt][2], A[rt][3]);
                    // half group: zero A slots 16..31, so whatever b1 holds there adds nothing
                    if (half) { A[rt][2] = 0u; A[rt][3] = 0u; }
                }
                // B: chunk k (bit positions 2k, 2k+1) = (b0, b1) of p = 2k, then of p = 2k + 1
                uint4 bq[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) bq[nt][k] = *reinterpret_cast<const uint4*>(smem + qk[nt][k] + 256 * G);
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const uint32_t msk = 0x01010101u << p;
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt) {
                        const uint32_t a0 = A[rt][0] & msk, a1 = A[rt][1] & msk;
                        const uint32_t a2 = A[rt][2] & msk, a3 = A[rt][3] & msk;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint4& v = bq[nt][p >> 1];
                            if (p & 1) ptx::mma_u8s8(D[rt][nt][p], a0, a1, a2, a3, v.z, v.w);
                            else       ptx::mma_u8s8(D[rt][nt][p], a0, a1, a2, a3, v.x, v.y);
                        }
                    }
                }
            };
            if (cb == kChunkBytes) {
                // full chunk: whole groups, straight-line code
#pragma unroll
                for (int G = 0; G < kGroups; ++G) group(G, false);
            } else {
                const int ng = (cb + 31) >> 5;             // groups of 256 columns in this chunk
#pragma unroll
                for (int G = 0; G < kGroups; ++G)
                    if (G < ng) group(G, (cb - 32 * G) == 16);
            }

            // ---- epilogue after the block's last k-chunk
            if (last_chunk) {
                // combine the bit-position accumulators: T = sum_p D_p * 2^(7-p) = 128 * S1
                int T[RT][NT][4];
#pragma unroll
                for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            int s = 0;
                            if ((r & 1) == 0 || m > 1) {
#pragma unroll
                                for (int p = 0; p < 8; ++p) s += D[rt][nt][p][r] << (7 - p);
                            }
                            T[rt][nt][r] = s;
                        }
                // lane -> (row of this warp, n-tile); D fragment of (row, token t) sits in
                // thread (row % 8) * 4 + (t % 8) / 2, register 2 * ((row / 8) % 2) + t % 2
                constexpr int kRowsW = 16 * RT;
                const int my_row = lane % kRowsW;
                const int my_nt = lane / kRowsW;            // 0, or 1 when RT = 1 and NT = 2
                const int rr = wrow0 + my_row;
                const bool row_ok = rr < nrows;
                const float* alpha_s = reinterpret_cast<const float*>(slot + R * kChunkBytes);
                const float* sa_s = alpha_s + R;
                const int4* wa_s = reinterpret_cast<const int4*>(slot + R * kChunkBytes + 8 * R);
                const float alpha = alpha_s[rr], sa = sa_s[rr];
                const WaRow wa = wa_row_from_int4(wa_s[rr]);
                const int jmax = NT == 1 ? m : 8;
                // j unrolled so every register index is a constant (no local-memory copy of T)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j >= jmax) break;
                    const int src = (my_row & 7) * 4 + (j >> 1);
                    int v_lo[RT][NT], v_hi[RT][NT];
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            v_lo[rt][nt] = __shfl_sync(0xffffffffu, T[rt][nt][j & 1], src);
                            v_hi[rt][nt] = __shfl_sync(0xffffffffu, T[rt][nt][2 + (j & 1)], src);
                        }
                    int val = 0;
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            if (rt == (my_row >> 4) && nt == my_nt) val = ((my_row >> 3) & 1) ? v_hi[rt][nt] : v_lo[rt][nt];
                    const int t = 8 * my_nt + j;
                    if (t < m && row_ok) {
                        const int acc = 2 * (val >> 7) - ts.sumq[t];
                        const float y = dequant(ts.sx[t], alpha, sa, acc, lora_dot(wa, ts.u[t]));
                        const int64_t idx = (int64_t)t * L.d_out + row0 + rr;
                        if (L.y_dtype == DFSSM_BF16)
                            reinterpret_cast<uint16_t*>(L.y)[idx] = f32_to_bf16_bits(y);
                        else
                            reinterpret_cast<float*>(L.y)[idx] = y;
                        if (L.dbg_acc) L.dbg_acc[idx] = acc;
                    }
                }
            }
        }
        // slot it % kStages is refilled by the next iteration; a wait that gave up ends the CTA
        if (__syncthreads_or(failed)) {
            if (tid == 0) {
                atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
                // let the loads still in flight into this CTA's shared memory land (bounded)
                for (int j = it; j < issued; ++j) ptx::mbar_wait(&dc.full[j % kStages], (uint32_t)((j / kStages) & 1), lim);
            }
            break;
        }
        cw.advance(a);
    }
    ptx::cp_async_wait<0>();
}

struct Geometry {
    int slot_bytes, q_region;
    size_t smem;
};

// Ring slots of R x 128 sign bytes + the block's alpha, s_A, W_A, each a multiple of 1 KB (the
// TMA swizzle pattern repeats every 1 KB); then the staged q, the per-token values and the
// control block; 1 KB for aligning the base.
template <int RT, int W>
Geometry geometry(int m, int max_d_in) {
    constexpr int R = 16 * RT * W;
    Geometry g;
    g.slot_bytes = (R * kChunkBytes + R * (4 + 4 + kRank) + 1023) & ~1023;
    g.q_region = (m * q_stride(max_d_in) + 127) & ~127;
    g.smem = 1024 + (size_t)kStages * g.slot_bytes + g.q_region + ((sizeof(TokShared) + 127) & ~(size_t)127) +
             sizeof(DecCtl);
    return g;
}

template <int RT, int NT, int W>
cudaError_t launch_cfg(const LaunchCtx& c) {
    constexpr int R = 16 * RT * W;
    constexpr int kThreads = W * 32;
    const Geometry geo = geometry<RT, W>(c.m, c.max_d_in);
    static_assert(R == 128 || R == 192, "work units exist for 128- and 192-row blocks");
    static_assert(kChunkBytes * 8 == kDecodeChunkCols, "kUnitChunk work units per k-chunk");
    int64_t total_units = 0;
    int blocks = 0;
    for (int i = 0; i < c.n; ++i) {
        total_units += decode_units(c.host_desc[i].d_in, c.host_desc[i].d_out, R);
        blocks += (c.host_desc[i].d_out + R - 1) / R;
    }
    int per_sm = 0;
    cudaError_t err =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<RT, NT, W>, kThreads, geo.smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (per_sm > kMaxCtasPerSm) per_sm = kMaxCtasPerSm;     // the plan's map slots
    int grid = c.sm_count * per_sm;
    if (grid > blocks) grid = blocks;
    DecodeArgs a;
    std::memset(&a.single_map, 0, sizeof(a.single_map));
    if (c.entries == nullptr) {
        if (!encode_sign_map(&a.single_map, c.single.w.sign, c.host_desc[0].d_in, c.host_desc[0].d_out, R))
            return cudaErrorInvalidValue;
    } else if (c.sign_tmpl == nullptr || c.map_slots == nullptr) {
        return cudaErrorInvalidValue;
    }
    a.tmpl = reinterpret_cast<const CUtensorMap*>(c.sign_tmpl) + (R == 128 ? 0 : c.tmpl_stride);
    a.map_slots = reinterpret_cast<CUtensorMap*>(c.map_slots);
    a.wait_limit_ns = c.wait_limit_ns;
    a.stall_test = c.stall_test;
    a.entries = c.entries;
    a.single = c.single;
    a.desc = c.desc;
    a.n = c.n;
    a.m = c.m;
    a.part = c.part;
    a.splits = quant_splits(c);
    a.slices = use_lora_slices(c) ? 1 : 0;
    a.total_units = total_units;
    a.ri = R == 128 ? 0 : 1;
    a.slot_bytes = geo.slot_bytes;
    a.q_region = geo.q_region;
    a.has_start = 0;
    a.err = c.err;
    // the grid's work ranges: range i starts at the first block at or after work unit
    // total_units * i / grid (as Walk::start finds it on the device) and runs up to range i + 1
    if (grid <= kStartTable && c.n < 65536) {
        bool fits = true;
        const int ri = R == 128 ? 0 : 1;
        const int64_t base = c.host_desc[0].work_begin[ri];
        int64_t pos[kStartTable + 1];      // first work unit of each range (its entry included)
        int l = 0;
        for (int i = 0; i < grid && fits; ++i) {
            const int64_t lo = total_units * i / grid;
            while (l + 1 < c.n && c.host_desc[l + 1].work_begin[ri] - base <= lo) ++l;
            const DevDesc& d = c.host_desc[l];
            const int bu = decode_block_units(d.d_in);
            const int nblocks = (d.d_out + R - 1) / R;
            const int64_t rel = lo - (d.work_begin[ri] - base) - kDecodeLinStart;
            int b = rel <= 0 ? 0 : (int)((rel + bu - 1) / bu);
            int sl = l;
            if (b >= nblocks) { b = 0; ++sl; }
            if (b > 0xFFFF) fits = false;
            a.start[i] = ((uint32_t)sl << 16) | (uint32_t)b;
            pos[i] = sl >= c.n ? total_units
                               : c.host_desc[sl].work_begin[ri] - base + (b > 0 ? kDecodeLinStart + (int64_t)b * bu : 0);
        }
        pos[grid] = total_units;
        a.has_start = fits ? 1 : 0;
        // Which CTA runs which range. Ranges end on block boundaries, so their costs differ by up
        // to a block (2 or 4 k-chunks in about 21 for the one-token stack), and a stack whose
        // linears repeat with the grid's period gives the CTAs that share an SM (CTAs i, i + S,
        // i + 2S, ... for S SMs when all are resident) equal ranges, so some SMs carry a whole
        // block per CTA more than others. Ranges are therefore dealt by cost, largest first, in
        // passes over the SMs that alternate direction; pass w goes to the CTAs i = w S + g, so
        // the first-launched CTA of an SM (the fastest of its CTAs in a per-CTA timing trace)
        // takes the largest.
        // The placement of CTAs on SMs is the hardware's: this only decides which range each CTA
        // index runs, so the results never depend on it.
        int order[kStartTable];
        for (int i = 0; i < grid; ++i) order[i] = i;
        const int S = c.sm_count;
        if (fits && grid == S * per_sm && per_sm > 1) {
            int64_t cost[kStartTable];
            for (int i = 0; i < grid; ++i) {
                const bool mid = (a.start[i] & 0xFFFFu) != 0;   // a CTA entering mid-linear quantises too
                cost[i] = pos[i + 1] - pos[i] + (mid ? kDecodeLinStart : 0);
            }
            std::stable_sort(order, order + grid, [&](int x, int y) { return cost[x] > cost[y]; });
            for (int w = 0; w < per_sm; ++w)
                for (int g = 0; g < S; ++g) a.perm[w * S + g] = (uint16_t)order[w * S + ((w & 1) ? S - 1 - g : g)];
        } else {
            for (int i = 0; i < grid; ++i) a.perm[i] = (uint16_t)i;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<RT, NT, W>, a);
}

}  // namespace

cudaError_t launch_decode(const LaunchCtx& c) {
    if (c.m <= 8) return launch_cfg<2, 1, 4>(c);
    return launch_cfg<1, 2, 12>(c);
}

// The decode kernel's tensor map over a linear's sign rows: d_out rows of d_in / 8 bytes, boxes of
// 128 bytes x `rows` (the block rows), 128-byte swizzle, zeros outside the matrix.
bool encode_sign_map(CUtensorMap* map, const void* sign, int d_in, int d_out, int rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const int rb = d_in / 8;
    cuuint64_t dims[2] = {(cuuint64_t)rb, (cuuint64_t)d_out};
    cuuint64_t strides[1] = {(cuuint64_t)rb};
    cuuint32_t box[2] = {(cuuint32_t)kChunkBytes, (cuuint32_t)rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(sign), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int decode_map_slots_per_sm() { return kMapSlots * kMaxCtasPerSm; }
int decode_block_rows(int m) { return m <= 8 ? 128 : 192; }

// The largest shared-memory carveout. Registers allow three decode CTAs per SM; with two ring
// slots three CTAs also fit in shared memory up to about 8 tokens (about 58 KB each at 4 tokens),
// beside the one-token slice kernel's CTA (34 KB) at one token. A third slot would leave two CTAs
// (8 warps) per SM from 2 tokens on, and the kernel is bound by issue latency, not by bytes in
// flight: measured on the 48-layer stack, 2 slots take 4 tokens from 90.5 to 77.7 us and 16
// tokens from 210 to 191 us, with one token unchanged (59.5 us).
cudaError_t set_decode_attr(int optin) {
    cudaError_t e = allow_dyn_smem(decode_kernel<2, 1, 4>, optin);
    if (e == cudaSuccess) e = allow_dyn_smem(decode_kernel<1, 2, 12>, optin);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_kernel<2, 1, 4>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_kernel<1, 2, 12>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    return e;
}

}  // namespace dfssm
