// Activation quantisation for many tokens (m > 16): the input stage of the
// tensor-core prefill.
//
// Same quantiser and LoRA down-projection as quant.cu ("Density Field State
// Space Models", gist.science technical summary, §2.B: int8 LoRA W_B with
// per-row scales; §2.C: int8 activations for the int8 x int8 -> int32
// scaffold matmul), arranged for throughput over a large activation matrix.
//
// Persistent kernel, one block of 16 warps per SM. Work items are T tokens of
// one linear, T = min(16, 32768 / d_in), so an item is at most 64 KB of bf16;
// the items of a linear are numbered in token order, the linears follow each
// other, and each block takes one contiguous range of items (so it meets few
// linears and keeps their W_B fragments in registers). Per item:
//   issue (warp 0, two items ahead, as soon as the tile is free): the item's
//     descriptor (shape, offsets, pointers, s_B; looked up in global memory
//     only when the linear changes) goes to a shared ring, and its rows (one
//     contiguous range of x) come in by a single bulk copy (TMA engine, no
//     tensor map, no multicast) into one of two shared x tiles: x is read from
//     HBM once, and the next item streams in while one is processed;
//   1. each thread loads its (up to two) 32-column groups of the tile into
//      registers and takes their max |x| as a 16-bit SIMD max over the bit
//      patterns (the unsigned order of |bf16| bits is the numeric order, NaN
//      above Inf, so a non-finite row is still seen); per token the maximum
//      is gathered by shuffles and a shared atomic max;
//   2. rint(x * inv) by adding 1.5 * 2^23 in round-to-nearest-even, exact here
//      because |x * inv| <= 127 * (1 + 2^-23); the low byte of the sum is q.
//      Each group's eight plane words (the plane-major order of the prefill's
//      activation rows) go to global memory (eight lanes fill one 32-byte
//      sector) and to a shared q tile in the same order;
//   3. h^T = W_B q^T on the warp MMA (m16n8k32, s8 x s8 -> s32): the 16 LoRA
//      rows are M and 8 tokens N, so T <= 8 takes one MMA per 32 bytes of K
//      and T = 16 two; the K order is the plane-major one of the shared tile,
//      so the W_B fragments are gathered in that order. sum q comes from dp4a
//      on the same q fragments. Warp w takes k-blocks w, w + 16, ...;
//   4. the 16 warp partials are added in shared memory; u = s_B h, s_x, sum q.
// Three barriers per item. No integer division per item: token and group of a
// thread come from an fp32 reciprocal of d_in / 32, exact at these sizes (the
// quotient's fractional part stays at least 1/512 away from an integer).
#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kConsumers = 512;             // all threads of the block
constexpr int kCWarps = kConsumers / 32;     // 16
constexpr int kThreads = kConsumers;
constexpr int kItemElems = 32768;            // bf16 values of one item at most (64 KB)
constexpr int kGroupsPerThread = kItemElems / 32 / kConsumers;   // 2
constexpr int kMaxT = 16;                    // tokens per item at most (two MMA n-tiles)
constexpr int kBufs = 2;                     // x tiles
constexpr int kInfos = kBufs + 2;            // item descriptors (stage 4 of item k runs beside the issue of k + 3)
constexpr int kIssueWarp = 15;               // issues items (stage 4 runs on warps 0..8)
// shared q rows: plane-major like the global rows, but segments 288 bytes apart (the plane words of
// the 4 segments a warp writes land on distinct banks) and rows 16 bytes longer than that (the 8
// token rows an ldmatrix reads land on distinct banks)
constexpr int kQsSegStride = kSegCols + 32;
constexpr int kQsRowPad = 16;
constexpr int kHCols = kRank + 1;            // h[0..15] and sum q
// largest T * (segments * 288 + 16) over d_in (T * d_in <= 32768)
constexpr int kQsBytes = 41984;
constexpr int kWbRegKb = 8;                  // k-blocks per warp whose W_B fragments stay in registers (d_in <= 4096)
constexpr uint32_t kBarConsumers = 1;        // named barrier of the 16 warps

struct ItemInfo {
    int lin, t0, nt, d_in;
    int T, qrow, usable, pad0;
    float rgpt, pad1;                        // 1 / (d_in / 32)
    int64_t q_off, st_off;
    const int8_t* wb;
    int8_t* dbg_q;
    int32_t* dbg_h;
    float* dbg_sx;
    float sb[kRank];
};

// Position in the item sequence and the linear of the last descriptor written.
struct Cursor {
    int lin, begin, count, tpi, info_lin;
    const uint16_t* x;
    int d_in, usable;
};

struct RowsShared {
    uint16_t x[kBufs][kItemElems];           // bf16 tiles, bulk-copy destinations
    int8_t q[kQsBytes];                      // q of the item, plane-major rows (see kQsSegStride)
    int h[kCWarps][kMaxT][kHCols];           // per-warp partial h and sum q
    ItemInfo info[kInfos];
    uint32_t amax_tok[2][kMaxT];             // max |x| per token (fp32 bit pattern), by item parity
    float sx[2][kMaxT];                      // s_x per token, by item parity
    Cursor cur;
    uint64_t full[kBufs];                    // tile and descriptor ready
};

__host__ __device__ inline int tokens_per_item(int d_in) {
    const int t = kItemElems / d_in;
    return t < kMaxT ? t : kMaxT;
}

constexpr int kStartTable = 256;            // blocks whose first item's linear the host supplies

struct RowsArgs {
    const dfssm_stack_entry* entries;
    dfssm_stack_entry single;
    const DevDesc* descs;
    int n;
    int m;
    int total;              // items over all linears
    int8_t* q_ws;
    TokStats* st_ws;
    uint32_t* err;
    // the linear of each block's first item and that linear's first item index, found on the host,
    // so a block does not walk the descriptors from the first linear (has_start = 0: it does)
    int has_start;
    int start_lin[kStartTable];
    int start_item[kStartTable];
};

__device__ __forceinline__ void consumer_sync() { ptx::named_barrier(kBarConsumers, kConsumers); }

// barrier of the consumer warps that also ORs a predicate over them
__device__ __forceinline__ bool consumer_sync_or(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "barrier.red.or.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r) : "r"((uint32_t)p), "r"(kBarConsumers), "r"(kConsumers) : "memory");
    return r != 0;
}

// two bf16 (one word) -> y = rint(x * inv) + 1.5 * 2^23 as fp32 bits, whose low byte is q. The
// rounding add is the scalar __fadd_rn, which is never merged with the product into an FMA (a fused
// x * inv + 1.5 * 2^23 would skip the product's own rounding and can move a tie).
__device__ __forceinline__ void quant_pair(uint32_t w, float inv, uint32_t& y_lo, uint32_t& y_hi) {
    constexpr float kRound = 12582912.0f;   // 1.5 * 2^23: ulp 1
    const float2 p = fmul2(make_float2(bf16_lo(w), bf16_hi(w)), make_float2(inv, inv));
    y_lo = __float_as_uint(__fadd_rn(p.x, kRound));
    y_hi = __float_as_uint(__fadd_rn(p.y, kRound));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int h) {
    return h == 0 ? v.x : h == 1 ? v.y : h == 2 ? v.z : v.w;
}

__device__ __forceinline__ void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t saddr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(saddr));
}

// A fragment (m16n8k32: rows = LoRA rows g, g + 8) of k-block kb in the plane-major K order of
// the shared q tile: K position 32 p + 4 c' + i of segment s is column 256 s + 32 c' + 8 i + p
// (p = kb % 8, s = kb / 8); columns past d_in (the absent half of a final half segment) are zero.
// f[0] = row g, c' = cq; f[1] = row g + 8, c' = cq; f[2] = row g, c' = cq + 4; f[3] = row g + 8, c' = cq + 4.
__device__ __forceinline__ void wb_fragment(const int8_t* wb, int d_in, int kb, int g, int cq, uint32_t (&f)[4]) {
    const int s = kb >> 3, p = kb & 7;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int row = g + 8 * (r & 1);
        const int col0 = 256 * s + 32 * (cq + 4 * (r >> 1)) + p;
        uint32_t v = 0u;
        if (col0 < d_in) {
            const uint8_t* src = reinterpret_cast<const uint8_t*>(wb) + (int64_t)row * d_in + col0;
            v = (uint32_t)__ldg(src) | ((uint32_t)__ldg(src + 8) << 8) | ((uint32_t)__ldg(src + 16) << 16) |
                ((uint32_t)__ldg(src + 24) << 24);
        }
        f[r] = v;
    }
}

// the fragments of k-blocks warp + 16 j, j < kWbRegKb
__device__ __forceinline__ void load_wb_fragments(const int8_t* wb, int d_in, int warp, int g, int cq,
                                                  uint32_t (&wbf)[kWbRegKb][4]) {
    const int nkb = (d_in + kSegCols - 1) / kSegCols * 8;
#pragma unroll
    for (int j = 0; j < kWbRegKb; ++j) {
        const int kb = warp + kCWarps * j;
        if (kb < nkb) wb_fragment(wb, d_in, kb, g, cq, wbf[j]);
    }
}

// (token, group) of group index G: token = G / gpt by the fp32 reciprocal (exact here)
__device__ __forceinline__ int div_by_recip(int G, float r) { return __float2int_rz(((float)G + 0.5f) * r); }

// this block's contiguous range of items
__device__ __forceinline__ void item_range(const RowsArgs& a, int& lo, int& hi) {
    lo = (int)((int64_t)blockIdx.x * a.total / gridDim.x);
    hi = (int)((int64_t)(blockIdx.x + 1) * a.total / gridDim.x);
}

// ------------------------------------------------------------------ item issue (warp 0)
__device__ __forceinline__ void cursor_start(const RowsArgs& a, Cursor& cur) {
    cur.lin = a.has_start ? a.start_lin[blockIdx.x] : 0;
    cur.begin = a.has_start ? a.start_item[blockIdx.x] : 0;
    cur.tpi = tokens_per_item(a.descs[cur.lin].d_in);
    cur.count = (a.m + cur.tpi - 1) / cur.tpi;
    cur.info_lin = -1;
    cur.x = nullptr;
    cur.d_in = 0;
    cur.usable = 0;
}

// Warp 0, all lanes: write the descriptor of the block's kk-th item (global index `item`) and
// start its bulk copy into tile kk % kBufs, which no thread still reads. Items arrive in
// increasing order; a descriptor repeats its predecessor's linear fields unless the linear changed.
__device__ void issue_item(const RowsArgs& a, RowsShared& sh, Cursor& cur, int kk, int item, int lane) {
    if (lane == 0) {
        while (item >= cur.begin + cur.count && cur.lin + 1 < a.n) {
            cur.begin += cur.count;
            ++cur.lin;
            cur.tpi = tokens_per_item(a.descs[cur.lin].d_in);
            cur.count = (a.m + cur.tpi - 1) / cur.tpi;
        }
    }
    __syncwarp();
    ItemInfo& inf = sh.info[kk % kInfos];
    if (cur.lin != cur.info_lin) {
        const dfssm_stack_entry& e = entry_at(a.entries, a.single, cur.lin);
        const DevDesc d = a.descs[cur.lin];
        const bool desc_ok = a.entries == nullptr || e.desc_index == cur.lin;
        const bool usable = desc_ok && entry_ptrs_ok(e);
        if (lane < kRank) inf.sb[lane] = usable ? e.w.sb[lane] : 0.0f;
        if (lane == 0) {
            inf.lin = cur.lin;
            inf.d_in = d.d_in;
            inf.T = cur.tpi;
            inf.qrow = d.qrow;
            inf.usable = usable;
            inf.rgpt = 1.0f / (float)(d.d_in >> 5);
            inf.q_off = d.q_off;
            inf.st_off = d.st_off;
            inf.wb = reinterpret_cast<const int8_t*>(e.w.wb);
            inf.dbg_q = e.dbg.q;
            inf.dbg_h = e.dbg.h;
            inf.dbg_sx = e.dbg.sx;
            if (!usable) atomicOr(a.err, desc_ok ? DFSSM_DEVERR_ENTRY_PTR : DFSSM_DEVERR_ENTRY_DESC);
        }
        __syncwarp();
        if (lane == 0) {
            cur.info_lin = cur.lin;
            cur.x = reinterpret_cast<const uint16_t*>(e.x);
            cur.d_in = d.d_in;
            cur.usable = usable;
        }
    } else {
        // the same linear: copy the previous descriptor (still intact: it is rewritten two items later)
        static_assert(sizeof(ItemInfo) % 4 == 0 && sizeof(ItemInfo) / 4 <= 64, "descriptor copy");
        const uint32_t* src = reinterpret_cast<const uint32_t*>(&sh.info[(kk + kInfos - 1) % kInfos]);
        uint32_t* dst = reinterpret_cast<uint32_t*>(&inf);
        for (int i = lane; i < (int)(sizeof(ItemInfo) / 4); i += 32) dst[i] = src[i];
    }
    __syncwarp();
    if (lane == 0) {
        const int t0 = (item - cur.begin) * cur.tpi;
        const int nt = min(cur.tpi, a.m - t0);
        inf.t0 = t0;
        inf.nt = nt;
        const int slot = kk % kBufs;
        uint64_t* bar = &sh.full[slot];
        if (cur.usable) {
            const uint32_t bytes = (uint32_t)nt * (uint32_t)cur.d_in * 2u;
            ptx::mbar_arrive_expect_tx(bar, bytes);   // release: the descriptor above is visible
            ptx::bulk_g2s(sh.x[slot], cur.x + (int64_t)t0 * cur.d_in, bytes, bar);
        } else {
            ptx::mbar_arrive(bar);                    // nothing to copy: complete the phase
        }
    }
    __syncwarp();
}

__global__ void __launch_bounds__(kThreads, 1) quant_rows_kernel(const __grid_constant__ RowsArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    RowsShared& sh = *reinterpret_cast<RowsShared*>(smem_raw);
    // let the dependent prefill kernel start streaming weights; it waits for this grid before reading q
    ptx::pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < 2 * kMaxT) sh.amax_tok[tid >> 4][tid & 15] = 0u;
    if (tid == 0) {
        for (int b = 0; b < kBufs; ++b) ptx::mbar_init(&sh.full[b], 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int lo, hi;
    item_range(a, lo, hi);
    const int n_items = hi - lo;
    if (n_items <= 0) return;
    Cursor& cur = sh.cur;     // the issuing warp's state (shared memory: no registers in the other warps)
    if (warp == kIssueWarp) {
        if (lane == 0) cursor_start(a, cur);
        __syncwarp();
        for (int k = 0; k < kBufs && k < n_items; ++k) issue_item(a, sh, cur, k, lo + k, lane);
    }

    const int g = lane >> 2, cq = lane & 3;
    // the 16-byte x loads in a lane-dependent order (chunk kk_j = (j + rot_r) % 4 at load j):
    // 8 consecutive lanes then read distinct banks
    const int rot_r = ((lane >> 1) ^ (lane >> 3)) & 3;
    // byte selector that puts the bytes of loads 0..3 (gathered as t01.b0, t01.b1, t23.b2, t23.b3)
    // at byte positions kk_0..kk_3 of a plane word
    const uint32_t plane_sel = (0u << (4 * (rot_r & 3))) | (1u << (4 * ((rot_r + 1) & 3))) |
                               (6u << (4 * ((rot_r + 2) & 3))) | (7u << (4 * ((rot_r + 3) & 3)));
    // ldmatrix (q as the B operand): this lane addresses token (lane & 7) + 8 (lane >> 4), bytes 16 ((lane >> 3) & 1)
    const int lm_tok = (lane & 7) + 8 * (lane >> 4), lm_off = 16 * ((lane >> 3) & 1);
    int wb_lin = -1;                       // linear whose W_B fragments are in wbf
    uint32_t wbf[kWbRegKb][4];             // A fragments of this warp's k-blocks (plane-major K order)
#pragma unroll
    for (int j = 0; j < kWbRegKb; ++j) wbf[j][0] = wbf[j][1] = wbf[j][2] = wbf[j][3] = 0u;
    uint4 xv[kGroupsPerThread][4];         // this thread's groups of the item in flight
    int tkg[kGroupsPerThread], cg[kGroupsPerThread];

    // ---- 1 (item k): wait for the tile, W_B fragments on a change of linear, load this thread's
    //      groups G = tid, tid + 512 (token G / gpt, group G % gpt) and gather max |x| per token
    auto stage1 = [&](int k) -> bool {
        const bool got = ptx::mbar_wait(&sh.full[k % kBufs], (uint32_t)(k / kBufs) & 1u);
        const ItemInfo& inf = sh.info[k % kInfos];
        if (!got || !inf.usable) return got;
        const int d_in = inf.d_in, nt = inf.nt, gpt = d_in >> 5;
        if (inf.lin != wb_lin) {
            wb_lin = inf.lin;
            load_wb_fragments(inf.wb, d_in, warp, g, cq, wbf);
        }
        const uint16_t* xt = sh.x[k % kBufs];
        uint32_t* amax_tok = sh.amax_tok[k & 1];
#pragma unroll
        for (int gi = 0; gi < kGroupsPerThread; ++gi) {
            const int G = tid + kConsumers * gi;
            const int tk = div_by_recip(G, inf.rgpt);
            tkg[gi] = tk;
            cg[gi] = G - tk * gpt;
            uint32_t ma = 0u, mb = 0u;         // two chains
            if (tk < nt) {
                const uint8_t* src = reinterpret_cast<const uint8_t*>(xt + tk * d_in + 32 * cg[gi]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    xv[gi][j] = *reinterpret_cast<const uint4*>(src + 16 * ((j + rot_r) & 3));
                    ma = __vmaxu2(ma, xv[gi][j].x & 0x7FFF7FFFu);
                    mb = __vmaxu2(mb, xv[gi][j].y & 0x7FFF7FFFu);
                    ma = __vmaxu2(ma, xv[gi][j].z & 0x7FFF7FFFu);
                    mb = __vmaxu2(mb, xv[gi][j].w & 0x7FFF7FFFu);
                }
            }
            const uint32_t m2 = __vmaxu2(ma, mb);
            uint32_t am = max(m2 & 0xFFFFu, m2 >> 16) << 16;
            if ((gpt & 31) == 0) {             // the warp's 32 groups belong to one token
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
                if (lane == 0 && tk < nt) atomicMax(&amax_tok[tk], am);
            } else if (tk < nt) {
                atomicMax(&amax_tok[tk], am);
            }
        }
        return true;
    };

    // ---- 2 (item k): quantise the groups held in registers
    auto stage2 = [&](int k) {
        const ItemInfo& inf = sh.info[k % kInfos];
        const int d_in = inf.d_in, nt = inf.nt, t0 = inf.t0;
        const int nseg = (d_in + kSegCols - 1) / kSegCols;
        const int qs_row = nseg * kQsSegStride + kQsRowPad;
#pragma unroll
        for (int gi = 0; gi < kGroupsPerThread; ++gi) {
            const int tk = tkg[gi], c = cg[gi];
            if (tk < nt) {
                const uint32_t amb = sh.amax_tok[k & 1][tk];
                const float am = __uint_as_float(amb);
                if (c == 0) {
                    sh.sx[k & 1][tk] = quant_sx(am);
                    if (amb >= 0x7F800000u) atomicOr(a.err, DFSSM_DEVERR_NONFINITE);
                }
                // plane p of this group: 4 bytes at 256 (c / 8) + 32 p + 4 (c % 8) of the token's row
                // (global), at 288 (c / 8) + 32 p + 4 (c % 8) of its shared row
                int8_t* dst = a.q_ws + inf.q_off + (int64_t)(t0 + tk) * inf.qrow + 256 * (c >> 3) + 4 * (c & 7);
                int8_t* qs = sh.q + tk * qs_row + kQsSegStride * (c >> 3) + 4 * (c & 7);
                uint32_t P[8];
                if (amb != 0u && amb < 0x7F800000u) {
                    const float inv = quant_inv(am);
                    // word h of every load: elements 2h, 2h + 1, i.e. planes 2h and 2h + 1 (the low
                    // byte of each y is q)
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        uint32_t ylo[4], yhi[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) quant_pair(word_of(xv[gi][j], h), inv, ylo[j], yhi[j]);
                        P[2 * h] = __byte_perm(__byte_perm(ylo[0], ylo[1], 0x0040u), __byte_perm(ylo[2], ylo[3], 0x4000u),
                                               plane_sel);
                        P[2 * h + 1] = __byte_perm(__byte_perm(yhi[0], yhi[1], 0x0040u),
                                                   __byte_perm(yhi[2], yhi[3], 0x4000u), plane_sel);
                    }
                    if (inf.dbg_q) {           // natural order: element e of load j is column 8 kk_j + e
                        int8_t* dq = inf.dbg_q + (int64_t)(t0 + tk) * d_in + 32 * c;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t y[8];
#pragma unroll
                            for (int h = 0; h < 4; ++h) quant_pair(word_of(xv[gi][j], h), inv, y[2 * h], y[2 * h + 1]);
                            const uint32_t lo4 = __byte_perm(__byte_perm(y[0], y[1], 0x0040u),
                                                             __byte_perm(y[2], y[3], 0x4000u), 0x7610u);
                            const uint32_t hi4 = __byte_perm(__byte_perm(y[4], y[5], 0x0040u),
                                                             __byte_perm(y[6], y[7], 0x4000u), 0x7610u);
                            *reinterpret_cast<uint2*>(dq + 8 * ((j + rot_r) & 3)) = make_uint2(lo4, hi4);
                        }
                    }
                } else {                       // amax 0: q = 0; Inf or NaN: q = 0 and the error bit
#pragma unroll
                    for (int p = 0; p < 8; ++p) P[p] = 0u;
                    if (inf.dbg_q) {
                        int8_t* dq = inf.dbg_q + (int64_t)(t0 + tk) * d_in + 32 * c;
#pragma unroll
                        for (int j = 0; j < 4; ++j) *reinterpret_cast<uint2*>(dq + 8 * j) = make_uint2(0u, 0u);
                    }
                }
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    *reinterpret_cast<uint32_t*>(dst + 32 * p) = P[p];
                    *reinterpret_cast<uint32_t*>(qs + 32 * p) = P[p];
                }
                // a final half segment: its absent half is zero in the shared tile (the MMA and
                // the dp4a sums read whole 32-byte k-blocks)
                if ((c >> 3) == nseg - 1 && (d_in & (kSegCols - 1)) != 0) {
#pragma unroll
                    for (int p = 0; p < 8; ++p) *reinterpret_cast<uint32_t*>(qs + 32 * p + 16) = 0u;
                }
            }
        }
    };

    // ---- 3 (item k): h^T = W_B q^T (M = 16 LoRA rows, N = 8 tokens per n-tile) and sum q by dp4a;
    //      k-block kb = (segment kb / 8, plane kb % 8), 32 bytes of the shared row
    auto stage3 = [&](int k) {
        const ItemInfo& inf = sh.info[k % kInfos];
        const int d_in = inf.d_in, nt = inf.nt;
        const int nseg = (d_in + kSegCols - 1) / kSegCols;
        const int qs_row = nseg * kQsSegStride + kQsRowPad;
        const bool two = inf.T > 8;                // a second n-tile (tokens 8..15)
        const int nkb = nseg * 8;
        int D0[4] = {0, 0, 0, 0}, D1[4] = {0, 0, 0, 0};
        int s0 = 0, s1 = 0;                        // sum q of tokens g and g + 8, this lane's k slices
        const uint32_t b_base = ptx::smem_u32(sh.q) + (uint32_t)(min(lm_tok, nt - 1) * qs_row + lm_off);
        const uint32_t m0 = g < nt ? 0xFFFFFFFFu : 0u, m1 = g + 8 < nt ? 0xFFFFFFFFu : 0u;
        auto kblock = [&](int kb, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
            const uint32_t off = (uint32_t)(kQsSegStride * (kb >> 3) + 32 * (kb & 7));
            uint32_t b0, b1, b2, b3;
            if (two) {
                ptx::ldmatrix_x4(b_base + off, b0, b1, b2, b3);
                b2 &= m1; b3 &= m1;
                mma_s8s8(D1, a0, a1, a2, a3, b2, b3);
                s1 = __dp4a((int)b2, 0x01010101, __dp4a((int)b3, 0x01010101, s1));
            } else {
                ldmatrix_x2(b_base + off, b0, b1);
            }
            b0 &= m0; b1 &= m0;
            mma_s8s8(D0, a0, a1, a2, a3, b0, b1);
            s0 = __dp4a((int)b0, 0x01010101, __dp4a((int)b1, 0x01010101, s0));
        };
#pragma unroll
        for (int j = 0; j < kWbRegKb; ++j) {
            const int kb = warp + kCWarps * j;
            if (kb < nkb) kblock(kb, wbf[j][0], wbf[j][1], wbf[j][2], wbf[j][3]);
        }
        // d_in > 4096: the remaining k-blocks gather W_B from global memory
        for (int kb = warp + kCWarps * kWbRegKb; kb < nkb; kb += kCWarps) {
            uint32_t f[4];
            wb_fragment(inf.wb, d_in, kb, g, cq, f);
            kblock(kb, f[0], f[1], f[2], f[3]);
        }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        // D: (LoRA row g, token 2cq), (g, 2cq + 1), (g + 8, 2cq), (g + 8, 2cq + 1); D1 for tokens + 8
        int (*hw)[kHCols] = sh.h[warp];
        hw[2 * cq][g] = D0[0];
        hw[2 * cq + 1][g] = D0[1];
        hw[2 * cq][g + 8] = D0[2];
        hw[2 * cq + 1][g + 8] = D0[3];
        hw[8 + 2 * cq][g] = D1[0];
        hw[8 + 2 * cq + 1][g] = D1[1];
        hw[8 + 2 * cq][g + 8] = D1[2];
        hw[8 + 2 * cq + 1][g + 8] = D1[3];
        if (cq == 0) {
            hw[g][kRank] = s0;
            hw[g + 8][kRank] = s1;
        }
    };

    // ---- 4 (item k): per-token results, thread (token tid / 17, column tid % 17)
    auto stage4 = [&](int k) {
        const ItemInfo& inf = sh.info[k % kInfos];
        const int nt = inf.nt;
        if (tid < nt * kHCols) {
            const int tk = tid / kHCols, col = tid - tk * kHCols;
            int s = 0;
#pragma unroll
            for (int w = 0; w < kCWarps; ++w) s += sh.h[w][tk][col];
            const int t = inf.t0 + tk;
            TokStats* st = a.st_ws + inf.st_off + t;
            if (col < kRank) {
                st->u[col] = __fmul_rn(inf.sb[col], (float)s);
                if (inf.dbg_h) inf.dbg_h[(int64_t)t * kRank + col] = s;
            } else {
                const float sx = sh.sx[k & 1][tk];
                st->sx = sx;
                st->sumq = s;
                if (inf.dbg_sx) inf.dbg_sx[t] = sx;
            }
        }
    };

    // Two barriers per item. Phase X(k): stage 2 of item k, stage 4 of item k - 1, issue of
    // item k + 2 (its tile was last read in stage 1 of item k). Phase Y(k): stage 3 of item k,
    // stage 1 of item k + 1.
    if (consumer_sync_or(!stage1(0))) {
        if (tid == 0) atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
        return;
    }
    for (int k = 0; k < n_items; ++k) {
        if (sh.info[k % kInfos].usable) stage2(k);
        if (k >= 1 && sh.info[(k - 1) % kInfos].usable) stage4(k - 1);
        if (warp == kIssueWarp && k + kBufs < n_items) issue_item(a, sh, cur, k + kBufs, lo + k + kBufs, lane);
        consumer_sync();
        if (sh.info[k % kInfos].usable) stage3(k);
        if (tid < kMaxT) sh.amax_tok[k & 1][tid] = 0u;   // item k + 2 gathers into it
        const bool got = k + 1 < n_items ? stage1(k + 1) : true;
        if (consumer_sync_or(!got)) {
            if (tid == 0) atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
            return;
        }
    }
    if (sh.info[(n_items - 1) % kInfos].usable) stage4(n_items - 1);
}

}  // namespace

cudaError_t launch_quant_rows(const LaunchCtx& c) {
    int total = 0;
    for (int i = 0; i < c.n; ++i) {
        const int tpi = tokens_per_item(c.host_desc[i].d_in);
        total += (c.m + tpi - 1) / tpi;
    }
    if (total == 0) return cudaSuccess;
    const int grid = min(total, c.sm_count);
    RowsArgs ra{c.entries, c.single, c.desc, c.n, c.m, total, c.q_ws, c.st_ws, c.err, 0, {}, {}};
    if (grid <= kStartTable) {
        // block b's items start at b * total / grid (item_range); its linear and that linear's first item
        int l = 0, begin = 0;
        for (int b = 0; b < grid; ++b) {
            const int lo = (int)((int64_t)b * total / grid);
            for (;;) {
                const int tpi = tokens_per_item(c.host_desc[l].d_in);
                const int count = (c.m + tpi - 1) / tpi;
                if (lo < begin + count || l + 1 == c.n) break;
                begin += count;
                ++l;
            }
            ra.start_lin[b] = l;
            ra.start_item[b] = begin;
        }
        ra.has_start = 1;
    }
    quant_rows_kernel<<<grid, kThreads, sizeof(RowsShared), c.stream>>>(ra);
    return cudaGetLastError();
}

cudaError_t set_quant_rows_attr(int optin) { return allow_dyn_smem(quant_rows_kernel, optin); }

}  // namespace dfssm
