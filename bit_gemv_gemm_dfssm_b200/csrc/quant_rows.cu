// Activation quantisation for many tokens (m > 16): the input stage of the
// tensor-core prefill.
//
// Same quantiser and LoRA down-projection as quant.cu ("Density Field State
// Space Models", gist.science technical summary, §2.B: int8 LoRA W_B with
// per-row scales; §2.C: int8 activations for the int8 x int8 -> int32
// scaffold matmul), arranged for throughput over a large activation matrix.
//
// Persistent kernel, one block per SM: 16 consumer warps and one producer warp.
// Work items are T tokens of one linear, T = min(16, 16384 / d_in), so an
// item is at most 32 KB of bf16; the items of a linear are numbered in token
// order and the linears follow each other.
//   producer   per item: looks up the linear, writes the item's descriptor
//              (shape, offsets, pointers, s_B) to a shared ring, and fetches
//              the item's rows (one contiguous range of x) with a single bulk
//              copy (TMA engine, no tensor map, no multicast) into one of three
//              shared x tiles. x is read from HBM once; two items stream in
//              while one is processed.
//   consumers  per item, with three barriers among the 16 warps:
//     1. amax per token from the shared tile: a 16-bit SIMD max over the |x|
//        bit patterns (the unsigned order of |bf16| bits is the numeric
//        order, NaN above Inf, so a non-finite row is still seen);
//     2. each thread quantises one 32-column group of one token.
//        rint(x * inv) is taken by adding 1.5 * 2^23 in round-to-nearest-even,
//        exact here because |x * inv| <= 127 * (1 + 2^-23); the low byte of
//        the sum is q. The group is written twice: in natural order to a
//        shared q tile, and in the plane-major order of the prefill's
//        activation rows straight to global memory (eight 4-byte plane words;
//        eight lanes fill one 32-byte sector);
//     3. h = q W_B^T and sum q on the warp MMA (m16n8k32, s8 x s8 -> s32)
//        from the shared q tile, a third n-tile of ones giving sum q; warp w
//        takes k-blocks w, w + 16, ... and keeps their W_B fragments in
//        registers for as long as the linear stays the same;
//     4. the 16 partials are added in shared memory; u = s_B h, s_x, sum q.
#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int kConsumers = 512;
constexpr int kCWarps = kConsumers / 32;     // 16
constexpr int kThreads = kConsumers + 32;    // + the producer warp
constexpr int kItemElems = 16384;            // bf16 values of one item at most (32 KB)
constexpr int kMaxT = 16;                    // tokens per item at most (the MMA's M)
constexpr int kBufs = 3;                     // x tiles
constexpr int kInfos = kBufs + 1;            // item descriptors (a descriptor outlives its tile)
constexpr int kQsPad = 16;                   // bytes of padding per shared q row (ldmatrix rows on distinct banks)
constexpr int kHCols = kRank + 1;            // h[0..15] and sum q
constexpr int kQsBytes = kItemElems + kMaxT * kQsPad;
constexpr int kWbRegKb = 8;                  // k-blocks per warp whose W_B fragments stay in registers (d_in <= 4096)
constexpr uint32_t kBarConsumers = 1;        // named barrier of the 16 consumer warps

struct ItemInfo {
    int lin, t0, nt, d_in;
    int qrow, usable, pad0, pad1;
    int64_t q_off, st_off;
    const int8_t* wb;
    int8_t* dbg_q;
    int32_t* dbg_h;
    float* dbg_sx;
    float sb[kRank];
};

struct RowsShared {
    uint16_t x[kBufs][kItemElems];           // bf16 tiles, bulk-copy destinations
    int8_t q[kQsBytes];                      // natural-order q of the item, rows of d_in + 16 bytes
    int h[kCWarps][kMaxT][kHCols];           // per-warp partial h and sum q
    ItemInfo info[kInfos];
    uint32_t amax[kCWarps];                  // per-warp partial max |x| (fp32 bit pattern)
    float sx[kMaxT];
    uint64_t full[kBufs];                    // producer -> consumers: tile and descriptor ready
    uint64_t empty[kBufs];                   // consumers -> producer: tile read
};

__host__ __device__ inline int tokens_per_item(int d_in) {
    const int t = kItemElems / d_in;
    return t < kMaxT ? t : kMaxT;
}

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

// two fp32 products in one instruction, each rounded like the scalar __fmul_rn
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// four bf16 (two words) -> four int8 (one word, little-endian), q = rint(x * inv). The
// rounding add is the scalar __fadd_rn, which is never merged with the product into an FMA
// (a fused x * inv + 1.5 * 2^23 would skip the product's own rounding and can move a tie).
__device__ __forceinline__ uint32_t quant_pack4(uint32_t wa, uint32_t wb, float inv) {
    constexpr float kRound = 12582912.0f;   // 1.5 * 2^23: ulp 1, low byte q
    const float2 iv = make_float2(inv, inv);
    const float2 pa = fmul2(make_float2(bf16_lo(wa), bf16_hi(wa)), iv);
    const float2 pb = fmul2(make_float2(bf16_lo(wb), bf16_hi(wb)), iv);
    const uint32_t y0 = __float_as_uint(__fadd_rn(pa.x, kRound)), y1 = __float_as_uint(__fadd_rn(pa.y, kRound));
    const uint32_t y2 = __float_as_uint(__fadd_rn(pb.x, kRound)), y3 = __float_as_uint(__fadd_rn(pb.y, kRound));
    return __byte_perm(__byte_perm(y0, y1, 0x0040u), __byte_perm(y2, y3, 0x4000u), 0x7610u);
}

// word r of the result = byte r of a, b, c, d (4x4 byte transpose)
__device__ __forceinline__ uint4 transpose4x4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    const uint32_t t0 = __byte_perm(a, b, 0x5140), t1 = __byte_perm(a, b, 0x7362);
    const uint32_t t2 = __byte_perm(c, d, 0x5140), t3 = __byte_perm(c, d, 0x7362);
    return make_uint4(__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632), __byte_perm(t1, t3, 0x5410),
                      __byte_perm(t1, t3, 0x7632));
}

__device__ __forceinline__ void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ producer warp
__device__ void produce(const RowsArgs& a, RowsShared& sh) {
    const int lane = threadIdx.x & 31;
    int lin = 0, begin = 0, tpi = tokens_per_item(a.descs[0].d_in);
    int count = (a.m + tpi - 1) / tpi;
    for (int kk = 0;; ++kk) {
        const int item = blockIdx.x + kk * gridDim.x;
        if (item >= a.total) break;
        while (item >= begin + count && lin + 1 < a.n) {   // items arrive in increasing order
            begin += count;
            ++lin;
            tpi = tokens_per_item(a.descs[lin].d_in);
            count = (a.m + tpi - 1) / tpi;
        }
        const int slot = kk % kBufs;
        bool ok = true;
        if (lane == 0) ok = ptx::mbar_wait(&sh.empty[slot], ((uint32_t)(kk / kBufs) & 1u) ^ 1u);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
            if (lane == 0) atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
            return;
        }
        const dfssm_stack_entry& e = entry_at(a.entries, a.single, lin);
        const DevDesc d = a.descs[lin];
        const bool desc_ok = a.entries == nullptr || e.desc_index == lin;
        const bool usable = desc_ok && entry_ptrs_ok(e);
        const int t0 = (item - begin) * tpi;
        const int nt = min(tpi, a.m - t0);
        ItemInfo& inf = sh.info[kk % kInfos];
        if (lane < kRank) inf.sb[lane] = usable ? e.w.sb[lane] : 0.0f;
        if (lane == 0) {
            inf.lin = lin;
            inf.t0 = t0;
            inf.nt = nt;
            inf.d_in = d.d_in;
            inf.qrow = d.qrow;
            inf.usable = usable;
            inf.q_off = d.q_off;
            inf.st_off = d.st_off;
            inf.wb = reinterpret_cast<const int8_t*>(e.w.wb);
            inf.dbg_q = e.dbg.q;
            inf.dbg_h = e.dbg.h;
            inf.dbg_sx = e.dbg.sx;
        }
        __syncwarp();
        if (lane == 0) {
            uint64_t* bar = &sh.full[slot];
            if (usable) {
                const uint32_t bytes = (uint32_t)nt * (uint32_t)d.d_in * 2u;
                ptx::mbar_arrive_expect_tx(bar, bytes);   // release: the descriptor above is visible
                ptx::bulk_g2s(sh.x[slot], reinterpret_cast<const uint16_t*>(e.x) + (int64_t)t0 * d.d_in, bytes,
                              bar);
            } else {
                atomicOr(a.err, desc_ok ? DFSSM_DEVERR_ENTRY_PTR : DFSSM_DEVERR_ENTRY_DESC);
                ptx::mbar_arrive(bar);                    // nothing to copy: complete the phase
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) quant_rows_kernel(const __grid_constant__ RowsArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    RowsShared& sh = *reinterpret_cast<RowsShared*>(smem_raw);
    // let the dependent prefill kernel start streaming weights; it waits for this grid before reading q
    ptx::pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int b = 0; b < kBufs; ++b) {
            ptx::mbar_init(&sh.full[b], 1);
            ptx::mbar_init(&sh.empty[b], 1);
        }
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (warp == kCWarps) {
        produce(a, sh);
        return;
    }

    // ------------------------------------------------------------------ consumers
    const int g = lane >> 2, cq = lane & 3;
    int wb_lin = -1;                       // linear whose W_B fragments are in wbf
    uint32_t wbf[kWbRegKb][4];
#pragma unroll
    for (int j = 0; j < kWbRegKb; ++j) wbf[j][0] = wbf[j][1] = wbf[j][2] = wbf[j][3] = 0u;
    for (int kk = 0;; ++kk) {
        const int item = blockIdx.x + kk * gridDim.x;
        if (item >= a.total) break;
        const int slot = kk % kBufs;
        const bool got = ptx::mbar_wait(&sh.full[slot], (uint32_t)(kk / kBufs) & 1u);
        const ItemInfo& inf = sh.info[kk % kInfos];
        const int usable = got ? inf.usable : 0;
        const int d_in = inf.d_in, nt = inf.nt, t0 = inf.t0;
        const int T = tokens_per_item(d_in);
        const int nkb = d_in >> 5;
        const uint16_t* xt = sh.x[slot];

        // W_B fragments of this warp's k-blocks (b00, b01: rank g; b10, b11: rank g + 8), on a change of linear
        if (usable && inf.lin != wb_lin) {
            wb_lin = inf.lin;
            const uint8_t* w0 = reinterpret_cast<const uint8_t*>(inf.wb) + (int64_t)g * d_in + 4 * cq;
            const uint8_t* w1 = w0 + (int64_t)8 * d_in;
#pragma unroll
            for (int j = 0; j < kWbRegKb; ++j) {
                const int col = 32 * (warp + kCWarps * j);
                if (col < d_in) {
                    wbf[j][0] = __ldg(reinterpret_cast<const uint32_t*>(w0 + col));
                    wbf[j][1] = __ldg(reinterpret_cast<const uint32_t*>(w0 + col + 16));
                    wbf[j][2] = __ldg(reinterpret_cast<const uint32_t*>(w1 + col));
                    wbf[j][3] = __ldg(reinterpret_cast<const uint32_t*>(w1 + col + 16));
                }
            }
        }

        // ---- 1: partial amax, warp w takes part w % parts of token w / parts
        const int parts = kCWarps / T;
        if (usable) {
            const int tk = warp / parts, part = warp - tk * parts;
            uint32_t m2 = 0u;
            if (tk < nt) {
                const uint4* row = reinterpret_cast<const uint4*>(xt + tk * d_in);
#pragma unroll 4
                for (int i = part * 32 + lane; i < (d_in >> 3); i += parts * 32) {
                    const uint4 v = row[i];
                    m2 = __vmaxu2(m2, v.x & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, v.y & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, v.w & 0x7FFF7FFFu);
                }
            }
            uint32_t am = max(m2 & 0xFFFFu, m2 >> 16) << 16;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (lane == 0) sh.amax[warp] = am;
        }
        if (consumer_sync_or(!got)) {
            if (tid == 0) atomicOr(a.err, DFSSM_DEVERR_TIMEOUT);
            break;
        }
        if (!usable) {                     // the producer recorded the error; just free the tile
            if (tid == 0) ptx::mbar_arrive(&sh.empty[slot]);
            continue;
        }

        // ---- 2: quantise one 32-column group per thread
        const int qs_row = d_in + kQsPad;
        {
            const int gpt = d_in >> 5;                 // groups per token
            const int tk = tid / gpt, c = tid - tk * gpt;
            if (tk < nt) {
                uint32_t amb = 0u;
                for (int p = 0; p < parts; ++p) amb = max(amb, sh.amax[tk * parts + p]);
                const float am = __uint_as_float(amb);
                const float inv = quant_inv(am);
                // amax 0: q = 0; Inf or NaN: q = 0 and the error bit (output undefined)
                const uint32_t keep = (amb != 0u && amb < 0x7F800000u) ? 0xFFFFFFFFu : 0u;
                if (c == 0) {
                    sh.sx[tk] = quant_sx(am);
                    if (amb >= 0x7F800000u) atomicOr(a.err, DFSSM_DEVERR_NONFINITE);
                }
                // the four 16-byte loads in a lane-dependent order: 8 (and 16) consecutive lanes
                // then touch distinct banks in the loads below and in the 8-byte q stores
                const int r = ((lane >> 1) ^ (lane >> 3)) & 3;
                const uint8_t* src = reinterpret_cast<const uint8_t*>(xt + tk * d_in + 32 * c);
                int8_t* qs = sh.q + tk * qs_row + 32 * c;
                int8_t* dq = inf.dbg_q ? inf.dbg_q + (int64_t)(t0 + tk) * d_in + 32 * c : nullptr;
                uint32_t w0[4], w1[4];       // load j: columns 8 kk .. 8 kk + 3 and 8 kk + 4 .. 8 kk + 7
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int kk8 = 8 * ((j + r) & 3);
                    const uint4 v = *reinterpret_cast<const uint4*>(src + 2 * kk8);
                    w0[j] = quant_pack4(v.x, v.y, inv) & keep;
                    w1[j] = quant_pack4(v.z, v.w, inv) & keep;
                    *reinterpret_cast<uint2*>(qs + kk8) = make_uint2(w0[j], w1[j]);
                    if (dq) *reinterpret_cast<uint2*>(dq + kk8) = make_uint2(w0[j], w1[j]);
                }
                // plane p of the group: columns 8 i + p (i = 0..3) as bytes i. The transposes give
                // byte j = load j; rotating left by r bytes puts it at i = (j + r) % 4.
                const uint4 lo = transpose4x4(w0[0], w0[1], w0[2], w0[3]);   // planes 0..3
                const uint4 hi = transpose4x4(w1[0], w1[1], w1[2], w1[3]);   // planes 4..7
                const uint32_t rot = 8u * (uint32_t)r;
                const uint32_t P[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                // plane p of segment c / 8: 4 bytes at 256 (c / 8) + 32 p + 4 (c % 8) of the token's row
                int8_t* dst = a.q_ws + inf.q_off + (int64_t)(t0 + tk) * inf.qrow + 256 * (c >> 3) + 4 * (c & 7);
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    *reinterpret_cast<uint32_t*>(dst + 32 * p) = __funnelshift_l(P[p], P[p], rot);
            }
        }
        consumer_sync();
        if (tid == 0) ptx::mbar_arrive(&sh.empty[slot]);   // the tile has been read

        // ---- 3: h = q W_B^T (two n-tiles) and sum q (n-tile of ones)
        {
            int D0[4] = {0, 0, 0, 0}, D1[4] = {0, 0, 0, 0}, D2[4] = {0, 0, 0, 0};
            const int mi = lane >> 3;                  // ldmatrix: this lane addresses row (lane & 7) of matrix mi
            const int row = min((lane & 7) + 8 * (mi & 1), nt - 1);
            const uint32_t a_base = ptx::smem_u32(sh.q) + (uint32_t)(row * qs_row + 16 * (mi >> 1));
            const uint32_t mA = g < nt ? 0xFFFFFFFFu : 0u, mB = g + 8 < nt ? 0xFFFFFFFFu : 0u;
#pragma unroll
            for (int j = 0; j < kWbRegKb; ++j) {
                const int kb = warp + kCWarps * j;
                if (kb < nkb) {
                    uint32_t a0, a1, a2, a3;
                    ptx::ldmatrix_x4(a_base + 32u * (uint32_t)kb, a0, a1, a2, a3);
                    a0 &= mA; a2 &= mA; a1 &= mB; a3 &= mB;
                    mma_s8s8(D0, a0, a1, a2, a3, wbf[j][0], wbf[j][1]);
                    mma_s8s8(D1, a0, a1, a2, a3, wbf[j][2], wbf[j][3]);
                    mma_s8s8(D2, a0, a1, a2, a3, 0x01010101u, 0x01010101u);
                }
            }
            // d_in > 4096: the remaining k-blocks read W_B from global memory
            const uint8_t* w0 = reinterpret_cast<const uint8_t*>(inf.wb) + (int64_t)g * d_in + 4 * cq;
            const uint8_t* w1 = w0 + (int64_t)8 * d_in;
            for (int kb = warp + kCWarps * kWbRegKb; kb < nkb; kb += kCWarps) {
                uint32_t a0, a1, a2, a3;
                ptx::ldmatrix_x4(a_base + 32u * (uint32_t)kb, a0, a1, a2, a3);
                a0 &= mA; a2 &= mA; a1 &= mB; a3 &= mB;
                const int col = 32 * kb;
                mma_s8s8(D0, a0, a1, a2, a3, __ldg(reinterpret_cast<const uint32_t*>(w0 + col)),
                         __ldg(reinterpret_cast<const uint32_t*>(w0 + col + 16)));
                mma_s8s8(D1, a0, a1, a2, a3, __ldg(reinterpret_cast<const uint32_t*>(w1 + col)),
                         __ldg(reinterpret_cast<const uint32_t*>(w1 + col + 16)));
                mma_s8s8(D2, a0, a1, a2, a3, 0x01010101u, 0x01010101u);
            }
            // D: (token g, n 2cq), (g, 2cq + 1), (g + 8, 2cq), (g + 8, 2cq + 1)
            int (*hw)[kHCols] = sh.h[warp];
            hw[g][2 * cq] = D0[0];
            hw[g][2 * cq + 1] = D0[1];
            hw[g + 8][2 * cq] = D0[2];
            hw[g + 8][2 * cq + 1] = D0[3];
            hw[g][8 + 2 * cq] = D1[0];
            hw[g][8 + 2 * cq + 1] = D1[1];
            hw[g + 8][8 + 2 * cq] = D1[2];
            hw[g + 8][8 + 2 * cq + 1] = D1[3];
            if (cq == 0) {
                hw[g][kRank] = D2[0];
                hw[g + 8][kRank] = D2[2];
            }
        }
        consumer_sync();

        // ---- 4: per-token results: thread (token tid / 17, column tid % 17)
        if (tid < nt * kHCols) {
            const int tk = tid / kHCols, col = tid - tk * kHCols;
            int s = 0;
#pragma unroll
            for (int w = 0; w < kCWarps; ++w) s += sh.h[w][tk][col];
            const int t = t0 + tk;
            TokStats* st = a.st_ws + inf.st_off + t;
            if (col < kRank) {
                st->u[col] = __fmul_rn(inf.sb[col], (float)s);
                if (inf.dbg_h) inf.dbg_h[(int64_t)t * kRank + col] = s;
            } else {
                st->sx = sh.sx[tk];
                st->sumq = s;
                if (inf.dbg_sx) inf.dbg_sx[t] = sh.sx[tk];
            }
        }
    }
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
    RowsArgs ra{c.entries, c.single, c.desc, c.n, c.m, total, c.q_ws, c.st_ws, c.err};
    quant_rows_kernel<<<grid, kThreads, sizeof(RowsShared), c.stream>>>(ra);
    return cudaGetLastError();
}

cudaError_t set_quant_rows_attr(int optin) { return allow_dyn_smem(quant_rows_kernel, optin); }

}  // namespace dfssm
