// Prefill path (many tokens): the scaffold contraction as a dense int8 GEMM on
// the 5th-generation tensor cores (tcgen05, accumulators in TMEM), with the
// LoRA up-projection and both dequantisation epilogues fused.
//
// "Density Field State Space Models" (gist.science technical summary), §2.C:
// packed 1-bit scaffold weights are expanded on the fly to int8 and multiplied
// on INT8 tensor cores. With many tokens the contraction is a dense GEMM
// (2 * d_in ops per token per output row), so here the expansion happens in
// shared memory, once per 128-row x 128-column weight block, and the block is
// reused by 256 tokens:
//
//   D[o, t] = sum_k b[o, k] * q[t, k]    (b = sign bit as 0/1, int32 in TMEM)
//   acc     = 2 * D - sum_k q[t, k]       (a +-1 weight is 2b - 1)
//
// Persistent kernel, one CTA per SM, 16 warps with fixed roles:
//   warp 0      TMA producer: 256-token x 128-byte tiles of the int8
//               activations (permuted column order, 128B swizzle), no multicast
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma.kind::i8, M=128 rows,
//               N=256 tokens, K=32 per instruction, 4 per 128-column block
//   warps 4-7   bit expansion: each thread owns one weight row of the tile,
//               loads the 32 sign bytes of a 256-column segment and writes, per
//               128-byte k-block (four bit planes of that segment, the activation
//               order of dfssm_internal.cuh), 128 0/1 bytes into the K-major
//               SWIZZLE_128B layout the MMA reads
//   warps 8-15  epilogue: tcgen05.ld of its 32 TMEM lanes (= output rows) and
//               half of the 256 token columns, acc = 2D - sum q, LoRA
//               up-projection and dequantisation, coalesced stores of y along
//               the output dimension; the per-token scalars of each 16-token
//               chunk are staged in a warp-private, double-buffered smem slice
// 4-stage shared-memory ring (mbarriers), two TMEM accumulator buffers of 256
// columns so the epilogue of one tile overlaps the main loop of the next.
// Every mbarrier wait is bounded; a timeout sets the plan's error word.
#include <cuda.h>

#include "dfssm_internal.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace dfssm {

namespace {

constexpr int BM = 128;            // output rows per tile (MMA M, TMEM lanes)
constexpr int BN = 256;            // tokens per tile (MMA N, TMEM columns)
constexpr int BK = 128;            // k (bytes) per stage
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;   // 16 KB
constexpr int B_STAGE = BN * BK;   // 32 KB
constexpr int NUM_THREADS = 16 * 32;
constexpr int EPI_WARPS = 8;                         // warps 8..15
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int STAT_CHUNK = 16 * (int)sizeof(TokStats);  // per-token scalars of 16 tokens (1280 B)
constexpr int STAT_BYTES = EPI_WARPS * 2 * STAT_CHUNK;  // double-buffered, one pair per epilogue warp
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE) + STAT_BYTES + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;

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

__device__ __forceinline__ TileCoord tile_coord(const DevDesc* desc, int n, int n_tt, int tile) {
    const int rt = tile / n_tt;                 // global 128-row tile index
    const int tt = tile - rt * n_tt;
    const int base = desc[0].rt_begin;
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (desc[mid].rt_begin - base <= rt) lo = mid; else hi = mid - 1;
    }
    TileCoord c;
    c.lin = lo;
    c.row0 = (rt - (desc[lo].rt_begin - base)) * BM;
    c.tok0 = tt * BN;
    return c;
}

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

__global__ void __launch_bounds__(NUM_THREADS, 1) prefill_kernel(const __grid_constant__ PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (SWIZZLE_128B atoms), offset from the __shared__ array so the
    // compiler keeps shared-memory addressing
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;
    uint8_t* sStat = sB + STAGES * B_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sStat + STAT_BYTES);
    uint64_t* full_a = bars;               // [STAGES], 128 arrivals (expansion threads)
    uint64_t* full_b = bars + STAGES;      // [STAGES], TMA transaction bytes
    uint64_t* empty = bars + 2 * STAGES;   // [STAGES], MMA commit
    uint64_t* acc_full = bars + 3 * STAGES;       // [2], MMA commit
    uint64_t* acc_empty = bars + 3 * STAGES + 2;  // [2], EPI_THREADS epilogue arrivals
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 4);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tt = (a.m + BN - 1) / BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&full_a[s], 128);
            ptx::mbar_init(&full_b[s], 1);
            ptx::mbar_init(&empty[s], 1);
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
                const TileCoord tc = tile_coord(a.desc, a.n, n_tt, tile);
                const CUtensorMap* tm = a.tmaps + tc.lin;
                const int nkb = a.desc[tc.lin].qrow / BK;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!ptx::mbar_wait(&empty[s], ph ^ 1u)) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; break; }
                    ptx::mbar_arrive_expect_tx(&full_b[s], B_STAGE);
                    ptx::tma_load_2d(sB + s * B_STAGE, tm, kb * BK, tc.tok0, &full_b[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x, ++tcount) {
                const TileCoord tc = tile_coord(a.desc, a.n, n_tt, tile);
                const int nkb = a.desc[tc.lin].qrow / BK;
                const int buf = tcount & 1;
                const uint32_t acc_ph = (uint32_t)(tcount >> 1) & 1u;
                if (!ptx::mbar_wait(&acc_empty[buf], acc_ph ^ 1u)) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!ptx::mbar_wait(&full_a[s], ph) || !ptx::mbar_wait(&full_b[s], ph)) {
                        set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; ok = false; break;
                    }
                    ptx::tc_fence_after();
                    const uint64_t adesc = sw128_desc(ptx::smem_u32(sA + s * A_STAGE));
                    const uint64_t bdesc = sw128_desc(ptx::smem_u32(sB + s * B_STAGE));
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)   // +32 bytes along K = +2 in the 16-byte address field
                        ptx::mma_i8(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, (kb | kk) != 0);
                    ptx::mma_commit(&empty[s]);
                }
                if (!ok) break;
                ptx::mma_commit(&acc_full[buf]);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ bit expansion (one weight row per thread)
        const int r = threadIdx.x - 128;
        int it = 0;
        for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x) {
            const TileCoord tc = tile_coord(a.desc, a.n, n_tt, tile);
            const DevDesc d = a.desc[tc.lin];
            const dfssm_stack_entry& e = entry_at(a.entries, a.single, tc.lin);
            const int nseg = d.qrow / kSegCols;
            const int rb = d.d_in >> 3;                 // sign bytes per row
            const int o = tc.row0 + r;
            const bool valid = o < d.d_out && entry_ptrs_ok(e);
            const uint8_t* src = e.w.sign + (int64_t)(valid ? o : 0) * rb;
            // segment sg of this row: words 0..3 and 4..7 (the second half is absent in a final half segment)
            auto load_seg = [&](int sg, uint4& lo, uint4& hi) {
                lo = make_uint4(0, 0, 0, 0);
                hi = make_uint4(0, 0, 0, 0);
                if (valid && sg < nseg) {
                    lo = __ldg(reinterpret_cast<const uint4*>(src + 32 * sg));
                    if (32 * sg + 16 < rb) hi = __ldg(reinterpret_cast<const uint4*>(src + 32 * sg + 16));
                }
            };
            // two segments of look-ahead
            uint4 c_lo, c_hi, n_lo, n_hi;
            load_seg(0, c_lo, c_hi);
            load_seg(1, n_lo, n_hi);
            // swizzled destination of this row: atom (r/8), row-in-atom (r%8)
            const uint32_t rrow = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
            const uint32_t xr = (uint32_t)(r & 7);
            bool ok = true;
            for (int sg = 0; sg < nseg && ok; ++sg) {
                const uint32_t w[8] = {c_lo.x, c_lo.y, c_lo.z, c_lo.w, c_hi.x, c_hi.y, c_hi.z, c_hi.w};
                c_lo = n_lo;
                c_hi = n_hi;
                load_seg(sg + 2, n_lo, n_hi);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    ++it;
                    // one lane polls, the warp follows
                    bool got = true;
                    if ((threadIdx.x & 31) == 0) got = ptx::mbar_wait(&empty[s], ph ^ 1u);
                    got = __shfl_sync(0xffffffffu, got, 0);
                    __syncwarp();
                    if (!got) { if ((threadIdx.x & 31) == 0) { set_err(a.err, DFSSM_DEVERR_TIMEOUT); *abort_flag = 1; } ok = false; break; }
                    uint8_t* dst = sA + s * A_STAGE + rrow;
                    // k-block 2 sg + h: bytes 32 p' + 4 c + i of plane p = 4 h + p' (0/1 bytes);
                    // 16-byte chunk 2 p' holds words c = 0..3, chunk 2 p' + 1 words 4..7
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp) {
                        const int p = 4 * h + pp;
                        const uint4 e0 = make_uint4((w[0] >> p) & 0x01010101u, (w[1] >> p) & 0x01010101u,
                                                    (w[2] >> p) & 0x01010101u, (w[3] >> p) & 0x01010101u);
                        const uint4 e1 = make_uint4((w[4] >> p) & 0x01010101u, (w[5] >> p) & 0x01010101u,
                                                    (w[6] >> p) & 0x01010101u, (w[7] >> p) & 0x01010101u);
                        *reinterpret_cast<uint4*>(dst + (((uint32_t)(2 * pp) ^ xr) << 4)) = e0;
                        *reinterpret_cast<uint4*>(dst + (((uint32_t)(2 * pp + 1) ^ xr) << 4)) = e1;
                    }
                    ptx::fence_proxy_async_smem();
                    ptx::mbar_arrive(&full_a[s]);
                }
            }
            if (!ok) break;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------ epilogue
        // warp 8 + 4h + q handles TMEM lanes 32q.. (output rows) and token columns [128h, 128h + 128)
        ptx::pdl_wait();
        const int q4 = warp & 3;
        const int half = (warp - 8) >> 2;
        const int r = q4 * 32 + lane;
        uint8_t* stat_buf = sStat + (warp - 8) * 2 * STAT_CHUNK;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < a.n_tiles && !*abort_flag; tile += gridDim.x, ++tcount) {
            const TileCoord tc = tile_coord(a.desc, a.n, n_tt, tile);
            const DevDesc d = a.desc[tc.lin];
            const dfssm_stack_entry& e = entry_at(a.entries, a.single, tc.lin);
            const int o = tc.row0 + r;
            const bool valid = o < d.d_out && entry_ptrs_ok(e);
            // entry fields in registers: the stores below must not force reloads
            void* const y_ptr = e.y;
            int32_t* const dbg_acc = e.dbg.acc;
            const bool y_bf16 = d.y_dtype == DFSSM_BF16;
            const int d_out = d.d_out;
            float alpha = 0.f, sa = 0.f;
            WaRow wa = wa_row_from_int4(make_int4(0, 0, 0, 0));
            if (valid) {
                alpha = e.w.alpha[o];
                sa = e.w.sa[o];
                wa = wa_row_from_int4(*reinterpret_cast<const int4*>(e.w.wa + (int64_t)o * kRank));
            }
            // per-token scalars: chunk ch covers tokens tok_base + 16 ch .. + 15 (80 x 16 bytes)
            const int tok_base = tc.tok0 + half * (BN / 2);
            const uint4* st_src = reinterpret_cast<const uint4*>(a.st_ws + d.st_off);
            auto load_chunk = [&](int ch, uint4 (&rg)[3]) {
#pragma unroll
                for (int u = 0; u < 3; ++u) {
                    const int idx = lane + 32 * u;                  // uint4 index inside the chunk
                    const int tok = tok_base + 16 * ch + idx / 5;
                    rg[u] = (idx < 80 && tok < a.m) ? st_src[(int64_t)(tok_base + 16 * ch) * 5 + idx]
                                                    : make_uint4(0u, 0u, 0u, 0u);
                }
            };
            auto store_chunk = [&](int buf_i, const uint4 (&rg)[3]) {
                uint4* dst = reinterpret_cast<uint4*>(stat_buf + buf_i * STAT_CHUNK);
#pragma unroll
                for (int u = 0; u < 3; ++u)
                    if (lane + 32 * u < 80) dst[lane + 32 * u] = rg[u];
            };
            uint4 rg[3];
            load_chunk(0, rg);
            store_chunk(0, rg);

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
            const uint32_t taddr = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(buf * BN + half * (BN / 2));
            constexpr int NCH = BN / 2 / 16;
            for (int ch = 0; ch < NCH; ++ch) {
                __syncwarp();
                const bool more = ch + 1 < NCH && tok_base + 16 * (ch + 1) < a.m;
                if (more) load_chunk(ch + 1, rg);
                uint32_t v[16];
                ptx::tmem_ld_32x32b_x16(taddr + (uint32_t)(16 * ch), v);
                ptx::tmem_ld_wait();
                const TokStats* stc = reinterpret_cast<const TokStats*>(stat_buf + (ch & 1) * STAT_CHUNK);
                const int t0c = tok_base + 16 * ch;
                if (t0c < a.m && valid) {
                    const int nj = min(16, a.m - t0c);
                    // element (t0c + j, o) of y / acc: base + j * d_out (32-bit offsets inside a chunk)
                    const int64_t base_idx = (int64_t)t0c * d_out + o;
                    if (y_bf16) {
                        uint16_t* yb = reinterpret_cast<uint16_t*>(y_ptr) + base_idx;
                        int32_t* ab = dbg_acc ? dbg_acc + base_idx : nullptr;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (j >= nj) break;
                            const TokStats& st = stc[j];
                            const int acc = 2 * (int)v[j] - st.sumq;
                            yb[j * d_out] = f32_to_bf16_bits(dequant(st.sx, alpha, sa, acc, lora_dot(wa, st.u)));
                            if (ab) ab[j * d_out] = acc;
                        }
                    } else {
                        float* yf = reinterpret_cast<float*>(y_ptr) + base_idx;
                        int32_t* ab = dbg_acc ? dbg_acc + base_idx : nullptr;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (j >= nj) break;
                            const TokStats& st = stc[j];
                            const int acc = 2 * (int)v[j] - st.sumq;
                            yf[j * d_out] = dequant(st.sx, alpha, sa, acc, lora_dot(wa, st.u));
                            if (ab) ab[j * d_out] = acc;
                        }
                    }
                }
                __syncwarp();
                if (more) store_chunk((ch + 1) & 1, rg);
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
