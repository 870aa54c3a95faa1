// Internal definitions shared by the libdfssm kernels (not part of the ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/dfssm.h"

namespace dfssm {

constexpr int kRank = 16;
constexpr int kMaxDIn = 8192;
constexpr int kMaxM = 65536;
constexpr int kMaxSplits = 8;        // d_in splits of the quantisation kernel for m <= 16
constexpr int kPartTok = 16;         // tokens covered by the split partials
constexpr int kPartInts = 20;        // ints per token in the split partials (16 partial h, padded)

// partial h of (linear lin, split sp of `splits`, token t, LoRA row k), written by the
// quantisation kernel for m <= 16 and added up by the decode kernel
__host__ __device__ inline int64_t part_index(int lin, int splits, int sp, int t, int k) {
    return (((int64_t)lin * splits + sp) * kPartTok + t) * kPartInts + k;
}

// Per-linear shape and workspace offsets, resident in device memory.
struct DevDesc {
    int32_t d_in;
    int32_t d_out;
    int32_t y_dtype;
    int32_t max_m;
    int64_t q_off;      // byte offset of this linear's activation rows (prefill) in the q workspace
    int64_t st_off;     // index of its first TokStats record
    int32_t qrow;       // activation bytes per token: d_in rounded up to a whole 256-column segment
    int32_t rt_begin;   // first 128-row tile of this linear in the flattened stack order
    int64_t work_begin[2]; // decode work units of all preceding linears, for 128- and 192-row blocks
};

// Per-token values the main kernels need after quantisation.
//   sx   : s_x = amax / 127 (fp32)
//   sumq : sum_j q[t,j] (int32). The scaffold kernels count sum_{bit=1} q and
//          form acc = 2 * that - sumq (exact integer identity for +-1 weights).
//   u[k] : s_B[k] * h[t,k] in fp32 (the LoRA bottleneck, not re-quantised)
struct alignas(16) TokStats {
    float sx;
    int32_t sumq;
    int32_t pad0, pad1;
    float u[kRank];
};
static_assert(sizeof(TokStats) == 80, "TokStats layout");
static_assert(sizeof(dfssm_stack_entry) == 104, "dfssm_stack_entry layout");

// Activation layout in the q workspace (the prefill's B operand). The columns of
// a row are taken in segments of 256 (a final half segment is padded to 256);
// inside a segment the int8 value of column 32c + 8i + p (c = 0..7: 32-bit word
// of the sign row, i = 0..3: byte of that word, p = 0..7: bit of that byte) sits
// at K position 32p + 4c + i. With this plane-major order the four bytes of
// bit plane p of sign word c meet four consecutive activation bytes, and the 32
// bytes of plane p form one K = 32 step of an int8 MMA. Token t, segment s is at
// q_off + t * qrow + 256 s (K-major rows, loaded by TMA with 128-byte swizzle).
// Decode work balance. The decode kernel splits the rows of all linears of a call over its CTAs
// in work units: kUnitChunk per k-chunk of a row block (kDecodeChunkCols columns of R rows, a
// partial last block counting in full), kUnitBlock for the block's epilogue, and
// kDecodeLinStart for entering a linear (the CTA quantises that linear's x first). A CTA's
// cost is close to linear in these units.
#ifndef DFSSM_UNIT_CHUNK
#define DFSSM_UNIT_CHUNK 5
#endif
#ifndef DFSSM_UNIT_BLOCK
#define DFSSM_UNIT_BLOCK 1
#endif
constexpr int kDecodeChunkCols = 1024;
constexpr int kUnitChunk = DFSSM_UNIT_CHUNK;       // one k-chunk of a block
constexpr int kUnitBlock = DFSSM_UNIT_BLOCK;       // the epilogue of a block
constexpr int kDecodeLinStart = 2 * kUnitChunk;    // entering a linear (its quantisation pass)
__host__ __device__ inline int decode_block_units(int d_in) {
    return (d_in + kDecodeChunkCols - 1) / kDecodeChunkCols * kUnitChunk + kUnitBlock;
}
__host__ __device__ inline int64_t decode_units(int d_in, int d_out, int rows) {
    return (int64_t)((d_out + rows - 1) / rows) * decode_block_units(d_in) + kDecodeLinStart;
}

constexpr int kSegCols = 256;
constexpr int kDecodeMaxTokens = 16;   // m up to this runs the decode kernel
__host__ __device__ inline int seg_qrow(int d_in) { return (d_in + kSegCols - 1) / kSegCols * kSegCols; }

// ---- launch wrappers implemented in the .cu files ---------------------------------

struct LaunchCtx {
    const dfssm_stack_entry* entries;  // device array, or nullptr for `single`
    dfssm_stack_entry single;          // used when entries == nullptr (n == 1)
    int n;                             // number of linears
    int m;                             // tokens per linear
    const DevDesc* desc;               // device descriptor table (n entries, index = position)
    const DevDesc* host_desc;          // host copy (same content)
    int8_t* q_ws;
    TokStats* st_ws;
    uint32_t* err;
    int* part;                         // split partials: n x kMaxSplits x 16 tokens x 20 ints
    const void* tmaps;                 // device array of CUtensorMap (prefill activation rows), one per desc
    const void* sign_tmpl;             // device CUtensorMap templates of the decode sign rows (stack calls):
                                       // [0, tmpl_stride) for 128-row blocks, [tmpl_stride, 2 tmpl_stride) for 64
    int tmpl_stride;
    void* map_slots;                   // device CUtensorMap slots edited by the decode CTAs (stack calls)
    int max_d_in;                      // largest d_in among the n linears
    int64_t total_rows;                // sum of d_out over the n linears
    int sm_count;
    uint64_t wait_limit_ns;            // bound of every in-kernel wait of the decode kernel
    int stall_test;                    // test hook of the decode kernel (0 in normal use)
    cudaStream_t stream;
};

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s

// One token: the LoRA down-projection h = W_B q runs as (linear, slice) items of
// kLoraSliceCols columns in a kernel small enough to share the SMs with the decode kernel;
// the decode kernel adds the slices' partial h (part_index with kLoraMaxSlices).
#ifndef DFSSM_LORA_SLICE_COLS
#define DFSSM_LORA_SLICE_COLS 2048
#endif
constexpr int kLoraSliceCols = DFSSM_LORA_SLICE_COLS;
constexpr int kLoraMaxSlices = kMaxDIn / kLoraSliceCols;
constexpr int kMaxSliceItems = 768;
static_assert(kLoraMaxSlices <= kMaxSplits, "slice partials fit the split partial buffer");
__host__ __device__ inline int lora_slices(int d_in) { return (d_in + kLoraSliceCols - 1) / kLoraSliceCols; }
inline int lora_slice_items(const LaunchCtx& c) {
    int items = 0;
    for (int i = 0; i < c.n; ++i) items += lora_slices(c.host_desc[i].d_in);
    return items;
}
inline bool use_lora_slices(const LaunchCtx& c) { return c.m == 1 && lora_slice_items(c) <= kMaxSliceItems; }
// CTAs of the slice kernel (one item each while they last, at most one per SM)
inline int lora_slice_grid(const LaunchCtx& c) {
    const int items = lora_slice_items(c);
    return items < c.sm_count ? items : c.sm_count;
}

// Arguments of the int8 table kernels (int8_table.cu).
struct Int8TableArgs {
    const int8_t* table;   // vocab x d int8
    const float* scale;    // vocab fp32
    int vocab, d;
    const int32_t* ids;    // embedding: m token ids
    const void* in;        // LM head: m x d bf16 hidden state
    int m;
    void* out;             // m x d (embedding) or m x vocab (LM head) of out_dtype
    int out_dtype;
    int32_t* acc;          // LM head: optional int32 sums
    uint32_t* err;         // embedding: optional error word
};
cudaError_t launch_embed(const Int8TableArgs& a, cudaStream_t s);
cudaError_t launch_lm_head(const Int8TableArgs& a, int sm_count, cudaStream_t s);

cudaError_t launch_pack_sign(const void* src, int src_dtype, int d_out, int d_in, uint8_t* packed,
                             cudaStream_t s);
cudaError_t launch_quant(const LaunchCtx& c);
int quant_splits(const LaunchCtx& c);   // d_in splits of the m <= 16 quantisation kernel
cudaError_t launch_decode(const LaunchCtx& c);
bool encode_sign_map(CUtensorMap* map, const void* sign, int d_in, int d_out, int rows);   // decode sign rows
int decode_map_slots_per_sm();                                                             // map slots the plan keeps per SM
int decode_block_rows(int m);                                                              // decode block rows for m tokens
cudaError_t launch_prefill(const LaunchCtx& c);

// ---- tensor maps (host side) ----------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver (nullptr if unavailable)
inline EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn) return fn;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
    return fn;
}

// Allow `kernel` the opt-in dynamic shared memory (minus its static shared memory).
template <typename K>
inline cudaError_t allow_dyn_smem(K kernel, int optin) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                optin - (int)fa.sharedSizeBytes);
}

// ---- small device helpers -----------------------------------------------------------

__device__ __forceinline__ const dfssm_stack_entry& entry_at(const dfssm_stack_entry* entries,
                                                            const dfssm_stack_entry& single, int i) {
    return entries ? entries[i] : single;
}

__device__ __forceinline__ bool ptr_ok(const void* p) {
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}
__device__ __forceinline__ bool opt_ptr_ok(const void* p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Every pointer of an entry is non-NULL (debug ones may be NULL) and 16-byte aligned.
// Entries of a stack call live in device memory, so the host cannot check them.
__device__ __forceinline__ bool entry_ptrs_ok(const dfssm_stack_entry& e) {
    return ptr_ok(e.w.sign) && ptr_ok(e.w.alpha) && ptr_ok(e.w.wa) && ptr_ok(e.w.sa) && ptr_ok(e.w.wb) &&
           ptr_ok(e.w.sb) && ptr_ok(e.x) && ptr_ok(e.y) && opt_ptr_ok(e.dbg.q) && opt_ptr_ok(e.dbg.sx) &&
           opt_ptr_ok(e.dbg.acc) && opt_ptr_ok(e.dbg.h);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

}  // namespace dfssm
