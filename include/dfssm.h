/*
 * dfssm.h - C ABI of libdfssm: the DF-SSM 1-bit scaffold + int8 LoRA linear on
 * NVIDIA B200 (sm_100a), and the parts of the model's decode step around it (the
 * int8 embedding / LM head, the Mamba-2 state step, the block frame), each
 * declared in its own section below.
 *
 * The layer ("Density Field State Space Models", gist.science technical
 * summary, §2.B "frozen scaffold with LoRA correction" and §2.C "optimised
 * inference pipeline"; arXiv 2606.10932 abstract): every Mamba-2 in_proj and
 * out_proj is a frozen 1-bit sign matrix plus a rank-16 int8 LoRA correction,
 * applied to int8-quantised activations. For token t and output row o:
 *
 *   q, s_x   : per-token symmetric absmax int8 quantisation of x (below)
 *   acc[t,o] = sum_j w[o,j] * q[t,j]        w[o,j] in {-1,+1}, int32
 *   h[t,k]   = sum_j W_B[k,j] * q[t,j]      k < 16, int32
 *   y[t,o]   = s_x[t] * ( alpha[o] * acc[t,o]
 *                         + s_A[o] * sum_k W_A[o,k] * (s_B[k] * h[t,k]) )
 *
 * Conventions the pages leave open, fixed here (and identical in the oracle):
 *   - sign bits: row-major, d_in/8 bytes per output row, no padding; column j
 *     of row o is bit (j % 8) of byte o*(d_in/8) + j/8 (LSB first);
 *     bit 1 -> +1, bit 0 -> -1.
 *   - quantiser, in IEEE fp32 with round-to-nearest: amax = max_j |x[t,j]|;
 *     amax == 0 -> q = 0, s_x = 0; otherwise inv = 127/amax,
 *     q = clamp(round_half_even(x * inv), -127, 127), s_x = amax/127
 *     (amax below 127/FLT_MAX overflows inv: nonzero entries give +-127, zeros 0;
 *     known issue: for m > 16 tokens the quantiser does not yet follow this case and
 *     gives 0 for nonzero entries and -1 for zeros of such a token).
 *   - alpha, s_A: one fp32 per output row; s_B: one fp32 per LoRA row.
 *   - s_x multiplies both terms; s_B * h stays in fp32 (not re-quantised).
 *
 * Memory: every tensor pointer is a DEVICE pointer owned by the caller (a
 * stack entry's y may also be the device address of mapped pinned host memory,
 * see dfssm_stack_entry); the library never frees it. Tensor pointers must be
 * 16-byte aligned. A plan owns
 * its workspace (device memory allocated by dfssm_linear_plan, freed by
 * dfssm_plan_destroy) and is tied to the device current at plan time.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream). Calls only enqueue work; they never synchronise, except
 * dfssm_plan_check. Caller buffers must stay valid until the stream has run
 * the work. x and y must not overlap. A plan's workspace is reused by every
 * call, so calls on one plan must be ordered (same stream, or synchronised);
 * a plan is not thread-safe.
 *
 * Errors: argument errors are returned synchronously and nothing is enqueued.
 * A failed launch returns DFSSM_ERR_CUDA. Conditions only the device can see
 * (a stack entry whose desc_index does not match its position or whose
 * pointers are NULL or misaligned, a non-finite amax, a bounded wait that gave
 * up) set the plan's device error word instead of trapping; read it with
 * dfssm_plan_check.
 */
#ifndef DFSSM_H
#define DFSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DFSSM_OK = 0,
    DFSSM_ERR_INVALID_ARG = 1,       /* NULL / misaligned pointer, bad enum, m out of range */
    DFSSM_ERR_UNSUPPORTED_SHAPE = 2, /* d_in % 128 != 0, d_in > 8192, rank != 16, ... */
    DFSSM_ERR_CUDA = 3,              /* a CUDA runtime call or launch failed */
    DFSSM_ERR_NO_MEMORY = 4,         /* workspace allocation failed */
    DFSSM_ERR_DEVICE_CHECK = 5       /* the device error word was set (dfssm_plan_check) */
} dfssm_status;

typedef enum { DFSSM_BF16 = 0, DFSSM_F32 = 1, DFSSM_I8 = 2 } dfssm_dtype;

/* Device error word bits (dfssm_plan_check). */
#define DFSSM_DEVERR_ENTRY_DESC 0x1u   /* stack entry i has desc_index != i */
#define DFSSM_DEVERR_NONFINITE  0x2u   /* a token's amax was Inf or NaN (output undefined) */
#define DFSSM_DEVERR_TIMEOUT    0x4u   /* a bounded in-kernel wait gave up (output undefined) */
#define DFSSM_DEVERR_ENTRY_PTR  0x8u   /* a stack entry holds a NULL or misaligned pointer (entry skipped) */
#define DFSSM_DEVERR_TOKEN_ID   0x10u  /* an embedding id outside [0, vocab) (its row is zeros) */

/* Shape of one linear. d_in % 128 == 0, 128 <= d_in <= 8192; 1 <= d_out <= 2^20;
 * rank == 16; 1 <= max_m <= 65536; y_dtype DFSSM_BF16 or DFSSM_F32; flags = 0. */
typedef struct {
    int32_t d_in;
    int32_t d_out;
    int32_t rank;
    int32_t max_m;
    int32_t y_dtype;
    uint32_t flags;
} dfssm_linear_desc;

/* Weights of one linear (device pointers, caller-owned, 16-byte aligned).
 *   sign  : d_out x (d_in/8) bytes, packed as above (see dfssm_pack_sign)
 *   alpha : d_out fp32 scaffold scale per output row
 *   wa    : d_out x 16 int8, row-major (LoRA up-projection W_A)
 *   sa    : d_out fp32 (per-row scale of W_A)
 *   wb    : 16 x d_in int8, row-major (LoRA down-projection W_B)
 *   sb    : 16 fp32 (per-row scale of W_B)
 * ("Density Field State Space Models", technical summary §2.B: W_A in
 * R^{d_out x r}, W_B in R^{r x d_in}, r = 16, int8 with per-channel/row scales.) */
typedef struct {
    const uint8_t* sign;
    const float* alpha;
    const int8_t* wa;
    const float* sa;
    const int8_t* wb;
    const float* sb;
} dfssm_linear_weights;

/* Optional exports for bit-exact checks (device pointers; any may be NULL):
 *   q   : m x d_in int8 (natural column order), sx : m fp32,
 *   acc : m x d_out int32 (scaffold sums), h : m x 16 int32 (LoRA down sums). */
typedef struct {
    int8_t* q;
    float* sx;
    int32_t* acc;
    int32_t* h;
} dfssm_debug;

/* One linear of a stack (this struct lives in DEVICE memory for
 * dfssm_linear_stack_fwd). x: m x d_in bf16 row-major; y: m x d_out of the
 * desc's y_dtype, row-major. desc_index must equal the entry's position.
 * y may be pinned host memory mapped for the device (its device address): the
 * kernels then write each output over the bus as they finish it, so the copy
 * back overlaps the compute. x is read several times and belongs in device
 * memory. */
typedef struct {
    dfssm_linear_weights w;
    const void* x;
    void* y;
    dfssm_debug dbg;
    int32_t desc_index;
    int32_t reserved;
} dfssm_stack_entry;

typedef struct dfssm_plan_s* dfssm_plan;

/* Create a plan for n_descs linears on the current device. For a stack, desc i
 * describes stack entry i (48 Mamba-2 layers = 96 descs: in_proj, out_proj,
 * ...). Allocates the workspace (int8 activations and per-token scales for
 * max_m tokens per linear, the prefill tensor maps and the error word).
 * On success *out receives the plan; on failure *out is NULL and nothing is
 * left allocated. */
dfssm_status dfssm_linear_plan(const dfssm_linear_desc* descs, int n_descs, dfssm_plan* out);

/* Free a plan and its workspace. Waits for the device to finish using it
 * (device synchronise). NULL is accepted. */
dfssm_status dfssm_plan_destroy(dfssm_plan plan);

/* Pack a frozen scaffold into sign bits (technical summary §2.B: the scaffold
 * is frozen at its rounded values; §2.C / §3: stored at 1 bit per weight).
 * src: d_out x d_in device tensor, row-major, of src_dtype DFSSM_I8 or
 * DFSSM_F32; value >= 0 (including -0.0) -> +1 -> bit 1, value < 0 -> bit 0.
 * A NaN in an fp32 source is outside the contract (its bit is unspecified).
 * packed: d_out x d_in/8 bytes, device. d_in % 128 == 0. */
dfssm_status dfssm_pack_sign(const void* src, int32_t src_dtype, int32_t d_out, int32_t d_in,
                             uint8_t* packed, void* stream);

/* y = layer(x) for one linear (the formula at the top of this file).
 * desc_index selects the shape; w is a HOST struct of device pointers;
 * x: m x d_in bf16 (device); y: m x d_out of the desc's y_dtype (device);
 * 1 <= m <= max_m. dbg may be NULL. */
dfssm_status dfssm_linear_fwd(dfssm_plan plan, int32_t desc_index, const dfssm_linear_weights* w,
                              const void* x, int32_t m, void* y, const dfssm_debug* dbg,
                              void* stream);

/* The layer for n_entries independent linears, in one pass (the pages capture
 * the whole 48-layer forward as one CUDA graph, technical summary §2.C).
 * entries_dev: DEVICE array of n_entries dfssm_stack_entry, entry i planned by
 * desc i; 1 <= n_entries <= n_descs; every entry uses the same m. */
dfssm_status dfssm_linear_stack_fwd(dfssm_plan plan, const dfssm_stack_entry* entries_dev,
                                    int32_t n_entries, int32_t m, void* stream);

/* The layer for one linear and a few tokens, allocating nothing.
 * No counterpart in the paper: this is for callers that cannot call cudaMalloc,
 * such as an embedder whose device allocator must not be re-entered from inside
 * the layer, or a host that fixes its device memory budget up front. It needs no
 * plan: its scratch (partial LoRA sums h, descriptor, error word) is a
 * file-scope device array of about 11 KB that every GPU using this library keeps
 * until the process exits; the descriptor is written there by a one-thread
 * kernel that receives it by value, so no host buffer outlives the call.
 * desc: HOST pointer to the linear's shape (rank 16, 128 <= d_in <= 8192,
 * d_in % 128 == 0; max_m is ignored); w: HOST struct of device pointers;
 * x: m x d_in bf16 (device); y: m x d_out of desc->y_dtype (device);
 * 1 <= m <= DFSSM_NOALLOC_MAX_M. Larger shapes return
 * DFSSM_ERR_UNSUPPORTED_SHAPE and enqueue nothing. All calls share the one
 * array, so calls that overlap on the GPU (unordered streams) race; the array
 * keeps the last call's contents, and what must start at zero is reset by the
 * kernels themselves. The first call on each device looks up the array's device
 * address and sets kernel attributes: make it before any stream capture. That
 * set-up lasts for the process, so cudaDeviceReset is not supported while this
 * entry point is in use. Device-side error conditions are not reported by this
 * entry point. */
#define DFSSM_NOALLOC_MAX_M 16
dfssm_status dfssm_linear_fwd_noalloc(const dfssm_linear_desc* desc, const dfssm_linear_weights* w,
                                      const void* x, int32_t m, void* y, void* stream);

/* Synchronise the plan's device, read and clear its error word.
 * Returns DFSSM_OK or DFSSM_ERR_DEVICE_CHECK (*bits, if not NULL, gets the word). */
dfssm_status dfssm_plan_check(dfssm_plan plan, uint32_t* bits);

/* An int8 table with one fp32 scale per row: the embedding and the LM head ("Density
 * Field State Space Models", technical summary §2.B: embedding / LM head quantised to
 * int8 with per-channel/row scales; §3: 37 % of the 278 MB model; Mamba ties the two, so
 * one table serves both). Device pointers, caller-owned, 16-byte aligned:
 *   table : vocab x d int8, row-major; d % 16 == 0, 16 <= d <= 8192; 1 <= vocab <= 2^24
 *   scale : vocab fp32 */
typedef struct {
    const int8_t* table;
    const float* scale;
    int32_t vocab;
    int32_t d;
} dfssm_int8_table;

/* Embedding rows: out[t, j] = scale[ids[t]] * table[ids[t], j], one fp32 product (exact
 * operands, one rounding), rounded to bf16 (nearest even) when out_dtype is DFSSM_BF16.
 * table: HOST struct of device pointers; ids: m int32 (device); out: m x d of out_dtype
 * (device); 1 <= m <= 65536. An id outside [0, vocab) gives a row of zeros and, if err (a
 * device uint32, may be NULL) is given, ORs DFSSM_DEVERR_TOKEN_ID into it. Allocates
 * nothing; the first call on a device sets kernel attributes (make it before any stream
 * capture). */
dfssm_status dfssm_embed_fwd(const dfssm_int8_table* table, const int32_t* ids, int32_t m, void* out,
                             int32_t out_dtype, uint32_t* err, void* stream);

/* LM head: logits[t, v] = s_x[t] * (scale[v] * sum_j table[v, j] * q[t, j]), the sum in
 * int32, where q, s_x are the layer's per-token int8 quantisation of h (as for every
 * linear above). table: HOST struct of device pointers; h: m x d bf16 (device),
 * 1 <= m <= 16; logits: m x vocab of out_dtype (device); acc: optional m x vocab int32
 * sums (device, may be NULL). Allocates nothing; the first call on a device sets kernel
 * attributes (make it before any stream capture). */
dfssm_status dfssm_lm_head_fwd(const dfssm_int8_table* table, const void* h, int32_t m, void* logits,
                               int32_t out_dtype, int32_t* acc, void* stream);

/* ---- decode step of the state operations between in_proj and out_proj -------------------
 * "Density Field State Space Models" (gist.science technical summary), §2.C, state
 * operations: the state shift register (causal convolution) and the SSM recurrence. The
 * step is Mamba-2's, for one group of B and C:
 *   in_proj output per token: [ z (d_inner) | xBC (conv_dim) | dt_raw (nheads) ],
 *     conv_dim = d_inner + 2 d_state, nheads = d_inner / headdim;
 *   shift register: window = (state[c][1..d_conv-1], xBC[c]) becomes the new state[c];
 *   xc[c] = silu(conv_b[c] + sum_k conv_w[c][k] window[k]); x, B, C = xc split;
 *   dt = softplus(dt_raw + dt_bias) (v itself above 20), dA = exp(-exp(a_log) dt);
 *   S[h][p][n] = S[h][p][n] dA_h + dt_h x[h headdim + p] B[n];
 *   y = sum_n S C[n] + d_skip_h x;  g = y silu(z);  out = g / sqrt(mean(g^2) + eps) norm_w.
 * Supported: headdim 64, d_state 128, d_conv 4, d_inner a multiple of 64 up to 16384. */
typedef struct {
    int32_t d_inner;
    int32_t headdim;    /* 64 */
    int32_t d_state;    /* 128 */
    int32_t d_conv;     /* 4 */
    float eps;          /* RMS-norm epsilon (Mamba-2: 1e-5) */
    int32_t out_dtype;  /* DFSSM_BF16 or DFSSM_F32 */
} dfssm_ssm_dims;

/* One layer (this struct lives in DEVICE memory for dfssm_ssm_step). Device pointers,
 * 16-byte aligned (zxbcdt: 2-byte aligned), caller-owned:
 *   zxbcdt     m x (2 d_inner + 2 d_state + nheads) bf16, row-major: the in_proj output;
 *   conv_state m x conv_dim x d_conv bf16, updated in place;
 *   ssm_state  m x nheads x headdim x d_state fp32, updated in place;
 *   conv_w     conv_dim x d_conv fp32; conv_b conv_dim fp32;
 *   dt_bias, a_log, d_skip  nheads fp32 each; norm_w d_inner fp32;
 *   out        m x d_inner of out_dtype: the out_proj input. */
typedef struct {
    const void* zxbcdt;
    void* conv_state;
    float* ssm_state;
    const float* conv_w;
    const float* conv_b;
    const float* dt_bias;
    const float* a_log;
    const float* d_skip;
    const float* norm_w;
    void* out;
} dfssm_ssm_layer;

/* Bytes of caller-owned device workspace one dfssm_ssm_step call of this shape needs. */
dfssm_status dfssm_ssm_workspace_bytes(const dfssm_ssm_dims* dims, int32_t n_layers, int32_t m, size_t* bytes);

/* One decode step for n_layers independent layers (layers_dev: DEVICE array of n_layers
 * dfssm_ssm_layer) and m tokens each, on `stream`, as two kernels (convolution, recurrence
 * and gate, one CTA per head, token and layer; then the B and C registers and the RMS norm
 * per token and layer). workspace: 256-byte aligned, at least dfssm_ssm_workspace_bytes,
 * zeroed once before its first use. Its first 4 bytes are a device error word that
 * gets DFSSM_DEVERR_ENTRY_PTR when a layer holds a NULL or misaligned pointer (that layer
 * is skipped); read and clear it with dfssm_ssm_read_error. Calls sharing a workspace must
 * be ordered. Allocates nothing. Argument errors return synchronously with no launch. */
dfssm_status dfssm_ssm_step(const dfssm_ssm_dims* dims, const dfssm_ssm_layer* layers_dev, int32_t n_layers,
                            int32_t m, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, return the workspace's error word in *bits and clear it;
 * DFSSM_ERR_DEVICE_CHECK if it was set. */
dfssm_status dfssm_ssm_read_error(void* workspace, uint32_t* bits, void* stream);

/* ---- the frame of a Mamba-2 block: residual add and RMS norm ------------------------------
 * "Density Field State Space Models" (gist.science technical summary), §2.B and §3: the
 * model is Mamba-2 1.3B (48 layers, d_model 2048) with in_proj / out_proj replaced by the
 * layer above. Around the layer each block keeps Mamba-2's frame: an fp32 residual stream r,
 *   r_new = r + delta            (delta: the previous block's out_proj output; NULL: none)
 *   out   = r_new / sqrt(mean(r_new^2) + eps) * norm_w      (the next in_proj's input,
 *                                                           or the LM head's after the last block)
 * per token, over d channels. r_new is one fp32 addition per element; the mean square is
 * summed in fp32 in a fixed order and the output rounded once (bf16 nearest even, or fp32).
 * Device pointers, caller-owned, 16-byte aligned: norm_w d fp32; resid_in, resid_out m x d
 * fp32 (resid_out may equal resid_in: in place); delta m x d of delta_dtype (DFSSM_BF16 or
 * DFSSM_F32) or NULL; out m x d of out_dtype (DFSSM_BF16 or DFSSM_F32). 8 <= d <= 8192,
 * d % 8 == 0, 1 <= m <= 65536 (else DFSSM_ERR_UNSUPPORTED_SHAPE); eps finite and >= 0.
 * One kernel (one CTA per token) on `stream`; allocates nothing; argument errors return
 * synchronously with no launch. */
dfssm_status dfssm_add_rmsnorm(const float* norm_w, int32_t d, float eps, const float* resid_in,
                               const void* delta, int32_t delta_dtype, int32_t m, float* resid_out,
                               void* out, int32_t out_dtype, void* stream);

/* Test of the error path of the decode kernel (m <= 16 tokens), which must end with an
 * error status and never hang. With flags & DFSSM_TEST_STALL, the first CTA of that
 * kernel waits on a barrier that nothing arrives on: the wait gives up after
 * wait_limit_ns, the CTA stops before reading or writing anything, and the plan's
 * device error word gets DFSSM_DEVERR_TIMEOUT (the other CTAs run as usual, so the
 * outputs of the first CTA's rows are undefined). wait_limit_ns also bounds every
 * other wait of that kernel; 0 means the default (1 s). flags = 0 turns the stall off.
 * Takes effect for later calls on this plan; returns DFSSM_ERR_INVALID_ARG for unknown
 * flags. */
#define DFSSM_TEST_STALL 0x1u
dfssm_status dfssm_plan_set_test_hooks(dfssm_plan plan, uint64_t wait_limit_ns, uint32_t flags);

/* Bytes of device workspace the plan holds. */
dfssm_status dfssm_plan_workspace_bytes(dfssm_plan plan, size_t* bytes);

/* Static description of a status code. */
const char* dfssm_status_string(dfssm_status status);

#ifdef __cplusplus
}
#endif

#endif /* DFSSM_H */
