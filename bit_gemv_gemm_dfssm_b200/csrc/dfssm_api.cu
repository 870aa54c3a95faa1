// libdfssm C ABI: plans, argument checks, workspace and dispatch.
//
// A call runs two kernels on the caller's stream:
//   1. quant_kernel: per-token int8 quantisation of x, sum q, and the rank-16
//      LoRA down-projection (quant.cu);
//   2. the scaffold contraction with the fused LoRA up-projection and
//      dequantisation: decode_kernel for m <= 16 tokens (decode.cu), the
//      tcgen05 prefill_kernel above that (prefill.cu).
// The second kernel uses programmatic dependent launch so its weight streaming
// overlaps the first kernel.
#include <cuda.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "dfssm_internal.cuh"

using namespace dfssm;

namespace dfssm {
cudaError_t set_quant_attr(int optin);
cudaError_t set_quant_rows_attr(int optin);
cudaError_t set_decode_attr(int optin);
cudaError_t set_prefill_attr(int optin);
cudaError_t set_int8_table_attr(int optin);
int prefill_box_tokens();
int prefill_box_bytes();

// Allow each kernel the opt-in shared memory size (a permission, not a reservation).
static cudaError_t set_kernel_attributes(int optin) {
    cudaError_t e = set_quant_attr(optin);
    if (e == cudaSuccess) e = set_quant_rows_attr(optin);
    if (e == cudaSuccess) e = set_decode_attr(optin);
    if (e == cudaSuccess) e = set_prefill_attr(optin);
    return e;
}
}

struct dfssm_plan_s {
    int device = -1;
    int sm_count = 0;
    int n = 0;
    std::vector<DevDesc> hdesc;
    DevDesc* ddesc = nullptr;
    int8_t* q_ws = nullptr;
    TokStats* st_ws = nullptr;
    uint32_t* err = nullptr;
    int* part = nullptr;
    CUtensorMap* tmaps = nullptr;       // prefill: activation rows of each linear
    CUtensorMap* sign_tmpl = nullptr;   // decode: sign rows of each linear (placeholder address), 128- then 192-row boxes
    CUtensorMap* map_slots = nullptr;   // decode: per-CTA slots for the device-edited sign maps
    uint64_t wait_limit_ns = kWaitLimitNs;
    int stall_test = 0;
    size_t ws_bytes = 0;
};

namespace {

constexpr int kDecodeMaxM = kDecodeMaxTokens;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

dfssm_status check_desc(const dfssm_linear_desc& d) {
    if (d.rank != kRank) return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (d.d_in < 128 || d.d_in > kMaxDIn || d.d_in % 128 != 0) return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (d.d_out < 1 || d.d_out > (1 << 20)) return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (d.max_m < 1 || d.max_m > kMaxM) return DFSSM_ERR_UNSUPPORTED_SHAPE;
    if (d.y_dtype != DFSSM_BF16 && d.y_dtype != DFSSM_F32) return DFSSM_ERR_INVALID_ARG;
    if (d.flags != 0) return DFSSM_ERR_INVALID_ARG;
    return DFSSM_OK;
}

dfssm_status check_weights(const dfssm_linear_weights& w) {
    const void* p[6] = {w.sign, w.alpha, w.wa, w.sa, w.wb, w.sb};
    for (const void* q : p)
        if (q == nullptr || !aligned16(q)) return DFSSM_ERR_INVALID_ARG;
    return DFSSM_OK;
}

dfssm_status check_dbg(const dfssm_debug& g) {
    const void* p[4] = {g.q, g.sx, g.acc, g.h};
    for (const void* q : p)
        if (q != nullptr && !aligned16(q)) return DFSSM_ERR_INVALID_ARG;
    return DFSSM_OK;
}


void free_plan(dfssm_plan_s* p) {
    if (!p) return;
    if (p->ddesc) cudaFree(p->ddesc);
    if (p->q_ws) cudaFree(p->q_ws);
    if (p->st_ws) cudaFree(p->st_ws);
    if (p->err) cudaFree(p->err);
    if (p->part) cudaFree(p->part);
    if (p->tmaps) cudaFree(p->tmaps);
    if (p->sign_tmpl) cudaFree(p->sign_tmpl);
    if (p->map_slots) cudaFree(p->map_slots);
    delete p;
}

dfssm_status run(dfssm_plan_s* p, LaunchCtx& c) {
    cudaError_t e = launch_quant(c);
    if (e != cudaSuccess) return DFSSM_ERR_CUDA;
    e = (c.m <= kDecodeMaxM) ? launch_decode(c) : launch_prefill(c);
    if (e != cudaSuccess) return DFSSM_ERR_CUDA;
    (void)p;
    return DFSSM_OK;
}

}  // namespace

extern "C" {

const char* dfssm_status_string(dfssm_status s) {
    switch (s) {
        case DFSSM_OK: return "ok";
        case DFSSM_ERR_INVALID_ARG: return "invalid argument";
        case DFSSM_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case DFSSM_ERR_CUDA: return "CUDA error";
        case DFSSM_ERR_NO_MEMORY: return "out of device memory";
        case DFSSM_ERR_DEVICE_CHECK: return "device-side check failed";
    }
    return "unknown status";
}

dfssm_status dfssm_linear_plan(const dfssm_linear_desc* descs, int n_descs, dfssm_plan* out) {
    if (out == nullptr) return DFSSM_ERR_INVALID_ARG;
    *out = nullptr;
    if (descs == nullptr || n_descs < 1 || n_descs > 4096) return DFSSM_ERR_INVALID_ARG;
    for (int i = 0; i < n_descs; ++i) {
        dfssm_status s = check_desc(descs[i]);
        if (s != DFSSM_OK) return s;
    }
    dfssm_plan_s* p = new (std::nothrow) dfssm_plan_s();
    if (!p) return DFSSM_ERR_NO_MEMORY;
    if (cudaGetDevice(&p->device) != cudaSuccess) { delete p; return DFSSM_ERR_CUDA; }
    int optin = 0;
    if (cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device) != cudaSuccess) {
        delete p;
        return DFSSM_ERR_CUDA;
    }
    p->n = n_descs;
    p->hdesc.resize(n_descs);
    int64_t q_bytes = 0, st_count = 0, units128 = 0, units192 = 0;
    int32_t rt = 0;
    for (int i = 0; i < n_descs; ++i) {
        DevDesc& d = p->hdesc[i];
        std::memset(&d, 0, sizeof(d));
        d.d_in = descs[i].d_in;
        d.d_out = descs[i].d_out;
        d.y_dtype = descs[i].y_dtype;
        d.max_m = descs[i].max_m;
        d.qrow = seg_qrow(d.d_in);
        // activation rows only for the prefill; every region is a multiple of 256 bytes
        d.q_off = q_bytes;
        if (d.max_m > kDecodeMaxM) q_bytes += (int64_t)d.max_m * d.qrow;
        d.st_off = st_count;
        d.rt_begin = rt;
        d.work_begin[0] = units128;
        d.work_begin[1] = units192;
        units128 += decode_units(d.d_in, d.d_out, 128);
        units192 += decode_units(d.d_in, d.d_out, 192);
        st_count += d.max_m;
        rt += (d.d_out + 127) / 128;
    }
    cudaError_t e = cudaSuccess;
    e = cudaMalloc(&p->ddesc, sizeof(DevDesc) * n_descs);
    if (e == cudaSuccess) e = cudaMalloc(&p->q_ws, (size_t)(q_bytes > 0 ? q_bytes : 256));
    if (e == cudaSuccess) e = cudaMalloc(&p->st_ws, sizeof(TokStats) * (size_t)st_count);
    if (e == cudaSuccess) e = cudaMalloc(&p->err, 16);
    if (e == cudaSuccess) e = cudaMalloc(&p->tmaps, sizeof(CUtensorMap) * n_descs);
    const size_t n_slots = (size_t)p->sm_count * decode_map_slots_per_sm();
    if (e == cudaSuccess) e = cudaMalloc(&p->sign_tmpl, sizeof(CUtensorMap) * 2 * n_descs);
    if (e == cudaSuccess) e = cudaMalloc(&p->map_slots, sizeof(CUtensorMap) * n_slots);
    const size_t part_bytes = sizeof(int) * (size_t)n_descs * kMaxSplits * kPartTok * 20;
    if (e == cudaSuccess) e = cudaMalloc(&p->part, part_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_plan(p);
        return e == cudaErrorMemoryAllocation ? DFSSM_ERR_NO_MEMORY : DFSSM_ERR_CUDA;
    }
    p->ws_bytes = sizeof(DevDesc) * n_descs + (size_t)q_bytes + sizeof(TokStats) * st_count + 16 +
                  sizeof(CUtensorMap) * (3 * (size_t)n_descs + n_slots) + part_bytes;

    // prefill: tensor maps over each linear's activation rows (B operand, 128-byte swizzle)
    std::vector<CUtensorMap> tm(n_descs);
    std::memset(tm.data(), 0, sizeof(CUtensorMap) * n_descs);
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) { free_plan(p); return DFSSM_ERR_CUDA; }
    for (int i = 0; i < n_descs; ++i) {
        const DevDesc& d = p->hdesc[i];
        if (d.max_m > kDecodeMaxM) {
            cuuint64_t dims[2] = {(cuuint64_t)d.qrow, (cuuint64_t)d.max_m};
            cuuint64_t strides[1] = {(cuuint64_t)d.qrow};
            cuuint32_t box[2] = {(cuuint32_t)prefill_box_bytes(), (cuuint32_t)prefill_box_tokens()};
            cuuint32_t estr[2] = {1, 1};
            CUresult r = enc(&tm[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->q_ws + d.q_off, dims, strides, box, estr,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) { free_plan(p); return DFSSM_ERR_CUDA; }
        }
    }
    // decode: each linear's sign map with a placeholder address (set per call on the device), for
    // the block rows of up to 8 tokens (first n) and of more (next n)
    std::vector<CUtensorMap> st(2 * (size_t)n_descs);
    for (int h = 0; h < 2; ++h)
        for (int i = 0; i < n_descs; ++i)
            if (!encode_sign_map(&st[(size_t)h * n_descs + i], p->ddesc, p->hdesc[i].d_in, p->hdesc[i].d_out,
                                 decode_block_rows(h == 0 ? 1 : kDecodeMaxM))) {
                free_plan(p);
                return DFSSM_ERR_CUDA;
            }
    e = cudaMemcpy(p->tmaps, tm.data(), sizeof(CUtensorMap) * n_descs, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(p->sign_tmpl, st.data(), sizeof(CUtensorMap) * 2 * n_descs, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(p->ddesc, p->hdesc.data(), sizeof(DevDesc) * n_descs, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(p->err, 0, 16);
    if (e == cudaSuccess) e = set_kernel_attributes(optin);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) { free_plan(p); return DFSSM_ERR_CUDA; }
    *out = p;
    return DFSSM_OK;
}

dfssm_status dfssm_plan_destroy(dfssm_plan plan) {
    if (!plan) return DFSSM_OK;
    DeviceGuard g(plan->device);
    cudaDeviceSynchronize();
    free_plan(plan);
    return DFSSM_OK;
}

dfssm_status dfssm_pack_sign(const void* src, int32_t src_dtype, int32_t d_out, int32_t d_in, uint8_t* packed,
                             void* stream) {
    if (src == nullptr || packed == nullptr || !aligned16(src) || !aligned16(packed)) return DFSSM_ERR_INVALID_ARG;
    if (src_dtype != DFSSM_I8 && src_dtype != DFSSM_F32) return DFSSM_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 128 || d_in % 128 != 0 || (int64_t)d_out * d_in > ((int64_t)1 << 40))
        return DFSSM_ERR_UNSUPPORTED_SHAPE;
    cudaError_t e = launch_pack_sign(src, src_dtype, d_out, d_in, packed, (cudaStream_t)stream);
    return e == cudaSuccess ? DFSSM_OK : DFSSM_ERR_CUDA;
}

dfssm_status dfssm_linear_fwd(dfssm_plan plan, int32_t desc_index, const dfssm_linear_weights* w, const void* x,
                              int32_t m, void* y, const dfssm_debug* dbg, void* stream) {
    if (!plan || !w || !x || !y) return DFSSM_ERR_INVALID_ARG;
    if (desc_index < 0 || desc_index >= plan->n) return DFSSM_ERR_INVALID_ARG;
    const DevDesc& hd = plan->hdesc[desc_index];
    if (m < 1 || m > hd.max_m) return DFSSM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return DFSSM_ERR_INVALID_ARG;
    dfssm_status s = check_weights(*w);
    if (s != DFSSM_OK) return s;
    dfssm_debug g = {nullptr, nullptr, nullptr, nullptr};
    if (dbg) {
        g = *dbg;
        if ((s = check_dbg(g)) != DFSSM_OK) return s;
    }
    DeviceGuard guard(plan->device);
    if (!guard.ok) return DFSSM_ERR_CUDA;
    LaunchCtx c{};
    c.entries = nullptr;
    c.single.w = *w;
    c.single.x = x;
    c.single.y = y;
    c.single.dbg = g;
    c.single.desc_index = desc_index;
    c.n = 1;
    c.m = m;
    c.desc = plan->ddesc + desc_index;
    c.host_desc = &plan->hdesc[desc_index];
    c.q_ws = plan->q_ws;
    c.st_ws = plan->st_ws;
    c.err = plan->err;
    c.part = plan->part + (size_t)desc_index * kMaxSplits * kPartTok * 20;
    c.tmaps = plan->tmaps + desc_index;
    c.wait_limit_ns = plan->wait_limit_ns;
    c.stall_test = plan->stall_test;
    c.max_d_in = hd.d_in;
    c.total_rows = hd.d_out;
    c.sm_count = plan->sm_count;
    c.stream = (cudaStream_t)stream;
    return run(plan, c);
}

dfssm_status dfssm_linear_stack_fwd(dfssm_plan plan, const dfssm_stack_entry* entries_dev, int32_t n_entries,
                                    int32_t m, void* stream) {
    if (!plan || !entries_dev || (reinterpret_cast<uintptr_t>(entries_dev) & 7u)) return DFSSM_ERR_INVALID_ARG;
    if (n_entries < 1 || n_entries > plan->n) return DFSSM_ERR_INVALID_ARG;
    int max_d_in = 0;
    int64_t rows = 0;
    for (int i = 0; i < n_entries; ++i) {
        const DevDesc& d = plan->hdesc[i];
        if (m < 1 || m > d.max_m) return DFSSM_ERR_INVALID_ARG;
        if (d.d_in > max_d_in) max_d_in = d.d_in;
        rows += d.d_out;
    }
    DeviceGuard guard(plan->device);
    if (!guard.ok) return DFSSM_ERR_CUDA;
    LaunchCtx c{};
    c.entries = entries_dev;
    c.n = n_entries;
    c.m = m;
    c.desc = plan->ddesc;
    c.host_desc = plan->hdesc.data();
    c.q_ws = plan->q_ws;
    c.st_ws = plan->st_ws;
    c.err = plan->err;
    c.part = plan->part;
    c.tmaps = plan->tmaps;
    c.sign_tmpl = plan->sign_tmpl;
    c.tmpl_stride = plan->n;
    c.map_slots = plan->map_slots;
    c.wait_limit_ns = plan->wait_limit_ns;
    c.stall_test = plan->stall_test;
    c.max_d_in = max_d_in;
    c.total_rows = rows;
    c.sm_count = plan->sm_count;
    c.stream = (cudaStream_t)stream;
    return run(plan, c);
}

dfssm_status dfssm_plan_check(dfssm_plan plan, uint32_t* bits) {
    if (!plan) return DFSSM_ERR_INVALID_ARG;
    DeviceGuard guard(plan->device);
    if (!guard.ok) return DFSSM_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DFSSM_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, plan->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DFSSM_ERR_CUDA;
    if (cudaMemset(plan->err, 0, 4) != cudaSuccess) return DFSSM_ERR_CUDA;
    if (bits) *bits = v;
    return v ? DFSSM_ERR_DEVICE_CHECK : DFSSM_OK;
}

// Per-device set-up of the plan-free int8 table calls (SM count, shared-memory limits).
namespace {
struct TableSetup {
    int sm_count = 0;
    bool ready = false;
};
TableSetup g_table_setup[64];
std::mutex g_table_mu;

dfssm_status table_setup(int* sm_count) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DFSSM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_table_mu);
    TableSetup& t = g_table_setup[dev];
    if (!t.ready) {
        int optin = 0;
        if (cudaDeviceGetAttribute(&t.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            set_int8_table_attr(optin) != cudaSuccess)
            return DFSSM_ERR_CUDA;
        t.ready = true;
    }
    *sm_count = t.sm_count;
    return DFSSM_OK;
}

dfssm_status check_table(const dfssm_int8_table* t) {
    if (!t || !t->table || !t->scale || !aligned16(t->table) || !aligned16(t->scale)) return DFSSM_ERR_INVALID_ARG;
    if (t->d < 16 || t->d > kMaxDIn || t->d % 16 != 0 || t->vocab < 1 || t->vocab > (1 << 24))
        return DFSSM_ERR_UNSUPPORTED_SHAPE;
    return DFSSM_OK;
}
}  // namespace

dfssm_status dfssm_embed_fwd(const dfssm_int8_table* table, const int32_t* ids, int32_t m, void* out,
                             int32_t out_dtype, uint32_t* err, void* stream) {
    dfssm_status s = check_table(table);
    if (s != DFSSM_OK) return s;
    if (!ids || !out || !aligned16(out) || (reinterpret_cast<uintptr_t>(ids) & 3u) || m < 1 || m > kMaxM)
        return DFSSM_ERR_INVALID_ARG;
    if ((out_dtype != DFSSM_BF16 && out_dtype != DFSSM_F32) || (reinterpret_cast<uintptr_t>(err) & 3u))
        return DFSSM_ERR_INVALID_ARG;
    int sms = 0;
    if ((s = table_setup(&sms)) != DFSSM_OK) return s;
    Int8TableArgs a{table->table, table->scale, table->vocab, table->d, ids, nullptr, m, out, out_dtype,
                    nullptr, err};
    return launch_embed(a, (cudaStream_t)stream) == cudaSuccess ? DFSSM_OK : DFSSM_ERR_CUDA;
}

dfssm_status dfssm_lm_head_fwd(const dfssm_int8_table* table, const void* h, int32_t m, void* logits,
                               int32_t out_dtype, int32_t* acc, void* stream) {
    dfssm_status s = check_table(table);
    if (s != DFSSM_OK) return s;
    if (!h || !logits || !aligned16(h) || !aligned16(logits) || !aligned16(acc) || m < 1 || m > 16)
        return DFSSM_ERR_INVALID_ARG;
    if (out_dtype != DFSSM_BF16 && out_dtype != DFSSM_F32) return DFSSM_ERR_INVALID_ARG;
    int sms = 0;
    if ((s = table_setup(&sms)) != DFSSM_OK) return s;
    Int8TableArgs a{table->table, table->scale, table->vocab, table->d, nullptr, h, m, logits, out_dtype, acc,
                    nullptr};
    return launch_lm_head(a, sms, (cudaStream_t)stream) == cudaSuccess ? DFSSM_OK : DFSSM_ERR_CUDA;
}

dfssm_status dfssm_plan_set_test_hooks(dfssm_plan plan, uint64_t wait_limit_ns, uint32_t flags) {
    if (!plan || (flags & ~DFSSM_TEST_STALL) != 0) return DFSSM_ERR_INVALID_ARG;
    plan->wait_limit_ns = wait_limit_ns ? wait_limit_ns : kWaitLimitNs;
    plan->stall_test = (flags & DFSSM_TEST_STALL) ? 1 : 0;
    return DFSSM_OK;
}

dfssm_status dfssm_plan_workspace_bytes(dfssm_plan plan, size_t* bytes) {
    if (!plan || !bytes) return DFSSM_ERR_INVALID_ARG;
    *bytes = plan->ws_bytes;
    return DFSSM_OK;
}

}  // extern "C"
