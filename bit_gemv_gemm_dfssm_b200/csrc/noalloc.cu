// dfssm_linear_fwd_noalloc: the layer for one linear and a few tokens without
// any device allocation.
//
// Some callers cannot call cudaMalloc: an embedder whose device allocator must
// not be re-entered from inside the layer, or a host that fixes its device
// memory budget up front. This entry point needs no plan: the quantisation and
// decode kernels run exactly as for dfssm_linear_fwd, with their scratch (the
// quantisation kernel's split partials, the linear's descriptor and the error
// word) in the file-scope device array below, which every GPU that loads this
// library keeps until the process exits. The descriptor is written into the
// array by a one-thread kernel that receives it by value, so no host buffer has
// to outlive the call.
//
// Limits: 1 <= m <= DFSSM_NOALLOC_MAX_M (16) tokens, 128 <= d_in <= 8192.
// Every call shares the array; calls that overlap on the GPU (different streams
// without ordering) race on it. The first call on a device looks up the array's
// device address (cudaGetSymbolAddress) and sets the kernels' shared-memory
// limits; make that first call before any stream capture. That set-up is kept
// for the life of the process, so cudaDeviceReset is not supported while this
// entry point is in use.
#include <cstring>
#include <mutex>

#include "dfssm_internal.cuh"

namespace dfssm {

cudaError_t set_quant_attr(int optin);
cudaError_t set_decode_attr(int optin);

namespace {

constexpr int kNoAllocMaxM = DFSSM_NOALLOC_MAX_M;
constexpr int kMaxDevices = 64;

// scratch layout (byte offsets, 256-byte aligned pieces)
constexpr size_t kOffDesc = 0;                                                      // DevDesc
constexpr size_t kOffErr = 256;                                                     // uint32 error word
constexpr size_t kOffPart = 512;                                                    // split partials of h
constexpr size_t kPartBytes = sizeof(int) * kMaxSplits * kPartTok * kPartInts;
constexpr size_t kScratchBytes = kOffPart + ((kPartBytes + 255) & ~(size_t)255);  // about 11 KB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

struct DeviceSetup {
    uint8_t* scratch = nullptr;   // device address of g_noalloc_scratch on this device
    int sm_count = 0;
    bool ready = false;
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mu;

// Once per device, with that device current: the array's device address (the
// host-side symbol is only a stand-in) and the kernels' shared-memory limits.
dfssm_status setup_device(int dev, DeviceSetup** out) {
    if (dev < 0 || dev >= kMaxDevices) return DFSSM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    DeviceSetup& s = g_setup[dev];
    if (!s.ready) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return DFSSM_ERR_CUDA;
        int optin = 0;
        if (cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            set_quant_attr(optin) != cudaSuccess || set_decode_attr(optin) != cudaSuccess)
            return DFSSM_ERR_CUDA;
        s.scratch = static_cast<uint8_t*>(ptr);
        s.ready = true;
    }
    *out = &s;
    return DFSSM_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// the linear's descriptor into the scratch (kernel arguments are passed by value)
__global__ void noalloc_set_desc(DevDesc* dst, const DevDesc v) { *dst = v; }

}  // namespace
}  // namespace dfssm

using namespace dfssm;

extern "C" dfssm_status dfssm_linear_fwd_noalloc(const dfssm_linear_desc* desc, const dfssm_linear_weights* w,
                                                 const void* x, int32_t m, void* y, void* stream) {
    if (!desc || !w || !x || !y || !aligned16(x) || !aligned16(y)) return DFSSM_ERR_INVALID_ARG;
    const void* wp[6] = {w->sign, w->alpha, w->wa, w->sa, w->wb, w->sb};
    for (const void* p : wp)
        if (!p || !aligned16(p)) return DFSSM_ERR_INVALID_ARG;
    if (desc->y_dtype != DFSSM_BF16 && desc->y_dtype != DFSSM_F32) return DFSSM_ERR_INVALID_ARG;
    if (desc->flags != 0 || m < 1) return DFSSM_ERR_INVALID_ARG;
    // sizes beyond the fixed scratch are refused
    if (desc->rank != kRank || desc->d_in < 128 || desc->d_in > kMaxDIn || desc->d_in % 128 != 0 ||
        desc->d_out < 1 || desc->d_out > (1 << 20) || m > kNoAllocMaxM)
        return DFSSM_ERR_UNSUPPORTED_SHAPE;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DFSSM_ERR_CUDA;
    DeviceSetup* s = nullptr;
    dfssm_status st = setup_device(dev, &s);
    if (st != DFSSM_OK) return st;

    DevDesc hd;
    std::memset(&hd, 0, sizeof(hd));
    hd.d_in = desc->d_in;
    hd.d_out = desc->d_out;
    hd.y_dtype = desc->y_dtype;
    hd.max_m = kNoAllocMaxM;
    hd.qrow = seg_qrow(desc->d_in);
    DevDesc* ddesc = reinterpret_cast<DevDesc*>(s->scratch + kOffDesc);
    noalloc_set_desc<<<1, 1, 0, (cudaStream_t)stream>>>(ddesc, hd);
    if (cudaGetLastError() != cudaSuccess) return DFSSM_ERR_CUDA;

    LaunchCtx c{};
    c.entries = nullptr;
    c.single.w = *w;
    c.single.x = x;
    c.single.y = y;
    c.single.desc_index = 0;
    c.n = 1;
    c.m = m;
    c.desc = ddesc;
    c.host_desc = &hd;
    c.q_ws = nullptr;     // the decode kernel quantises into shared memory; no activation rows are stored
    c.st_ws = nullptr;     // the decode path reads only the split partials
    c.err = reinterpret_cast<uint32_t*>(s->scratch + kOffErr);
    c.part = reinterpret_cast<int*>(s->scratch + kOffPart);
    c.tmaps = nullptr;
    c.wait_limit_ns = kWaitLimitNs;
    c.max_d_in = desc->d_in;
    c.total_rows = desc->d_out;
    c.sm_count = s->sm_count;
    c.stream = (cudaStream_t)stream;
    if (launch_quant(c) != cudaSuccess) return DFSSM_ERR_CUDA;
    if (launch_decode(c) != cudaSuccess) return DFSSM_ERR_CUDA;
    return DFSSM_OK;
}
