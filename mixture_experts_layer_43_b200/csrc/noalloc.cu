// noalloc.cu -- moe_route_noalloc: the decode-regime routing step for
// callers that must not allocate device memory.
//
// Some host programs cannot call cudaMalloc when they want to route a batch:
// an engine that hands the library only pre-planned memory and forbids
// allocations on its serving path, a plugin interface whose enqueue step may
// only launch work, or code that runs where the allocator is locked.  For them
// this entry point needs no plan: the router kernel's scratch (fp32 logits,
// the last-CTA ticket, the work list, the slot-token map, the error word)
// lives in the file-scope device array below instead of a plan workspace.
// The caller still passes every input and output.
//
// The array is a module global: every GPU that loads the library holds its
// own copy (kNoAllocScratchBytes) until the process exits, and every call on
// that GPU shares it.  The ticket is cleared before each launch; the error
// word is sticky until moe_route_noalloc_status reads it; the rest is fully
// rewritten by each call, so the array keeps only the last call's contents.
// Two calls whose work overlaps on the GPU (other streams, other threads)
// race on the array and must be serialised by the caller.
//
// The array's device address is resolved once per CUDA context (the first
// call in a context, with its device current) and cached with the context's
// id: after a cudaDeviceReset, or in another context on the same device, the
// module global lives at a different address, and the cache is refreshed.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

constexpr size_t kNoAllocScratchBytes = 64 * 1024;

static __device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

struct NoAllocDevice {
    bool ready = false;
    unsigned long long ctx_id = 0;  // CUDA context the address below belongs to
    uint8_t* scratch = nullptr;     // device address of g_route_scratch in that context
    int num_sms = 0;
};

std::mutex g_mu;
NoAllocDevice g_dev[kMaxDevices];

// Scratch layout (byte offsets into g_route_scratch).
constexpr size_t kOffLogits = 0;                                             // [8][1024] f32
constexpr size_t kOffSlotTok = kOffLogits + 4ull * kDecodeTok * kMaxExperts;  // [128] i32
constexpr size_t kOffSlotW = kOffSlotTok + 4ull * kDecodeTok * kMaxTopK;      // [128] f32
constexpr size_t kOffItems = kOffSlotW + 4ull * kDecodeTok * kMaxTopK;        // [E+S] items
constexpr size_t kOffNItems = kOffItems + sizeof(WorkItem) * (kMaxExperts + kMaxShared);
constexpr size_t kOffTicket = kOffNItems + 16;
constexpr size_t kOffErr = kOffTicket + 16;
constexpr size_t kScratchUsed = kOffErr + 16;
static_assert(kScratchUsed <= kNoAllocScratchBytes, "scratch layout exceeds the array");

// Id of the calling thread's current CUDA context, through the driver entry
// points (the library links no driver stub).  0 when it cannot be read.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1{}, q2{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        cudaGetLastError();
        resolved = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// First call in a context (its device current): resolve the array's device
// address and the SM count.  Neither allocates.  A context id that cannot be
// read (0) resolves the address again on every call.
moe_status_t setup_device(int dev, NoAllocDevice** out) {
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    NoAllocDevice& d = g_dev[dev];
    const unsigned long long ctx = current_context_id();
    if (!d.ready || ctx == 0 || ctx != d.ctx_id) {
        d.ready = false;
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        d.scratch = static_cast<uint8_t*>(ptr);
        d.num_sms = sms;
        d.ctx_id = ctx;
        d.ready = true;
    }
    *out = &d;
    return MOE_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_route_noalloc(const moe_config_t* cfg, const moe_weights_t* w,
                                          const void* x, int32_t T, float* out,
                                          moe_routing_t* routing, void* stream) {
    if (!cfg || !w || !routing) return MOE_ERR_INVALID_ARG;
    const int d = cfg->d_model, E = cfg->n_experts, k = cfg->top_k, S = cfg->n_shared;
    if (d < 128 || d % 128 != 0 || E < 1 || E > kMaxExperts || k < 1 || k > E ||
        k > kMaxTopK || S < 0 || S > kMaxShared)
        return MOE_ERR_INVALID_ARG;
    // the scratch holds at most MOE_DECODE_MAX_T tokens
    if (T < 0 || T > MOE_DECODE_MAX_T) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !out || !al16(x) || !al16(out) || !w->router_w || !al16(w->router_w))
        return MOE_ERR_INVALID_ARG;
    if (w->router_b && (reinterpret_cast<uintptr_t>(w->router_b) & 3u)) return MOE_ERR_INVALID_ARG;
    if (!routing->ids || !routing->weights || !routing->counts || !routing->offsets ||
        !routing->slot_pair)
        return MOE_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    NoAllocDevice* nd = nullptr;
    moe_status_t s = setup_device(dev, &nd);
    if (s) return s;

    uint8_t* sc = nd->scratch;
    RouteArgs r{};
    r.x = static_cast<const uint16_t*>(x);
    r.wr = w->router_w;
    r.br = w->router_b;
    r.out = out;
    r.ws.logits = reinterpret_cast<float*>(sc + kOffLogits);
    r.ws.ids = routing->ids;
    r.ws.wts = routing->weights;
    r.ws.counts = routing->counts;
    r.ws.offsets = routing->offsets;
    r.ws.slot_pair = routing->slot_pair;
    r.ws.slot_token = reinterpret_cast<int32_t*>(sc + kOffSlotTok);
    r.ws.slot_w = reinterpret_cast<float*>(sc + kOffSlotW);
    r.ws.items = reinterpret_cast<WorkItem*>(sc + kOffItems);
    r.ws.n_items = reinterpret_cast<int32_t*>(sc + kOffNItems);
    r.ws.ticket = reinterpret_cast<uint32_t*>(sc + kOffTicket);
    r.ws.err = reinterpret_cast<uint32_t*>(sc + kOffErr);
    r.T = T;
    r.d = d;
    r.E = E;
    r.k = k;
    r.S = S;
    int epc = 1;
    while (epc < 8 && (E + epc - 1) / epc > nd->num_sms) epc *= 2;
    r.experts_per_cta = epc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the last-CTA ticket must start at zero (the error word stays sticky)
    if (cudaMemsetAsync(sc + kOffTicket, 0, 16, st) != cudaSuccess) return MOE_ERR_CUDA;
    return launch_decode_route(r, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_route_noalloc_status(void) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    NoAllocDevice* nd = nullptr;
    moe_status_t s = setup_device(dev, &nd);
    if (s) return s;
    uint32_t v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(&v, nd->scratch + kOffErr, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (v && cudaMemset(nd->scratch + kOffErr, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
    return v ? MOE_ERR_DEVICE_FLAG : MOE_OK;
}
