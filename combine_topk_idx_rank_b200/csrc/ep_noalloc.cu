// ep_dispatch_noalloc: dispatch for callers that cannot allocate device memory.
//
// ep_dispatch needs a device workspace for its routing scratch (per-chunk
// histograms, column totals, the padding map and a grid-barrier counter).
// Some callers have no way to provide one: code that runs where cudaMalloc is
// not allowed or not wanted -- inside a region that must not allocate (for
// example while a memory pool is frozen or under a strict allocator that only
// hands out the tensors the caller already owns), plugins that receive only
// their input and output pointers from a host framework, or runtimes without
// an allocator of their own.  For them this file keeps the scratch in a
// static device array that exists for as long as the library is loaded, and
// forwards to ep_dispatch with that array as the workspace.
//
// Properties a caller must know:
//   - The array holds kScratchBytes (2 MiB) on every GPU that loads the
//     library, until the process exits.  Sizes whose scratch would not fit are
//     rejected with EP_ERR_INVALID_ARG and a message on stderr; nothing runs.
//   - The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it beside
//     the ID of the device's current CUDA context; make that first call
//     before any stream capture.  A later call in another context of that
//     device (after cudaDeviceReset, or with the primary context released
//     and created again) finds a different context ID and looks the address
//     up again, so a stale address from a destroyed context is never used;
//     that call, too, should come before any stream capture.
//   - All calls share the one array per device and it keeps the last call's
//     contents.  Dispatch rewrites every part of the scratch it reads in each
//     call (and clears its barrier counter itself), so nothing needs clearing
//     between calls -- but calls whose kernels overlap on the GPU (two
//     streams, or two host threads) race on the array and corrupt each other;
//     serialise them on one stream.
//   - No cudaMalloc, cudaFree or allocating library routine is called.
#include <cuda.h>   // CUcontext / CUresult types; the driver calls are resolved at run time
#include <mutex>
#include <stdio.h>

#include "ep_internal.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;   // 2 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_dispatch_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
struct ScratchAddr {
    unsigned long long ctx_id;   // ID of the context the address belongs to (0 = none yet)
    void* addr;                  // device address of g_dispatch_scratch in that context
};
ScratchAddr g_scratch[kMaxDevices] = {};

// Driver calls resolved through the runtime (the library links no driver
// library): the current context and its unique ID.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// ID of the context current on this thread, or 0 if there is none or the
// driver cannot say.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {   // called with g_scratch_mutex held
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        void* f1 = nullptr;
        void* f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f2);
        resolved = true;
    }
    if (get_current == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// The device address of the static scratch on the current device.  In host
// code `g_dispatch_scratch` names a host-side stand-in, not device memory, so
// the address must come from the runtime: it is looked up once per device and
// context, and again whenever the device's current context has changed.
ep_status_t scratch_on_current_device(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        fprintf(stderr, "libep: ep_dispatch_noalloc: cudaGetDevice failed (%s)\n", cudaGetErrorString(e));
        return EP_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return EP_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchAddr& c = g_scratch[dev];
    const unsigned long long id = current_context_id();
    if (c.addr == nullptr || id == 0 || id != c.ctx_id) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (e != cudaSuccess || p == nullptr) {
            fprintf(stderr, "libep: ep_dispatch_noalloc: cudaGetSymbolAddress failed on device %d (%s)\n", dev,
                    cudaGetErrorString(e));
            c.addr = nullptr;
            return EP_ERR_CUDA;
        }
        c.addr = p;
        c.ctx_id = current_context_id();   // the lookup makes the device's context current if it was not
    }
    *out = c.addr;
    return EP_OK;
}

}  // namespace

extern "C" ep_status_t ep_dispatch_noalloc(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                                           const float* topk_weights, int32_t K, int32_t E, int32_t R,
                                           const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                                           int32_t* recv_topk_idx, float* recv_topk_weights,
                                           int64_t recv_capacity, ep_handle_t* handle,
                                           int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                                           uint8_t* is_token_in_rank, void* stream) {
    const size_t need = ep_workspace_bytes(T, K, E, R);
    if (need == 0) return EP_ERR_INVALID_ARG;   // sizes ep_dispatch would reject
    if (need > kScratchBytes) {
        fprintf(stderr,
                "libep: ep_dispatch_noalloc: T=%d K=%d E=%d R=%d needs %zu bytes of scratch, more than its "
                "static maximum of %zu bytes; use ep_dispatch with a caller workspace\n",
                (int)T, (int)K, (int)E, (int)R, need, kScratchBytes);
        return EP_ERR_INVALID_ARG;
    }
    void* ws = nullptr;
    const ep_status_t s = scratch_on_current_device(&ws);
    if (s != EP_OK) return s;
    return ep_dispatch(x, T, H, topk_idx, topk_weights, K, E, R, opts, recv_x, recv_scales, recv_topk_idx,
                       recv_topk_weights, recv_capacity, handle, num_tokens_per_rank, num_tokens_per_expert,
                       is_token_in_rank, ws, kScratchBytes, stream);
}
