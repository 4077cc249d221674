// scan_noalloc.cu -- ramnet_scan_forward_noalloc: the prefill scan with its scratch in a
// fixed array that is part of the library's device image, for callers that cannot hand
// over device memory of their own.
//
// Who needs it: a caller with no device allocator at hand (plain C host code that links
// this library and owns only the tensors it passes in), or a caller that must not allocate
// on its hot path because an allocation may block on the driver or fail part way through a
// run.  Such a caller cannot provide the `workspace` that ramnet_scan_forward requires.
//
// How: the scratch is `g_scan_scratch`, a file-scope static device array of
// RAMNET_NOALLOC_SCRATCH_BYTES bytes, 256-byte aligned.  The first call on a device (that
// device being current) looks up the array's device address with cudaGetSymbolAddress
// and caches it together with the identity of the current CUDA context; later calls in the
// same context reuse the cached address, and a call in a new context (after a device reset,
// or once the primary context was destroyed and created again, which reloads the module)
// looks it up again.  The call then runs the same route and scan kernels as
// ramnet_scan_forward with that address as the workspace.  Nothing here, or in what it
// calls, allocates device or host memory.
//
// Contents: nothing in the array has to start at zero.  Each call writes every event the
// scan reads (event decode) and resets the read accumulator itself before the scan adds
// into it.
//
// Sharing: there is one array per device and per loaded copy of the library.  Two calls
// whose kernels can be in flight at the same time (different streams, or different host
// threads each with its own stream) use the same array and race; issue such calls on one
// stream, one after the other, or use ramnet_scan_forward with separate workspaces.
#include <cstdio>
#include <mutex>

#include "../../include/ramnet.h"

namespace {

static __device__ __align__(256) unsigned char g_scan_scratch[RAMNET_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;

struct CachedScratch {
    void* addr;
    unsigned long long ctx_id;  // context the address belongs to (0: unknown)
};
CachedScratch g_scratch[kMaxDevices] = {};

// Identity of the calling thread's current CUDA context (driver entry points resolved
// through the runtime, so the library does not link the driver library itself).  False if
// there is no current context or the driver does not provide the calls.
bool current_context_id(unsigned long long* id)
{
    using GetCurrent = int (*)(void**);
    using GetId = int (*)(void*, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess && cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) ==
                                                     cudaSuccess && q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        resolved = true;
    }
    if (get_current == nullptr || get_id == nullptr) return false;
    void* ctx = nullptr;
    if (get_current(&ctx) != 0 || ctx == nullptr) return false;
    return get_id(ctx, id) == 0 && *id != 0;
}

}  // namespace

namespace ramnet {
// error text for ramnet_last_error (defined with the rest of the ABI)
ramnet_status set_last_error(ramnet_status s, const char* msg);
}  // namespace ramnet

extern "C" ramnet_status ramnet_scan_forward_noalloc(const ramnet_config* cfg, int32_t B, int32_t T, int32_t H,
                                                     ramnet_dtype in_dt, const void* k_logits,
                                                     const void* q_logits, const void* v, const void* g,
                                                     const void* z, const float* norm_w, const uint8_t* cape_mask,
                                                     const int32_t* pos0, const float* S_in, const float* m_in,
                                                     void* y, ramnet_dtype out_dt, float* S_out, float* m_out,
                                                     void* stream)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ramnet::set_last_error(RAMNET_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return ramnet::set_last_error(RAMNET_ERR_UNSUPPORTED, "scan_forward_noalloc: device ordinal above 63");
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        unsigned long long id = 0;
        const bool have_id = current_context_id(&id);
        CachedScratch& cs = g_scratch[dev];
        if (cs.addr == nullptr || !have_id || cs.ctx_id != id) {
            void* addr = nullptr;
            e = cudaGetSymbolAddress(&addr, g_scan_scratch);
            if (e != cudaSuccess || addr == nullptr)
                return ramnet::set_last_error(RAMNET_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                                                 : "static scratch has no address");
            // the lookup makes the device's context current if there was none yet
            unsigned long long id2 = 0;
            cs.addr = addr;
            cs.ctx_id = current_context_id(&id2) ? id2 : 0ull;
        }
        scratch = cs.addr;
    }
    // 0 means invalid arguments: ramnet_scan_forward reports which one
    const size_t need = ramnet_scan_workspace_bytes(cfg, B, T, H);
    if (need > RAMNET_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "scan_forward_noalloc: these sizes need %zu bytes of scratch, the static scratch holds %zu; "
                 "use ramnet_scan_forward with a workspace",
                 need, static_cast<size_t>(RAMNET_NOALLOC_SCRATCH_BYTES));
        return ramnet::set_last_error(RAMNET_ERR_UNSUPPORTED, msg);
    }
    return ramnet_scan_forward(cfg, B, T, H, in_dt, k_logits, q_logits, v, g, z, norm_w, cape_mask, pos0, S_in,
                               m_in, y, out_dt, S_out, m_out, scratch, RAMNET_NOALLOC_SCRATCH_BYTES, stream);
}
