// gdn_noalloc.cu -- gdn_forward_noalloc: the GDN forward for callers that
// cannot allocate device memory themselves.
//
// gdn_forward needs a caller-provided device workspace for its intermediates
// (prepared q/k/v, gates, per-block UT operands, per-segment states).  Some
// callers have no way to get one: code that runs where cudaMalloc is not
// allowed or not wanted -- inside a host callback or another library's
// allocation-free hot loop, a process whose memory pool is fully reserved by
// a framework that does not lend it out, or a plugin ABI that hands over only
// input and output pointers.  For them this entry point takes its workspace
// from one fixed array that lives in this library's device image: it calls no
// cudaMalloc/cudaFree and no allocating library routine.
//
// The array has a fixed maximum size (GDN_NOALLOC_SCRATCH_BYTES); every GPU
// that loads the library holds it until the process exits.  Plans whose
// workspace does not fit are rejected before anything is enqueued.  All calls
// on a device share the one array, so calls whose work may overlap on the GPU
// (different streams without ordering, or host threads) race on it; calls on
// one stream are ordered and safe.  The array keeps the last call's contents:
// the forward itself zeroes the only value that must start at zero (the
// device status word) at the start of each call.
//
// In host code the array's name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress and cached per device together
// with the unique id of the CUDA context it belongs to.  A later call in another
// context (after cudaDeviceReset, or from a thread with another context current)
// sees a different id and looks the address up again, since the array's address
// in a new context need not be the old one.  The first call on a device, and the
// first after a reset, should come before any stream capture.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_gdn_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
    unsigned long long ctx_id;  // cuCtxGetId of the context `ptr` belongs to
    void *ptr;                  // nullptr: not looked up in any context yet
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array in the current device's current context.
gdn_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    unsigned long long id = 0;
    bool have_id = gdn::current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchEntry &e = g_scratch[dev];
    if (have_id && e.ptr && e.ctx_id == id) {
        *out = e.ptr;
        return GDN_OK;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gdn_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
    }
    if (!have_id) have_id = gdn::current_context_id(&id);  // the lookup made the device's context current
    e.ctx_id = have_id ? id : 0;
    e.ptr = have_id ? p : nullptr;                      // without an id nothing is cached
    *out = p;
    return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_forward_noalloc(gdn_plan_t plan, const gdn_inputs *in, void *y, gdn_stream_t stream) {
    if (!plan || !in || !y) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::plan_workspace_bytes(plan);
    if (need > static_cast<size_t>(GDN_NOALLOC_SCRATCH_BYTES)) return GDN_ERR_UNSUPPORTED;
    void *ws = nullptr;
    const gdn_status st = scratch_address(&ws);
    if (st != GDN_OK) return st;
    return gdn_forward(plan, in, y, ws, stream);
}
