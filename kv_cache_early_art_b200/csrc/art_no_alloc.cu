// art_no_alloc.cu -- art_decode_attention_no_alloc: the workspace walk
// (merge_cta = 2) with its scratch in a fixed device array of this library,
// for callers that cannot allocate device memory.
//
// The array is zero when the library's device code is loaded onto a GPU and
// then keeps whatever the last call left in it.  Nothing in it has to start
// at zero: every control word the walk reads (merged counts, fetch counts,
// ready tags) carries a 32-bit tag of the call that wrote it, so words an
// earlier call left behind never read as this call's; the block states are
// written before they are read.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/art.h"
#include "art_host.h"

namespace {

static __device__ __align__(256) unsigned char g_art_scratch[ART_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_art_scratch, per device; null until set up

// The device address of the scratch array on the current device.  In host
// code g_art_scratch names a host-side stand-in, so the address is asked of
// the runtime, once per device, with that device current.
art_status_t scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return ART_ERR_LAUNCH;
    }
    if (dev < 0 || dev >= kMaxDevices)
        return ART_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_art_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return ART_ERR_LAUNCH;
        }
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return ART_OK;
}

}  // namespace

extern "C" art_status_t art_decode_attention_no_alloc(const art_params_t *p, art_stream_t stream)
{
    if (!p)
        return ART_ERR_NULL;
    if (p->workspace || p->workspace_bytes || (p->merge_cta != 0 && p->merge_cta != 2))
        return ART_ERR_PARAM;
    art_params_t q = *p;
    q.merge_cta = 2;
    const int64_t need = art_host::gr_min_workspace_bytes(&q);
    if (need < 0)
        return static_cast<art_status_t>(need);
    if (need == 0)
        return ART_ERR_UNSUPPORTED;
    if (need > (int64_t)ART_NO_ALLOC_SCRATCH_BYTES)
        return ART_ERR_SCRATCH_SIZE;
    void *scratch = nullptr;
    art_status_t st = scratch_address(&scratch);
    if (st != ART_OK)
        return st;
    q.workspace = scratch;
    q.workspace_bytes = ART_NO_ALLOC_SCRATCH_BYTES;
    return art_decode_attention_ex(&q, stream);
}
