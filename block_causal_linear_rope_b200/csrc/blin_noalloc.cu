// blin_prefill_static: blin_prefill for callers that cannot allocate device
// memory.  Some callers have no device allocator of their own, for instance a
// plugin loaded into a host framework that owns all device memory and hands
// out no scratch buffers, so they cannot provide the workspace blin_prefill
// needs.  This entry point uses a fixed scratch area that lives in the
// library's own device memory instead and allocates nothing.
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/blin.h"
#include "blin_internal.cuh"

namespace {

// Upper bound of the workspace this entry point can serve (see the header).
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB

// The scratch area.  Every GPU that loads the library holds it until the
// process exits, and every call on that GPU shares it.
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch in each CUDA context.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress with that context current.  A module's device variables
// exist once per context (not once per device ordinal): a host framework may
// make a context of its own current, and cudaDeviceReset replaces the primary
// context, so the cache is keyed by the context's unique id.
blin::ContextCache<void *> g_scratch_addr;

blin_status scratch_for_current_context(void **out, char *msg, size_t msg_len) {
    const unsigned long long ctx = blin::current_context_id();
    if (ctx == 0) {
        snprintf(msg, msg_len, "no CUDA context is current (or the driver cannot name it)");
        return BLIN_ERR_CUDA;
    }
    void *p = nullptr;
    if (g_scratch_addr.get(ctx, &p)) {
        *out = p;
        return BLIN_OK;
    }
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) {
        snprintf(msg, msg_len, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
        return BLIN_ERR_CUDA;
    }
    g_scratch_addr.put(ctx, p);
    *out = p;
    return BLIN_OK;
}

}  // namespace

extern "C" {

size_t blin_prefill_static_capacity(void) { return kStaticScratchBytes; }

blin_status blin_prefill_static(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B,
                                int H, int d, const blin_geom *g, blin_state *st, blin_stream stream) {
    if (g == nullptr) return blin_prefill(q, k, v, o, dt, B, H, d, g, st, nullptr, 0, stream);  // reports it
    char msg[256];
    const size_t need = blin_prefill_workspace_size(B, H, d, g);
    if (need == 0)  // an invalid shape: blin_prefill rejects it with its own message
        return blin_prefill(q, k, v, o, dt, B, H, d, g, st, nullptr, 0, stream);
    if (need > kStaticScratchBytes) {
        // A clear error instead of a silent overrun: the shape needs more than
        // the fixed scratch area holds.
        snprintf(msg, sizeof msg,
                 "blin_prefill_static: this shape needs %zu bytes of scratch, the static area holds %zu; "
                 "use blin_prefill with a caller-provided workspace",
                 need, kStaticScratchBytes);
        return blin::set_last_error(BLIN_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    const blin_status rc = scratch_for_current_context(&scratch, msg, sizeof msg);
    if (rc != BLIN_OK) return blin::set_last_error(rc, msg);
    return blin_prefill(q, k, v, o, dt, B, H, d, g, st, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
