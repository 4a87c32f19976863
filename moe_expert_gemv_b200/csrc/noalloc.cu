// noalloc.cu -- moe_expert_qmlp for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory for a workspace: code that
// runs where allocation is forbidden or unavailable (a plugin or embedded
// runtime handed only a stream and tensor pointers, a host framework whose
// memory pool may not be touched from the calling thread, a real-time path
// that must not call into the allocator).  For them the library carries its
// own scratch buffer: a file-scope __device__ array that every GPU loading the
// library holds until the process exits.
//
// The kernels see the buffer through its device address, which host code
// obtains with cudaGetSymbolAddress (the array's name in host code is only a
// host-side stand-in).  The address is looked up on every call, with the
// device that is current at the call, so a new context (after a device reset)
// or another current device gets its own address; nothing is cached.  Only
// the arrival counters must start at zero; every call checks all of its
// arguments first and only then clears them on the stream.  All calls share
// the one buffer, so calls that overlap on the GPU (two streams, or two
// devices' worth of work issued to the same device at once) race and must be
// avoided.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {
namespace {

// Maximum scratch: 1 MiB covers top_k <= 16 with hidden <= 8192 and
// inter <= 4096 (and the decode layer of hidden 2816 / inter 704 many times).
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current device's context.
qmoe_status noalloc_scratch(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
        return QMOE_ERR_CUDA;
    *out = p;
    return QMOE_OK;
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

extern "C" qmoe_status moe_expert_qmlp_noalloc(const qmoe_moe_layer *L, const uint16_t *x,
                                               const int32_t *idx, const float *weights,
                                               int32_t top_k, uint16_t *y, int32_t *status_dev,
                                               void *stream)
{
    // every argument check first: a rejected call enqueues nothing on the
    // stream, so it cannot clear the counters of a call still in flight
    qmoe_status s = validate_expert_qmlp(L, x, idx, weights, top_k, y, status_dev);
    if (s != QMOE_OK)
        return s;
    const size_t need = moe_expert_workspace_bytes(L, top_k);
    if (need == 0)
        return QMOE_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes)
        return QMOE_ERR_WORKSPACE;   // beyond the built-in scratch: use moe_expert_qmlp
    void *scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != QMOE_OK)
        return s;
    ExpertWorkspace ws;
    expert_workspace_layout(L->hidden, L->inter, top_k, scratch, &ws);
    if (cudaMemsetAsync(ws.counters, 0, (size_t)(L->hidden / 16) * sizeof(int32_t),
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return QMOE_ERR_CUDA;
    return moe_expert_qmlp(L, x, idx, weights, top_k, y, scratch, need, status_dev, stream);
}
