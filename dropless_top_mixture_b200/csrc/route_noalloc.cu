// moe_route_noalloc: the route step with its scratch memory owned by the
// library, for callers that cannot allocate device memory.
//
// Who needs it: code that runs where no allocator is available or allowed —
// for example an enqueue callback of a host framework that hands over only
// input/output pointers and a stream, or a serving loop whose memory pool has
// reserved the device and where a cudaMalloc would synchronise the device or
// fail. moe_route needs a caller-provided workspace; this variant needs none.
//
// The scratch is one file-scope device array of MOE_ROUTE_NOALLOC_SCRATCH_BYTES
// (8 MiB). Every GPU that loads this library keeps that much memory reserved
// until the process exits. Host code cannot use the array's name as a device
// address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it; later calls
// on that device reuse the cached address.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace noalloc {

static __device__ __align__(256) unsigned char g_route_scratch[MOE_ROUTE_NOALLOC_SCRATCH_BYTES];

// Device address of g_route_scratch on the current device, or nullptr if the
// lookup failed. Looked up once per device.
static void* scratch_address() {
    static void* cached[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cached[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
        cached[dev] = p;
    }
    return cached[dev];
}

}  // namespace noalloc
}  // namespace moe

using namespace moe;

extern "C" int moe_route_noalloc(const float* logits, const void* x, const void* Wr, int dtype,
                                 int64_t T, int64_t d, int64_t E, int k, int renorm,
                                 float* logits_out, int32_t* idx, float* gate, int32_t* counts,
                                 int32_t* offsets, int32_t* slot, int32_t* tile_offsets,
                                 void* stream) {
    if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID;
    const int from_x = (logits == nullptr && T > 0) ? 1 : 0;
    const size_t need = moe_route_workspace_size(T, E, from_x);
    if (need > (size_t)MOE_ROUTE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
    void* scratch = noalloc::scratch_address();
    if (!scratch) return MOE_ERR_CUDA;
    // The existing route kernels run unchanged on the library-owned scratch.
    // They never read scratch they did not write in the same call, and the one
    // word that must start at zero (the scan's completion counter) is cleared
    // on the stream before use, so leftovers of an earlier call do no harm.
    return moe_route(logits, x, Wr, dtype, T, d, E, k, renorm, logits_out, idx, gate, counts,
                     offsets, slot, tile_offsets, scratch, (size_t)MOE_ROUTE_NOALLOC_SCRATCH_BYTES,
                     stream);
}
