// k_select_noalloc.cu -- lsa_select_noalloc: the selection entry point for
// callers that cannot allocate device memory.
//
// Some callers have no way to obtain device scratch at the point where they
// select keys: a plug-in whose host only hands it input and output buffers, a
// serving loop whose device memory was divided up once at start-up by another
// runtime, or a host program that links this library but no device
// allocator.  lsa_select needs a caller workspace for its candidate lists and
// its exact-fallback scores; this variant keeps that scratch in one
// file-scope device array instead, so the caller passes only inputs and
// outputs.
//
// The array is a fixed-size part of the loaded module: every device that
// loads the library holds it until the process exits.  Its name is only a
// host-side stand-in in host code, so its device address is looked up with
// cudaGetSymbolAddress, once per device, on the first call made on that
// device (make that first call before any stream capture).  All calls share
// the array and it keeps the last call's contents: the candidate lists and
// the fallback scores are rewritten by every call, and the one value that
// must start at zero -- the fallback counter -- is zeroed by the first kernel
// of every call.  Calls that overlap on the GPU (different streams, or
// different host threads without ordering) race on the array.
#include <mutex>

#include "lsa_internal.cuh"

namespace lsa {

constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)8 << 20;   // 8 MiB

static __device__ __align__(256) unsigned char g_select_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_select_scratch on the current device (set-up on first use).
static cudaError_t noalloc_scratch(void** out)
{
    constexpr int MAXDEV = 64;
    static void* addr[MAXDEV] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAXDEV) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

size_t noalloc_scratch_bytes() { return NOALLOC_SCRATCH_BYTES; }

cudaError_t noalloc_select(const IndexView& ix, int64_t n_blk, const void* latent_Q,
                           const int32_t* positions, int64_t Nq, lsa_select_params sp,
                           int32_t* indices, int32_t* counts, int s_max, bool use_tc,
                           cudaStream_t st)
{
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
    const SelectWs ws = select_ws_carve(scratch, ix, Nq);
    return launch_select(ix, n_blk, latent_Q, PosSrc{positions, 0}, Nq, sp, indices, counts,
                         s_max, ws, use_tc, st);
}

}  // namespace lsa
