// gdn_noalloc.cu -- gdn_chunk_forward for callers that cannot allocate.
//
// Some callers have no way to obtain device memory for a workspace: a
// plugin inside a host runtime that hands it only the tensors' pointers and
// no allocator, or serving code whose memory is fixed up front and which
// must not call cudaMalloc on the request path (cudaMalloc can synchronise
// the device and stall every stream).  For them this file keeps the
// prefill's scratch (the schedule tables and the status word) in a fixed
// device array that the library owns, so the call needs only inputs and
// outputs.
//
// The array lives in every GPU that loads the library, for the life of the
// process, and is shared by all calls on that device: calls that overlap on
// the GPU (different streams, or host threads racing) overwrite each
// other's scratch and give wrong results.  Each call re-initialises what it
// needs (the schedule kernel rewrites the tables, the status word and the
// work counter before the prefill kernel reads them), so stale contents from
// an earlier call do no harm.
#include <cstdio>

#include "gdn_internal.cuh"

namespace gdn {

// Scratch of the prefill schedule for up to kNoAllocMaxSeqs sequences:
// a 256-byte header plus three int32 tables of that length.
constexpr int32_t kNoAllocMaxSeqs = 16384;
constexpr size_t kNoAllocScratchBytes = 256 + 3 * 4 * size_t(kNoAllocMaxSeqs);
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the current device's context,
// looked up on every call with that device current.  The host-side symbol is
// only a stand-in and must never be passed to a kernel; and an address kept
// from an earlier call could belong to another context (after
// cudaDeviceReset the module is loaded anew, and a caller's own driver-API
// context holds its own instance of the module), so nothing is cached.  The
// lookup is a host-side query (no synchronisation); the first one in a
// context may load the library's device code.
static cudaError_t scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace gdn

extern "C" GDN_API gdn_status_t gdn_chunk_forward_noalloc(const gdn_shape_t *shape, const void *q, const void *k,
                                                          const void *v, const float *g, const float *beta,
                                                          const float *initial_state, const int32_t *cu_seqlens,
                                                          void *o, float *final_state, void *stream) {
    using namespace gdn;
    if (shape && shape->num_seqs > kNoAllocMaxSeqs) {
        char msg[160];
        snprintf(msg, sizeof(msg),
                 "gdn_chunk_forward_noalloc handles at most %d sequences per call (got %d); "
                 "use gdn_chunk_forward with a caller-allocated workspace",
                 int(kNoAllocMaxSeqs), int(shape->num_seqs));
        return set_error(GDN_ERR_UNSUPPORTED, msg);
    }
    void *scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof(msg), "resolving the device address of the built-in scratch array failed: %s",
                 cudaGetErrorString(e));
        return set_error(GDN_ERR_CUDA, msg);
    }
    // the single-kernel path: its scratch is the schedule tables alone
    if (!shape) return gdn_chunk_forward(shape, q, k, v, g, beta, initial_state, cu_seqlens, o, final_state,
                                         scratch, kNoAllocScratchBytes, stream);
    gdn_shape_t one = *shape;
    one.flags |= GDN_FLAG_ONE_KERNEL;
    return gdn_chunk_forward(&one, q, k, v, g, beta, initial_state, cu_seqlens, o, final_state, scratch,
                             kNoAllocScratchBytes, stream);
}

extern "C" GDN_API gdn_status_t gdn_noalloc_read_device_status(int32_t *device_status, void *stream) {
    using namespace gdn;
    if (!device_status) return set_error(GDN_ERR_INVALID_ARGUMENT, "device_status is NULL");
    void *scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof(msg), "resolving the device address of the built-in scratch array failed: %s",
                 cudaGetErrorString(e));
        return set_error(GDN_ERR_CUDA, msg);
    }
    // the array starts with the same header a caller's workspace does
    return gdn_read_device_status(scratch, device_status, stream);
}
