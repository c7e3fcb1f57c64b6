// noalloc.cu -- kda_chunk_fwd_noalloc: the chunked prefill with its scratch memory taken from a
// device array that the library owns, so that the call allocates nothing.
//
// Who needs it: a caller that cannot call cudaMalloc at the point where it runs the prefill.
// Examples are a serving runtime whose memory pool has already reserved all free device memory,
// a plug-in that is handed only tensor pointers and no allocator, and a latency-critical path
// where cudaMalloc's implicit device-wide synchronisation is not acceptable. kda_chunk_fwd asks
// such a caller for a ~72 MB workspace; this entry point uses a file-scope __device__ array of
// that size instead.
//
// The tensor-core prefill hands each chunk's operands from its producer CTAs to its consumer CTA
// through per-SM rings in global memory: that is the scratch memory. The ring carries no state
// from one call to the next (every slot is written before it is read, and the flags live in
// shared memory), so nothing needs clearing between calls.
//
// The array's name in host code is only a host-side stand-in, not a device address, so the
// address is looked up once per device with cudaGetSymbolAddress (with that device current) and
// cached. The first call on a device does this set-up; make that first call before any stream
// capture. The array is one per device and process, and every GPU that loads the library holds
// it until the process exits (with CUDA's lazy module loading it is reserved when this module is
// first used on the device). Calls that overlap on the GPU race on the array: run them on one
// stream, or otherwise one after another.
#include "kda.h"

#include <mutex>
#include <stdint.h>

#include "launchers.h"

#define KDA_API extern "C" __attribute__((visibility("default")))

namespace {

// Maximum scratch of one call: the prefill's ring tables (160 SM ids x 6 slots x 74752 bytes).
constexpr size_t kStaticWorkspaceBytes = kda::kTcxWorkspaceBytes;
static_assert(kStaticWorkspaceBytes % 256 == 0, "array size");
static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_device_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device (looked up on first use), or null.
void* static_workspace() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_device_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess) return nullptr;
        g_device_ptr[dev] = p;
    }
    return g_device_ptr[dev];
}

}  // namespace

KDA_API kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                         const float* beta, float scale, const float* h0, float* ht,
                                         void* o, const int32_t* cu_seqlens,
                                         const int32_t* cu_seqlens_host, int B, int T, int N, int H,
                                         int dk, int dv, int chunk, kda_io_dtype io, void* stream) {
    // The scratch size depends only on the element type, head sizes and chunk length; every
    // other argument is checked by kda_chunk_fwd itself.
    size_t need = 0;
    const kda_status qs = kda_chunk_fwd_workspace_size(0, 0, 1, dk, dv, chunk, io, &need);
    if (qs != KDA_OK) return qs;
    if (need > kStaticWorkspaceBytes) return KDA_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0 && (ws = static_workspace()) == nullptr) {
        // no device array to use: argument errors still take precedence, as in kda_chunk_fwd
        const kda_status s = kda_chunk_fwd(q, k, v, g, beta, scale, h0, ht, o, cu_seqlens,
                                           cu_seqlens_host, B, T, N, H, dk, dv, chunk, io, nullptr,
                                           0, stream);
        return (s == KDA_ERR_INVALID_ARG || s == KDA_ERR_UNSUPPORTED) ? s : KDA_ERR_CUDA;
    }
    return kda_chunk_fwd(q, k, v, g, beta, scale, h0, ht, o, cu_seqlens, cu_seqlens_host, B, T, N, H,
                         dk, dv, chunk, io, ws, need > 0 ? kStaticWorkspaceBytes : 0, stream);
}
