// noalloc.cu -- kda_chunk_fwd_noalloc: the chunked prefill with its workspace taken from a
// device array that the library itself owns, so that the caller allocates nothing.
//
// The tensor-core prefill hands each chunk's operands from its producer CTAs to its consumer
// CTA through per-SM rings in global memory (the workspace that kda_chunk_fwd takes from its
// caller). Here that memory is a file-scope __device__ array, reserved when the module is
// loaded; its address comes from cudaGetSymbolAddress on the current device. The array is one
// per device and process: calls on one device must not run concurrently (the same rule as for
// one caller-owned workspace).
#include "kda.h"

#include <stdint.h>

#define KDA_API extern "C" __attribute__((visibility("default")))

namespace {
// Ring tables for 160 SM ids x 6 slots x 58368 bytes: what kda_chunk_fwd_workspace_size reports
// for the bf16, dk = dv = 128, chunk-64 prefill (checked at every call).
constexpr size_t kStaticWorkspaceBytes = (size_t)160 * 6 * 58368;
__device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];
}  // namespace

KDA_API kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                         const float* beta, float scale, const float* h0, float* ht,
                                         void* o, const int32_t* cu_seqlens,
                                         const int32_t* cu_seqlens_host, int B, int T, int N, int H,
                                         int dk, int dv, int chunk, kda_io_dtype io, void* stream) {
    size_t need = 0;
    int64_t T_tot = (int64_t)B * T;
    const kda_status qs = kda_chunk_fwd_workspace_size(N > 0 ? N : B, T_tot, H, dk, dv, chunk, io, &need);
    if (qs != KDA_OK) return qs;
    if (need > kStaticWorkspaceBytes) return KDA_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0 && cudaGetSymbolAddress(&ws, g_static_workspace) != cudaSuccess) {
        // no device array to use: argument errors still take precedence, as in kda_chunk_fwd
        const kda_status s = kda_chunk_fwd(q, k, v, g, beta, scale, h0, ht, o, cu_seqlens,
                                           cu_seqlens_host, B, T, N, H, dk, dv, chunk, io, nullptr,
                                           0, stream);
        return (s == KDA_ERR_INVALID_ARG || s == KDA_ERR_UNSUPPORTED) ? s : KDA_ERR_CUDA;
    }
    return kda_chunk_fwd(q, k, v, g, beta, scale, h0, ht, o, cu_seqlens, cu_seqlens_host, B, T, N, H,
                         dk, dv, chunk, io, ws, need > 0 ? kStaticWorkspaceBytes : 0, stream);
}
