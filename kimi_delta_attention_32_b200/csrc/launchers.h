// launchers.h -- host-side launch entry points of the libkda kernels (internal).
// Arguments are validated by api.cu before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

enum class Io { F32 = 0, BF16 = 1 };

struct ConvArgs {
    const void* x[3];        // q_raw, k_raw, v_raw
    const float* w[3];       // [H*d, K]
    void* y[3];              // outputs
    void* conv_state;        // [N, H*(2dk+dv), K-1] or null
    const int32_t* cu;       // device cu_seqlens or null (padded)
    int64_t T_tot;
    int T_pad;               // tokens per sequence when cu == null
    int N, H, dk, dv;
    float eps;
    Io io;
};
cudaError_t launch_conv(const ConvArgs& a, cudaStream_t stream);

struct StepArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    float scale;
    float* state;
    void* o;
    int N, H, dk, dv;
    Io io;
};
cudaError_t launch_recurrent_step(const StepArgs& a, cudaStream_t stream);

struct ChunkArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    float scale;
    const float* h0;
    float* ht;
    void* o;
    const int32_t* cu;       // device cu_seqlens or null (padded)
    const int32_t* cu_host;  // host copy or null (padded)
    int64_t T_tot;
    int T_pad;
    int N, H, dk, dv, chunk;
    Io io;
};
cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream);

// Tensor-core (tcgen05) prefill: bf16 I/O, dk = dv = 128, chunk 64.
bool chunk_tc_supported(const ChunkArgs& a);
cudaError_t launch_chunk_tc(const ChunkArgs& a, unsigned int* err, cudaStream_t stream);
// Same math as a producer/consumer pipeline in one 4-CTA cluster per (sequence, head). Needs a
// device workspace of chunk_tcx_workspace_bytes() (16-byte aligned): the per-SM hand-off rings.
size_t chunk_tcx_workspace_bytes();
cudaError_t launch_chunk_tcx(const ChunkArgs& a, void* workspace, size_t workspace_bytes,
                             unsigned int* err, cudaStream_t stream);

}  // namespace kda
