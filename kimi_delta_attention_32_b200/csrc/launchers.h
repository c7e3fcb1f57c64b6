// launchers.h -- host-side launch entry points of the libkda kernels (internal).
// Arguments are validated by api.cu before any of these is called.
#pragma once

#include <cuda_bf16.h>
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
// Only the cache update of the prefill form: conv_state <- the last K-1 raw inputs of each
// sequence's extended history (the cache followed by x).
cudaError_t launch_conv_cache(const ConvArgs& a, cudaStream_t stream);

struct StepArgs {
    const void *q, *k, *v;           // formed q, k, v, or the raw inputs when conv_state is set
    const float *g, *beta;
    float scale;
    float* state;
    void* o;
    int N, H, dk, dv;
    Io io;
    // conv prologue fused into the step (conv_state non-null): weights [H*d, 4], the width-3
    // history [N, H*(2dk+dv), 3] advanced in place, and the L2-norm epsilon of q and k
    const float* w[3] = {nullptr, nullptr, nullptr};
    void* conv_state = nullptr;
    float eps = 0.f;
    // gate from raw logits (A_log non-null): g_raw [N,H,dk] and beta_raw [N,H] in the io
    // dtype, A_log [H], dt_bias [H*dk]; then g and beta above are unused. Optional output
    // gated RMSNorm: z [N,H,dv] io dtype (null: none), w_norm [dv], norm_eps.
    const void* g_raw = nullptr;
    const void* beta_raw = nullptr;
    const float* A_log = nullptr;
    const float* dt_bias = nullptr;
    const void* z = nullptr;
    const float* w_norm = nullptr;
    float norm_eps = 0.f;
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
    // tensor-core path only: gate and beta from raw logits (g_raw non-null: bf16 g_raw
    // [T_tot,H,dk] and beta_raw [T_tot,H], A_log [H], dt_bias [H*dk]; g and beta unused), and
    // the output's gated RMSNorm (z non-null: bf16 z [T_tot,H,dv], w_norm [dv], norm_eps)
    const void* g_raw = nullptr;
    const void* beta_raw = nullptr;
    const float* A_log = nullptr;
    const float* dt_bias = nullptr;
    const void* z = nullptr;
    const float* w_norm = nullptr;
    float norm_eps = 0.f;
    // conv prologue in the producers' load stage (wconv[0] non-null): q, k, v are raw; conv
    // weights [H*d, 4]; conv_state [N, H*(2dk+dv), 3] bf16 history (null: zero), read only here
    const float* wconv[3] = {nullptr, nullptr, nullptr};
    const void* conv_state = nullptr;
    float l2_eps = 0.f;
    // tensor-core path only, plain inputs: a stretch launch (mt non-null, or o null) forms each
    // unit's end state (ht) and output (o, may be null) and, in as many extra clusters as units,
    // its transition M into mt [N, H, dk, dk] fp32 and the output of the transition's run,
    // scale M_t^T q_t, into o_trans [T_tot, H, dk] bf16 (may be null)
    float* mt = nullptr;
    void* o_trans = nullptr;
};
cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream);

// Hand-off rings of the cluster prefill (bf16 I/O, dk = dv = 128, chunk 64): one ring of
// kTcxRingSlots slots per SM id below kTcxRingSms, each slot one chunk's factors.
constexpr int kTcxRingSms = 160;                 // a B200 has 148 SMs
constexpr int kTcxRingSlots = 6;
constexpr size_t kTcxSlotBytes = 74752;
constexpr size_t kTcxWorkspaceBytes = (size_t)kTcxRingSms * kTcxRingSlots * kTcxSlotBytes;

// Tensor-core (tcgen05) prefill for bf16 I/O, dk = dv = 128, chunk 64: a producer/consumer
// pipeline in one 4-CTA cluster per (sequence, head). Needs a device workspace of
// chunk_tcx_workspace_bytes() (16-byte aligned): the per-SM hand-off rings.
inline bool chunk_tc_supported(const ChunkArgs& a) {
    return a.io == Io::BF16 && a.dk == 128 && a.dv == 128 && a.chunk == 64;
}
size_t chunk_tcx_workspace_bytes();
// Clusters of the prefill kernel that can be resident at once on the current device (0 if the
// query fails); cached per device.
int chunk_tcx_cluster_slots();
// Bound (SM cycles) of every device-side wait of later prefill launches; 0 restores the default.
extern long long g_chunk_wait_cycles;
cudaError_t launch_chunk_tcx(const ChunkArgs& a, void* workspace, size_t workspace_bytes,
                             unsigned int* err, cudaStream_t stream);

// Splits every sequence of a batch into P stretches of whole chunks (the last one ragged):
// stretch p of sequence n is stretch index n * P + p, and seg_cu [N * P + 1] receives their
// bounds in packed form. cu: device cu_seqlens, or null for a padded batch of N x T_pad tokens.
cudaError_t launch_split_stretches(const int32_t* cu, int T_pad, int N, int P, int32_t* seg_cu,
                                   cudaStream_t stream);

struct ScanArgs {
    const float* m;          // [*, H, dk, dk] stretch transitions
    const float* s_zero;     // [*, H, dk, dv] stretch end states from zero
    const float* h0;         // [N, H, dk, dv] or null (zero)
    float* h_start;          // [*, H, dk, dv] the state entering each stretch, or null
    float* ht;               // [N, H, dk, dv] the state after each sequence's last stretch, or null
    int N, P, H, dk, dv;
    int64_t seq_stride, seg_stride;   // stretch p of sequence n is index n * seq_stride + p * seg_stride
};
cudaError_t launch_state_scan(const ScanArgs& a, cudaStream_t stream);

// o[t, h, :] += w[t, h, :] h_ent[j, h] over the tokens t of every stretch j (d = 128; bf16 o, w;
// fp32 h_ent [n_stretch, H, 128, 128]); stretch j covers tokens [seg_cu[j], seg_cu[j+1]).
struct CorrectArgs {
    const __nv_bfloat16* w;
    const float* h_ent;
    __nv_bfloat16* o;
    const int32_t* seg_cu;
    int n_stretch, H, P;
    int64_t max_len;         // longest stretch (tokens)
    bool skip_first;         // stretches j with j % P == 0 enter with a zero state
    int blocks_per_stretch;  // (set by the launcher)
};
cudaError_t launch_stretch_correct(const CorrectArgs& a, cudaStream_t stream);

}  // namespace kda
