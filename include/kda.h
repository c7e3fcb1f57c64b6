/*
 * kda.h -- C ABI of libkda, a B200 (sm_100a) implementation of the Kimi Delta
 * Attention (KDA) linear-attention core.
 *
 * What the operations compute comes from pages about the AliceAI-Foundation-
 * 80B-A3B-Base model:
 *  - sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base: MoE-модель,
 *    обученная с нуля", section "Что именно изменилось": KDA keeps a fixed-size
 *    state; for each token it reads the value the state holds for the token's
 *    key, compares it with the new value and writes back only the difference;
 *    it forgets with one coefficient per state row (Gated DeltaNet has one
 *    coefficient for the whole state).
 *  - m.lqnn.cn/news/205170, section "KDA 与 Gated Attention：每 4 层只留 1 层
 *    全注意力": q/k/v first pass a kernel-4 causal convolution with a cache that
 *    is advanced per step; the recurrence is state = state * exp(gate) + delta
 *    with delta = prediction residual x sigmoid(beta); beta in (0, 1).
 *  - m.lqnn.cn/news/255115, section "二、第一关：配置文件": the conv kernel is at
 *    least 2 and the chunk size positive.
 *
 * Per (sequence, head), with state S (dk x dv, row i = key channel i) and token t:
 *     S   <- diag(exp(g_t)) S                       per-row forgetting
 *     u_t  = v_t - S^T k_t                          read-out and residual
 *     S   <- S + beta_t k_t u_t^T                   write only the correction
 *     o_t  = scale * S^T q_t                        output from the updated state
 *
 * Conventions shared by every call
 *  - All tensor pointers are caller-owned DEVICE memory, row-major and dense,
 *    16-byte aligned except beta (4-byte aligned is enough). Host pointers are
 *    marked "host".
 *  - Token-major layouts: q, k, g : [T_tot, H, dk];  v, o : [T_tot, H, dv];
 *    beta : [T_tot, H];  state : [N, H, dk, dv] fp32.
 *  - io selects the element type of q, k, v, o (and of the conv tensors):
 *    KDA_IO_F32 (float) or KDA_IO_BF16 (__nv_bfloat16). g, beta, state and conv
 *    weights are always fp32.
 *  - Batches: padded (cu_seqlens == NULL): B sequences of T tokens each, so
 *    N = B and T_tot = B*T; packed (cu_seqlens != NULL): N sequences, sequence n
 *    is tokens [cu[n], cu[n+1]), T_tot = cu[N]; cu_seqlens (device, int32 [N+1])
 *    and cu_seqlens_host (host copy) must both be given and hold the same values.
 *  - stream is a cudaStream_t (NULL = the legacy default stream). Every call is
 *    asynchronous on it; results are valid once the stream has been synchronised.
 *    The library allocates nothing, frees nothing and never synchronises (except
 *    kda_last_device_error, which says so).
 *  - Errors: arguments are checked on the host before anything is launched; a
 *    failing check launches nothing and returns KDA_ERR_INVALID_ARG or
 *    KDA_ERR_UNSUPPORTED. A launch failure returns KDA_ERR_CUDA. No call aborts
 *    or throws. Preconditions that are NOT checked: g <= 0, beta in (0, 1),
 *    finite inputs, and that cu_seqlens matches cu_seqlens_host.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* a null, misaligned, negative or inconsistent argument */
    KDA_ERR_UNSUPPORTED = 2,   /* a valid size this build has no kernel for */
    KDA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the query says */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime error while launching */
    KDA_ERR_TIMEOUT = 5        /* a bounded device-side wait gave up (see kda_last_device_error) */
} kda_status;

typedef enum { KDA_IO_F32 = 0, KDA_IO_BF16 = 1 } kda_io_dtype;

/* Static English text for a status; never NULL. */
const char* kda_status_string(kda_status status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int kda_version(void);

/*
 * kda_conv_fwd -- fused short causal depthwise convolution + SiLU (+ L2 norm of q, k).
 * (m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...": kernel-4 causal
 *  conv of q, k and v with a cache advanced per step; m.lqnn.cn/news/255115,
 *  section "二、第一关：配置文件": kernel >= 2.)
 *
 * For each channel c of x in {q_raw, k_raw, v_raw} (channel c = h*d + i):
 *     y[t, c] = silu( sum_{j=0}^{K-1} w[c, j] * x[t-(K-1)+j, c] ),  silu(z) = z / (1 + e^-z)
 * where positions before a sequence's first token read the conv history of
 * that sequence (conv_state, oldest first) or zero when conv_state is NULL.
 * Then each dk-vector of the q and k outputs is divided by sqrt(sum y^2 + l2_eps).
 * No bias. The conv never crosses a sequence boundary.
 *
 *  q_raw, k_raw : [T_tot, H, dk] io dtype      v_raw : [T_tot, H, dv] io dtype
 *  w_q, w_k     : [H*dk, K] fp32               w_v   : [H*dv, K] fp32 (tap K-1 = current token)
 *  q_out, k_out, v_out : same shapes as the inputs; must not overlap any input.
 *  conv_state   : [N, H*(2*dk+dv), K-1] io dtype, channels ordered q, then k, then v,
 *                 or NULL. In: the K-1 raw inputs preceding each sequence (oldest
 *                 first). Out (overwritten in place): the last K-1 raw inputs of the
 *                 history followed by this call's tokens. Decode is the padded
 *                 case with T == 1.
 *  Supported: dk, dv in {64, 128}; K == 4; io F32 or BF16.
 */
kda_status kda_conv_fwd(const void* q_raw, const void* k_raw, const void* v_raw,
                        const float* w_q, const float* w_k, const float* w_v,
                        void* q_out, void* k_out, void* v_out, void* conv_state,
                        const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                        int B, int T, int N, int H, int dk, int dv, int K, float l2_eps,
                        kda_io_dtype io, void* stream);

/*
 * kda_chunk_fwd_workspace_size -- bytes of device workspace kda_chunk_fwd needs
 * for these sizes (written to *bytes, host). Zero means none; the call then
 * accepts workspace == NULL. The bf16, dk = dv = 128, chunk-64 prefill needs a
 * fixed ~71.8 MB whatever the batch: per-SM hand-off rings through which the
 * kernel's producer CTAs pass each chunk's operands to its consumer CTA via L2.
 * The contents need no initialisation and are dead after the call; one
 * workspace may serve consecutive calls on one stream, not concurrent ones.
 */
kda_status kda_chunk_fwd_workspace_size(int N, int64_t T_tot, int H, int dk, int dv, int chunk,
                                        kda_io_dtype io, size_t* bytes);

/*
 * kda_chunk_fwd -- chunked prefill of the KDA recurrence over a padded or packed batch.
 * (sarnas.ru, section "Что именно изменилось"; m.lqnn.cn/news/205170, section
 *  "KDA 与 Gated Attention ..."; chunk > 0 from m.lqnn.cn/news/255115.)
 *
 * Computes, for every token, exactly the per-token recurrence above; the chunk
 * length only changes the order of the arithmetic (the result is the same up to
 * rounding). o[t] = scale * S_t^T q_t with S_t the state after token t.
 *
 *  q, k : [T_tot, H, dk] io dtype   v : [T_tot, H, dv] io dtype   o : [T_tot, H, dv] io dtype
 *  g    : [T_tot, H, dk] fp32 per-channel log-decay (<= 0)
 *  beta : [T_tot, H] fp32 write strength in (0, 1)
 *  scale: multiplies the output (1.0 for no scaling)
 *  h0   : [N, H, dk, dv] fp32 initial states, or NULL for zero states
 *  ht   : [N, H, dk, dv] fp32 final states, or NULL to skip; may alias h0
 *  chunk: tokens per chunk; this build supports 64.
 *  workspace: device memory of at least kda_chunk_fwd_workspace_size() bytes,
 *         16-byte aligned, owned by the caller (KDA_ERR_WORKSPACE otherwise);
 *         may be NULL when that size is 0.
 *  Supported: dk, dv each in {64, 128}, chunk 64 (bf16 with dk = dv = 128 runs on the tensor
 *  cores, every other combination on CUDA cores in fp32).
 *  Empty sequences are allowed (their final state is the initial state).
 */
kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, float scale, const float* h0, float* ht, void* o,
                         const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                         int B, int T, int N, int H, int dk, int dv, int chunk,
                         kda_io_dtype io, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * kda_chunk_states -- a prefill's pieces for a split into stretches of tokens (context
 * parallelism), joined by kda_state_scan: per sequence its end state, output and transition,
 * and the queries carried back to its start.
 * (sarnas.ru, section "Что именно изменилось", and m.lqnn.cn/news/205170, section "KDA 与
 *  Gated Attention ...": the per-token update state = state*exp(gate) + delta is affine in the
 *  state, S -> (I - beta k k^T) diag(exp(g)) S + beta k v^T; sarnas.ru, section "Как проходило
 *  обучение": the model is trained at 8K, 32K and 256K contexts, which a split spreads over more
 *  SMs or GPUs.)
 *
 * For each (sequence n, head h) of the batch, with M_t the product over the sequence's tokens
 * up to t, latest on the left, of (I - beta k k^T) diag(exp(g)) (dk x dk):
 *   ht[n,h] = the state after the sequence, started from h0[n,h] (zero when h0 is NULL), as
 *             kda_chunk_fwd returns it;
 *   o       = the output from that start, as kda_chunk_fwd returns it;
 *   m[n,h]  = the transition M = M_T of the whole sequence (fp32, row i = key channel i), so
 *             that started from any S the sequence ends in M S + (ht from zero);
 *   w[t,h]  = scale * M_t^T q_t, so that started from any S the output is
 *             o_t(from zero) + S^T w_t.
 * Each output may be NULL, not all. m and w come from as many extra clusters as (sequence,
 * head) pairs in the same launch. Inputs, layouts, workspace and errors as for kda_chunk_fwd.
 *  o : [T_tot, H, dv] bf16 or NULL   m : [N, H, dk, dk] fp32 or NULL   w : [T_tot, H, dk] bf16
 *  or NULL.   Supported: bf16 I/O, dk == dv == 128, chunk 64.
 */
kda_status kda_chunk_states(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, float scale, const float* h0, float* ht, void* o,
                            float* m, void* w, const int32_t* cu_seqlens,
                            const int32_t* cu_seqlens_host, int B, int T, int N, int H, int dk,
                            int dv, int chunk, kda_io_dtype io, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * kda_state_scan -- joins the stretches of a split prefill in order (same sources as
 * kda_chunk_states): for every sequence n and head h,
 *     H_0 = h0[n,h] (zero when h0 is NULL),  H_{p+1} = M_p H_p + Z_p  for p = 0 .. P-1,
 * with stretch p of sequence n at index j = n*seq_stride + p*seg_stride of m (M_j) and s_zero
 * (Z_j, the stretch's end state from zero). h_start[j] receives H_p (the state entering
 * stretch p) and ht[n] receives H_P; either may be NULL. fp32 throughout.
 *  m : [*, H, dk, dk]   s_zero, h_start : [*, H, dk, dv]   h0, ht : [N, H, dk, dv]
 *  (* = every index j reached). h_start must not overlap m, s_zero or h0.
 *  Supported: dk, dv in {64, 128}.
 */
kda_status kda_state_scan(const float* m, const float* s_zero, const float* h0, float* h_start,
                          float* ht, int N, int P, int H, int dk, int dv, int64_t seq_stride,
                          int64_t seg_stride, void* stream);

/*
 * kda_output_correct -- adds the entering state's share to outputs formed from a zero state
 * (same sources as kda_chunk_states): for every sequence n, head h and token t of it,
 *     o[t,h,:] += h[n,h]^T w[t,h,:]
 * with w from kda_chunk_states and h[n,h] the state the sequence was entered with (from
 * kda_state_scan). The product runs on the tensor cores in bf16 with fp32 accumulation; h is
 * split into two bf16 halves, which keep 16 of its mantissa bits (relative error below 2^-16
 * per product).
 *  w : [T_tot, H, dk] bf16   h : [N, H, dk, dv] fp32   o : [T_tot, H, dv] bf16, updated in place.
 *  Packed batches only (cu_seqlens and cu_seqlens_host given; KDA_ERR_UNSUPPORTED otherwise).
 *  Supported: bf16 I/O, dk == dv == 128.
 */
kda_status kda_output_correct(const void* w, const float* h, void* o, const int32_t* cu_seqlens,
                              const int32_t* cu_seqlens_host, int B, int T, int N, int H, int dk,
                              int dv, kda_io_dtype io, void* stream);

/*
 * kda_chunk_fwd_split_workspace_size -- stretches per sequence and workspace bytes of
 * kda_chunk_fwd_split for this batch. Host-only, except that n_split == 0 asks the current
 * device, once per device, how many of the prefill's 4-SM clusters it holds at once
 * (cudaOccupancyMaxActiveClusters; KDA_ERR_CUDA if that query fails).
 *  cu_seqlens_host, B, T, N: the batch as for kda_chunk_fwd (host data only).
 *  n_split: stretches per sequence, or 0 to choose: the split is taken when the (sequence,
 *  head) pairs leave most of those clusters idle and the cost model (serial chunks per
 *  stretch, waves of clusters, the join and the output correction) gains more than 10%; 1
 *  otherwise.
 *  n_split_out: host, receives the stretch count; bytes: host, receives the size.
 */
kda_status kda_chunk_fwd_split_workspace_size(const int32_t* cu_seqlens_host, int B, int T,
                                              int N, int H, int dk, int dv, int chunk,
                                              kda_io_dtype io, int n_split, int* n_split_out,
                                              size_t* bytes);

/*
 * kda_chunk_fwd_split_plan -- kda_chunk_fwd_split_workspace_size for a device that holds
 * resident_clusters of the prefill's 4-SM clusters at once (33 on a B200), with no device
 * query: host-only, so a batch can be planned away from the GPU that runs it.
 *  resident_clusters: > 0 when n_split == 0 (KDA_ERR_INVALID_ARG otherwise); unused when
 *  n_split > 0. Other arguments and results as for kda_chunk_fwd_split_workspace_size.
 */
kda_status kda_chunk_fwd_split_plan(const int32_t* cu_seqlens_host, int B, int T, int N, int H,
                                    int dk, int dv, int chunk, kda_io_dtype io, int n_split,
                                    int resident_clusters, int* n_split_out, size_t* bytes);

/*
 * kda_chunk_fwd_split -- kda_chunk_fwd with every sequence split into stretches of whole
 * chunks that run side by side (context parallelism inside one GPU; same sources as
 * kda_chunk_states). Four launches on the stream: the stretch bounds; every stretch from a
 * zero state, with its output, end state, transition and carried-back queries
 * (kda_chunk_states); the join (kda_state_scan), which gives each stretch's entering state H;
 * and the correction o_t += H^T w_t of every stretch's output (a dense product on the tensor
 * cores). Results equal kda_chunk_fwd's up to rounding: the entering states pass through the
 * bf16 products of the transitions, and the output from zero and w are rounded to bf16 before
 * the correction.
 *  n_split: as for kda_chunk_fwd_split_workspace_size (0 = choose; 1 = kda_chunk_fwd).
 *  workspace: at least kda_chunk_fwd_split_workspace_size() bytes for the same batch and
 *  n_split, 16-byte aligned.
 * Other arguments, results and errors as for kda_chunk_fwd; also KDA_ERR_UNSUPPORTED when the
 * batch has 2^31 tokens or more. Supported: bf16 I/O, dk == dv == 128, chunk 64.
 */
kda_status kda_chunk_fwd_split(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, float scale, const float* h0, float* ht,
                               void* o, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                               int B, int T, int N, int H, int dk, int dv, int chunk,
                               kda_io_dtype io, int n_split, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd_fused -- kda_chunk_fwd with the surrounding steps of the KDA layer fused into the
 * prefill kernel, each optional:
 *  - conv prologue (w_q, w_k, w_v given): q, k, v are the RAW projections; each is passed
 *    through the kernel-4 causal depthwise conv and SiLU, and q, k through the L2 norm, exactly
 *    as kda_conv_fwd computes them, in the producers' load stage (no HBM round trip). The history
 *    before each sequence is conv_state (or zero when NULL); when conv_state is given it is
 *    overwritten with the new history afterwards (the last K-1 raw inputs, as kda_conv_fwd does).
 *  - gate from raw logits (g_raw given): g = -exp(A_log[h]) * softplus(g_raw + dt_bias[h, c]) and
 *    beta = sigmoid(beta_raw), in the producers' fold; otherwise g and beta are taken as given.
 *  - gated RMSNorm of the output (z given): o' = o / sqrt(mean_j o_j^2 + norm_eps) * w_norm *
 *    sigmoid(z), before the store.
 * (m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...": kernel-4 causal conv with a
 *  cache, the gate from a_log_bias and dt_bias, delta = residual * sigmoid(beta); sarnas.ru,
 *  section "Отвергнутые решения": every norm except the QK norms is a gated RMSNorm.)
 *
 *  q, k, v     : as kda_chunk_fwd (raw projections with the conv)
 *  w_q, w_k, w_v: [H*d, K] fp32 conv weights, all NULL or all given; conv_state: [N, H*(2dk+dv),
 *                K-1] bf16 or NULL (only with the conv); l2_eps: the q, k L2-norm epsilon
 *  g, beta     : as kda_chunk_fwd, used when g_raw is NULL
 *  g_raw       : [T_tot, H, dk] bf16   beta_raw : [T_tot, H] bf16 (2-byte aligned)
 *  A_log       : [H] fp32              dt_bias  : [H*dk] fp32 (with g_raw)
 *  z           : [T_tot, H, dv] bf16 or NULL        w_norm : [dv] fp32 (with z)
 *  other arguments, the workspace and the errors as for kda_chunk_fwd.
 *  Supported: bf16 I/O, dk == dv == 128, chunk 64, K == 4 (KDA_ERR_UNSUPPORTED otherwise).
 */
kda_status kda_chunk_fwd_fused(const void* q, const void* k, const void* v, const float* w_q,
                               const float* w_k, const float* w_v, const void* conv_state,
                               float l2_eps, const float* g, const float* beta, const void* g_raw,
                               const void* beta_raw, const float* A_log, const float* dt_bias,
                               const void* z, const float* w_norm, float norm_eps, float scale,
                               const float* h0, float* ht, void* o, const int32_t* cu_seqlens,
                               const int32_t* cu_seqlens_host, int B, int T, int N, int H, int dk,
                               int dv, int K, int chunk, kda_io_dtype io, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate device memory.
 * (The pages have no counterpart: this is a library convenience, not a step of the method.)
 *
 * kda_chunk_fwd needs a caller-owned workspace of kda_chunk_fwd_workspace_size() bytes
 * (~72 MB for the bf16, dk = dv = 128 prefill). Some callers cannot cudaMalloc one where they
 * run the prefill: a runtime whose memory pool already holds all free device memory, a plug-in
 * handed only tensor pointers, or a latency-critical path that cannot afford cudaMalloc's
 * implicit device synchronisation. This entry point uses instead a device array owned by the
 * library (a file-scope __device__ array of exactly that maximum size, one per device, held by
 * every GPU that loads libkda until the process exits), so the call allocates nothing; the
 * caller still passes every input and output.
 *
 * Arguments, layouts, results and errors are those of kda_chunk_fwd. A size whose workspace
 * would exceed the array returns KDA_ERR_WORKSPACE; if the array's device address cannot be
 * obtained the call returns KDA_ERR_CUDA (argument errors are still reported first).
 * Set-up: the first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any stream capture.
 * Sharing: every call on a device uses the same array, which keeps the last call's contents
 * (no call needs it cleared); calls that overlap on the GPU race, so run them one after another.
 */
kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, float scale, const float* h0, float* ht,
                                 void* o, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                 int B, int T, int N, int H, int dk, int dv, int chunk,
                                 kda_io_dtype io, void* stream);

/*
 * kda_recurrent_step -- one decode token per (sequence, head), state updated in place.
 * (sarnas.ru, section "Что именно изменилось"; m.lqnn.cn/news/205170, section
 *  "KDA 与 Gated Attention ...": the per-token loop state = state*exp(gate)+delta.)
 *
 *  q, k : [N, H, dk] io dtype   v, o : [N, H, dv] io dtype
 *  g    : [N, H, dk] fp32   beta : [N, H] fp32
 *  state: [N, H, dk, dv] fp32, read and overwritten with the state after the token.
 *  o    : must not overlap any input.
 *  Supported: dk, dv in {64, 128}.
 */
kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, float scale, float* state, void* o,
                              int N, int H, int dk, int dv, kda_io_dtype io, void* stream);

/*
 * kda_conv_recurrent_step -- one decode token per (sequence, head) from RAW q, k, v: the conv
 * prologue and the state update in one kernel, with the conv cache advanced in place.
 * (m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...": q/k/v pass a kernel-4 causal
 *  conv whose cache is advanced per step, then the loop state = state*exp(gate)+delta;
 *  sarnas.ru, section "Что именно изменилось".)
 *
 * Computes exactly kda_conv_fwd in decode form (T == 1 per sequence) followed by
 * kda_recurrent_step, except that the conv outputs stay in fp32 inside the kernel instead of
 * being rounded to the io dtype and written out (they are not returned).
 *
 *  q_raw, k_raw : [N, H, dk] io dtype   v_raw : [N, H, dv] io dtype (this step's raw inputs)
 *  w_q, w_k     : [H*dk, K] fp32        w_v   : [H*dv, K] fp32 (tap K-1 = current token)
 *  conv_state   : [N, H*(2*dk+dv), K-1] io dtype, channels q, k, v; read and overwritten with
 *                 the last K-1 raw inputs (required: the decode history)
 *  g    : [N, H, dk] fp32   beta : [N, H] fp32   scale: multiplies the output
 *  state: [N, H, dk, dv] fp32, read and overwritten with the state after the token
 *  o    : [N, H, dv] io dtype; must not overlap any input
 *  l2_eps: the epsilon of the q, k L2 norm (x / sqrt(sum x^2 + eps))
 *  Supported: dk, dv in {64, 128}; K == 4.
 */
kda_status kda_conv_recurrent_step(const void* q_raw, const void* k_raw, const void* v_raw,
                                   const float* w_q, const float* w_k, const float* w_v,
                                   void* conv_state, const float* g, const float* beta,
                                   float scale, float* state, void* o, int N, int H, int dk,
                                   int dv, int K, float l2_eps, kda_io_dtype io, void* stream);

/*
 * kda_fused_recurrent_step -- the whole decode step of a KDA layer from raw projections, in one
 * kernel: conv prologue (cache advanced in place), gate activation, the state update, and
 * optionally the gated RMSNorm of the output.
 * (m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...": kernel-4 causal conv with a
 *  cache advanced per step; the gate is computed from a_log_bias and dt_bias; delta is the
 *  residual times sigmoid(beta). sarnas.ru, section "Отвергнутые решения": every norm except
 *  the QK norms is a gated RMSNorm.)
 *
 * As kda_conv_recurrent_step, except that the gate and beta arrive as raw logits:
 *     g[n, h, c] = -exp(A_log[h]) * softplus(g_raw[n, h, c] + dt_bias[h * dk + c]),
 *     beta[n, h] = sigmoid(beta_raw[n, h]),
 * and, when z is not NULL, the output is o' = o / sqrt(mean_j o_j^2 + norm_eps) * w_norm *
 * sigmoid(z) over the dv channels of each (sequence, head).
 *
 *  g_raw   : [N, H, dk] io dtype        beta_raw : [N, H] io dtype (element-aligned)
 *  A_log   : [H] fp32                   dt_bias  : [H*dk] fp32
 *  z       : [N, H, dv] io dtype or NULL (no output norm)   w_norm : [dv] fp32 (with z)
 *  other arguments as for kda_conv_recurrent_step.
 *  Supported: dk, dv in {64, 128}; K == 4.
 */
kda_status kda_fused_recurrent_step(const void* q_raw, const void* k_raw, const void* v_raw,
                                    const void* g_raw, const void* beta_raw, const float* w_q,
                                    const float* w_k, const float* w_v, void* conv_state,
                                    const float* A_log, const float* dt_bias, const void* z,
                                    const float* w_norm, float norm_eps, float scale,
                                    float* state, void* o, int N, int H, int dk, int dv, int K,
                                    float l2_eps, kda_io_dtype io, void* stream);

/*
 * kda_set_wait_limit -- bound, in SM clock cycles, of every device-side wait of the prefill
 * kernels launched after this call on any device (0 restores the default of ~2 s). A wait that
 * runs out sets the device error word (KDA_ERR_TIMEOUT from kda_last_device_error) and the
 * kernel ends without finishing the call; its outputs are then undefined. A diagnostic for
 * failure handling: a short bound makes the cross-CTA hand-off waits give up. Not thread-safe
 * against concurrent launches. KDA_ERR_INVALID_ARG for a negative bound.
 */
kda_status kda_set_wait_limit(int64_t cycles);

/*
 * kda_last_device_error -- synchronises `stream`, then returns and clears the
 * device-side error word that kernels set when a bounded wait gives up
 * (KDA_ERR_TIMEOUT) -- KDA_OK if none. Returns KDA_ERR_CUDA if the stream
 * reports a CUDA error.
 */
kda_status kda_last_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
