// api.cu -- the C ABI of libkda: argument checks, then the kernel launches.
// Checks mirror the model's hard configuration validation (m.lqnn.cn/news/255115,
// section "二、第一关：配置文件": conv kernel >= 2, chunk size > 0, head counts
// that divide) and the library's own layout rules; nothing is launched when a
// check fails.
#include "kda.h"

#include <stdint.h>

#define KDA_API extern "C" __attribute__((visibility("default")))

#include "common.cuh"
#include "launchers.h"

namespace kda {
__device__ unsigned int g_device_error = 0;
}

namespace {

constexpr int kVersion = 100;   // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }
bool ok_req(const void* p) { return p != nullptr && aligned16(p); }
bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Resolves padded/packed batch geometry; returns false on inconsistent input.
bool batch_geometry(const int32_t* cu, const int32_t* cu_host, int B, int T, int N,
                    int64_t* T_tot, int* N_out) {
    if ((cu == nullptr) != (cu_host == nullptr)) return false;
    if (cu == nullptr) {
        if (B < 0 || T < 0) return false;
        *T_tot = (int64_t)B * T;
        *N_out = B;
        return true;
    }
    if (N < 0 || cu_host[0] != 0) return false;
    for (int n = 0; n < N; ++n)
        if (cu_host[n + 1] < cu_host[n]) return false;
    *T_tot = cu_host[N];
    *N_out = N;
    return true;
}

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// The bf16, dk = dv = 128, chunk-64 prefill runs on the cluster pipeline, which needs a workspace.
bool cluster_prefill_path(kda_io_dtype io, int dk, int dv, int chunk) {
    return io == KDA_IO_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

// Device address of the error word on the current device.
unsigned int* device_error_word() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, kda::g_device_error) != cudaSuccess) return nullptr;
    return static_cast<unsigned int*>(p);
}

// A prefill split into P stretches per sequence: the layout of its workspace after the rings.
struct SplitLayout {
    size_t seg_cu, m, z, hs, w, total;
};
SplitLayout split_layout(int N, int64_t T_tot, int P, int H, int dk, int dv) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t stretches = (size_t)N * P * H;
    SplitLayout l;
    l.seg_cu = up(kda::chunk_tcx_workspace_bytes());
    l.m = l.seg_cu + up(sizeof(int32_t) * ((size_t)N * P + 1));
    l.z = l.m + up(sizeof(float) * stretches * dk * dk);
    l.hs = l.z + up(sizeof(float) * stretches * dk * dv);
    l.w = l.hs + up(sizeof(float) * stretches * dk * dv);
    l.total = l.w + up(sizeof(uint16_t) * (size_t)T_tot * H * dk);
    return l;
}

// Stretches per sequence for a split prefill. The per-head recurrence is serial over chunks,
// and one cluster of 4 SMs carries one (stretch, head) at a time; `clusters` of them fit on the
// GPU at once (33 on a B200: clusters are placed within GPCs). The split runs 2 U P units
// (outputs and end states from zero, and the transitions) over stretches P times shorter; it
// pays when U = N H units leave most clusters idle. Cost in chunk steps (~2 us each):
//  - per wave of clusters, the longest stretch plus the pipeline's fill and drain (measured:
//    a 128-chunk prefill spans 141 steps of its steady period, so 12 per wave);
//  - one step per stretch for the join;
//  - the output correction, an HBM-bound pass of 768 bytes per token and head (~1/16384 step).
// The cheapest count is taken if it gains more than 10% over one stretch.
int auto_split(int64_t longest, int64_t T_tot, int H, int64_t units, int clusters) {
    constexpr int64_t kFill = 12;
    if (units <= 0 || longest <= 0 || clusters <= 0) return 1;
    const int64_t chunks = (longest + 63) / 64;
    auto waves = [&](int64_t u) { return (u + clusters - 1) / clusters; };
    const int64_t correct = T_tot * H / 16384 + 1;
    const int64_t unsplit = waves(units) * (chunks + kFill);
    int best_p = 1;
    int64_t best = unsplit;
    for (int P = 2; P <= 64; ++P) {
        const int64_t per = (chunks + P - 1) / P;
        if (per < 2) break;
        const int64_t cost = waves(2 * units * P) * (per + kFill) + P + correct;
        if (cost < best) {
            best = cost;
            best_p = P;
        }
    }
    return 10 * best < 9 * unsplit ? best_p : 1;
}

}  // namespace

KDA_API const char* kda_status_string(kda_status status) {
    switch (status) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported size or option";
        case KDA_ERR_WORKSPACE: return "workspace missing or too small";
        case KDA_ERR_CUDA: return "CUDA error";
        case KDA_ERR_TIMEOUT: return "a bounded device wait timed out";
    }
    return "unknown status";
}

KDA_API int kda_version(void) { return kVersion; }

KDA_API kda_status kda_conv_fwd(const void* q_raw, const void* k_raw, const void* v_raw,
                        const float* w_q, const float* w_k, const float* w_v,
                        void* q_out, void* k_out, void* v_out, void* conv_state,
                        const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                        int B, int T, int N, int H, int dk, int dv, int K, float l2_eps,
                        kda_io_dtype io, void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || dk <= 0 || dv <= 0 || K < 2 || !(l2_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    int64_t T_tot = 0;
    int Nn = 0;
    if (!batch_geometry(cu_seqlens, cu_seqlens_host, B, T, N, &T_tot, &Nn)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q_raw, k_raw, v_raw, w_q, w_k, w_v, q_out, k_out, v_out};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (!ok_opt(conv_state) || !ok_opt(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (K != 4 || !head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    kda::ConvArgs a;
    a.x[0] = q_raw; a.x[1] = k_raw; a.x[2] = v_raw;
    a.w[0] = w_q; a.w[1] = w_k; a.w[2] = w_v;
    a.y[0] = q_out; a.y[1] = k_out; a.y[2] = v_out;
    a.conv_state = conv_state;
    a.cu = cu_seqlens;
    a.T_tot = T_tot;
    a.T_pad = cu_seqlens ? 0 : T;
    a.N = Nn; a.H = H; a.dk = dk; a.dv = dv;
    a.eps = l2_eps;
    a.io = io == KDA_IO_BF16 ? kda::Io::BF16 : kda::Io::F32;
    return from_cuda(kda::launch_conv(a, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_chunk_fwd_workspace_size(int N, int64_t T_tot, int H, int dk, int dv, int chunk,
                                        kda_io_dtype io, size_t* bytes) {
    if (bytes == nullptr || N < 0 || T_tot < 0 || H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0)
        return KDA_ERR_INVALID_ARG;
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    *bytes = cluster_prefill_path(io, dk, dv, chunk) ? kda::chunk_tcx_workspace_bytes() : 0;
    return KDA_OK;
}

KDA_API kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, float scale, const float* h0, float* ht, void* o,
                         const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                         int B, int T, int N, int H, int dk, int dv, int chunk,
                         kda_io_dtype io, void* workspace, size_t workspace_bytes,
                         void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0) return KDA_ERR_INVALID_ARG;
    int64_t T_tot = 0;
    int Nn = 0;
    if (!batch_geometry(cu_seqlens, cu_seqlens_host, B, T, N, &T_tot, &Nn)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q, k, v, g, o};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    if (!ok_opt(h0) || !ok_opt(ht) || !ok_opt(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (chunk != 64 || !head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.scale = scale;
    a.h0 = h0; a.ht = ht; a.o = o;
    a.cu = cu_seqlens; a.cu_host = cu_seqlens_host;
    a.T_tot = T_tot;
    a.T_pad = cu_seqlens ? 0 : T;
    a.N = Nn; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.io = io == KDA_IO_BF16 ? kda::Io::BF16 : kda::Io::F32;
    if (kda::chunk_tc_supported(a)) {
        if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0 ||
            workspace_bytes < kda::chunk_tcx_workspace_bytes())
            return KDA_ERR_WORKSPACE;
        unsigned int* err = device_error_word();
        if (err == nullptr) return KDA_ERR_CUDA;
        return from_cuda(kda::launch_chunk_tcx(a, workspace, workspace_bytes, err,
                                               static_cast<cudaStream_t>(stream)));
    }
    return from_cuda(kda::launch_chunk_simt(a, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_chunk_states(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, float scale, const float* h0, float* ht,
                                    void* o, float* m, void* w, const int32_t* cu_seqlens,
                                    const int32_t* cu_seqlens_host, int B, int T, int N, int H,
                                    int dk, int dv, int chunk, kda_io_dtype io, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0) return KDA_ERR_INVALID_ARG;
    int64_t T_tot = 0;
    int Nn = 0;
    if (!batch_geometry(cu_seqlens, cu_seqlens_host, B, T, N, &T_tot, &Nn)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q, k, v, g};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    if (!ok_opt(h0) || !ok_opt(ht) || !ok_opt(m) || !ok_opt(o) || !ok_opt(w) || !ok_opt(cu_seqlens))
        return KDA_ERR_INVALID_ARG;
    if (ht == nullptr && m == nullptr && o == nullptr && w == nullptr) return KDA_ERR_INVALID_ARG;
    if (!cluster_prefill_path(io, dk, dv, chunk)) return KDA_ERR_UNSUPPORTED;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < kda::chunk_tcx_workspace_bytes())
        return KDA_ERR_WORKSPACE;
    unsigned int* err = device_error_word();
    if (err == nullptr) return KDA_ERR_CUDA;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.scale = scale;
    a.h0 = h0; a.ht = ht; a.o = o; a.mt = m; a.o_trans = w;
    a.cu = cu_seqlens; a.cu_host = cu_seqlens_host;
    a.T_tot = T_tot;
    a.T_pad = cu_seqlens ? 0 : T;
    a.N = Nn; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.io = kda::Io::BF16;
    return from_cuda(kda::launch_chunk_tcx(a, workspace, workspace_bytes, err,
                                           static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_state_scan(const float* m, const float* s_zero, const float* h0,
                                  float* h_start, float* ht, int N, int P, int H, int dk, int dv,
                                  int64_t seq_stride, int64_t seg_stride, void* stream) {
    if (N < 0 || P < 1 || H <= 0 || dk <= 0 || dv <= 0 || seq_stride < 0 || seg_stride < 0)
        return KDA_ERR_INVALID_ARG;
    if (!ok_req(m) || !ok_req(s_zero) || !ok_opt(h0) || !ok_opt(h_start) || !ok_opt(ht))
        return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    kda::ScanArgs a;
    a.m = m; a.s_zero = s_zero; a.h0 = h0; a.h_start = h_start; a.ht = ht;
    a.N = N; a.P = P; a.H = H; a.dk = dk; a.dv = dv;
    a.seq_stride = seq_stride; a.seg_stride = seg_stride;
    return from_cuda(kda::launch_state_scan(a, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_output_correct(const void* w, const float* h, void* o,
                                      const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                      int B, int T, int N, int H, int dk, int dv, kda_io_dtype io,
                                      void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    int64_t T_tot = 0;
    int Nn = 0;
    if (!batch_geometry(cu_seqlens, cu_seqlens_host, B, T, N, &T_tot, &Nn)) return KDA_ERR_INVALID_ARG;
    if (!ok_req(w) || !ok_req(h) || !ok_req(o) || !ok_opt(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (io != KDA_IO_BF16 || dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
    if (T_tot > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens == nullptr) return KDA_ERR_UNSUPPORTED;      // packed batches (the split's form)
    int64_t longest = 0;
    for (int n = 0; n < Nn; ++n) {
        const int64_t len = (int64_t)cu_seqlens_host[n + 1] - cu_seqlens_host[n];
        if (len > longest) longest = len;
    }
    kda::CorrectArgs c;
    c.w = static_cast<const __nv_bfloat16*>(w);
    c.h_ent = h;
    c.o = static_cast<__nv_bfloat16*>(o);
    c.seg_cu = cu_seqlens;
    c.n_stretch = Nn; c.H = H; c.P = 1;
    c.max_len = longest;
    c.skip_first = false;
    c.blocks_per_stretch = 0;
    return from_cuda(kda::launch_stretch_correct(c, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_chunk_fwd_split_plan(const int32_t* cu_seqlens_host, int B, int T, int N,
                                            int H, int dk, int dv, int chunk, kda_io_dtype io,
                                            int n_split, int resident_clusters, int* n_split_out,
                                            size_t* bytes) {
    if (bytes == nullptr || n_split_out == nullptr || n_split < 0 || H <= 0 || dk <= 0 || dv <= 0 ||
        chunk <= 0 || (n_split == 0 && resident_clusters <= 0))
        return KDA_ERR_INVALID_ARG;
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host == nullptr ? (B < 0 || T < 0) : N < 0) return KDA_ERR_INVALID_ARG;
    if (!cluster_prefill_path(io, dk, dv, chunk)) return KDA_ERR_UNSUPPORTED;
    const int Nn = cu_seqlens_host ? N : B;
    int64_t longest = cu_seqlens_host ? 0 : T;
    const int64_t T_tot = cu_seqlens_host ? (int64_t)cu_seqlens_host[N] : (int64_t)B * T;
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0) return KDA_ERR_INVALID_ARG;
        for (int n = 0; n < N; ++n) {
            const int64_t len = (int64_t)cu_seqlens_host[n + 1] - cu_seqlens_host[n];
            if (len < 0) return KDA_ERR_INVALID_ARG;
            if (len > longest) longest = len;
        }
    }
    const int P = n_split > 0 ? n_split : auto_split(longest, T_tot, H, (int64_t)Nn * H, resident_clusters);
    *n_split_out = P;
    *bytes = P == 1 ? kda::chunk_tcx_workspace_bytes() : split_layout(Nn, T_tot, P, H, dk, dv).total;
    return KDA_OK;
}

KDA_API kda_status kda_chunk_fwd_split_workspace_size(const int32_t* cu_seqlens_host, int B, int T,
                                                      int N, int H, int dk, int dv, int chunk,
                                                      kda_io_dtype io, int n_split, int* n_split_out,
                                                      size_t* bytes) {
    // the resident cluster count matters only for n_split == 0 on the cluster path
    int slots = 1;
    if (n_split == 0 && H > 0 && cluster_prefill_path(io, dk, dv, chunk)) {
        slots = kda::chunk_tcx_cluster_slots();
        if (slots == 0) return KDA_ERR_CUDA;
    }
    return kda_chunk_fwd_split_plan(cu_seqlens_host, B, T, N, H, dk, dv, chunk, io, n_split, slots,
                                    n_split_out, bytes);
}

KDA_API kda_status kda_chunk_fwd_split(const void* q, const void* k, const void* v, const float* g,
                                       const float* beta, float scale, const float* h0, float* ht,
                                       void* o, const int32_t* cu_seqlens,
                                       const int32_t* cu_seqlens_host, int B, int T, int N, int H,
                                       int dk, int dv, int chunk, kda_io_dtype io, int n_split,
                                       void* workspace, size_t workspace_bytes, void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0 || n_split < 0) return KDA_ERR_INVALID_ARG;
    int64_t T_tot = 0;
    int Nn = 0;
    if (!batch_geometry(cu_seqlens, cu_seqlens_host, B, T, N, &T_tot, &Nn)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q, k, v, g, o};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    if (!ok_opt(h0) || !ok_opt(ht) || !ok_opt(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (!cluster_prefill_path(io, dk, dv, chunk)) return KDA_ERR_UNSUPPORTED;
    if (T_tot > INT32_MAX) return KDA_ERR_UNSUPPORTED;        // stretch bounds are int32
    int P = 0;
    size_t need = 0;
    const kda_status ws = kda_chunk_fwd_split_workspace_size(cu_seqlens_host, B, T, N, H, dk, dv,
                                                             chunk, io, n_split, &P, &need);
    if (ws != KDA_OK) return ws;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    unsigned int* err = device_error_word();
    if (err == nullptr) return KDA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.scale = scale;
    a.h0 = h0; a.ht = ht; a.o = o;
    a.cu = cu_seqlens; a.cu_host = cu_seqlens_host;
    a.T_tot = T_tot;
    a.T_pad = cu_seqlens ? 0 : T;
    a.N = Nn; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.io = kda::Io::BF16;
    const size_t ring = kda::chunk_tcx_workspace_bytes();
    if (P == 1) return from_cuda(kda::launch_chunk_tcx(a, workspace, ring, err, st));
    if (Nn == 0) return KDA_OK;
    // (1) stretch bounds; (2) every stretch from a zero state: its output, its end state Z, and
    // in as many extra clusters its transition M and the queries carried back to its start W;
    // (3) the join, giving each stretch's entering state H and the final states; (4) the
    // output correction o += W H
    const SplitLayout l = split_layout(Nn, T_tot, P, H, dk, dv);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    int32_t* seg_cu = reinterpret_cast<int32_t*>(base + l.seg_cu);
    float* m = reinterpret_cast<float*>(base + l.m);
    float* z = reinterpret_cast<float*>(base + l.z);
    float* hs = reinterpret_cast<float*>(base + l.hs);
    void* w = base + l.w;
    cudaError_t e = kda::launch_split_stretches(cu_seqlens, cu_seqlens ? 0 : T, Nn, P, seg_cu, st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    kda::ChunkArgs s = a;
    s.cu = seg_cu; s.cu_host = nullptr; s.T_pad = 0; s.N = Nn * P;
    s.h0 = nullptr; s.ht = z; s.mt = m; s.o_trans = w;
    if ((e = kda::launch_chunk_tcx(s, workspace, ring, err, st)) != cudaSuccess) return KDA_ERR_CUDA;
    kda::ScanArgs j;
    j.m = m; j.s_zero = z; j.h0 = h0; j.h_start = hs; j.ht = ht;
    j.N = Nn; j.P = P; j.H = H; j.dk = dk; j.dv = dv;
    j.seq_stride = P; j.seg_stride = 1;
    if ((e = kda::launch_state_scan(j, st)) != cudaSuccess) return KDA_ERR_CUDA;
    int64_t longest = cu_seqlens_host ? 0 : T;
    for (int n = 0; cu_seqlens_host && n < Nn; ++n) {
        const int64_t len = (int64_t)cu_seqlens_host[n + 1] - cu_seqlens_host[n];
        if (len > longest) longest = len;
    }
    kda::CorrectArgs c;
    c.w = static_cast<const __nv_bfloat16*>(w);
    c.h_ent = hs;
    c.o = static_cast<__nv_bfloat16*>(o);
    c.seg_cu = seg_cu;
    c.n_stretch = Nn * P; c.H = H; c.P = P;
    c.max_len = (((longest + 63) / 64 + P - 1) / P) * 64;
    c.skip_first = (h0 == nullptr);
    c.blocks_per_stretch = 0;
    return from_cuda(kda::launch_stretch_correct(c, st));
}

KDA_API kda_status kda_chunk_fwd_fused(
    const void* q, const void* k, const void* v, const float* w_q, const float* w_k,
    const float* w_v, const void* conv_state, float l2_eps, const float* g, const float* beta,
    const void* g_raw, const void* beta_raw, const float* A_log, const float* dt_bias,
    const void* z, const float* w_norm, float norm_eps, float scale, const float* h0, float* ht,
    void* o, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int B, int T, int N,
    int H, int dk, int dv, int K, int chunk, kda_io_dtype io, void* workspace,
    size_t workspace_bytes, void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0 || K < 2) return KDA_ERR_INVALID_ARG;
    int64_t T_tot = 0;
    int Nn = 0;
    if (!batch_geometry(cu_seqlens, cu_seqlens_host, B, T, N, &T_tot, &Nn)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q, k, v, o};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (!ok_opt(h0) || !ok_opt(ht) || !ok_opt(cu_seqlens) || !ok_opt(z) || !ok_opt(conv_state))
        return KDA_ERR_INVALID_ARG;
    const bool conv = (w_q != nullptr || w_k != nullptr || w_v != nullptr);
    if (conv && (!ok_req(w_q) || !ok_req(w_k) || !ok_req(w_v) || !(l2_eps >= 0.f)))
        return KDA_ERR_INVALID_ARG;
    if (!conv && conv_state != nullptr) return KDA_ERR_INVALID_ARG;
    const bool gate = (g_raw != nullptr);
    if (gate) {
        if (!ok_req(g_raw) || A_log == nullptr || !aligned4(A_log) || dt_bias == nullptr ||
            !aligned4(dt_bias) || beta_raw == nullptr || (reinterpret_cast<uintptr_t>(beta_raw) & 1u) != 0)
            return KDA_ERR_INVALID_ARG;
    } else if (!ok_req(g) || beta == nullptr || !aligned4(beta)) {
        return KDA_ERR_INVALID_ARG;
    }
    if (z != nullptr && (w_norm == nullptr || !aligned4(w_norm) || !(norm_eps >= 0.f)))
        return KDA_ERR_INVALID_ARG;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.scale = scale;
    a.h0 = h0; a.ht = ht; a.o = o;
    a.cu = cu_seqlens; a.cu_host = cu_seqlens_host;
    a.T_tot = T_tot;
    a.T_pad = cu_seqlens ? 0 : T;
    a.N = Nn; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.io = io == KDA_IO_BF16 ? kda::Io::BF16 : kda::Io::F32;
    if (gate) { a.g_raw = g_raw; a.beta_raw = beta_raw; a.A_log = A_log; a.dt_bias = dt_bias; }
    a.z = z; a.w_norm = w_norm; a.norm_eps = norm_eps;
    if (conv) {
        a.wconv[0] = w_q; a.wconv[1] = w_k; a.wconv[2] = w_v;
        a.conv_state = conv_state;
        a.l2_eps = l2_eps;
    }
    if (!kda::chunk_tc_supported(a) || K != 4) return KDA_ERR_UNSUPPORTED;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0 ||
        workspace_bytes < kda::chunk_tcx_workspace_bytes())
        return KDA_ERR_WORKSPACE;
    unsigned int* err = device_error_word();
    if (err == nullptr) return KDA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = kda::launch_chunk_tcx(a, workspace, workspace_bytes, err, st);
    if (e != cudaSuccess || !conv || conv_state == nullptr) return from_cuda(e);
    // the new conv cache: the last three raw inputs of each sequence's history
    kda::ConvArgs c;
    c.x[0] = q; c.x[1] = k; c.x[2] = v;
    c.w[0] = w_q; c.w[1] = w_k; c.w[2] = w_v;
    c.y[0] = c.y[1] = c.y[2] = nullptr;
    c.conv_state = const_cast<void*>(conv_state);
    c.cu = cu_seqlens;
    c.T_tot = T_tot;
    c.T_pad = cu_seqlens ? 0 : T;
    c.N = Nn; c.H = H; c.dk = dk; c.dv = dv;
    c.eps = l2_eps;
    c.io = a.io;
    return from_cuda(kda::launch_conv_cache(c, st));
}

KDA_API kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, float scale, float* state, void* o,
                              int N, int H, int dk, int dv, kda_io_dtype io, void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q, k, v, g, state, o};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    kda::StepArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.scale = scale;
    a.state = state; a.o = o;
    a.N = N; a.H = H; a.dk = dk; a.dv = dv;
    a.io = io == KDA_IO_BF16 ? kda::Io::BF16 : kda::Io::F32;
    return from_cuda(kda::launch_recurrent_step(a, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_conv_recurrent_step(const void* q_raw, const void* k_raw, const void* v_raw,
                                           const float* w_q, const float* w_k, const float* w_v,
                                           void* conv_state, const float* g, const float* beta,
                                           float scale, float* state, void* o, int N, int H, int dk,
                                           int dv, int K, float l2_eps, kda_io_dtype io,
                                           void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || K < 2 || !(l2_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q_raw, k_raw, v_raw, w_q, w_k, w_v, conv_state, g, state, o};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    if (beta == nullptr || !aligned4(beta)) return KDA_ERR_INVALID_ARG;
    if (K != 4 || !head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    kda::StepArgs a;
    a.q = q_raw; a.k = k_raw; a.v = v_raw; a.g = g; a.beta = beta; a.scale = scale;
    a.state = state; a.o = o;
    a.N = N; a.H = H; a.dk = dk; a.dv = dv;
    a.io = io == KDA_IO_BF16 ? kda::Io::BF16 : kda::Io::F32;
    a.w[0] = w_q; a.w[1] = w_k; a.w[2] = w_v;
    a.conv_state = conv_state;
    a.eps = l2_eps;
    return from_cuda(kda::launch_recurrent_step(a, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_fused_recurrent_step(
    const void* q_raw, const void* k_raw, const void* v_raw, const void* g_raw,
    const void* beta_raw, const float* w_q, const float* w_k, const float* w_v, void* conv_state,
    const float* A_log, const float* dt_bias, const void* z, const float* w_norm, float norm_eps,
    float scale, float* state, void* o, int N, int H, int dk, int dv, int K, float l2_eps,
    kda_io_dtype io, void* stream) {
    if (io != KDA_IO_F32 && io != KDA_IO_BF16) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || K < 2 || !(l2_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    const void* req[] = {q_raw, k_raw, v_raw, g_raw, w_q, w_k, w_v, conv_state, A_log, dt_bias,
                         state, o};
    for (const void* p : req)
        if (!ok_req(p)) return KDA_ERR_INVALID_ARG;
    const uintptr_t esz = io == KDA_IO_BF16 ? 2u : 4u;     // beta_raw: element alignment
    if (beta_raw == nullptr || (reinterpret_cast<uintptr_t>(beta_raw) & (esz - 1)) != 0)
        return KDA_ERR_INVALID_ARG;
    if (!ok_opt(z) || (z != nullptr && (w_norm == nullptr || !(norm_eps >= 0.f))))
        return KDA_ERR_INVALID_ARG;
    if (K != 4 || !head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    kda::StepArgs a;
    a.q = q_raw; a.k = k_raw; a.v = v_raw; a.g = nullptr; a.beta = nullptr; a.scale = scale;
    a.state = state; a.o = o;
    a.N = N; a.H = H; a.dk = dk; a.dv = dv;
    a.io = io == KDA_IO_BF16 ? kda::Io::BF16 : kda::Io::F32;
    a.w[0] = w_q; a.w[1] = w_k; a.w[2] = w_v;
    a.conv_state = conv_state;
    a.eps = l2_eps;
    a.g_raw = g_raw; a.beta_raw = beta_raw; a.A_log = A_log; a.dt_bias = dt_bias;
    a.z = z; a.w_norm = w_norm; a.norm_eps = norm_eps;
    return from_cuda(kda::launch_recurrent_step(a, static_cast<cudaStream_t>(stream)));
}

KDA_API kda_status kda_set_wait_limit(int64_t cycles) {
    if (cycles < 0) return KDA_ERR_INVALID_ARG;
    kda::g_chunk_wait_cycles = cycles;
    return KDA_OK;
}

KDA_API kda_status kda_last_device_error(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, kda::g_device_error, sizeof(word)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(kda::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
            return KDA_ERR_CUDA;
        return KDA_ERR_TIMEOUT;
    }
    return KDA_OK;
}
