// recurrent_step.cu -- one decode token of the KDA recurrence per (sequence, head).
//
// Per (sequence, head) with fp32 state S (dk x dv, row i = key channel i):
//   S <- diag(exp(g)) S;  u = v - S^T k;  S <- S + beta k u^T;  o = scale S^T q
// (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...", section
//  "Что именно изменилось": read the stored value, write only the correction,
//  one forgetting coefficient per state row; m.lqnn.cn/news/205170, section
//  "KDA 与 Gated Attention ...": state = state * exp(gate) + delta.)
//
// The fully fused step (kda_fused_recurrent_step) also forms the gate from raw logits,
// g = -exp(A_log[h]) softplus(x + dt_bias) and beta = sigmoid(b) (m.lqnn.cn/news/205170: the
// gate comes from a_log_bias and dt_bias, delta is the residual times sigmoid(beta)), and can
// pass the output through the gated RMSNorm o / sqrt(mean(o^2) + eps) * w * sigmoid(z)
// (sarnas.ru, section "Отвергнутые решения": every norm but the QK norms is a gated RMSNorm).
//
// With the conv prologue fused (kda_conv_recurrent_step), the CTA first advances the
// (sequence, head)'s width-3 conv cache and forms q, k, v from the raw inputs itself: causal
// depthwise conv (kernel 4, tap 3 on the current token), SiLU, and the L2 norm of q and k
// (m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...": the conv cache is advanced per
// step), so q, k, v never make a round trip through HBM and stay in fp32.
//
// The step is bound by HBM: each (sequence, head) streams its 64 KiB state in and
// out once. One CTA of 8 warps owns one state. Lane l holds columns
// [l*CPL, l*CPL+CPL) of R = dk/8 consecutive rows in registers, so every row read
// is one coalesced 128-bit (dv=128) or 64-bit (dv=64) access per lane. The two
// reductions over rows (S^T k and S^T q) are in-register across a thread's rows,
// then across the 8 warps through shared memory; the rank-1 update is in registers.
#include "common.cuh"
#include "launchers.h"

namespace kda {
namespace {

constexpr int kStepWarps = 8;

// The conv prologue's inputs (null when q, k, v arrive already formed), and the raw-logit
// gate and output norm of the fully fused step.
struct StepConv {
    const float* w[3];       // [H*d, 4] weights of q, k, v
    void* cache;             // [N, H*(2dk+dv), 3] conv history, in/out
    float eps;
    int H;
    const float* A_log;      // [H]: g = -exp(A_log[h]) softplus(g_raw + dt_bias)
    const float* dt_bias;    // [H*dk]
    const void* z;           // [N, H, dv] gate of the output norm, or null: no norm
    const float* w_norm;     // [dv] weight of the output norm
    float norm_eps;
};

// softplus(x) = log(1 + e^x), for x > 20 equal to x within fp32 rounding.
__device__ __forceinline__ float softplus_f(float x) { return x > 20.f ? x : log1pf(expf(x)); }

// silu(z) = z sigmoid(z) = h + h tanh(h), h = z / 2 (one tanh.approx, relative error below
// 2^-10) for bf16 I/O; exp and divide for fp32 I/O, held to the tighter bar.
template <typename T>
__device__ __forceinline__ float silu_step(float z) {
    if constexpr (sizeof(T) == 2) {
        const float hz = 0.5f * z;
        float th;
        asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(hz));
        return fmaf(hz, th, hz);
    } else {
        return __fdividef(z, 1.f + __expf(-z));
    }
}

// CONV: q, k, v are raw inputs (conv prologue). GATE: g and beta are raw logits in the io
// dtype (g = -exp(A_log) softplus(g + dt_bias), beta = sigmoid(beta)), and the output passes
// the gated RMSNorm when cv.z is set.
template <typename T, int DK, int DV, bool CONV, bool GATE>
__global__ void __launch_bounds__(kStepWarps * 32, 2)
recurrent_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const void* __restrict__ g_in, const void* __restrict__ beta_in, float scale,
                      float* __restrict__ state, T* __restrict__ o, const StepConv cv) {
    constexpr int R = DK / kStepWarps;   // rows per warp
    constexpr int CPL = DV / 32;         // columns per lane
    const int64_t pair = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
    __shared__ float s_red[kStepWarps][DV];

    float* S = state + pair * (DK * DV);
    const int col = lane * CPL;

    // Issue every state load first: R independent vector loads per lane.
    float s[R][CPL];
#pragma unroll
    for (int r = 0; r < R; ++r) Vec<float, CPL>::load(S + (warp * R + r) * DV + col, s[r]);

    // per-key-channel decay exp(g), with GATE from the raw logit
    auto decay = [&](int i) -> float {
        if constexpr (GATE) {
            const int h = (int)(pair % cv.H);
            const float x = to_f32(static_cast<const T*>(g_in)[pair * DK + i]) + cv.dt_bias[h * DK + i];
            return expf(-expf(cv.A_log[h]) * softplus_f(x));
        } else {
            return expf(static_cast<const float*>(g_in)[pair * DK + i]);
        }
    };
    if constexpr (CONV) {
        // conv step of this (sequence, head)'s 2 DK + DV channels: q, then k, then v
        __shared__ float s_inv[2];
        const int H = cv.H, h = (int)(pair % H);
        const int64_t n = pair / H;
        const int64_t Ctot = (int64_t)H * (2 * DK + DV);
        T* cache = static_cast<T*>(cv.cache);
        for (int c = threadIdx.x; c < 2 * DK + DV; c += blockDim.x) {
            const int z = c < DK ? 0 : (c < 2 * DK ? 1 : 2);
            const int ch = c - z * DK, D = z < 2 ? DK : DV;
            const T* x = z == 0 ? q : (z == 1 ? k : v);
            const float* wz = z == 0 ? cv.w[0] : (z == 1 ? cv.w[1] : cv.w[2]);
            const float4 w = *reinterpret_cast<const float4*>(wz + (int64_t)(h * D + ch) * 4);
            T* cs = cache + (n * Ctot + (int64_t)z * H * DK + (int64_t)h * D + ch) * 3;
            const T x0 = cs[0], x1 = cs[1], x2 = cs[2], xt = x[pair * D + ch];
            if (c < DK) s_a[c] = decay(c);             // (its loads overlap the conv's)
            float zc = w.x * to_f32(x0);
            zc = fmaf(w.y, to_f32(x1), zc);
            zc = fmaf(w.z, to_f32(x2), zc);
            zc = fmaf(w.w, to_f32(xt), zc);
            const float y = silu_step<T>(zc);
            cs[0] = x1;
            cs[1] = x2;
            cs[2] = xt;
            (z == 0 ? s_q : (z == 1 ? s_k : s_v))[ch] = y;
        }
        __syncthreads();
        if (warp < 2) {              // L2 norms of q (warp 0) and k (warp 1)
            const float* arr = warp == 0 ? s_q : s_k;
            float ss = 0.f;
            for (int i = lane; i < DK; i += 32) ss = fmaf(arr[i], arr[i], ss);
            ss = warp_sum(ss);
            if (lane == 0) s_inv[warp] = rsqrtf(ss + cv.eps);
        }
        __syncthreads();
        for (int i = threadIdx.x; i < DK; i += blockDim.x) {
            s_q[i] *= s_inv[0];
            s_k[i] *= s_inv[1];
        }
    } else {
        // every per-pair input in one pass (a thread: q, k and the gate of one key channel, or
        // one value), so that the loads' latencies overlap
        for (int i = threadIdx.x; i < DK + DV; i += blockDim.x) {
            if (i < DK) {
                const float kv = to_f32(k[pair * DK + i]), qv = to_f32(q[pair * DK + i]);
                s_a[i] = decay(i);
                s_k[i] = kv;
                s_q[i] = qv;
            } else {
                s_v[i - DK] = to_f32(v[pair * DV + (i - DK)]);
            }
        }
    }
    float b;
    if constexpr (GATE) b = 1.f / (1.f + expf(-to_f32(static_cast<const T*>(beta_in)[pair])));
    else b = static_cast<const float*>(beta_in)[pair];
    __syncthreads();

    // Decay rows, then partial read-out S^T k over this warp's rows.
    float part[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) part[c] = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int i = warp * R + r;
        const float a = s_a[i], kk = s_k[i];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            s[r][c] *= a;
            part[c] = fmaf(s[r][c], kk, part[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) s_red[warp][col + c] = part[c];
    __syncthreads();

    float u[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kStepWarps; ++w) acc += s_red[w][col + c];
        u[c] = s_v[col + c] - acc;
    }
    __syncthreads();   // s_red is reused below

    // Rank-1 correction, write the state back, partial output S^T q.
#pragma unroll
    for (int c = 0; c < CPL; ++c) part[c] = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int i = warp * R + r;
        const float bk = b * s_k[i], qq = s_q[i];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            s[r][c] = fmaf(bk, u[c], s[r][c]);
            part[c] = fmaf(s[r][c], qq, part[c]);
        }
        Vec<float, CPL>::store(S + i * DV + col, s[r]);
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) s_red[warp][col + c] = part[c];
    __syncthreads();

    if (warp == 0) {
        float out[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < kStepWarps; ++w) acc += s_red[w][col + c];
            out[c] = scale * acc;
        }
        if constexpr (GATE) {
            if (cv.z != nullptr) {       // gated RMSNorm over the dv outputs of this (seq, head)
                float ss = 0.f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) ss = fmaf(out[c], out[c], ss);
                ss = warp_sum(ss);
                const float inv = rsqrtf(ss * (1.f / DV) + cv.norm_eps);
                const T* zz = static_cast<const T*>(cv.z) + pair * DV + col;
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    out[c] = out[c] * inv * cv.w_norm[col + c] / (1.f + expf(-to_f32(zz[c])));
            }
        }
        Vec<T, CPL>::store(o + pair * DV + col, out);
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_step_t(const StepArgs& a, cudaStream_t stream) {
    const int64_t pairs = (int64_t)a.N * a.H;
    if (pairs == 0) return cudaSuccess;
    StepConv cv;
    cv.w[0] = a.w[0]; cv.w[1] = a.w[1]; cv.w[2] = a.w[2];
    cv.cache = a.conv_state;
    cv.eps = a.eps;
    cv.H = a.H;
    cv.A_log = a.A_log;
    cv.dt_bias = a.dt_bias;
    cv.z = a.z;
    cv.w_norm = a.w_norm;
    cv.norm_eps = a.norm_eps;
    const T* q = static_cast<const T*>(a.q);
    const T* k = static_cast<const T*>(a.k);
    const T* v = static_cast<const T*>(a.v);
    T* o = static_cast<T*>(a.o);
    const unsigned grid = (unsigned)pairs, block = kStepWarps * 32;
    if (a.A_log != nullptr)
        recurrent_step_kernel<T, DK, DV, true, true><<<grid, block, 0, stream>>>(
            q, k, v, a.g_raw, a.beta_raw, a.scale, a.state, o, cv);
    else if (a.conv_state != nullptr)
        recurrent_step_kernel<T, DK, DV, true, false><<<grid, block, 0, stream>>>(
            q, k, v, a.g, a.beta, a.scale, a.state, o, cv);
    else
        recurrent_step_kernel<T, DK, DV, false, false><<<grid, block, 0, stream>>>(
            q, k, v, a.g, a.beta, a.scale, a.state, o, cv);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_step(const StepArgs& a, cudaStream_t stream) {
    if (a.dk == 128 && a.dv == 128) return launch_step_t<T, 128, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_step_t<T, 128, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_step_t<T, 64, 128>(a, stream);
    if (a.dk == 64 && a.dv == 64) return launch_step_t<T, 64, 64>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent_step(const StepArgs& a, cudaStream_t stream) {
    return a.io == Io::BF16 ? dispatch_step<__nv_bfloat16>(a, stream)
                            : dispatch_step<float>(a, stream);
}

}  // namespace kda
