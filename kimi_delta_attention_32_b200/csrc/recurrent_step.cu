// recurrent_step.cu -- one decode token of the KDA recurrence per (sequence, head).
//
// Per (sequence, head) with fp32 state S (dk x dv, row i = key channel i):
//   S <- diag(exp(g)) S;  u = v - S^T k;  S <- S + beta k u^T;  o = scale S^T q
// (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...", section
//  "Что именно изменилось": read the stored value, write only the correction,
//  one forgetting coefficient per state row; m.lqnn.cn/news/205170, section
//  "KDA 与 Gated Attention ...": state = state * exp(gate) + delta.)
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

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kStepWarps * 32, 2)
recurrent_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ g, const float* __restrict__ beta, float scale,
                      float* __restrict__ state, T* __restrict__ o) {
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

    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
        s_k[i] = to_f32(k[pair * DK + i]);
        s_q[i] = to_f32(q[pair * DK + i]);
        s_a[i] = expf(g[pair * DK + i]);
    }
    for (int j = threadIdx.x; j < DV; j += blockDim.x) s_v[j] = to_f32(v[pair * DV + j]);
    const float b = beta[pair];
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
        Vec<T, CPL>::store(o + pair * DV + col, out);
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_step_t(const StepArgs& a, cudaStream_t stream) {
    const int64_t pairs = (int64_t)a.N * a.H;
    if (pairs == 0) return cudaSuccess;
    recurrent_step_kernel<T, DK, DV><<<(unsigned)pairs, kStepWarps * 32, 0, stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.g,
        a.beta, a.scale, a.state, static_cast<T*>(a.o));
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
