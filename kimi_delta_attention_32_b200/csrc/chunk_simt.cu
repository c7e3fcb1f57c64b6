// chunk_simt.cu -- chunked KDA prefill on CUDA cores, all arithmetic in fp32.
//
// This is the fp32-I/O path (its tolerance needs fp32 products throughout); the
// bf16 path uses the tensor-core kernel. Same recurrence as the per-token loop
// (sarnas.ru, section "Что именно изменилось"; m.lqnn.cn/news/205170, section
// "KDA 与 Gated Attention ...": decay each state row, read the stored value,
// write only the beta-scaled correction, read the output from the updated state),
// regrouped per chunk of C = 64 tokens with the state S at the chunk start and
// gamma_r = sum_{s<=r} g_s the in-chunk cumulative log-decay per key channel:
//   A[r,i] = sum_c k_rc k_ic exp(gamma_rc - gamma_ic)   (i < r)
//   P[r,i] = sum_c q_rc k_ic exp(gamma_rc - gamma_ic)   (i <= r)
//   [W | U] = (I + diag(beta) A)^-1 diag(beta) [k*exp(gamma) | v]     (forward substitution)
//   Ut = U - W S                 (row r = beta_r times the residual of token r)
//   O  = scale ((q*exp(gamma)) S + P Ut)
//   S  = diag(exp(gamma_last)) S + (k*exp(gamma_last - gamma))^T Ut
// Every exponent above is <= 0, so nothing overflows. A CTA owns one (sequence,
// head, block of kDVB value columns); value columns are independent, so dk and dv are free.
#include "common.cuh"
#include "launchers.h"

namespace kda {
namespace {

constexpr int kC = 64;          // chunk length
constexpr int kDVB = 32;        // value columns per CTA
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2eS = 1.4426950408889634f;   // log2(e): gamma is kept in log2 units

template <int DK>
struct SimtSmem {
    float q[kC][DK];
    float k[kC][DK];
    float gam[kC][DK];
    float W[kC][DK];
    float A[kC][kC + 1];
    float P[kC][kC + 1];
    float U[kC][kDVB];
    float S[DK][kDVB];
    float beta[kC];
};

template <typename T, int DK>
__global__ void __launch_bounds__(kThreads)
chunk_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ g, const float* __restrict__ beta, float scale,
                  const float* __restrict__ h0, float* __restrict__ ht, T* __restrict__ o,
                  const int32_t* __restrict__ cu, int T_pad, int H, int dv) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem<DK>& sm = *reinterpret_cast<SimtSmem<DK>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int j0 = blockIdx.y * kDVB;
    const int64_t bos = cu ? (int64_t)cu[n] : (int64_t)n * T_pad;
    const int64_t eos = cu ? (int64_t)cu[n + 1] : bos + T_pad;
    const int64_t sbase = ((int64_t)n * H + h) * DK * dv;

    for (int e = tid; e < DK * kDVB; e += kThreads) {
        const int i = e / kDVB, j = e % kDVB;
        sm.S[i][j] = h0 ? h0[sbase + (int64_t)i * dv + j0 + j] : 0.f;
    }

    for (int64_t c0 = bos; c0 < eos; c0 += kC) {
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
        __syncthreads();   // previous chunk finished with every buffer
        // ---- load the chunk; rows r >= L are zero (g = 0 keeps gamma flat) ----
        for (int e = tid; e < kC * DK; e += kThreads) {
            const int r = e / DK, c = e % DK;
            const int64_t off = ((c0 + r) * H + h) * DK + c;
            const bool ok = r < L;
            sm.q[r][c] = ok ? to_f32(q[off]) : 0.f;
            sm.k[r][c] = ok ? to_f32(k[off]) : 0.f;
            sm.gam[r][c] = ok ? g[off] : 0.f;
        }
        for (int e = tid; e < kC * kDVB; e += kThreads) {
            const int r = e / kDVB, j = e % kDVB;
            const bool ok = r < L;
            const float b = ok ? beta[(c0 + r) * H + h] : 0.f;
            sm.U[r][j] = ok ? b * to_f32(v[((c0 + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        for (int r = tid; r < kC; r += kThreads) sm.beta[r] = r < L ? beta[(c0 + r) * H + h] : 0.f;
        __syncthreads();
        // ---- gamma = in-chunk cumulative sum of g, per channel, in log2 units ----
        for (int c = tid; c < DK; c += kThreads) {
            float acc = 0.f;
            for (int r = 0; r < kC; ++r) { acc += sm.gam[r][c]; sm.gam[r][c] = acc * kLog2eS; }
        }
        __syncthreads();
        // ---- A and P: one thread per (r, i) pair (i <= r), channels visited from a per-lane
        //      offset so that the row-strided reads of a warp fall in different banks ----
        for (int pidx = tid; pidx < kC * (kC + 1) / 2; pidx += kThreads) {
            int r = (int)((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
            while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
            while (r * (r + 1) / 2 > pidx) --r;
            const int i = pidx - r * (r + 1) / 2;
            float a = 0.f, pp = 0.f;
#pragma unroll 8
            for (int cc = 0; cc < DK; ++cc) {
                const int c = (cc + lane) & (DK - 1);
                const float ki = sm.k[i][c] * exp2f(sm.gam[r][c] - sm.gam[i][c]);
                a = fmaf(sm.k[r][c], ki, a);
                pp = fmaf(sm.q[r][c], ki, pp);
            }
            sm.A[r][i] = (i < r) ? a : 0.f;
            sm.P[r][i] = pp;
            if (i < r) sm.P[i][r] = 0.f;
            sm.A[i][r] = 0.f;
        }
        __syncthreads();
        // ---- W rhs = beta_r k_r exp(gamma_r); q <- q exp(gamma); k <- k exp(gamma_last - gamma) ----
        for (int e = tid; e < kC * DK; e += kThreads) {
            const int r = e / DK, c = e % DK;
            const float gr = sm.gam[r][c];
            const float er = exp2f(gr);
            sm.W[r][c] = sm.beta[r] * sm.k[r][c] * er;
            sm.q[r][c] *= er;
            sm.k[r][c] *= exp2f(sm.gam[kC - 1][c] - gr);
        }
        __syncthreads();
        // ---- forward substitution X_r -= beta_r sum_{i<r} A[r,i] X_i: columns of [W | U] are
        //      independent, so one thread solves one column in registers, with no barrier
        //      between rows (rows past L have beta = 0 and stay zero) ----
        for (int col = tid; col < DK + kDVB; col += kThreads) {
            const bool wcol = col < DK;
            float* const xs = wcol ? &sm.W[0][col] : &sm.U[0][col - DK];
            const int ld = wcol ? DK : kDVB;
            float x[kC];
#pragma unroll
            for (int r = 0; r < kC; ++r) x[r] = xs[r * ld];
#pragma unroll
            for (int r = 1; r < kC; ++r) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int i = 0; i + 1 < r; i += 2) {
                    a0 = fmaf(sm.A[r][i], x[i], a0);
                    a1 = fmaf(sm.A[r][i + 1], x[i + 1], a1);
                }
                if (r & 1) a0 = fmaf(sm.A[r][r - 1], x[r - 1], a0);
                x[r] -= sm.beta[r] * (a0 + a1);
            }
#pragma unroll
            for (int r = 0; r < kC; ++r) xs[r * ld] = x[r];
        }
        __syncthreads();
        // ---- Ut = U - W S  (thread: column j = lane, rows warp + 8m) ----
        {
            const int j = lane;
            for (int r = warp; r < kC; r += kWarps) {
                float acc = 0.f;
                for (int c = 0; c < DK; ++c) acc = fmaf(sm.W[r][c], sm.S[c][j], acc);
                sm.U[r][j] -= acc;
            }
        }
        __syncthreads();
        // ---- O = scale (Qhat S + P Ut) ----
        {
            const int j = lane;
            for (int r = warp; r < L; r += kWarps) {
                float acc = 0.f;
                for (int c = 0; c < DK; ++c) acc = fmaf(sm.q[r][c], sm.S[c][j], acc);
                for (int i = 0; i <= r; ++i) acc = fmaf(sm.P[r][i], sm.U[i][j], acc);
                o[((c0 + r) * H + h) * dv + j0 + j] = from_f32<T>(scale * acc);
            }
        }
        __syncthreads();
        // ---- S = diag(exp(gamma_last)) S + Ktilde^T Ut ----
        {
            const int j = lane;
            for (int c = warp; c < DK; c += kWarps) {
                const float gl = sm.gam[kC - 1][c];
                float acc = exp2f(gl) * sm.S[c][j];
                for (int r = 0; r < L; ++r) acc = fmaf(sm.k[r][c], sm.U[r][j], acc);
                sm.S[c][j] = acc;
            }
        }
    }
    __syncthreads();
    if (ht) {
        for (int e = tid; e < DK * kDVB; e += kThreads) {
            const int i = e / kDVB, j = e % kDVB;
            ht[sbase + (int64_t)i * dv + j0 + j] = sm.S[i][j];
        }
    }
}

template <typename T, int DK>
cudaError_t launch_t(const ChunkArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem<DK>);
    auto kern = chunk_simt_kernel<T, DK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((int64_t)a.N * a.H), (unsigned)(a.dv / kDVB));
    kern<<<grid, kThreads, smem, stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.g,
        a.beta, a.scale, a.h0, a.ht, static_cast<T*>(a.o), a.cu, a.T_pad, a.H, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs& a, cudaStream_t stream) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    if (a.dv % kDVB != 0) return cudaErrorInvalidValue;
    if (a.io == Io::BF16) {
        if (a.dk == 128) return launch_t<__nv_bfloat16, 128>(a, stream);
        if (a.dk == 64) return launch_t<__nv_bfloat16, 64>(a, stream);
    } else {
        if (a.dk == 128) return launch_t<float, 128>(a, stream);
        if (a.dk == 64) return launch_t<float, 64>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
