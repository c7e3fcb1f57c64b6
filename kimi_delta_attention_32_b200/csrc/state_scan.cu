// state_scan.cu -- joining a prefill that was split into stretches of tokens.
//
// The KDA recurrence (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...",
// section "Что именно изменилось"; m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...":
// state = state * exp(gate) + delta) maps the state affinely at every token, so a stretch of
// tokens started from S ends in M S + Z, where M (dk x dk) is the stretch's transition and Z its
// end state from zero. A long sequence (the model trains at 8K, 32K and 256K contexts: sarnas.ru,
// section "Как проходило обучение") can therefore be cut into stretches whose (M, Z) are formed
// independently, on more SMs or on more GPUs, then joined here in order:
//     H_0 = h0,   H_{p+1} = M_p H_p + Z_p,
// and each stretch's output recomputed from its own entering state H_p.
//
// The join is small (one dk x dk by dk x dv product per stretch) and serial only over the
// stretches of a sequence. Columns of the state evolve independently (M acts on rows), so each
// CTA owns 32 value columns of one (sequence, head): its 128 x 32 slice of H stays in registers
// and shared memory, and every stretch's M is staged once in shared memory, rows padded by one
// word so that the 16 rows a warp reads fall in 16 different banks.
#include "common.cuh"
#include "launchers.h"

namespace kda {
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanCols = 32;       // value columns per CTA

template <int DK>
__global__ void __launch_bounds__(kScanThreads) state_scan_kernel(const ScanArgs a) {
    constexpr int kTpr = kScanThreads / DK;     // threads per state row: 2 (dk 128) or 4 (dk 64)
    constexpr int kCpt = kScanCols / kTpr;      // columns per thread: 16 or 8
    extern __shared__ float smem[];
    float* sM = smem;                            // [DK][DK + 1]
    float* sH = smem + DK * (DK + 1);            // [DK][kScanCols]

    const int blocks_per_state = a.dv / kScanCols;
    const int cb = blockIdx.x % blocks_per_state;
    const int nh = blockIdx.x / blocks_per_state;
    const int n = nh / a.H, h = nh % a.H;
    const int i = threadIdx.x / kTpr;            // state row (key channel)
    const int c0 = (threadIdx.x % kTpr) * kCpt;  // first column within the CTA's 32
    const int col = cb * kScanCols + c0;         // first column within the state
    const size_t dkdv = (size_t)DK * a.dv;

    float hr[kCpt];
    {
        const float* src = a.h0 ? a.h0 + ((size_t)n * a.H + h) * dkdv + (size_t)i * a.dv + col : nullptr;
#pragma unroll
        for (int c = 0; c < kCpt; ++c) hr[c] = src ? src[c] : 0.f;
    }
    for (int p = 0; p < a.P; ++p) {
        const int64_t j = (int64_t)n * a.seq_stride + (int64_t)p * a.seg_stride;
        const size_t sbase = ((size_t)j * a.H + h) * dkdv + (size_t)i * a.dv + col;
        if (a.h_start) {
#pragma unroll
            for (int c = 0; c < kCpt; ++c) a.h_start[sbase + c] = hr[c];
        }
        __syncthreads();                         // the previous stretch's reads are done
#pragma unroll
        for (int c = 0; c < kCpt; ++c) sH[i * kScanCols + c0 + c] = hr[c];
        const float* mj = a.m + ((size_t)j * a.H + h) * (size_t)DK * DK;
        for (int e = threadIdx.x; e < DK * DK; e += kScanThreads) sM[(e / DK) * (DK + 1) + e % DK] = mj[e];
        __syncthreads();
        const float* zj = a.s_zero + sbase;
#pragma unroll
        for (int c = 0; c < kCpt; ++c) hr[c] = zj[c];
        for (int kk = 0; kk < DK; ++kk) {
            const float mik = sM[i * (DK + 1) + kk];
            const float* hrow = sH + kk * kScanCols + c0;
#pragma unroll
            for (int c = 0; c < kCpt; ++c) hr[c] = fmaf(mik, hrow[c], hr[c]);
        }
    }
    if (a.ht) {
        float* dst = a.ht + ((size_t)n * a.H + h) * dkdv + (size_t)i * a.dv + col;
#pragma unroll
        for (int c = 0; c < kCpt; ++c) dst[c] = hr[c];
    }
}

__global__ void split_stretches_kernel(const int32_t* __restrict__ cu, int T_pad, int N, int P,
                                       int32_t* __restrict__ seg_cu) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const int64_t bos = cu ? cu[n] : (int64_t)n * T_pad;
    const int64_t eos = cu ? cu[n + 1] : (int64_t)(n + 1) * T_pad;
    const int64_t len = eos - bos;
    const int64_t chunks = (len + 63) / 64;
    const int64_t per = (chunks + P - 1) / P;   // whole chunks per stretch
    for (int p = 0; p < P; ++p) {
        const int64_t off = (int64_t)p * per * 64;
        seg_cu[(int64_t)n * P + p] = (int32_t)(bos + (off < len ? off : len));
    }
    if (n == N - 1) seg_cu[(int64_t)N * P] = (int32_t)eos;
}

template <int DK>
cudaError_t launch_scan_t(const ScanArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(float) * ((size_t)DK * (DK + 1) + (size_t)DK * kScanCols);
    cudaError_t e = cudaFuncSetAttribute(state_scan_kernel<DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)a.N * a.H * (a.dv / kScanCols);
    state_scan_kernel<DK><<<(unsigned)blocks, kScanThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_split_stretches(const int32_t* cu, int T_pad, int N, int P, int32_t* seg_cu,
                                   cudaStream_t stream) {
    if (N == 0) return cudaSuccess;
    split_stretches_kernel<<<(N + 127) / 128, 128, 0, stream>>>(cu, T_pad, N, P, seg_cu);
    return cudaGetLastError();
}

cudaError_t launch_state_scan(const ScanArgs& a, cudaStream_t stream) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    if (a.dv % kScanCols != 0) return cudaErrorInvalidValue;
    if (a.dk == 128) return launch_scan_t<128>(a, stream);
    if (a.dk == 64) return launch_scan_t<64>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace kda
