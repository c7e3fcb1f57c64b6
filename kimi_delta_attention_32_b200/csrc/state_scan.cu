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

// ---------------------------------------------------------------------------------------------
// Output correction of a split prefill. A stretch's output from its entering state H is
//     o_t = o_t(from zero) + H^T w_t,   w_t = scale M_t^T q_t,
// with M_t the transition through token t (the output of the stretch's transition run), so each
// stretch's output from zero takes one dense product with its entering state:
//     O[t, :] += W[t, :] H   (W: tokens x dk bf16, H: dk x dv fp32).
// HBM-bound (read W and O, write O: 768 bytes per token and head for d = 128), on the warp
// tensor-core MMA (bf16 in, fp32 accumulate). H is split as H = Hhi + Hlo with both halves
// bf16, which keeps 16 of its mantissa bits (each product within 2^-16 of exact, against 2^-8
// for H in one bf16); W and O are bf16 in memory anyway.
// One 256-thread CTA takes up to kCorrTiles tiles of 64 tokens of one (stretch, head): it
// converts H once into shared memory, then streams the W tiles (cp.async, double-buffered).
// 8 warps as 4 (16 tokens) x 2 (64 value columns); each warp runs 8 k-steps of 16 channels.
// ---------------------------------------------------------------------------------------------
constexpr int kCorrThreads = 256;
constexpr int kCorrRows = 64;             // tokens per tile
constexpr int kCorrTiles = 16;            // tiles per CTA
constexpr int kPitch = 136;               // bf16 per shared row (128 + 8: 272 B, conflict-free)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
                 "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kCorrThreads) stretch_correct_kernel(const CorrectArgs a) {
    extern __shared__ __align__(16) __nv_bfloat16 csm[];
    __nv_bfloat16* sHi = csm;                          // [128][kPitch]  (k = channel, n = value)
    __nv_bfloat16* sLo = sHi + 128 * kPitch;
    __nv_bfloat16* sW = sLo + 128 * kPitch;            // 2 x [kCorrRows][kPitch]
    const int H = a.H;
    const int blocks = a.blocks_per_stretch;
    const int b = blockIdx.x % blocks;
    const int jh = blockIdx.x / blocks;
    const int j = jh / H, h = jh % H;
    if (a.skip_first && j % a.P == 0) return;          // entering state zero: nothing to add
    const int64_t bos = a.seg_cu[j], eos = a.seg_cu[j + 1];
    const int64_t t_begin = bos + (int64_t)b * kCorrTiles * kCorrRows;
    if (t_begin >= eos) return;
    const int64_t t_end = eos < t_begin + kCorrTiles * kCorrRows ? eos : t_begin + kCorrTiles * kCorrRows;
    const int ntiles = (int)((t_end - t_begin + kCorrRows - 1) / kCorrRows);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // W tile loader: 64 rows x 256 B = 1024 16-byte pieces, 4 per thread (rows past the end are
    // not loaded; their products are never stored)
    auto load_tile = [&](int tile, int buf) {
        const int64_t t0 = t_begin + (int64_t)tile * kCorrRows;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int piece = tid + e * kCorrThreads;
            const int r = piece >> 4, c = piece & 15;
            if (t0 + r < t_end)
                cp_async16(smem_addr(sW + (buf * kCorrRows + r) * kPitch + 8 * c),
                           a.w + ((t0 + r) * H + h) * 128 + 8 * c);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    load_tile(0, 0);
    // H = Hhi + Hlo, both bf16
    const float* Hg = a.h_ent + ((size_t)j * H + h) * 128 * 128;
    for (int e = tid; e < 128 * 32; e += kCorrThreads) {
        const int r = e >> 5, c4 = e & 31;
        const float4 v = reinterpret_cast<const float4*>(Hg + r * 128)[c4];
        const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(x[u]);
            sHi[r * kPitch + 4 * c4 + u] = hi;
            sLo[r * kPitch + 4 * c4 + u] = __float2bfloat16_rn(x[u] - __bfloat162float(hi));
        }
    }
    const int wr = warp & 3, wc = warp >> 2;           // 16-token row block, 64-column half
    for (int tile = 0; tile < ntiles; ++tile) {
        const int buf = tile & 1;
        if (tile + 1 < ntiles) {
            load_tile(tile + 1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                               // tile `tile` (and H) visible to all
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[nt][u] = 0.f;
        const __nv_bfloat16* wt = sW + buf * kCorrRows * kPitch;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t af[4];
            ldsm_x4(smem_addr(wt + (16 * wr + (lane & 15)) * kPitch + 16 * ks + 8 * (lane >> 4)),
                    af[0], af[1], af[2], af[3]);
            const int krow = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
            for (int np = 0; np < 4; ++np) {           // pairs of 8-column tiles
                const int ncol = 64 * wc + 16 * np + 8 * (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(smem_addr(sHi + krow * kPitch + ncol), b0, b1, b2, b3);
                mma_bf16_16816(acc[2 * np], af, b0, b1);
                mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
                ldsm_x4_t(smem_addr(sLo + krow * kPitch + ncol), b0, b1, b2, b3);
                mma_bf16_16816(acc[2 * np], af, b0, b1);
                mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
            }
        }
        // O[t, :] += acc (C fragment: rows lane/4 and lane/4 + 8, columns 2 (lane % 4) + {0, 1});
        // all 16 reads are issued before the first write, so the tile pays one round trip
        const int64_t t0 = t_begin + (int64_t)tile * kCorrRows + 16 * wr + (lane >> 2);
        uint32_t* orow[2];
        uint32_t ov[2][8];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int64_t t = t0 + 8 * half;
            orow[half] = t < t_end ? reinterpret_cast<uint32_t*>(a.o + (t * H + h) * 128) : nullptr;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                ov[half][nt] = orow[half] ? __ldcs(orow[half] + ((64 * wc + 8 * nt + 2 * (lane & 3)) >> 1)) : 0u;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            if (orow[half] == nullptr) continue;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                __nv_bfloat162 o2 = *reinterpret_cast<__nv_bfloat162*>(&ov[half][nt]);
                const float2 o0 = __bfloat1622float2(o2);
                o2 = __floats2bfloat162_rn(o0.x + acc[nt][2 * half], o0.y + acc[nt][2 * half + 1]);
                __stcs(orow[half] + ((64 * wc + 8 * nt + 2 * (lane & 3)) >> 1),
                       *reinterpret_cast<uint32_t*>(&o2));
            }
        }
        __syncthreads();                               // buffer `buf` is reloaded next
    }
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

cudaError_t launch_stretch_correct(const CorrectArgs& a, cudaStream_t stream) {
    if (a.n_stretch == 0 || a.H == 0 || a.max_len == 0) return cudaSuccess;
    const size_t smem = sizeof(__nv_bfloat16) * (size_t)kPitch * (2 * 128 + 2 * kCorrRows);
    cudaError_t e = cudaFuncSetAttribute(stretch_correct_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    CorrectArgs c = a;
    c.blocks_per_stretch = (int)((a.max_len + kCorrTiles * kCorrRows - 1) / (kCorrTiles * kCorrRows));
    const int64_t blocks = (int64_t)a.n_stretch * a.H * c.blocks_per_stretch;
    stretch_correct_kernel<<<(unsigned)blocks, kCorrThreads, smem, stream>>>(c);
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
