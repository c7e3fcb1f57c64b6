// conv.cu -- fused short causal depthwise convolution (kernel 4) + SiLU (+ L2 norm of q, k).
//
// (m.lqnn.cn/news/205170, section "KDA 与 Gated Attention：每 4 层只留 1 层全注意力":
//  q, k and v each pass a kernel-4 causal convolution whose cache is advanced per
//  step; m.lqnn.cn/news/255115, section "二、第一关：配置文件": kernel >= 2.)
//
//   y[t, c] = silu( sum_{j=0..3} w[c, j] * x[t-3+j, c] ),   q and k then / sqrt(sum y^2 + eps)
//
// Work unit: one warp = one head-vector of one tensor over a tile of kTile
// consecutive packed tokens. Lane l owns channels [l*CPL, l*CPL+CPL) of the head,
// keeps the previous three inputs of those channels in registers (each input is
// read from HBM once) and finishes the L2 norm with a warp reduction. A tile may
// cross a sequence boundary; the history is then reset from that sequence's conv
// cache (or zero). The cache is only READ by this kernel in prefill mode; a second
// small kernel writes the new cache afterwards, so an in-place cache is never read
// after it was overwritten. Decode (one token per sequence) reads and writes the
// cache in the same warp, so it needs no second kernel.
#include "common.cuh"
#include "launchers.h"

namespace kda {
namespace {

constexpr int kTaps = 4;
constexpr int kHist = kTaps - 1;
constexpr int kTile = 16;
constexpr int kConvWarps = 4;

struct ConvParams {
    const void* x[3];
    const float* w[3];
    void* y[3];
    void* conv_state;
    const int32_t* cu;
    int64_t T_tot;
    int T_pad;
    int N, H, dk, dv;
    int Ctot;
    float eps;
    int step_mode;       // one token per sequence: read and write the cache here
};

// Register image of CPL consecutive elements of type T (8 or 16 bytes), and its unpacking.
template <typename T, int CPL>
struct RawVec;
template <>
struct RawVec<__nv_bfloat16, 4> {
    using Word = uint2;
    static __device__ __forceinline__ void unpack(const Word& w, float* o) {
        o[0] = __uint_as_float(w.x << 16); o[1] = __uint_as_float(w.x & 0xffff0000u);
        o[2] = __uint_as_float(w.y << 16); o[3] = __uint_as_float(w.y & 0xffff0000u);
    }
};
template <>
struct RawVec<__nv_bfloat16, 2> {
    using Word = uint32_t;
    static __device__ __forceinline__ void unpack(const Word& w, float* o) {
        o[0] = __uint_as_float(w << 16); o[1] = __uint_as_float(w & 0xffff0000u);
    }
};
template <>
struct RawVec<float, 4> {
    using Word = uint4;
    static __device__ __forceinline__ void unpack(const Word& w, float* o) {
        o[0] = __uint_as_float(w.x); o[1] = __uint_as_float(w.y);
        o[2] = __uint_as_float(w.z); o[3] = __uint_as_float(w.w);
    }
};
template <>
struct RawVec<float, 2> {
    using Word = uint2;
    static __device__ __forceinline__ void unpack(const Word& w, float* o) {
        o[0] = __uint_as_float(w.x); o[1] = __uint_as_float(w.y);
    }
};

// silu(z) = z sigmoid(z) = h + h tanh(h) with h = z / 2: one SFU operation (tanh.approx,
// relative error below 2^-10) for bf16 outputs instead of an exponential and a division; the
// fp32 path, held to a tighter bar, keeps exp and divide.
template <typename T>
__device__ __forceinline__ float silu(float z) {
    if constexpr (sizeof(T) == 2) {
        const float hz = 0.5f * z;
        float th;
        asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(hz));
        return fmaf(hz, th, hz);
    } else {
        return __fdividef(z, 1.f + __expf(-z));
    }
}

// The general tile: sequence boundaries inside the tile or its history, the conv cache, and the
// decode form. Out of line, so that the common tile's code stays small.
template <typename T, int D>
__device__ __noinline__ void conv_unit(const ConvParams& p, int z, int h, int64_t t0) {
    constexpr int CPL = D / 32;
    using Word = typename RawVec<T, CPL>::Word;
    const int lane = threadIdx.x & 31;
    // selects rather than p.x[z]: indexing the parameter arrays at run time would copy them
    // to local memory
    const T* __restrict__ x = static_cast<const T*>(z == 0 ? p.x[0] : z == 1 ? p.x[1] : p.x[2]);
    T* __restrict__ y = static_cast<T*>(z == 0 ? p.y[0] : z == 1 ? p.y[1] : p.y[2]);
    const float* wz = z == 0 ? p.w[0] : z == 1 ? p.w[1] : p.w[2];
    T* cache = static_cast<T*>(p.conv_state);
    const int H = p.H;
    const int cl = lane * CPL;                                    // channel within the head
    const int cstate = (z == 0 ? 0 : z == 1 ? H * p.dk : 2 * H * p.dk) + h * D + cl;
    const int64_t t1 = t0 + kTile < p.T_tot ? t0 + kTile : p.T_tot;
    const int ntok = (int)(t1 - t0);

    // Issue every load of the tile first: the three tokens before it and its kTile tokens.
    Word raw[kHist + kTile];
#pragma unroll
    for (int m = 0; m < kHist + kTile; ++m) {
        const int64_t t = t0 - kHist + m;
        raw[m] = Word{};
        if (t >= 0 && t < t1) raw[m] = *reinterpret_cast<const Word*>(x + (t * H + h) * D + cl);
    }
    float w[CPL][kTaps];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const float4 wv = *reinterpret_cast<const float4*>(wz + (int64_t)(h * D + cl + c) * kTaps);
        w[c][0] = wv.x; w[c][1] = wv.y; w[c][2] = wv.z; w[c][3] = wv.w;
    }

    int n;
    int64_t bos, eos;
    if (p.cu) {
        n = find_seq(p.cu, p.N, t0);
        bos = p.cu[n];
        eos = p.cu[n + 1];
    } else {
        n = (int)(t0 / p.T_pad);
        bos = (int64_t)n * p.T_pad;
        eos = bos + p.T_pad;
    }

    // hist[m] = input at position t-3+m (m = 0 oldest) of the current sequence.
    float hist[kHist][CPL];
    T* yrow = y + (t0 * H + h) * D + cl;
    const bool norm = (z < 2);
#pragma unroll
    for (int tt = 0; tt < kTile; ++tt) {
        if (tt >= ntok) break;
        const int64_t t = t0 + tt;
        if (tt == 0 || t >= eos) {
            if (t >= eos) {                       // crossed into the next non-empty sequence
                if (p.cu) {
                    do { ++n; } while (p.cu[n + 1] <= t);
                    bos = p.cu[n];
                    eos = p.cu[n + 1];
                } else {
                    ++n;
                    bos = eos;
                    eos = bos + p.T_pad;
                }
            }
#pragma unroll
            for (int m = 0; m < kHist; ++m) {
                const int64_t tp = t - kHist + m;
                if (tp >= bos) {
                    RawVec<T, CPL>::unpack(raw[tt + m], hist[m]);
                } else if (cache) {
                    const int slot = kHist - (int)(bos - tp);           // oldest first
#pragma unroll
                    for (int c = 0; c < CPL; ++c)
                        hist[m][c] = to_f32(cache[((int64_t)n * p.Ctot + cstate + c) * kHist + slot]);
                } else {
#pragma unroll
                    for (int c = 0; c < CPL; ++c) hist[m][c] = 0.f;
                }
            }
        }
        float xt[CPL], out[CPL];
        RawVec<T, CPL>::unpack(raw[kHist + tt], xt);
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            float zc = w[c][0] * hist[0][c];
            zc = fmaf(w[c][1], hist[1][c], zc);
            zc = fmaf(w[c][2], hist[2][c], zc);
            zc = fmaf(w[c][3], xt[c], zc);
            const float sv = silu<T>(zc);
            out[c] = sv;
            ss = fmaf(sv, sv, ss);
        }
        if (norm) {
            ss = warp_sum(ss);
            const float inv = rsqrtf(ss + p.eps);
#pragma unroll
            for (int c = 0; c < CPL; ++c) out[c] *= inv;
        }
        Vec<T, CPL>::store(yrow, out);
        yrow += (int64_t)H * D;
        if (p.step_mode && cache) {
            // decode: new cache = the two newest history entries, then this token
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                T* cs = cache + ((int64_t)n * p.Ctot + cstate + c) * kHist;
                cs[0] = from_f32<T>(hist[1][c]);
                cs[1] = from_f32<T>(hist[2][c]);
                cs[2] = from_f32<T>(xt[c]);
            }
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            hist[0][c] = hist[1][c];
            hist[1][c] = hist[2][c];
            hist[2][c] = xt[c];
        }
    }
}

// The common tile: kTile tokens and their three predecessors all in one sequence, prefill form.
// No branch per token; the weights are halved once so that SiLU is h + h tanh(h) straight from
// the sum (bf16 outputs; the fp32 path keeps its exact SiLU).
template <typename T, int D>
__device__ __forceinline__ void conv_tile_inner(const ConvParams& p, int z, int h, int64_t t0) {
    constexpr int CPL = D / 32;
    constexpr bool kHalf = sizeof(T) == 2;
    using Word = typename RawVec<T, CPL>::Word;
    const int lane = threadIdx.x & 31;
    const T* __restrict__ x = static_cast<const T*>(z == 0 ? p.x[0] : z == 1 ? p.x[1] : p.x[2]);
    T* __restrict__ y = static_cast<T*>(z == 0 ? p.y[0] : z == 1 ? p.y[1] : p.y[2]);
    const float* wz = z == 0 ? p.w[0] : z == 1 ? p.w[1] : p.w[2];
    const int H = p.H;
    const int cl = lane * CPL;
    const int64_t rs = (int64_t)H * D;                             // elements per token
    const T* xp = x + ((t0 - kHist) * H + h) * D + cl;
    Word raw[kHist + kTile];
#pragma unroll
    for (int m = 0; m < kHist + kTile; ++m) raw[m] = *reinterpret_cast<const Word*>(xp + m * rs);
    float w[CPL][kTaps];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const float4 wv = *reinterpret_cast<const float4*>(wz + (int64_t)(h * D + cl + c) * kTaps);
        const float sc = kHalf ? 0.5f : 1.f;
        w[c][0] = wv.x * sc; w[c][1] = wv.y * sc; w[c][2] = wv.z * sc; w[c][3] = wv.w * sc;
    }
    float hist[kHist][CPL];
#pragma unroll
    for (int m = 0; m < kHist; ++m) RawVec<T, CPL>::unpack(raw[m], hist[m]);
    T* yrow = y + (t0 * H + h) * D + cl;
    const bool norm = (z < 2);
#pragma unroll
    for (int tt = 0; tt < kTile; ++tt) {
        float xt[CPL], out[CPL];
        RawVec<T, CPL>::unpack(raw[kHist + tt], xt);
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            float zc = w[c][0] * hist[0][c];
            zc = fmaf(w[c][1], hist[1][c], zc);
            zc = fmaf(w[c][2], hist[2][c], zc);
            zc = fmaf(w[c][3], xt[c], zc);
            float sv;
            if constexpr (kHalf) {                                  // zc is already z / 2
                float th;
                asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(zc));
                sv = fmaf(zc, th, zc);
            } else {
                sv = silu<T>(zc);
            }
            out[c] = sv;
            ss = fmaf(sv, sv, ss);
        }
        if (norm) {
            ss = warp_sum(ss);
            const float inv = rsqrtf(ss + p.eps);
#pragma unroll
            for (int c = 0; c < CPL; ++c) out[c] *= inv;
        }
        Vec<T, CPL>::store(yrow, out);
        yrow += rs;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            hist[0][c] = hist[1][c];
            hist[1][c] = hist[2][c];
            hist[2][c] = xt[c];
        }
    }
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kConvWarps * 32)
conv_kernel(const ConvParams p) {
    const int z = blockIdx.z;
    const int h = blockIdx.y * kConvWarps + (threadIdx.x >> 5);
    const int64_t t0 = (int64_t)blockIdx.x * kTile;
    if (h >= p.H || t0 >= p.T_tot) return;
    bool inner = !p.step_mode && t0 >= kHist && t0 + kTile <= p.T_tot;
    if (inner) {                       // the tile and its history within one sequence?
        if (p.cu) {
            const int n = find_seq(p.cu, p.N, t0);
            inner = t0 - kHist >= p.cu[n] && t0 + kTile <= p.cu[n + 1];
        } else {
            inner = (t0 - kHist) / p.T_pad == (t0 + kTile - 1) / p.T_pad;
        }
    }
    if (z < 2) {
        if (inner) conv_tile_inner<T, DK>(p, z, h, t0);
        else conv_unit<T, DK>(p, z, h, t0);
    } else {
        if (inner) conv_tile_inner<T, DV>(p, z, h, t0);
        else conv_unit<T, DV>(p, z, h, t0);
    }
}

// Prefill mode: new cache[n, c, p] = ext[L + p], ext = (old cache of n, then x of n).
template <typename T>
__global__ void conv_cache_kernel(const ConvParams p) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.N * p.Ctot) return;
    const int n = (int)(idx / p.Ctot);
    const int c = (int)(idx % p.Ctot);
    const int64_t bos = p.cu ? (int64_t)p.cu[n] : (int64_t)n * p.T_pad;
    const int64_t L = p.cu ? (int64_t)p.cu[n + 1] - bos : (int64_t)p.T_pad;
    int z, ch, D;
    if (c < p.H * p.dk) { z = 0; ch = c; D = p.dk; }
    else if (c < 2 * p.H * p.dk) { z = 1; ch = c - p.H * p.dk; D = p.dk; }
    else { z = 2; ch = c - 2 * p.H * p.dk; D = p.dv; }
    (void)D;
    const T* x = static_cast<const T*>(z == 0 ? p.x[0] : z == 1 ? p.x[1] : p.x[2]);
    T* cs = static_cast<T*>(p.conv_state) + idx * kHist;
    const int rowlen = (z < 2 ? p.dk : p.dv) * p.H;           // channels per token of x[z]
    T old[kHist], nw[kHist];
#pragma unroll
    for (int m = 0; m < kHist; ++m) old[m] = cs[m];
#pragma unroll
    for (int m = 0; m < kHist; ++m) {
        const int64_t e = L + m;                             // index into ext
        nw[m] = (e < kHist) ? old[e] : x[(bos + e - kHist) * rowlen + ch];
    }
#pragma unroll
    for (int m = 0; m < kHist; ++m) cs[m] = nw[m];
}

template <typename T>
cudaError_t launch_conv_t(const ConvParams& p, cudaStream_t stream) {
    if (p.T_tot > 0) {
        dim3 grid((unsigned)((p.T_tot + kTile - 1) / kTile), (unsigned)((p.H + kConvWarps - 1) / kConvWarps), 3);
        if (p.dk == 128 && p.dv == 128) conv_kernel<T, 128, 128><<<grid, kConvWarps * 32, 0, stream>>>(p);
        else if (p.dk == 128 && p.dv == 64) conv_kernel<T, 128, 64><<<grid, kConvWarps * 32, 0, stream>>>(p);
        else if (p.dk == 64 && p.dv == 128) conv_kernel<T, 64, 128><<<grid, kConvWarps * 32, 0, stream>>>(p);
        else if (p.dk == 64 && p.dv == 64) conv_kernel<T, 64, 64><<<grid, kConvWarps * 32, 0, stream>>>(p);
        else return cudaErrorInvalidValue;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.conv_state && !p.step_mode && p.N > 0) {
        const int64_t total = (int64_t)p.N * p.Ctot;
        conv_cache_kernel<T><<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_conv_cache(const ConvArgs& a, cudaStream_t stream) {
    ConvParams p;
    for (int i = 0; i < 3; ++i) { p.x[i] = a.x[i]; p.w[i] = a.w[i]; p.y[i] = a.y[i]; }
    p.conv_state = a.conv_state;
    p.cu = a.cu;
    p.T_tot = a.T_tot;
    p.T_pad = a.T_pad;
    p.N = a.N; p.H = a.H; p.dk = a.dk; p.dv = a.dv;
    p.Ctot = a.H * (2 * a.dk + a.dv);
    p.eps = a.eps;
    p.step_mode = 0;
    if (p.conv_state == nullptr || p.N == 0) return cudaSuccess;
    const int64_t total = (int64_t)p.N * p.Ctot;
    if (a.io == Io::BF16)
        conv_cache_kernel<__nv_bfloat16><<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p);
    else
        conv_cache_kernel<float><<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_conv(const ConvArgs& a, cudaStream_t stream) {
    ConvParams p;
    for (int i = 0; i < 3; ++i) { p.x[i] = a.x[i]; p.w[i] = a.w[i]; p.y[i] = a.y[i]; }
    p.conv_state = a.conv_state;
    p.cu = a.cu;
    p.T_tot = a.T_tot;
    p.T_pad = a.T_pad;
    p.N = a.N; p.H = a.H; p.dk = a.dk; p.dv = a.dv;
    p.Ctot = a.H * (2 * a.dk + a.dv);
    p.eps = a.eps;
    p.step_mode = (a.cu == nullptr && a.T_pad == 1) ? 1 : 0;
    return a.io == Io::BF16 ? launch_conv_t<__nv_bfloat16>(p, stream)
                            : launch_conv_t<float>(p, stream);
}

}  // namespace kda
