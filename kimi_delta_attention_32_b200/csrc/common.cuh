// common.cuh -- small device helpers shared by the libkda kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Bit set (atomicOr) in the device-side error word when a bounded wait gives up.
// The word lives in api.cu; kernels that wait receive its address as an argument.
constexpr unsigned int kErrTimeout = 1u;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load / store n consecutive elements (n = 2 or 4) of type T as fp32.
template <typename T, int n>
struct Vec;

template <>
struct Vec<float, 4> {
    static __device__ __forceinline__ void load(const float* p, float* out) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* in) {
        *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
    }
};
template <>
struct Vec<float, 2> {
    static __device__ __forceinline__ void load(const float* p, float* out) {
        float2 v = *reinterpret_cast<const float2*>(p);
        out[0] = v.x; out[1] = v.y;
    }
    static __device__ __forceinline__ void store(float* p, const float* in) {
        *reinterpret_cast<float2*>(p) = make_float2(in[0], in[1]);
    }
};
template <>
struct Vec<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* out) {
        uint2 raw = *reinterpret_cast<const uint2*>(p);
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        out[0] = fa.x; out[1] = fa.y; out[2] = fb.x; out[3] = fb.y;
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* in) {
        __nv_bfloat162 a = __floats2bfloat162_rn(in[0], in[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(in[2], in[3]);
        uint2 raw;
        raw.x = *reinterpret_cast<uint32_t*>(&a);
        raw.y = *reinterpret_cast<uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = raw;
    }
};
template <>
struct Vec<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* out) {
        float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        out[0] = f.x; out[1] = f.y;
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* in) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(in[0], in[1]);
    }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Index of the sequence containing packed token t: largest n with cu[n] <= t.
__device__ __forceinline__ int find_seq(const int32_t* cu, int N, int64_t t) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Phase timestamps for performance work: a no-op unless the library is built with
// -DKDA_TRACE, which records %globaltimer (ns) for the first cluster's CTAs into
// g_trace[cta][chunk][mark] of the including translation unit.
#ifdef KDA_TRACE
static __device__ unsigned long long g_trace[4][512][16];
__device__ __forceinline__ void trace_mark(int cta, int chunk, int mark, int who = 0) {
    if (threadIdx.x == who && blockIdx.x < 4 && chunk < 512) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_trace[cta][chunk][mark] = t;
    }
}
__device__ __forceinline__ void trace_value(int cta, int chunk, int slot, unsigned long long v) {
    if (threadIdx.x == 0 && blockIdx.x < 4 && chunk < 512) g_trace[cta][chunk][slot] = v;
}
#else
__device__ __forceinline__ void trace_mark(int, int, int, int = 0) {}
__device__ __forceinline__ void trace_value(int, int, int, unsigned long long) {}
#endif

}  // namespace kda
