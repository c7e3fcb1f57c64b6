// chunk_tc.cu -- chunked KDA prefill on the sm_100a tensor cores (tcgen05 + TMEM), bf16 I/O,
// dk = dv = 128, chunk C = 64, fp32 state.
//
// The recurrence (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...",
// section "Что именно изменилось": per-row forgetting, read the stored value, write only
// the correction; m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...":
// state = state * exp(gate) + delta, delta = residual * sigmoid(beta)) regrouped per chunk,
// with S the state at the chunk start and gamma_r = sum_{s<=r} g_s per key channel:
//   A[r,i] = sum_c k_rc k_ic e^{gamma_rc - gamma_ic} (i < r),  P[r,i] likewise with q_r (i <= r)
//   T' = (I + diag(beta) A)^-1 diag(beta);   W = T' (k e^gamma);   U = T' v
//   Ut = U - W S;   O = scale ((q e^gamma) S + P Ut);   S' = diag(e^{gamma_C}) S + (k e^{gamma_C - gamma})^T Ut
//
// Mapping to the hardware. One CTA (8 warps) owns one (sequence, head). Every product is
// written transposed so that its M dimension is a 128-wide channel index and its
// accumulator row is a TMEM lane (tcgen05.mma M=128, cta_group::1):
//   A|P  : [k e^{gamma-gamma_m} ; q e^{gamma-gamma_m}] (128 x 128ch) . (k e^{gamma_m-gamma})^T
//   W^T  = Khat^T T'^T,  U^T = V^T T'^T,  O^T = S^T Qhat^T + Ut^T P^T,
//   Ut^T = U^T - S^T W^T (A operand negated in the instruction descriptor),
//   dS^T = Ut^T Ktilde.
// gamma_m is the cumulative decay at the middle of the chunk (token 31), so the folded
// factors stay within e^{+-80} whenever both half-chunk decays are above -80 per channel;
// a chunk that fails this test computes A and P exactly on CUDA cores instead.
// The fp32 master state lives in registers (thread (j, half) holds S[64*half .. +64][j]);
// its bf16 copy is the A operand of the state products. The triangular inverse is done
// in fp32 on CUDA cores (16x16 diagonal blocks by substitution, then block merges).
#include "common.cuh"
#include "launchers.h"
#include "tc.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr float kHalfRange = 80.f;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at the boost clock

// TMEM columns (fp32 accumulators, lane = M row)
constexpr uint32_t COL_AP = 0, COL_W = 64, COL_X = 128, COL_O = 192, COL_S = 256;
constexpr uint32_t kTmemCols = 512;

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_XQ = 0;                   // raw q [64][128] bf16      | Tm, Y (fp32) for the inverse
constexpr uint32_t OFF_XK = OFF_XQ + 16384;      // raw k [64][128] bf16
constexpr uint32_t OFF_XG = OFF_XK + 16384;      // raw g / gamma [64][128] f32 | N = diag(beta) A (fp32 [64][65])
constexpr uint32_t OFF_VT = OFF_XG + 32768;      // V^T  : A, MN-major, K = 64 tokens, M = 128
constexpr uint32_t OFF_LS = OFF_VT + 16384;      // [Lk;Lq]: A, MN-major, K = 128 ch, M = 128 | exact-A fp32 | W^T (B) + Ut^T (A)
constexpr uint32_t OFF_RT = OFF_LS + 32768;      // R^T  : B, MN-major, K = 128 ch, N = 64   | P (B, K-major) + T' (B, K-major)
constexpr uint32_t OFF_KH = OFF_RT + 16384;      // Khat^T: A, K-major, rows = ch, K = 64 tokens
constexpr uint32_t OFF_QH = OFF_KH + 16384;      // Qhat^T: B, MN-major, K = 128 ch, N = 64 tokens
constexpr uint32_t OFF_KT = OFF_QH + 16384;      // Ktilde: B, K-major, rows = ch (N = 128), K = 64 tokens
constexpr uint32_t OFF_ST = OFF_KT + 16384;      // S^T  : A, K-major, rows = value ch, K = 128 key ch
constexpr uint32_t OFF_MISC = OFF_ST + 32768;
constexpr uint32_t OFF_WOP = OFF_LS;             // W^T  : B, MN-major, K = 128 ch, N = 64 tokens
constexpr uint32_t OFF_UOP = OFF_LS + 16384;     // Ut^T : A, K-major, rows = value ch, K = 64 tokens
constexpr uint32_t OFF_POP = OFF_RT;             // P    : B, K-major, rows = r, K = 64 (i)
constexpr uint32_t OFF_TOP = OFF_RT + 8192;      // T'   : B, K-major, rows = r, K = 64 (i)
constexpr uint32_t kSmemBytes = OFF_MISC + 2048 + 1024;   // + alignment slack

constexpr int kLd = 65;                          // fp32 row stride of the 64x64 scratch matrices

__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ float bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                const float* __restrict__ beta, float scale, const float* __restrict__ h0,
                float* __restrict__ ht, __nv_bfloat16* __restrict__ o,
                const int32_t* __restrict__ cu, int T_pad, int H, unsigned int* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
    const uint32_t lane_sel = (uint32_t)(32 * (warp & 3)) << 16;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int64_t bos = cu ? (int64_t)cu[n] : (int64_t)n * T_pad;
    const int64_t eos = cu ? (int64_t)cu[n + 1] : bos + T_pad;

    float* s_beta = reinterpret_cast<float*>(sm + OFF_MISC);      // [64]
    float* s_gsum = s_beta + 64;                                   // [2][128]
    float* s_eC = s_gsum + 256;                                    // [128] e^{gamma_C}
    uint64_t* s_bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC + 1792);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC + 1800);

    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) mbar_init(s_bar, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;
    uint32_t phase = 0;
    bool aborted = false;

    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(s_bar, phase, kWaitCycles);
        phase ^= 1u;
        if (!ok) atomicOr(err, kErrTimeout);
        return __syncthreads_or(!ok) == 0;
    };

    // ---- master state: thread (j = row, half = wg) holds S[64*wg + cc][j] ----
    const int j = row;
    const int64_t sbase = ((int64_t)n * H + h) * kD * kD;
    float sreg[64];
#pragma unroll
    for (int cc = 0; cc < 64; ++cc)
        sreg[cc] = h0 ? h0[sbase + (int64_t)(64 * wg + cc) * kD + j] : 0.f;

    auto write_state_operand = [&]() {
#pragma unroll
        for (int qq = 0; qq < 8; ++qq) {
            uint4 pk;
            pk.x = pack_bf16(sreg[8 * qq + 0], sreg[8 * qq + 1]);
            pk.y = pack_bf16(sreg[8 * qq + 2], sreg[8 * qq + 3]);
            pk.z = pack_bf16(sreg[8 * qq + 4], sreg[8 * qq + 5]);
            pk.w = pack_bf16(sreg[8 * qq + 6], sreg[8 * qq + 7]);
            st16(sm, OFF_ST + kmaj_chunk(j, qq, wg, 128), pk);
        }
    };
    write_state_operand();

    for (int64_t c0 = bos; c0 < eos && !aborted; c0 += kC) {
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);

        // ================= P0: load the chunk (rows >= L are zero) =================
        for (int e = tid; e < kC * 16; e += kThreads) {
            const int r = e >> 4, jj = e & 15;
            uint4 vq = make_uint4(0, 0, 0, 0), vk = vq, vv = vq;
            if (r < L) {
                const int64_t off = ((c0 + r) * H + h) * kD + jj * 8;
                vq = ld16(q + off);
                vk = ld16(k + off);
                vv = ld16(v + off);
            }
            st16(sm, OFF_XQ + r * 256 + jj * 16, vq);
            st16(sm, OFF_XK + r * 256 + jj * 16, vk);
            st16(sm, OFF_VT + mnmaj_chunk(r, jj & 7, jj >> 3, 8), vv);
        }
        for (int e = tid; e < kC * 32; e += kThreads) {
            const int r = e >> 5, jj = e & 31;
            uint4 vg = make_uint4(0, 0, 0, 0);
            if (r < L) vg = ld16(g + ((c0 + r) * H + h) * kD + jj * 4);
            st16(sm, OFF_XG + r * 512 + jj * 16, vg);
        }
        if (tid < kC) s_beta[tid] = tid < L ? beta[(c0 + tid) * H + h] : 0.f;
        __syncthreads();

        // ================= P1: cumulative decay and folded operands =================
        // thread (c = row, half = wg) owns channel c for tokens [32*wg, 32*wg + 32)
        const int c = row;
        float* Xg = reinterpret_cast<float*>(sm + OFF_XG);
        const __nv_bfloat16* Xq = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_XQ);
        const __nv_bfloat16* Xk = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_XK);
        float gam[32];
        {
            float acc = 0.f;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                acc += Xg[(32 * wg + t) * kD + c];
                gam[t] = acc;
            }
            s_gsum[wg * 128 + c] = acc;
        }
        __syncthreads();
        const float gA = s_gsum[c], gB = s_gsum[128 + c];
        if (wg) {
#pragma unroll
            for (int t = 0; t < 32; ++t) gam[t] += gA;
        }
        const float gm = gA, gC = gA + gB;          // gamma at token 31 and at the chunk end
        const int bad = __syncthreads_or((gA < -kHalfRange) || (gB < -kHalfRange));
        if (bad) {
#pragma unroll
            for (int t = 0; t < 32; ++t) Xg[(32 * wg + t) * kD + c] = gam[t];
        }
        if (wg) s_eC[c] = expf(gC);
        {
            const float e_m = expf(gm), e_Cm = expf(gC - gm);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint32_t lk[4], lq[4], rr[4], kh[4], qh[4], kt[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    float vlk[2], vlq[2], vr[2], vkh[2], vqh[2], vkt[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int t = 8 * qq + 2 * p + u;
                        const int r = 32 * wg + t;
                        const float kx = bf(Xk + r * kD + c), qx = bf(Xq + r * kD + c);
                        if (!bad) {
                            const float a = expf(gam[t] - gm), b = expf(gm - gam[t]);
                            vlk[u] = kx * a;
                            vlq[u] = qx * a;
                            vr[u] = kx * b;
                            vkh[u] = vlk[u] * e_m;
                            vqh[u] = vlq[u] * e_m;
                            vkt[u] = vr[u] * e_Cm;
                        } else {
                            const float e1 = expf(gam[t]), e2 = expf(gC - gam[t]);
                            vlk[u] = vlq[u] = vr[u] = 0.f;
                            vkh[u] = kx * e1;
                            vqh[u] = qx * e1;
                            vkt[u] = kx * e2;
                        }
                    }
                    lk[p] = pack_bf16(vlk[0], vlk[1]);
                    lq[p] = pack_bf16(vlq[0], vlq[1]);
                    rr[p] = pack_bf16(vr[0], vr[1]);
                    kh[p] = pack_bf16(vkh[0], vkh[1]);
                    qh[p] = pack_bf16(vqh[0], vqh[1]);
                    kt[p] = pack_bf16(vkt[0], vkt[1]);
                }
                const int ch = 4 * wg + qq;           // 8-token chunk index within the 64 tokens
                if (!bad) {
                    st16(sm, OFF_LS + mnmaj_chunk(c, ch, 0, 16), make_uint4(lk[0], lk[1], lk[2], lk[3]));
                    st16(sm, OFF_LS + mnmaj_chunk(c, ch, 1, 16), make_uint4(lq[0], lq[1], lq[2], lq[3]));
                    st16(sm, OFF_RT + mnmaj_chunk(c, ch, 0, 16), make_uint4(rr[0], rr[1], rr[2], rr[3]));
                }
                st16(sm, OFF_KH + kmaj_chunk(c, ch, 0, 128), make_uint4(kh[0], kh[1], kh[2], kh[3]));
                st16(sm, OFF_QH + mnmaj_chunk(c, ch, 0, 16), make_uint4(qh[0], qh[1], qh[2], qh[3]));
                st16(sm, OFF_KT + kmaj_chunk(c, ch, 0, 128), make_uint4(kt[0], kt[1], kt[2], kt[3]));
            }
        }
        fence_async_smem();
        __syncthreads();

        // ================= P2: A and P =================
        float* Nm = reinterpret_cast<float*>(sm + OFF_XG);       // diag(beta) A, fp32 [64][65]
        if (!bad) {
            if (tid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, true, true);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tm + COL_AP, make_desc(sb + OFF_LS + s * 2048, 16384, 1024),
                             make_desc(sb + OFF_RT + s * 2048, 16384, 1024), id, s > 0);
                mma_commit(s_bar);
            }
            if (!wait_mma()) { aborted = true; break; }
            tc_fence_after();
            float val[32];
            tmem_ld32(tm + lane_sel + COL_AP + 32 * wg, val);
            const int i0 = 32 * wg;
            if (row < 64) {
                const int r = row;
                const float br = s_beta[r];
#pragma unroll
                for (int ii = 0; ii < 32; ++ii) Nm[r * kLd + i0 + ii] = (i0 + ii < r) ? br * val[ii] : 0.f;
            } else {
                const int r = row - 64;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint32_t pk[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const int i = i0 + 8 * qq + 2 * p;
                        pk[p] = pack_bf16(i <= r ? val[8 * qq + 2 * p] : 0.f,
                                          i + 1 <= r ? val[8 * qq + 2 * p + 1] : 0.f);
                    }
                    st16(sm, OFF_POP + kmaj_chunk(r, (i0 >> 3) + qq, 0, 64),
                         make_uint4(pk[0], pk[1], pk[2], pk[3]));
                }
            }
        } else {
            // exact A and P on CUDA cores: one warp per (r, i) pair, lanes over channels
            float* Aex = reinterpret_cast<float*>(sm + OFF_LS);
            __nv_bfloat16* Pop = reinterpret_cast<__nv_bfloat16*>(sm + OFF_POP);
            const int lane = tid & 31;
            for (int pidx = warp; pidx < kC * (kC + 1) / 2; pidx += kThreads / 32) {
                int r = (int)((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
                while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
                while (r * (r + 1) / 2 > pidx) --r;
                const int i = pidx - r * (r + 1) / 2;
                float a = 0.f, pp = 0.f;
                for (int cc = lane; cc < kD; cc += 32) {
                    const float ki = bf(Xk + i * kD + cc) * expf(Xg[r * kD + cc] - Xg[i * kD + cc]);
                    a = fmaf(bf(Xk + r * kD + cc), ki, a);
                    pp = fmaf(bf(Xq + r * kD + cc), ki, pp);
                }
                a = warp_sum(a);
                pp = warp_sum(pp);
                if (lane == 0) {
                    Aex[r * kLd + i] = a;
                    const uint32_t po = kmaj_chunk(r, i >> 3, 0, 64) + (i & 7) * 2;
                    Pop[po / 2] = __float2bfloat16_rn(pp);
                    if (i < r) {
                        const uint32_t pu = kmaj_chunk(i, r >> 3, 0, 64) + (r & 7) * 2;
                        Pop[pu / 2] = __float2bfloat16_rn(0.f);
                    }
                }
            }
            __syncthreads();
            for (int e = tid; e < kC * kC; e += kThreads) {
                const int r = e >> 6, i = e & 63;
                Nm[r * kLd + i] = (i < r) ? s_beta[r] * Aex[r * kLd + i] : 0.f;
            }
        }
        __syncthreads();

        // ================= P3: T' = (I + N)^-1 diag(beta), fp32 =================
        {
            float* Tm = reinterpret_cast<float*>(sm + OFF_XQ);
            float* Y = Tm + kC * kLd;                             // [3][16][17]
            if (tid < 64) {
                const int b = tid >> 4, i = tid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s = 0.f;
#pragma unroll
                    for (int m = 0; m < r; ++m) s = fmaf(Nm[(16 * b + r) * kLd + 16 * b + m], x[m], s);
                    x[r] = (r < i) ? 0.f : (r == i ? 1.f : -s);
                    Tm[(16 * b + r) * kLd + 16 * b + i] = x[r];
                }
            }
            __syncthreads();
            const int rr = tid >> 4, ii = tid & 15;
#pragma unroll
            for (int d = 1; d <= 3; ++d) {
                for (int b = 0; b + d <= 3; ++b) {
                    float s = 0.f;
                    for (int jb = b; jb < b + d; ++jb) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            s = fmaf(Nm[(16 * (b + d) + rr) * kLd + 16 * jb + m],
                                     Tm[(16 * jb + m) * kLd + 16 * b + ii], s);
                    }
                    Y[b * 272 + rr * 17 + ii] = s;
                }
                __syncthreads();
                for (int b = 0; b + d <= 3; ++b) {
                    float s = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        s = fmaf(Tm[(16 * (b + d) + rr) * kLd + 16 * (b + d) + m], Y[b * 272 + m * 17 + ii], s);
                    Tm[(16 * (b + d) + rr) * kLd + 16 * b + ii] = -s;
                }
                __syncthreads();
            }
            for (int e = tid; e < kC * 8; e += kThreads) {
                const int r = e >> 3, q8 = e & 7;
                uint32_t pk[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    float w2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int i = 8 * q8 + 2 * p + u;
                        w2[u] = (i < r) ? Tm[r * kLd + i] * s_beta[i] : (i == r ? s_beta[r] : 0.f);
                    }
                    pk[p] = pack_bf16(w2[0], w2[1]);
                }
                st16(sm, OFF_TOP + kmaj_chunk(r, q8, 0, 64), make_uint4(pk[0], pk[1], pk[2], pk[3]));
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ================= P4: W^T, U^T, O^T = S^T Qhat^T =================
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_kk = idesc_bf16(128, 64, false, false);
            const uint32_t id_mk = idesc_bf16(128, 64, true, false);
            const uint32_t id_km = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t bT = make_desc(sb + OFF_TOP + s * 32, 16, 1024);
                mma_bf16(tm + COL_W, make_desc(sb + OFF_KH + s * 32, 16, 1024), bT, id_kk, s > 0);
                mma_bf16(tm + COL_X, make_desc(sb + OFF_VT + s * 2048, 8192, 1024), bT, id_mk, s > 0);
            }
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tm + COL_O, make_desc(sb + OFF_ST + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                         make_desc(sb + OFF_QH + s * 2048, 16384, 1024), id_km, s > 0);
            mma_commit(s_bar);
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();

        // ================= P5: W^T -> bf16 B operand =================
        {
            float val[32];
            tmem_ld32(tm + lane_sel + COL_W + 32 * wg, val);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint4 pk;
                pk.x = pack_bf16(val[8 * qq + 0], val[8 * qq + 1]);
                pk.y = pack_bf16(val[8 * qq + 2], val[8 * qq + 3]);
                pk.z = pack_bf16(val[8 * qq + 4], val[8 * qq + 5]);
                pk.w = pack_bf16(val[8 * qq + 6], val[8 * qq + 7]);
                st16(sm, OFF_WOP + mnmaj_chunk(row, 4 * wg + qq, 0, 16), pk);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ================= P6: Ut^T = U^T - S^T W^T =================
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, true, true);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tm + COL_X, make_desc(sb + OFF_ST + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                         make_desc(sb + OFF_WOP + s * 2048, 16384, 1024), id, 1);
            mma_commit(s_bar);
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();

        // ================= P7: Ut^T -> bf16 A operand =================
        {
            float val[32];
            tmem_ld32(tm + lane_sel + COL_X + 32 * wg, val);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint4 pk;
                pk.x = pack_bf16(val[8 * qq + 0], val[8 * qq + 1]);
                pk.y = pack_bf16(val[8 * qq + 2], val[8 * qq + 3]);
                pk.z = pack_bf16(val[8 * qq + 4], val[8 * qq + 5]);
                pk.w = pack_bf16(val[8 * qq + 6], val[8 * qq + 7]);
                st16(sm, OFF_UOP + kmaj_chunk(row, 4 * wg + qq, 0, 128), pk);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ================= P8: O^T += Ut^T P^T;  dS^T = Ut^T Ktilde =================
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_s = idesc_bf16(128, 128, false, false);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t aU = make_desc(sb + OFF_UOP + s * 32, 16, 1024);
                mma_bf16(tm + COL_O, aU, make_desc(sb + OFF_POP + s * 32, 16, 1024), id_o, 1);
                mma_bf16(tm + COL_S, aU, make_desc(sb + OFF_KT + s * 32, 16, 1024), id_s, s > 0);
            }
            mma_commit(s_bar);
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();

        // ================= P9: outputs, state update =================
        {
            float val[32];
            tmem_ld32(tm + lane_sel + COL_O + 32 * wg, val);
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int r = 32 * wg + t;
                if (r < L) o[((c0 + r) * H + h) * kD + j] = __float2bfloat16_rn(scale * val[t]);
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tm + lane_sel + COL_S + 64 * wg + 32 * half, val);
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const int cc = 32 * half + t;
                    sreg[cc] = fmaf(s_eC[64 * wg + cc], sreg[cc], val[t]);
                }
            }
            write_state_operand();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (ht && !aborted) {
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) ht[sbase + (int64_t)(64 * wg + cc) * kD + j] = sreg[cc];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a) {
    return a.io == Io::BF16 && a.dk == kD && a.dv == kD && a.chunk == kC;
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, unsigned int* err, cudaStream_t stream) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<<<(unsigned)((int64_t)a.N * a.H), kThreads, kSmemBytes, stream>>>(
        static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
        static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.scale, a.h0, a.ht,
        static_cast<__nv_bfloat16*>(a.o), a.cu, a.T_pad, a.H, err);
    return cudaGetLastError();
}

}  // namespace kda
