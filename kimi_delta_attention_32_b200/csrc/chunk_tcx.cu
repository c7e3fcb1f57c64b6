// chunk_tcx.cu -- chunked KDA prefill, bf16 I/O, dk = dv = 128, chunk 64, as a producer /
// consumer pipeline inside one thread-block cluster per (sequence, head).
//
// Same per-chunk algebra as the sequential kernel (sarnas.ru, "Яндекс открыл веса
// AliceAI-Foundation-80B-A3B-Base ...", section "Что именно изменилось"; m.lqnn.cn/news/205170,
// section "KDA 与 Gated Attention ..."), with the decay folded around a per-chunk reference
// gamma_ref (the chunk middle, or the chunk start when the range test fails):
//   Lk = k e^{gamma - gamma_ref},  Lq = q e^{gamma - gamma_ref},  R = k e^{gamma_ref2 - gamma}
//   [A ; P] = [Lk ; Lq] R^T                                   (gamma_ref2 = gamma_ref)
//   T' = (I + diag(beta) A)^-1 diag(beta),   Z = Lk^T T'^T      (= e^{-gamma_ref} W^T)
//   Sm = (diag(e^{gamma_ref}) S)^T
//   Ut^T = V^T T'^T - Sm Z,   O^T = Sm Lq^T + Ut^T P^T,   dS^T = Ut^T R
//   S' = diag(e^{gamma_C}) S + diag(e^{gamma_C - gamma_ref2}) dS
// A chunk whose half-chunk decay exceeds 80 in some channel takes gamma_ref = 0 and
// gamma_ref2 = gamma_C, and forms A and P exactly on CUDA cores; every factor is then <= 1.
//
// Cluster of 4 CTAs: rank 0 is the consumer -- it owns the fp32 state and runs only the
// sequential chain (U^T, Ut^T, O^T, dS^T on tcgen05, state update); ranks 1..3 are producers,
// each preparing every third chunk (loads, cumulative decay, folded operands, A|P on
// tcgen05, fp32 triangular inverse, Z on tcgen05) and writing the chunk's operands straight
// into a two-slot ring in the consumer's shared memory over DSMEM. Flow control is by
// cluster-scope mbarriers: "full" in the consumer (one producer arrival per chunk) and
// "free" in each producer (one consumer arrival per chunk it may write). All waits are bounded.
#include "common.cuh"
#include "launchers.h"
#include "tc.cuh"
#include "tma_host.h"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr int kProducers = 3;
constexpr int kCluster = 1 + kProducers;
constexpr float kHalfRange = 80.f;
constexpr long long kWaitCycles = 4000000000LL;
constexpr int kLd = 68;                // fp32 row stride of the 64x64 scratch (16-byte rows)
constexpr int kLdY = 24;               // row stride of the per-warp 16x16 merge scratch

// ---- consumer shared memory: two ring slots, then the state operands ----
// A slot holds one chunk's operands. The order inside a slot alternates so that the wide
// MMAs see adjacent B operands matching adjacent TMEM accumulators:
//   slot 0: [Z | Lq] (MN-major, N = 128) -> [X0 | O0];  [P | R] (K-major rows, N = 192) -> [O0 | S]
//   slot 1: [Lq | Z]                      -> [O1 | X1];  [R | P]                      -> [S | O1]
constexpr uint32_t kSlotBytes = 83968;
struct SlotMap { uint32_t zo, lq, po, rt; };
__device__ __forceinline__ SlotMap slot_map(int slot) {
    return slot == 0 ? SlotMap{0u, 16384u, 32768u, 40960u} : SlotMap{16384u, 0u, 49152u, 32768u};
}
constexpr uint32_t S_TP = 57344;      // T'   : B, K-major rows token r, K = token i
constexpr uint32_t S_VT = 65536;      // V^T  : A, MN-major, K = token, M = value ch (2 blocks)
constexpr uint32_t kFacBytes = 1536;  // per chunk: eRef[128], eC[128], eCR[128] (fp32)
constexpr uint32_t C_SLOT0 = 0;
constexpr uint32_t C_ST = 2 * kSlotBytes;       // Sm  : A, K-major rows value ch, K = key ch (2 atom cols)
constexpr uint32_t C_UT = C_ST + 32768;         // Ut^T: A, K-major rows value ch, K = token
constexpr uint32_t C_FAC = C_UT + 16384;        // factor ring: chunk n in entry n % 3, so a
                                                // ring slot can be released before they are read
constexpr uint32_t C_MISC = C_FAC + 3 * kFacBytes;
// ---- producer shared memory ----
constexpr uint32_t P_XQ = 0;          // raw q [64][128] bf16
constexpr uint32_t P_XK = 16384;      // raw k [64][128] bf16
constexpr uint32_t P_LK = 32768;      // Lk: first M block of the A|P A operand; K-major A of Z
constexpr uint32_t P_HS = 49152;      // two hand-off sets (alternate tasks), each:
constexpr uint32_t H_LQ = 0;          //   Lq (second M block of the A|P A operand)
constexpr uint32_t H_RT = 16384;      //   R
constexpr uint32_t H_ZO = 32768;      //   Z (exact path: A in fp32 until the inverse starts)
constexpr uint32_t H_TP = 49152;      //   T'
constexpr uint32_t H_PO = 57344;      //   P
constexpr uint32_t H_FAC = 65536;     //   eRef, eC, eCR
constexpr uint32_t kHsBytes = 67584;
constexpr uint32_t kHandoffTx = 16384 * 3 + 8192 * 2 + 1536;   // bytes bulk-copied per chunk
constexpr uint32_t P_SCR = P_HS + 2 * kHsBytes;   // raw g / gamma [64][128] f32, then
                                                  // Nm [64][68], Tm [64][68], Y [3][16][24] (fp32)
constexpr uint32_t P_XG = P_SCR;
constexpr uint32_t P_MISC = P_SCR + 40960;
constexpr uint32_t kMiscBytes = 2560;   // barriers, beta[64], decay sums [4][128]
constexpr uint32_t kSmemBytes = (P_MISC > C_MISC ? P_MISC : C_MISC) + kMiscBytes + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(320 + 4 * 128 * 4 <= kMiscBytes, "misc area");

// misc area (relative to the role's misc base)
constexpr uint32_t M_BAR_MMA = 0;     // own MMA completions
constexpr uint32_t M_BAR_A = 8;       // consumer: full[0]; producer: free
constexpr uint32_t M_BAR_B = 16;      // consumer: full[1]
constexpr uint32_t M_TMEM = 24;
constexpr uint32_t M_TMP = 32;
constexpr uint32_t M_BAR_C = 40;      // producer: q, k tiles landed; consumer: V tile of slot 0
constexpr uint32_t M_BAR_D = 48;      // producer: g tile landed;    consumer: V tile of slot 1
constexpr uint32_t M_BETA = 64;       // producer: beta[64]
constexpr uint32_t M_GSUM = 320;      // producer: [4][128] token-quarter decay sums

// consumer TMEM columns: [X0 | O0 | S(128) | .. | O1 | X1]; producer: [A|P | Z]
constexpr uint32_t TC_X0 = 0, TC_O0 = 64, TC_S = 128, TC_O1 = 256, TC_X1 = 320, kTmemC = 512;
constexpr uint32_t TP_AP = 0, TP_Z = 64, kTmemP = 128;

struct Params {
    CUtensorMap tq, tk, tg, tv, to;   // TMA maps: q, k, o [T,H,128] bf16 and g [T,H,128] f32 in
                                      // (128, 1, 64) boxes; v in (64, 1, 64) boxes, 128B swizzle
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const float* g;
    const float* beta;
    float scale;
    const float* h0;
    float* ht;
    __nv_bfloat16* o;
    const int32_t* cu;
    int T_pad;
    int N, H;
    unsigned int* err;
};

__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ float bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                      pack_bf16(v[6], v[7]));
}

// Sequence / head of this cluster. Packed batches with at most 256 sequences are processed
// longest first: cluster u takes the sequence of descending-length rank u / H (ties by index).
// Every thread of the CTA must call this (it synchronises the CTA once).
__device__ void unit_of(const Params& p, int unit, int* s_tmp, int& n, int& h, int64_t& bos,
                        int64_t& eos) {
    h = unit % p.H;
    const int rank = unit / p.H;
    n = rank;
    if (p.cu != nullptr && p.N <= kThreads) {
        const int i = threadIdx.x;
        if (i < p.N) {
            const int li = p.cu[i + 1] - p.cu[i];
            int r = 0;
            for (int j2 = 0; j2 < p.N; ++j2) {
                const int lj = p.cu[j2 + 1] - p.cu[j2];
                r += (lj > li) || (lj == li && j2 < i);
            }
            if (r == rank) *s_tmp = i;
        }
        __syncthreads();
        n = *s_tmp;
    }
    if (p.cu == nullptr) {
        bos = (int64_t)n * p.T_pad;
        eos = bos + p.T_pad;
    } else {
        bos = p.cu[n];
        eos = p.cu[n + 1];
    }
}

// ============================== producer ==============================
__device__ void producer(const Params& p, uint8_t* sm, uint32_t sb, int prank, int h,
                         int64_t bos, int64_t eos, bool& aborted) {
    const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
    const uint32_t lane_sel = (uint32_t)(32 * (warp & 3)) << 16;
    uint8_t* misc = sm + P_MISC;
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(misc + M_BAR_MMA);
    uint64_t* bar_free = reinterpret_cast<uint64_t*>(misc + M_BAR_A);
    float* s_beta = reinterpret_cast<float*>(misc + M_BETA);
    float* s_gsum = reinterpret_cast<float*>(misc + M_GSUM);
    const uint32_t tm = *reinterpret_cast<uint32_t*>(misc + M_TMEM);
    const int H = p.H;
    const int nchunks = (int)((eos - bos + kC - 1) / kC);
    uint32_t ph_mma = 0, ph_free = 0;

    const uint32_t c_misc = map_to_rank(sb + C_MISC, 0);
    const uint32_t c_slot0 = map_to_rank(sb + C_SLOT0, 0);
    const uint32_t c_fac = map_to_rank(sb + C_FAC, 0);

    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitCycles);
        ph_mma ^= 1u;
        if (!ok) atomicOr(p.err, kErrTimeout);
        return __syncthreads_or(!ok) == 0;
    };
    // Raw q, k tiles (staging, free after the folds) and g tile (in the inverse's scratch,
    // free once T' is written) of a chunk, by TMA from one thread. Rows past the sequence are
    // masked where they are read; rows past the whole batch arrive as zeros.
    uint64_t* bar_qk = reinterpret_cast<uint64_t*>(misc + M_BAR_C);
    uint64_t* bar_g = reinterpret_cast<uint64_t*>(misc + M_BAR_D);
    uint32_t ph_qk = 0, ph_g = 0;
    auto issue_loads = [&](int64_t c0, int) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_qk, 32768u);
            tma_load_3d(sb + P_XQ, &p.tq, 0, h, (int)c0, bar_qk);
            tma_load_3d(sb + P_XK, &p.tk, 0, h, (int)c0, bar_qk);
        }
    };
    auto issue_g = [&](int64_t c0) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_g, 32768u);
            tma_load_3d(sb + P_XG, &p.tg, 0, h, (int)c0, bar_g);
        }
    };
    auto wait_load = [&](uint64_t* bar, uint32_t& ph) -> bool {
        const bool ok = mbar_wait_bounded(bar, ph, kWaitCycles);
        ph ^= 1u;
        if (!ok) atomicOr(p.err, kErrTimeout);
        return __syncthreads_or(!ok) == 0;
    };

    int n = prank - 1;
    if (n < nchunks) {
        const int64_t c0 = bos + (int64_t)n * kC;
        issue_loads(c0, 0);
        issue_g(c0);
    }
    for (int task = 0; n < nchunks && !aborted; n += kProducers, ++task) {
        const int64_t c0 = bos + (int64_t)n * kC;
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
        const int slot = n & 1;
        const uint32_t hs = P_HS + (uint32_t)(task & 1) * kHsBytes;     // this task's hand-off set
        float* fac = reinterpret_cast<float*>(sm + hs + H_FAC);
        if (tid < kC) s_beta[tid] = tid < L ? p.beta[(c0 + tid) * H + h] : 0.f;
        if (!wait_load(bar_qk, ph_qk) || !wait_load(bar_g, ph_g)) { aborted = true; break; }
        trace_mark(prank, n, 0);

        // ---- cumulative decay (thread: channels 2*cp, 2*cp+1; tokens [16*tq, 16*tq+16)) ----
        // kept in log2 units so that every decay factor is one ex2.approx
        const int cp = tid & 63, tq = tid >> 6;
        const int c = row;                      // channel owned for the factors below
        float* Xg = reinterpret_cast<float*>(sm + P_XG);
        const uint32_t* Xq2 = reinterpret_cast<const uint32_t*>(sm + P_XQ);
        const uint32_t* Xk2 = reinterpret_cast<const uint32_t*>(sm + P_XK);
        const __nv_bfloat16* Xq = reinterpret_cast<const __nv_bfloat16*>(sm + P_XQ);
        const __nv_bfloat16* Xk = reinterpret_cast<const __nv_bfloat16*>(sm + P_XK);
        constexpr float kLog2e = 1.4426950408889634f;
        float gam0[16], gam1[16];
        {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int r = 16 * tq + t;
                const float2 gv = r < L ? *reinterpret_cast<const float2*>(Xg + r * kD + 2 * cp)
                                        : make_float2(0.f, 0.f);
                a0 = fmaf(gv.x, kLog2e, a0);
                a1 = fmaf(gv.y, kLog2e, a1);
                gam0[t] = a0;
                gam1[t] = a1;
            }
            s_gsum[tq * 128 + 2 * cp] = a0;
            s_gsum[tq * 128 + 2 * cp + 1] = a1;
        }
        __syncthreads();
        float off0 = 0.f, off1 = 0.f;           // decay of the earlier token quarters
        for (int k2 = 0; k2 < tq; ++k2) { off0 += s_gsum[k2 * 128 + 2 * cp]; off1 += s_gsum[k2 * 128 + 2 * cp + 1]; }
#pragma unroll
        for (int t = 0; t < 16; ++t) { gam0[t] += off0; gam1[t] += off1; }
        // per channel c (thread row): half-chunk decays, in log2 units
        const float gA2 = s_gsum[c] + s_gsum[128 + c];                 // tokens 0..31
        const float gB2 = s_gsum[256 + c] + s_gsum[384 + c];           // tokens 32..63
        const float kHalf2 = kHalfRange * kLog2e;
        const int bad = __syncthreads_or((gA2 < -kHalf2) || (gB2 < -kHalf2));
        // references per channel pair (this thread's channels), log2 units
        const float gm0 = s_gsum[2 * cp] + s_gsum[128 + 2 * cp], gm1 = s_gsum[2 * cp + 1] + s_gsum[128 + 2 * cp + 1];
        const float gC0 = gm0 + s_gsum[256 + 2 * cp] + s_gsum[384 + 2 * cp];
        const float gC1 = gm1 + s_gsum[256 + 2 * cp + 1] + s_gsum[384 + 2 * cp + 1];
        const float gr0 = bad ? 0.f : gm0, gr1 = bad ? 0.f : gm1;      // reference for Lk / Lq
        const float gs0 = bad ? gC0 : gm0, gs1 = bad ? gC1 : gm1;      // reference for R
        if (tq == 0) {
            fac[2 * cp] = ex2_approx(gr0);
            fac[2 * cp + 1] = ex2_approx(gr1);
            fac[128 + 2 * cp] = ex2_approx(gC0);
            fac[128 + 2 * cp + 1] = ex2_approx(gC1);
            fac[256 + 2 * cp] = ex2_approx(gC0 - gs0);
            fac[256 + 2 * cp + 1] = ex2_approx(gC1 - gs1);
        }
        if (bad) {                              // natural-log gamma for the exact path
#pragma unroll
            for (int t = 0; t < 16; ++t)
                *reinterpret_cast<float2*>(Xg + (16 * tq + t) * kD + 2 * cp) =
                    make_float2(gam0[t] * (1.f / kLog2e), gam1[t] * (1.f / kLog2e));
        }
        // ---- folded operands Lk, Lq (A of A|P), R (B of A|P) ----
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
            float lk0[8], lq0[8], rr0[8], lk1[8], lq1[8], rr1[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = 8 * qq + u;
                const int r = 16 * tq + t;
                const bool ok = r < L;
                const uint32_t kw = ok ? Xk2[r * 64 + cp] : 0u, qw = ok ? Xq2[r * 64 + cp] : 0u;
                const float k0 = __uint_as_float(kw << 16), k1 = __uint_as_float(kw & 0xffff0000u);
                const float q0 = __uint_as_float(qw << 16), q1 = __uint_as_float(qw & 0xffff0000u);
                const float a0 = ex2_approx(gam0[t] - gr0), b0 = ex2_approx(gs0 - gam0[t]);
                const float a1 = ex2_approx(gam1[t] - gr1), b1 = ex2_approx(gs1 - gam1[t]);
                lk0[u] = k0 * a0; lq0[u] = q0 * a0; rr0[u] = k0 * b0;
                lk1[u] = k1 * a1; lq1[u] = q1 * a1; rr1[u] = k1 * b1;
            }
            const int ch = 2 * tq + qq;         // 8-token chunk index within the 64 tokens
            st16(sm, P_LK + mnmaj_chunk(2 * cp, ch, 0, 16), pack8(lk0));
            st16(sm, P_LK + mnmaj_chunk(2 * cp + 1, ch, 0, 16), pack8(lk1));
            st16(sm, hs + H_LQ + mnmaj_chunk(2 * cp, ch, 0, 16), pack8(lq0));
            st16(sm, hs + H_LQ + mnmaj_chunk(2 * cp + 1, ch, 0, 16), pack8(lq1));
            st16(sm, hs + H_RT + mnmaj_chunk(2 * cp, ch, 0, 16), pack8(rr0));
            st16(sm, hs + H_RT + mnmaj_chunk(2 * cp + 1, ch, 0, 16), pack8(rr1));
        }
        fence_async_smem();
        __syncthreads();
        trace_mark(prank, n, 1);

        float* Nm = reinterpret_cast<float*>(sm + P_SCR);
        __nv_bfloat16* Pop = reinterpret_cast<__nv_bfloat16*>(sm + hs + H_PO);
        if (!bad) {
            // raw inputs are no longer needed: prefetch this producer's next chunk
            if (n + kProducers < nchunks) {
                const int64_t c1 = c0 + (int64_t)kProducers * kC;
                issue_loads(c1, (int)(eos - c1 < kC ? eos - c1 : kC));
            }
            trace_mark(prank, n, 9);
            if (warp == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, true, true);
                const uint64_t a0 = make_desc(sb + P_LK, hs + H_LQ - P_LK, 1024);
                const uint64_t b0 = make_desc(sb + hs + H_RT, 16384, 1024);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    warp_mma(tm + TP_AP, desc_add(a0, s * 2048), desc_add(b0, s * 2048), id, s > 0);
                warp_commit(bar_mma);
                trace_mark(prank, n, 10);
            }
            if (!wait_mma()) { aborted = true; break; }
            trace_mark(prank, n, 2);
            tc_fence_after();
            float val[32];
            tmem_ld32(tm + lane_sel + TP_AP + 32 * wg, val);
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
                    float pv[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) pv[u] = (i0 + 8 * qq + u <= r) ? val[8 * qq + u] : 0.f;
                    st16(sm, hs + H_PO + kmaj_chunk(r, (i0 >> 3) + qq, 0, 64), pack8(pv));
                }
            }
        } else {
            // exact A and P on CUDA cores (one warp per (r, i) pair, lanes over channels)
            const int lane = tid & 31;
            for (int pidx = warp; pidx < kC * (kC + 1) / 2; pidx += kThreads / 32) {
                int r = (int)((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
                while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
                while (r * (r + 1) / 2 > pidx) --r;
                const int i = pidx - r * (r + 1) / 2;
                float a = 0.f, pp = 0.f;
                for (int cc = lane; cc < kD && r < L; cc += 32) {
                    const float ki = bf(Xk + i * kD + cc) * expf(Xg[r * kD + cc] - Xg[i * kD + cc]);
                    a = fmaf(bf(Xk + r * kD + cc), ki, a);
                    pp = fmaf(bf(Xq + r * kD + cc), ki, pp);
                }
                a = warp_sum(a);
                pp = warp_sum(pp);
                if (lane == 0) {
                    float* Aex = reinterpret_cast<float*>(sm + hs + H_ZO);     // [64][64]
                    Aex[r * 64 + i] = (i < r) ? s_beta[r] * a : 0.f;
                    Aex[i * 64 + r] = (i < r) ? 0.f : Aex[i * 64 + r];
                    Pop[(kmaj_chunk(r, i >> 3, 0, 64) + (i & 7) * 2) / 2] = __float2bfloat16_rn(pp);
                    if (i < r) Pop[(kmaj_chunk(i, r >> 3, 0, 64) + (r & 7) * 2) / 2] = __float2bfloat16_rn(0.f);
                }
            }
            __syncthreads();
            if (n + kProducers < nchunks) {
                const int64_t c1 = c0 + (int64_t)kProducers * kC;
                issue_loads(c1, (int)(eos - c1 < kC ? eos - c1 : kC));
            }
            // gamma (in the scratch) is dead: move diag(beta) A into place
            const float* Aex = reinterpret_cast<const float*>(sm + hs + H_ZO);
            for (int e = tid; e < kC * kC; e += kThreads) Nm[(e >> 6) * kLd + (e & 63)] = Aex[e];
        }
        __syncthreads();
        trace_mark(prank, n, 3);

        // ---- T' = (I + N)^-1 diag(beta) in fp32 ----
        // 16x16 diagonal blocks by column substitution (fp32), then the block merges
        // T[b+d][b] = -T[b+d][b+d] * sum_{j=b}^{b+d-1} N[b+d][j] T[j][b] as warp-level
        // tensor-core products (TF32 inputs, fp32 accumulation); T' is rounded to bf16 afterwards.
        {
            float* Tm = Nm + kC * kLd;
            float* Y = Tm + kC * kLd;                     // [3 warps][16][kLdY]
            if (tid < 64) {
                const int b = tid >> 4, i = tid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s0 = 0.f, s1 = 0.f;
#pragma unroll
                    for (int m = 0; m + 1 < r; m += 2) {
                        s0 = fmaf(Nm[(16 * b + r) * kLd + 16 * b + m], x[m], s0);
                        s1 = fmaf(Nm[(16 * b + r) * kLd + 16 * b + m + 1], x[m + 1], s1);
                    }
                    if (r & 1) s0 = fmaf(Nm[(16 * b + r) * kLd + 16 * b + r - 1], x[r - 1], s0);
                    x[r] = (r < i) ? 0.f : (r == i ? 1.f : -(s0 + s1));
                    Tm[(16 * b + r) * kLd + 16 * b + i] = x[r];
                }
            }
            __syncthreads();
            trace_mark(prank, n, 11);
            // block merges on the tensor cores: warp w < 4 - d owns block (w + d, w)
            for (int d = 1; d <= 3; ++d) {
                if (warp < 4 - d) {
                    const int b = warp, B = warp + d;
                    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    for (int jb = b; jb < B; ++jb)
                        warp_block_mma16(acc, Nm + (16 * B) * kLd + 16 * jb, kLd, Tm + (16 * jb) * kLd + 16 * b, kLd);
                    float* Yw = Y + warp * 16 * kLdY;
                    warp_block_store16(Yw, kLdY, acc, 1.f);
                    __syncwarp();
                    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                    warp_block_mma16(acc2, Tm + (16 * B) * kLd + 16 * B, kLd, Yw, kLdY);
                    warp_block_store16(Tm + (16 * B) * kLd + 16 * b, kLd, acc2, -1.f);
                }
                __syncthreads();
                if (d == 1) trace_mark(prank, n, 14);
                if (d == 3) trace_mark(prank, n, 15);
            }
            // T' = T diag(beta): 8 consecutive columns per item from two 16-byte reads
            for (int e = tid; e < kC * 8; e += kThreads) {
                const int r = e >> 3, q8 = e & 7;
                const float4 t0 = *reinterpret_cast<const float4*>(Tm + r * kLd + 8 * q8);
                const float4 t1 = *reinterpret_cast<const float4*>(Tm + r * kLd + 8 * q8 + 4);
                const float4 b0 = *reinterpret_cast<const float4*>(s_beta + 8 * q8);
                const float4 b1 = *reinterpret_cast<const float4*>(s_beta + 8 * q8 + 4);
                const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                float w8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = 8 * q8 + u;
                    w8[u] = (i < r) ? tv[u] * bv[u] : (i == r ? bv[u] : 0.f);
                }
                st16(sm, hs + H_TP + kmaj_chunk(r, q8, 0, 64), pack8(w8));
            }
        }
        __syncthreads();
        if (n + kProducers < nchunks) issue_g(c0 + (int64_t)kProducers * kC);
        trace_mark(prank, n, 4);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- Z = Lk^T T'^T ----
        if (warp == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false);
            const uint64_t a0 = make_desc(sb + P_LK, 16, 1024);
            const uint64_t b0 = make_desc(sb + hs + H_TP, 16, 1024);
#pragma unroll
            for (int s = 0; s < 4; ++s) warp_mma(tm + TP_Z, desc_add(a0, s * 32), desc_add(b0, s * 32), id, s > 0);
            warp_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        trace_mark(prank, n, 5);
        tc_fence_after();

        // ---- Z -> bf16 into the hand-off set (local), then hand the chunk over ----
        {
            float val[32];
            tmem_ld32(tm + lane_sel + TP_Z + 32 * wg, val);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
                st16(sm, hs + H_ZO + mnmaj_chunk(row, 4 * wg + qq, 0, 16), pack8(val + 8 * qq));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        trace_mark(prank, n, 12);
        if (n >= 2) {                           // ring slot n % 2 must have been released
            const bool ok = mbar_wait_cluster_bounded(bar_free, ph_free, kWaitCycles);
            ph_free ^= 1u;
            if (!ok) atomicOr(p.err, kErrTimeout);
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        trace_mark(prank, n, 6);
        if (warp == 0) {
            // one arrival announcing the bytes, then the bulk copies into the consumer's slot
            // (one per lane); together they complete that slot's "full" barrier
            const int lane = tid & 31;
            const uint32_t dst = c_slot0 + (uint32_t)slot * kSlotBytes;
            const SlotMap mp = slot_map(slot);
            const uint32_t full = c_misc + (slot ? M_BAR_B : M_BAR_A);
            // relaxed: the bytes travel in the bulk copies, which complete the barrier themselves
            if (lane == 0) mbar_arrive_expect_tx_remote_relaxed(full, kHandoffTx);
            __syncwarp();
            if (lane == 0) bulk_copy_to_peer(dst + mp.lq, sb + hs + H_LQ, 16384, full);
            if (lane == 1) bulk_copy_to_peer(dst + mp.zo, sb + hs + H_ZO, 16384, full);
            if (lane == 2) bulk_copy_to_peer(dst + mp.rt, sb + hs + H_RT, 16384, full);
            if (lane == 3) bulk_copy_to_peer(dst + S_TP, sb + hs + H_TP, 8192, full);
            if (lane == 4) bulk_copy_to_peer(dst + mp.po, sb + hs + H_PO, 8192, full);
            if (lane == 5) bulk_copy_to_peer(c_fac + (uint32_t)(n % 3) * kFacBytes, sb + hs + H_FAC, kFacBytes, full);
        }
        trace_mark(prank, n, 7);
    }
}

// ============================== consumer ==============================
__device__ void consumer(const Params& p, uint8_t* sm, uint32_t sb, int n_seq, int h,
                         int64_t bos, int64_t eos, bool& aborted) {
    const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, j = tid & 127;
    const uint32_t lane_sel = (uint32_t)(32 * (warp & 3)) << 16;
    uint8_t* misc = sm + C_MISC;
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(misc + M_BAR_MMA);
    uint64_t* bar_full0 = reinterpret_cast<uint64_t*>(misc + M_BAR_A);
    uint64_t* bar_full1 = reinterpret_cast<uint64_t*>(misc + M_BAR_B);
    const uint32_t tm = *reinterpret_cast<uint32_t*>(misc + M_TMEM);
    const int H = p.H;
    const int nchunks = (int)((eos - bos + kC - 1) / kC);
    uint32_t ph_mma = 0, ph_full0 = 0, ph_full1 = 0;   // scalars: no run-time indexed arrays
    const int64_t sbase = ((int64_t)n_seq * H + h) * kD * kD;

    float sreg[64];                     // S[64*wg + cc][j]
#pragma unroll
    for (int cc = 0; cc < 64; ++cc)
        sreg[cc] = p.h0 ? p.h0[sbase + (int64_t)(64 * wg + cc) * kD + j] : 0.f;

    // V tile of chunk nn into its slot by TMA: two (64 channels x 64 tokens) boxes whose
    // 128B-swizzled image is exactly the MN-major operand layout. Rows past the sequence do
    // not matter (the matching columns of T' are zero).
    uint64_t* bar_v0 = reinterpret_cast<uint64_t*>(misc + M_BAR_C);
    uint64_t* bar_v1 = reinterpret_cast<uint64_t*>(misc + M_BAR_D);
    uint32_t ph_v0 = 0, ph_v1 = 0;
    auto issue_v = [&](int nn) {
        if (tid == 0) {
            uint64_t* bv = (nn & 1) ? bar_v1 : bar_v0;
            const uint32_t base = sb + C_SLOT0 + (nn & 1) * kSlotBytes + S_VT;
            const int c0 = (int)(bos + (int64_t)nn * kC);
            mbar_arrive_expect_tx(bv, 16384u);
            tma_load_3d(base, &p.tv, 0, h, c0, bv);
            tma_load_3d(base + 8192, &p.tv, 64, h, c0, bv);
        }
    };
    auto wait_v = [&](int nn) -> bool {
        const int sl = nn & 1;
        const bool ok = mbar_wait_bounded(sl ? bar_v1 : bar_v0, sl ? ph_v1 : ph_v0, kWaitCycles);
        if (sl) ph_v1 ^= 1u; else ph_v0 ^= 1u;
        if (!ok) atomicOr(p.err, kErrTimeout);
        return __syncthreads_or(!ok) == 0;
    };
    // Output epilogue: O of chunk nn goes from TMEM to a row-major [token][channel] bf16
    // staging tile (the Ut^T buffer, free once the chunk's last MMAs completed), then to HBM
    // as one TMA tile store (a ragged last chunk: one bulk copy per valid token, so rows of the
    // next sequence are never touched), overlapping the next chunk.
    float oval[32];
    auto load_o = [&](int nn) { tmem_ld32(tm + lane_sel + ((nn & 1) ? TC_O1 : TC_O0) + 32 * wg, oval); };
    auto stage_o = [&]() {
        __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(sm + C_UT);
#pragma unroll
        for (int t = 0; t < 32; ++t) st[(32 * wg + t) * kD + j] = __float2bfloat16_rn(p.scale * oval[t]);
    };
    auto store_o = [&](int nn) {               // warp 1, after the staging writes are fenced
        const int64_t c0 = bos + (int64_t)nn * kC;
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
        const int lane = tid & 31;
        if (L == kC) {
            if (lane == 0) tma_store_3d(&p.to, 0, h, (int)c0, sb + C_UT);
        } else {
            for (int r = lane; r < L; r += 32)
                bulk_store(p.o + ((c0 + r) * H + h) * kD, sb + C_UT + r * 256, 256);
        }
        bulk_commit();
    };
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitCycles);
        ph_mma ^= 1u;
        if (!ok) atomicOr(p.err, kErrTimeout);
        return __syncthreads_or(!ok) == 0;
    };
    auto wait_full = [&](int nn) -> bool {
        const int sl = nn & 1;
        const bool ok = mbar_wait_cluster_bounded(sl ? bar_full1 : bar_full0,
                                                  sl ? ph_full1 : ph_full0, kWaitCycles);
        if (sl) ph_full1 ^= 1u; else ph_full0 ^= 1u;
        if (!ok) atomicOr(p.err, kErrTimeout);
        return __syncthreads_or(!ok) == 0;
    };
    // -U^T = -(V^T T'^T) of chunk nn into its X accumulator (one converged warp).
    auto issue_u = [&](int nn) {
        const uint32_t so = C_SLOT0 + (nn & 1) * kSlotBytes;
        tc_fence_after();
        const uint32_t id_u = idesc_bf16(128, 64, true, false, true);
        const uint64_t a0 = make_desc(sb + so + S_VT, 8192, 1024);
        const uint64_t b0 = make_desc(sb + so + S_TP, 16, 1024);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            warp_mma(tm + ((nn & 1) ? TC_X1 : TC_X0), desc_add(a0, s * 2048), desc_add(b0, s * 32), id_u, s > 0);
    };
    // Sm(nn) = (diag(e^{gamma_ref(nn)}) S)^T as the bf16 A operand (S already updated).
    auto write_sm = [&](int nn) {
        const float* fac = reinterpret_cast<const float*>(sm + C_FAC + (nn % 3) * kFacBytes);
        const float4* fac4 = reinterpret_cast<const float4*>(fac + 64 * wg);
#pragma unroll
        for (int qq = 0; qq < 8; ++qq) {
            const float4 e0 = fac4[2 * qq], e1 = fac4[2 * qq + 1];
            const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
            float w8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) w8[u] = sreg[8 * qq + u] * ev[u];
            st16(sm, C_ST + kmaj_chunk(j, qq, wg, 128), pack8(w8));
        }
    };

    // prologue: operands of chunk 0 (and the V tile of chunk 1)
    if (nchunks > 0) {
        issue_v(0);
        if (nchunks > 1) issue_v(1);
        if (!wait_v(0)) aborted = true;
        if (!aborted && !wait_full(0)) aborted = true;
        if (!aborted) {
            write_sm(0);
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (warp == 0) issue_u(0);
        }
    }

    for (int n = 0; n < nchunks && !aborted; ++n) {
        const int slot = n & 1;
        const uint32_t so = C_SLOT0 + slot * kSlotBytes;
        const SlotMap mp = slot_map(slot);
        const float* fac = reinterpret_cast<const float*>(sm + C_FAC + (n % 3) * kFacBytes);
        const uint32_t tX = slot ? TC_X1 : TC_X0;
        trace_mark(0, n, 0);

        // ---- [X | O] (+)= Sm [Z | Lq]: X = -Ut^T, O = Sm Lq^T ----
        if (warp == 0) {
            tc_fence_after();
            const uint32_t id64 = idesc_bf16(128, 64, false, true);
            const uint32_t id128 = idesc_bf16(128, 128, false, true);
            const uint64_t aS = make_desc(sb + C_ST, 16, 1024);
            const uint64_t bZ = make_desc(sb + so + mp.zo, 16384, 1024);
            const uint64_t bQ = make_desc(sb + so + mp.lq, 16384, 1024);
            // first K step: X accumulates onto -U^T, O starts from zero
            warp_mma(tm + tX, aS, bZ, id64, 1);
            warp_mma(tm + (slot ? TC_O1 : TC_O0), aS, bQ, id64, 0);
            const uint64_t bW = slot ? bQ : bZ;           // the lower of the two adjacent B blocks
            const uint32_t dW = slot ? TC_O1 : TC_X0;
#pragma unroll
            for (int s = 1; s < 8; ++s)
                warp_mma(tm + dW, desc_add(aS, (s >> 2) * 16384 + (s & 3) * 32), desc_add(bW, s * 2048), id128, 1);
            warp_commit(bar_mma);
        }
        trace_mark(0, n, 1);
        // the staging tile of O(n - 1) is rewritten below: its TMA store must have read it
        if (warp == 1) bulk_wait_read0();
        trace_mark(0, n, 2);
        if (!wait_mma()) { aborted = true; break; }
        trace_mark(0, n, 10);
        tc_fence_after();
        {
            float val[32];
            tmem_ld32(tm + lane_sel + tX + 32 * wg, val);
#pragma unroll
            for (int t = 0; t < 32; ++t) val[t] = -val[t];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) st16(sm, C_UT + kmaj_chunk(j, 4 * wg + qq, 0, 128), pack8(val + 8 * qq));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        trace_mark(0, n, 3);

        // ---- [O | dS^T] (+)= Ut^T [P | R] ----
        if (warp == 0) {
            tc_fence_after();
            const uint32_t id64 = idesc_bf16(128, 64, false, false);
            const uint32_t id128 = idesc_bf16(128, 128, false, false);
            const uint32_t id192 = idesc_bf16(128, 192, false, false);
            const uint64_t aU = make_desc(sb + C_UT, 16, 1024);
            const uint64_t bP = make_desc(sb + so + mp.po, 16, 1024);
            const uint64_t bR = make_desc(sb + so + mp.rt, 16, 1024);
            warp_mma(tm + (slot ? TC_O1 : TC_O0), aU, bP, id64, 1);
            warp_mma(tm + TC_S, aU, bR, id128, 0);
            const uint64_t bW = slot ? bR : bP;
            const uint32_t dW = slot ? TC_S : TC_O0;
#pragma unroll
            for (int s = 1; s < 4; ++s) warp_mma(tm + dW, desc_add(aU, s * 32), desc_add(bW, s * 32), id192, 1);
            warp_commit(bar_mma);
        }
        // the V tile of this slot was consumed by -U^T (complete): fetch the one of chunk n + 2
        if (n + 2 < nchunks) issue_v(n + 2);
        trace_mark(0, n, 4);
        if (!wait_mma()) { aborted = true; break; }
        // every MMA that reads ring slot n % 2 has completed (the chunk's factors live in the
        // factor ring): tell the producer of chunk n + 2 it may write the slot
        if (tid == 0 && n + 2 < nchunks)
            mbar_arrive_remote_relaxed(map_to_rank(sb + P_MISC + M_BAR_A, 1 + (n + 2) % kProducers));
        trace_mark(0, n, 5);
        const bool more = n + 1 < nchunks;
        if (more) {
            // operands of chunk n + 1 (its V tile was requested one chunk earlier)
            if (!wait_v(n + 1)) { aborted = true; break; }
            if (!wait_full(n + 1)) { aborted = true; break; }
        }
        trace_mark(0, n, 6);
        tc_fence_after();
        {
            float val[32];
            const float4* eC4 = reinterpret_cast<const float4*>(fac + 128 + 64 * wg);
            const float4* eR4 = reinterpret_cast<const float4*>(fac + 256 + 64 * wg);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tm + lane_sel + TC_S + 64 * wg + 32 * half, val);
#pragma unroll
                for (int t4 = 0; t4 < 8; ++t4) {
                    const float4 ec = eC4[8 * half + t4], er = eR4[8 * half + t4];
                    const float ecv[4] = {ec.x, ec.y, ec.z, ec.w}, erv[4] = {er.x, er.y, er.z, er.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int cc = 32 * half + 4 * t4 + u;
                        sreg[cc] = fmaf(ecv[u], sreg[cc], erv[u] * val[4 * t4 + u]);
                    }
                }
            }
        }
        load_o(n);
        stage_o();
        if (more) write_sm(n + 1);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        trace_mark(0, n, 7);
        if (more && warp == 0) issue_u(n + 1);
        if (warp == 1) store_o(n);
    }
    if (warp == 1) bulk_wait0();
    if (p.ht && !aborted) {
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) p.ht[sbase + (int64_t)(64 * wg + cc) * kD + j] = sreg[cc];
    }
}

__global__ void __launch_bounds__(kThreads, 1) chunk_tcx_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    const int warp = threadIdx.x >> 5;
    const uint32_t crank = cluster_rank();
    const bool is_consumer = (crank == 0);
    uint8_t* misc = sm + (is_consumer ? C_MISC : P_MISC);

    int n_seq, h;
    int64_t bos, eos;
    unit_of(p, (int)(blockIdx.x / kCluster), reinterpret_cast<int*>(misc + M_TMP), n_seq, h, bos, eos);

    const uint32_t ncols = is_consumer ? kTmemC : kTmemP;
    if (warp == 0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), ncols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(reinterpret_cast<uint64_t*>(misc + M_BAR_MMA), 1);
        // consumer "full" barriers: one producer arrival + the bulk bytes; producer "free"
        // barrier: one consumer arrival
        mbar_init(reinterpret_cast<uint64_t*>(misc + M_BAR_A), 1);
        mbar_init(reinterpret_cast<uint64_t*>(misc + M_BAR_B), 1);
        mbar_init(reinterpret_cast<uint64_t*>(misc + M_BAR_C), 1);
        mbar_init(reinterpret_cast<uint64_t*>(misc + M_BAR_D), 1);
    }
    tc_fence_before();
    cluster_sync();                     // barriers of every CTA exist before any remote arrive
    tc_fence_after();

    bool aborted = false;
    if (is_consumer) consumer(p, sm, sb, n_seq, h, bos, eos, aborted);
    else producer(p, sm, sb, (int)crank, h, bos, eos, aborted);

    tc_fence_before();
    __syncthreads();
    cluster_sync();                     // no CTA leaves while a peer may still write to it
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*reinterpret_cast<uint32_t*>(misc + M_TMEM), ncols);
    }
}

}  // namespace

cudaError_t launch_chunk_tcx(const ChunkArgs& a, unsigned int* err, cudaStream_t stream) {
    const int64_t units = (int64_t)a.N * a.H;
    if (units == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(chunk_tcx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    Params p;
    const bool maps_ok =
        make_tmap_thd(&p.tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.T_tot, a.H, kD, kD, kC, false) &&
        make_tmap_thd(&p.tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.T_tot, a.H, kD, kD, kC, false) &&
        make_tmap_thd(&p.tg, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.T_tot, a.H, kD, kD, kC, false) &&
        make_tmap_thd(&p.tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.T_tot, a.H, kD, 64, kC, true) &&
        make_tmap_thd(&p.to, a.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.T_tot, a.H, kD, kD, kC, false);
    if (!maps_ok) return cudaErrorInvalidValue;
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.v = static_cast<const __nv_bfloat16*>(a.v);
    p.g = a.g;
    p.beta = a.beta;
    p.scale = a.scale;
    p.h0 = a.h0;
    p.ht = a.ht;
    p.o = static_cast<__nv_bfloat16*>(a.o);
    p.cu = a.cu;
    p.T_pad = a.T_pad;
    p.N = a.N;
    p.H = a.H;
    p.err = err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * kCluster), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, chunk_tcx_kernel, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace kda

#ifdef KDA_TRACE
// Copies the prefill phase timestamps (see trace_mark) to `host` (4 * 512 * 16 uint64).
extern "C" __attribute__((visibility("default"))) int kda_trace_dump(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, kda::g_trace, sizeof(kda::g_trace));
}
#endif
