// chunk_tcx.cu -- chunked KDA prefill, bf16 I/O, dk = dv = 128, chunk 64, as a producer /
// consumer pipeline inside one thread-block cluster per (sequence, head).
//
// The recurrence (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...", section
// "Что именно изменилось"; m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...") is
// linear in the state, so one chunk maps the state at its start, S, to the state at its end by
// S' = M S + N with M, N built from the chunk's inputs alone. This kernel splits along that
// line: producers build the chunk's factors, which do not depend on S; the consumer applies
// them. With gamma the within-chunk cumulative log-decay, gamma_C its last row and gamma_ref a
// per-chunk reference (the chunk middle, or 0 when a half chunk decays by more than 80 in some
// channel), per chunk:
//   Lk = k e^{gamma - gamma_ref},  Lq = q e^{gamma - gamma_ref}
//   R = k e^{gamma_ref - gamma},   Rh = k e^{gamma_C - gamma}              (every Rh <= |k|)
//   [A ; P] = [Lk ; Lq] R^T   (strictly / inclusively lower triangular parts)
//   T' = (I + diag(beta) A)^-1 diag(beta)
//   Yh^T = Rh^T T',  Wh^T = P T'
// and with Sm = S^T diag(e^{gamma_ref}) (bf16), on the consumer:
//   X = Sm Lk^T,  U = V^T - X                            (the part of V the state misses)
//   S'^T = S^T diag(e^{gamma_C}) + U Yh                  (fp32 state, fp32 decay term)
//   O^T  = scale (Sm Lq^T + U Wh)
// A chunk that fails the range test forms A and P exactly on CUDA cores (gamma_ref = 0, so
// every factor is <= 1).
//
// Cluster of 4 CTAs: rank 0 is the consumer, ranks 1..3 are producers, each preparing every
// third chunk. Per chunk the consumer runs two tensor-core groups with the A operand in tensor
// memory: Sm [Lk^T | Lq^T] into [X | O], then, once U is written back, U [Yh | Wh] into the
// state delta and O. It keeps the fp32 state in registers; O leaves through a TMA store. A
// chunk's factors (57 KB) travel through L2, not DSMEM (bulk copies between SMs of a cluster
// move ~30-60 GB/s, TMA loads from L2 150-220 GB/s): the producer bulk-stores them into a
// six-slot ring in global memory owned by the consumer's SM (Lk and Lq straight from its own
// A|P operand tiles, which have the consumer's layout), and the consumer TMA-loads them two
// chunks ahead into a two-slot ring in its shared memory. Only the flags use cluster
// barriers: "gfull" (ring slot written) in the consumer, "gfree" (ring slot read) in each
// producer. Every wait is bounded.
#include "common.cuh"
#include "launchers.h"
#include "tc.cuh"
#include "tma_host.h"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 512;          // 16 warps: latency hiding for the CUDA-core phases
constexpr int kProducers = 3;
constexpr int kCluster = 1 + kProducers;
constexpr float kHalfRange = 80.f;
constexpr long long kWaitCycles = 4000000000LL;
constexpr int kLd = 68;                // fp32 row stride of the 64x64 scratch (16-byte rows)
constexpr int kLdY = 24;               // row stride of the per-warp 16x16 merge scratch

// ---- one chunk's hand-off (identical image in a global ring slot and a consumer slot) ----
constexpr uint32_t S_LK = 0;          // [Lk | Lq]: MN-major (K = key ch, N = token), two
constexpr uint32_t S_LQ = 16384;      //   64-wide N atoms; the producer's A|P operand image
constexpr uint32_t S_YW = 32768;      // [Yh^T (rows key ch 0..127) | Wh^T (rows token 0..63)]:
                                      //   K-major (K = token), one 128B-swizzled atom column
constexpr uint32_t S_FAC = 57344;     // e^{gamma_ref}[128], e^{gamma_C}[128] (fp32)
constexpr uint32_t kSlotBytes = 58368;
constexpr int kRing = 6;                                // global ring slots per consumer SM

// ---- consumer shared memory ----
constexpr uint32_t C_SLOT0 = 0;                       // two slots
constexpr uint32_t C_V = 2 * kSlotBytes;              // V ring, 3 x (two 64-ch SW128 boxes)
constexpr uint32_t C_OST = C_V + 3 * 16384;           // O staging [64 tokens][128 ch] bf16
constexpr uint32_t C_MISC = C_OST + 16384;
// ---- producer shared memory ----
constexpr uint32_t P_X = 0;           // raw q, k [64][128] bf16 (folds), then the inverse's
                                      // scratch Nm, Tm [64][68], Y [3][16][24] (fp32)
constexpr uint32_t P_LK = 40960;      // Lk : rows key ch, N = token (A|P A block 0, MN-major)
constexpr uint32_t P_LQ = 57344;      // Lq : same layout (A|P A block 1)
constexpr uint32_t P_RT = 73728;      // R  : B of A|P. Raw g (fp32, 32 KB) spans P_RT..P_RH
constexpr uint32_t P_RH = 90112;      // Rh : K-major A of Yh^T
constexpr uint32_t P_PO = 106496;     // P' : rows token, K = token (K-major A of Wh^T; the
                                      //      M = 128 padding rows read T' below)
constexpr uint32_t P_TP = 114688;     // T' : rows token, columns token (MN-major B)
constexpr uint32_t P_AEX = 122880;    // exact path: diag(beta) A, fp32 [64][64]
constexpr uint32_t P_GX = 139264;     // exact path: natural-log gamma, fp32 [64][128]
constexpr uint32_t P_ST = 172032;     // hand-off staging: [Yh^T | Wh^T], then the factors
constexpr uint32_t P_MISC = P_ST + (kSlotBytes - S_YW);
constexpr uint32_t kMiscBytes = 2560;
constexpr uint32_t kSmemBytes = (P_MISC > C_MISC ? P_MISC : C_MISC) + kMiscBytes + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(2 * kC * kLd * 4 + 4 * 16 * kLdY * 4 <= P_LK, "inverse scratch");
static_assert(P_LQ - P_LK == S_LQ - S_LK && S_LQ + 16384 == S_YW && S_FAC - S_YW == 24576 &&
              P_GX + kC * kD * 4 <= P_ST, "producer layout");
static_assert(kSlotBytes % 1024 == 0 && S_FAC + 1024 <= kSlotBytes, "slot layout");

// misc areas: 16 mbarriers at 8-byte steps, then scalars
constexpr uint32_t kBars = 16;
constexpr uint32_t M_TMEM = 128;
constexpr uint32_t M_TMP = 132;       // unit_of scratch
constexpr uint32_t M_SMID = 136;      // consumer: its SM id (selects the global ring)
// consumer
constexpr uint32_t M_BAR_S = 0;       // U Yh (the state delta) done
constexpr uint32_t M_BAR_O = 8;       // U Wh (the output) done
constexpr uint32_t M_LFULL = 16;      // shared slot [2] loaded from the ring
constexpr uint32_t M_BAR_V = 32;      // V ring [3]
constexpr uint32_t M_BAR_X = 56;      // Sm [Lk^T | Lq^T] done
constexpr uint32_t M_GFULL = 80;      // global ring slot [kRing] written (producer arrival)
// producer
constexpr uint32_t M_BAR_MMA = 0;
constexpr uint32_t M_BAR_QK = 8;
constexpr uint32_t M_BAR_G = 16;
constexpr uint32_t M_GFREE = 24;      // [kRing] per ring slot: its previous chunk was read (one barrier
                                      // per slot, so arrivals for later chunks never overrun)
constexpr uint32_t M_BETA = 192;      // beta[64]
constexpr uint32_t M_GSUM = 448;      // [4][128] token-quarter decay sums
static_assert(M_GSUM + 4 * 128 * 4 <= kMiscBytes && M_GFULL + 8 * kRing <= 8 * kBars &&
              M_GFREE + 8 * kRing <= M_GFULL && M_BAR_X + 8 <= M_GFULL, "misc area");

// consumer TMEM columns: [X | O] (64 + 64) for even and odd chunks, the state delta (128),
// Sm (64 columns of bf16 pairs), U (32 columns of bf16 pairs)
constexpr uint32_t TXO0 = 0, TXO1 = 128, TC_DS = 256, TC_SM = 384, TC_U = 448, kTmemC = 512;
// producer TMEM columns
constexpr uint32_t TP_AP = 0, TP_Y = 64, TP_W = 128, kTmemP = 256;

struct Params {
    CUtensorMap tq, tk, tg, tv, to;   // TMA maps: q, k, o [T,H,128] bf16 and g [T,H,128] f32 in
                                      // (128, 1, 64) boxes; v in (64, 1, 64) boxes, 128B swizzle
    const float* beta;
    float scale;
    const float* h0;
    float* ht;
    __nv_bfloat16* o;
    const int32_t* cu;
    uint8_t* ring;                    // workspace: ring_sms x kRing x kSlotBytes
    int ring_sms;
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

// Block-wide bounded wait for the phase of `bar` with the given parity: one thread polls (the
// other 15 warps sleep in the block barrier instead of taking issue slots from the warp that
// issues MMAs); false for every thread if the wait gave up.
constexpr int kPoller = kThreads - 32;
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, bool cluster_scope,
                                           unsigned int* err) {
    int fail = 0;
    if (threadIdx.x == kPoller) {
        const bool ok = cluster_scope ? mbar_wait_cluster_bounded(bar, parity, kWaitCycles)
                                      : mbar_wait_bounded(bar, parity, kWaitCycles);
        if (!ok) {
            atomicOr(err, kErrTimeout);
            fail = 1;
        }
    }
    return __syncthreads_or(fail) == 0;
}

// The same with a flag of the caller's that is OR-ed into the result.
__device__ __forceinline__ bool block_wait_or(uint64_t* bar, uint32_t parity, int fail,
                                              unsigned int* err) {
    if (threadIdx.x == kPoller && !mbar_wait_bounded(bar, parity, kWaitCycles)) {
        atomicOr(err, kErrTimeout);
        fail = 1;
    }
    return __syncthreads_or(fail) == 0;
}
// Named barrier 1 over warps 1..15 (warp 0 issues the consumer's MMAs meanwhile), with an
// OR-reduction of `pred`.
constexpr int kGroupThreads = kThreads - 32;
__device__ __forceinline__ int group_sync_or(int pred) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, 1, %2, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred), "n"(kGroupThreads)
        : "memory");
    return r;
}
__device__ __forceinline__ void group_sync() {
    asm volatile("barrier.cta.sync 1, %0;" ::"n"(kGroupThreads) : "memory");
}
// Bounded wait of warps 1..15 for up to two barriers (the poller is in warp 15).
__device__ __forceinline__ bool group_wait(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1,
                                           unsigned int* err) {
    int fail = 0;
    if (threadIdx.x == kPoller) {
        const bool ok = mbar_wait_bounded(b0, p0, kWaitCycles) &&
                        (b1 == nullptr || mbar_wait_bounded(b1, p1, kWaitCycles));
        if (!ok) {
            atomicOr(err, kErrTimeout);
            fail = 1;
        }
    }
    return group_sync_or(fail) == 0;
}
// Bounded wait of warp 0 on its own (every lane observes the barrier).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned int* err) {
    const bool ok = mbar_wait_bounded(bar, parity, kWaitCycles);
    if (!ok && (threadIdx.x & 31) == 0) atomicOr(err, kErrTimeout);
    return __all_sync(0xffffffffu, ok);
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

// Exact A and P on CUDA cores for a chunk whose decay fails the range test (one warp per (r, i)
// pair, lanes over channels): A (times beta) into an fp32 [64][64] scratch, P into its bf16
// operand. Rare, so kept out of line, away from the common path's
// instruction stream. Every thread of the CTA calls it.
__device__ __noinline__ void exact_ap(uint8_t* sm, const float* s_beta, int L) {
    const int tid = threadIdx.x, warp = tid >> 5;
    const __nv_bfloat16* Xq = reinterpret_cast<const __nv_bfloat16*>(sm + P_X);
    const __nv_bfloat16* Xk = reinterpret_cast<const __nv_bfloat16*>(sm + P_X + 16384);
    __nv_bfloat16* Pop = reinterpret_cast<__nv_bfloat16*>(sm + P_PO);
    const float* Gx = reinterpret_cast<const float*>(sm + P_GX);
    float* Aex = reinterpret_cast<float*>(sm + P_AEX);              // [64][64]
    const int lane = tid & 31;
    for (int pidx = warp; pidx < kC * (kC + 1) / 2; pidx += kThreads / 32) {
        int r = (int)((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
        while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
        while (r * (r + 1) / 2 > pidx) --r;
        const int i = pidx - r * (r + 1) / 2;
        float a = 0.f, pp = 0.f;
        for (int cc = lane; cc < kD && r < L; cc += 32) {
            const float ki = bf(Xk + i * kD + cc) * expf(Gx[r * kD + cc] - Gx[i * kD + cc]);
            a = fmaf(bf(Xk + r * kD + cc), ki, a);
            pp = fmaf(bf(Xq + r * kD + cc), ki, pp);
        }
        a = warp_sum(a);
        pp = warp_sum(pp);
        if (lane == 0) {
            Aex[r * 64 + i] = (i < r) ? s_beta[r] * a : 0.f;
            Aex[i * 64 + r] = (i < r) ? 0.f : Aex[i * 64 + r];
            Pop[(kmaj_chunk(r, i >> 3, 0, 64) + (i & 7) * 2) / 2] = __float2bfloat16_rn(pp);
            if (i < r) Pop[(kmaj_chunk(i, r >> 3, 0, 64) + (r & 7) * 2) / 2] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();
}

// ============================== producer ==============================
__device__ void producer(const Params& p, uint8_t* sm, uint32_t sb, int prank, int h,
                         int64_t bos, int64_t eos, bool& aborted) {
    const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
    const uint32_t lane_sel = (uint32_t)(32 * (warp & 3)) << 16;
    uint8_t* misc = sm + P_MISC;
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(misc + M_BAR_MMA);
    uint64_t* bar_qk = reinterpret_cast<uint64_t*>(misc + M_BAR_QK);
    uint64_t* bar_g = reinterpret_cast<uint64_t*>(misc + M_BAR_G);
    uint64_t* bar_gfree = reinterpret_cast<uint64_t*>(misc + M_GFREE);
    float* s_beta = reinterpret_cast<float*>(misc + M_BETA);
    float* s_gsum = reinterpret_cast<float*>(misc + M_GSUM);
    const uint32_t tm = *reinterpret_cast<uint32_t*>(misc + M_TMEM);
    const int H = p.H;
    const int nchunks = (int)((eos - bos + kC - 1) / kC);
    uint32_t ph_mma = 0, ph_qk = 0, ph_g = 0, ph_gfree = 0;   // ph_gfree: bit per ring slot

    const uint32_t c_misc = map_to_rank(sb + C_MISC, 0);
    uint8_t* ring = p.ring + (size_t)ld_cluster_u32(c_misc + M_SMID) * (kRing * kSlotBytes);
    // Chunk whose ring stores were issued but not yet announced (-1: none). Thread 0 stores a
    // chunk as two bulk groups, [Lk | Lq] from the A|P operand tiles right after the folds and
    // [Yh^T | Wh^T | factors] from the staging at the end of the task, and announces it in the
    // producer's next task once only that task's first group may still be in flight: it
    // then arrives on the consumer's "gfull" barrier of that ring slot.
    int pending = -1;
    auto announce = [&](bool last) {
        if (tid == 0 && pending >= 0) {
            if (last) bulk_wait0();
            else asm volatile("cp.async.bulk.wait_group 1;" ::: "memory");
            fence_proxy_async_global();
            mbar_arrive_remote(c_misc + M_GFULL + 8u * (uint32_t)(pending % kRing));
        }
        pending = -1;
    };

    auto wait_local = [&](uint64_t* bar, uint32_t& ph) -> bool {
        const bool ok = block_wait(bar, ph, false, p.err);
        ph ^= 1u;
        return ok;
    };
    // raw q, k tiles of a chunk (into P_X) and its g tile (into P_RT..P_RH), by TMA from one
    // thread. Rows past the sequence are masked where they are read; rows past the whole
    // batch arrive as zeros.
    auto issue_qk = [&](int64_t c0) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_qk, 32768u);
            tma_load_3d(sb + P_X, &p.tq, 0, h, (int)c0, bar_qk);
            tma_load_3d(sb + P_X + 16384, &p.tk, 0, h, (int)c0, bar_qk);
        }
    };
    auto issue_g = [&](int64_t c0) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_g, 32768u);
            tma_load_3d(sb + P_RT, &p.tg, 0, h, (int)c0, bar_g);
        }
    };

    int n = prank - 1;
    float beta_nx = 0.f;                    // beta of the next task, loaded a task ahead
    if (n < nchunks) {
        const int64_t c0 = bos + (int64_t)n * kC;
        issue_qk(c0);
        issue_g(c0);
        if (tid < kC && c0 + tid < eos) beta_nx = p.beta[(c0 + tid) * H + h];
    }
    for (int task = 0; n < nchunks && !aborted; n += kProducers, ++task) {
        const int64_t c0 = bos + (int64_t)n * kC;
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
        const bool has_next = n + kProducers < nchunks;
        const int64_t c_next = c0 + (int64_t)kProducers * kC;
        trace_mark(prank, n, 14);
        if (tid < kC) s_beta[tid] = beta_nx;    // (zero past the sequence)
        beta_nx = 0.f;
        if (has_next && tid < kC && c_next + tid < eos) beta_nx = p.beta[(c_next + tid) * H + h];
        if (!wait_local(bar_qk, ph_qk) || !wait_local(bar_g, ph_g)) { aborted = true; break; }
        // ring slot n % kRing must have been read by the consumer (chunk n - kRing)
        if (n >= kRing) {
            const int rs = n % kRing;
            const bool ok = block_wait(bar_gfree + rs, (ph_gfree >> rs) & 1u, true, p.err);
            ph_gfree ^= 1u << rs;
            if (!ok) { aborted = true; break; }
        }
        uint8_t* slot = ring + (size_t)(n % kRing) * kSlotBytes;
        // the previous task's [Lk | Lq] store must have read the operand tiles before the folds
        // below overwrite them (its second group may still be in flight)
        if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        trace_mark(prank, n, 0);

        // ---- cumulative decay (thread: channel c = row, tokens [16*qt, 16*qt + 16)) ----
        // kept in log2 units so that every decay factor is one ex2.approx. Lanes run over
        // consecutive channels, so every 16-byte store below hits 8 distinct swizzled bank groups.
        const int c = row, qt = wg;
        const float* Xg = reinterpret_cast<const float*>(sm + P_RT);
        const __nv_bfloat16* Xq = reinterpret_cast<const __nv_bfloat16*>(sm + P_X);
        const __nv_bfloat16* Xk = reinterpret_cast<const __nv_bfloat16*>(sm + P_X + 16384);
        constexpr float kLog2e = 1.4426950408889634f;
        float gam[16];
        {
            float a0 = 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int r = 16 * qt + t;
                a0 = fmaf(r < L ? Xg[r * kD + c] : 0.f, kLog2e, a0);
                gam[t] = a0;
            }
            s_gsum[qt * 128 + c] = a0;
        }
        __syncthreads();                        // the g tile is dead from here on
        const float q0s = s_gsum[c], q1s = s_gsum[128 + c], q2s = s_gsum[256 + c], q3s = s_gsum[384 + c];
        const float off = qt == 0 ? 0.f : (qt == 1 ? q0s : (qt == 2 ? q0s + q1s : q0s + q1s + q2s));
#pragma unroll
        for (int t = 0; t < 16; ++t) gam[t] += off;
        const float gA = q0s + q1s, gB = q2s + q3s;           // half-chunk decays (log2)
        const float kHalf2 = kHalfRange * kLog2e;
        const int bad = __syncthreads_or((gA < -kHalf2) || (gB < -kHalf2));
        const float gC = gA + gB;
        const float gr = bad ? 0.f : gA;        // reference for Lk, Lq, R (token 31, or 0)
        const float gs = bad ? gC : gA;         // R's reference (the exact path does not use R)
        const float rhf = ex2_approx(gC - gs);  // Rh = R * rhf
        const float fac_r = ex2_approx(gr), fac_c = ex2_approx(gC);   // staged with Yh, Wh
        if (bad) {                              // exact path: natural-log gamma
            float* Gx = reinterpret_cast<float*>(sm + P_GX);
#pragma unroll
            for (int t = 0; t < 16; ++t) Gx[(16 * qt + t) * kD + c] = gam[t] * (1.f / kLog2e);
        }
        // ---- folded operands Lk, Lq (A of A|P, and the consumer's B of Sm [Lk^T | Lq^T]),
        // R (B of A|P), Rh: 8 tokens per 16-byte store ----
#pragma unroll
        for (int q8 = 0; q8 < 2; ++q8) {
            float lk[8], lq[8], rr[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = 8 * q8 + u;
                const int r = 16 * qt + t;
                const bool ok = r < L;
                const float kv = ok ? __bfloat162float(Xk[r * kD + c]) : 0.f;
                const float qv = ok ? __bfloat162float(Xq[r * kD + c]) : 0.f;
                const float a = ex2_approx(gam[t] - gr), b = ex2_approx(gs - gam[t]);
                lk[u] = kv * a; lq[u] = qv * a; rr[u] = kv * b;
            }
            const int ch = 2 * qt + q8;         // 8-token chunk index within the 64 tokens
            const uint32_t o16 = mnmaj_chunk(c, ch, 0, 16);
            st16(sm, P_LK + o16, pack8(lk));
            st16(sm, P_LQ + o16, pack8(lq));
            st16(sm, P_RT + o16, pack8(rr));
#pragma unroll
            for (int u = 0; u < 8; ++u) rr[u] *= rhf;
            st16(sm, P_RH + o16, pack8(rr));
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {                         // first group: [Lk | Lq]
            bulk_store(slot + S_LK, sb + P_LK, S_YW - S_LK);
            bulk_commit();
        }
        trace_mark(prank, n, 1);

        float* Nm = reinterpret_cast<float*>(sm + P_X);
        if (!bad) {
            if (warp == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, true, true);
                const uint64_t a0 = make_desc(sb + P_LK, P_LQ - P_LK, 1024);
                const uint64_t b0 = make_desc(sb + P_RT, 16384, 1024);
                if (elect_one()) {
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        mma_bf16(tm + TP_AP, desc_add(a0, s * 2048), desc_add(b0, s * 2048), id, s > 0);
                    mma_commit(bar_mma);
                }
                __syncwarp();
            }
            if (!wait_local(bar_mma, ph_mma)) { aborted = true; break; }
            trace_mark(prank, n, 2);
            tc_fence_after();
            float val[16];
            tmem_ld16(tm + lane_sel + TP_AP + 16 * wg, val);
            const int i0 = 16 * wg;
            if (row < 64) {
                const int r = row;
                const float br = s_beta[r];
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    float4 w;
                    w.x = (i0 + 4 * i4 + 0 < r) ? br * val[4 * i4 + 0] : 0.f;
                    w.y = (i0 + 4 * i4 + 1 < r) ? br * val[4 * i4 + 1] : 0.f;
                    w.z = (i0 + 4 * i4 + 2 < r) ? br * val[4 * i4 + 2] : 0.f;
                    w.w = (i0 + 4 * i4 + 3 < r) ? br * val[4 * i4 + 3] : 0.f;
                    *reinterpret_cast<float4*>(Nm + r * kLd + i0 + 4 * i4) = w;
                }
            } else {
                const int r = row - 64;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    float pv[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) pv[u] = (i0 + 8 * qq + u <= r) ? val[8 * qq + u] : 0.f;
                    st16(sm, P_PO + kmaj_chunk(r, (i0 >> 3) + qq, 0, 64), pack8(pv));
                }
            }
        } else {
            exact_ap(sm, s_beta, L);
            const float* Aex = reinterpret_cast<const float*>(sm + P_AEX);
            // the raw tiles are dead: move diag(beta) A into the inverse's scratch
            for (int e = tid; e < kC * kC; e += kThreads) Nm[(e >> 6) * kLd + (e & 63)] = Aex[e];
        }
        __syncthreads();
        trace_mark(prank, n, 3);

        // ---- T' = (I + N)^-1 diag(beta) in fp32, N = diag(beta) A ----
        // Block recursion on the unit lower triangular matrix: the inverse of [[A, 0], [B, C]]
        // is [[A^-1, 0], [-C^-1 B A^-1, C^-1]]. 8x8 diagonal blocks by column substitution,
        // then 8 -> 16 on CUDA cores (fp32), 16 -> 32 -> 64 as warp-level tensor-core products
        // (TF32 inputs, fp32 sums). T' is rounded to bf16 afterwards.
        {
            float* Tm = Nm + kC * kLd;
            float* Y = Tm + kC * kLd;                     // [4][16][kLdY] products / [4][8][8]
            if (tid < 64) {                               // level 0: block b, column i
                const int b = tid >> 3, i = tid & 7;
                const float* Nb = Nm + (8 * b) * kLd + 8 * b;
                float x[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    float s0 = 0.f;
#pragma unroll
                    for (int m = 0; m < r; ++m) s0 = fmaf(Nb[r * kLd + m], x[m], s0);
                    x[r] = (r < i) ? 0.f : (r == i ? 1.f : -s0);
                    Tm[(8 * b + r) * kLd + 8 * b + i] = x[r];
                }
            }
            __syncthreads();
            trace_mark(prank, n, 4);
            if (tid < 256) {                              // level 1: 16-block blk, element (r, j)
                const int blk = tid >> 6, r = (tid >> 3) & 7, j = tid & 7, o = 16 * blk;
                float y = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) y = fmaf(Nm[(o + 8 + r) * kLd + o + m], Tm[(o + m) * kLd + o + j], y);
                Y[blk * 64 + r * 8 + j] = y;
                Tm[(o + r) * kLd + o + 8 + j] = 0.f;      // upper-right 8x8 of the 16-block
            }
            __syncthreads();
            if (tid < 256) {
                const int blk = tid >> 6, r = (tid >> 3) & 7, j = tid & 7, o = 16 * blk;
                float t = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) t = fmaf(Tm[(o + 8 + r) * kLd + o + 8 + m], Y[blk * 64 + m * 8 + j], t);
                Tm[(o + 8 + r) * kLd + o + j] = -t;
            }
            __syncthreads();
            // level 2: 32-blocks g = 0, 1 on warps 0, 1; the other warps zero their upper-right 16x16
            if (warp < 2) {
                const int o = 32 * warp;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                warp_block_mma16(acc, Nm + (o + 16) * kLd + o, kLd, Tm + o * kLd + o, kLd);
                warp_block_store16(Y + warp * 16 * kLdY, kLdY, acc, 1.f);
            } else {
                for (int e = tid - 64; e < 512; e += kThreads - 64) {
                    const int g2 = e >> 8, r = (e >> 4) & 15, j = e & 15;
                    Tm[(32 * g2 + r) * kLd + 32 * g2 + 16 + j] = 0.f;
                }
            }
            __syncthreads();
            if (warp < 2) {
                const int o = 32 * warp;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                warp_block_mma16(acc, Tm + (o + 16) * kLd + o + 16, kLd, Y + warp * 16 * kLdY, kLdY);
                warp_block_store16(Tm + (o + 16) * kLd + o, kLd, acc, -1.f);
            }
            __syncthreads();
            // level 3: the lower-left 32x32 as 2x2 blocks of 16, warp w = (a, b)
            if (warp < 4) {
                const int a = warp >> 1, b = warp & 1;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int k2 = b; k2 < 2; ++k2)            // Y_ab = sum_k N21_ak T11_kb
                    warp_block_mma16(acc, Nm + (32 + 16 * a) * kLd + 16 * k2, kLd, Tm + (16 * k2) * kLd + 16 * b, kLd);
                warp_block_store16(Y + warp * 16 * kLdY, kLdY, acc, 1.f);
            }
            __syncthreads();
            if (warp < 4) {
                const int a = warp >> 1, b = warp & 1;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int k2 = 0; k2 <= a; ++k2)           // T21_ab = -sum_k T22_ak Y_kb
                    warp_block_mma16(acc, Tm + (32 + 16 * a) * kLd + 32 + 16 * k2, kLd, Y + (2 * k2 + b) * 16 * kLdY, kLdY);
                warp_block_store16(Tm + (32 + 16 * a) * kLd + 16 * b, kLd, acc, -1.f);
            }
            __syncthreads();
            trace_mark(prank, n, 5);
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
                st16(sm, P_TP + kmaj_chunk(r, q8, 0, 64), pack8(w8));
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (has_next) issue_qk(c_next);         // the inverse's scratch is dead
        announce(false);                        // the previous chunk, stored a task ago
        trace_mark(prank, n, 6);

        // ---- Yh^T = Rh^T T' (M = key ch) and Wh^T = P' T' (M = token, 64 rows of 128) ----
        if (warp == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, true);
            const uint64_t aY = make_desc(sb + P_RH, 16, 1024);
            const uint64_t aW = make_desc(sb + P_PO, 16, 1024);
            const uint64_t bT = make_desc(sb + P_TP, 8192, 1024);
            if (elect_one()) {
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tm + TP_Y, desc_add(aY, s * 32), desc_add(bT, s * 2048), id, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tm + TP_W, desc_add(aW, s * 32), desc_add(bT, s * 2048), id, s > 0);
                mma_commit(bar_mma);
            }
            __syncwarp();
        }
        // the staging is free once the previous chunk's second group has read it
        if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        if (!wait_local(bar_mma, ph_mma)) { aborted = true; break; }
        trace_mark(prank, n, 7);
        if (has_next) issue_g(c_next);          // R and Rh are dead
        tc_fence_after();
        {
            float val[16];
            tmem_ld16(tm + lane_sel + TP_Y + 16 * wg, val);
#pragma unroll
            for (int qq = 0; qq < 2; ++qq)
                st16(sm, P_ST + kmaj_chunk(row, 2 * wg + qq, 0, 0), pack8(val + 8 * qq));
            if ((warp & 3) < 2) {               // lanes 0..63 hold Wh^T
                tmem_ld16(tm + lane_sel + TP_W + 16 * wg, val);
#pragma unroll
                for (int qq = 0; qq < 2; ++qq)
                    st16(sm, P_ST + kmaj_chunk(128 + row, 2 * wg + qq, 0, 0), pack8(val + 8 * qq));
            }
            if (qt == 0) {
                float* fs = reinterpret_cast<float*>(sm + P_ST + (S_FAC - S_YW));
                fs[c] = fac_r;
                fs[128 + c] = fac_c;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {                         // second group: [Yh^T | Wh^T | factors]
            bulk_store(slot + S_YW, sb + P_ST, kSlotBytes - S_YW);
            bulk_commit();
        }
        pending = n;
        trace_mark(prank, n, 8);
    }
    if (!aborted) announce(true);
    if (tid == 0) bulk_wait0();
}

// ============================== consumer ==============================
__device__ void consumer(const Params& p, uint8_t* sm, uint32_t sb, int n_seq, int h,
                         int64_t bos, int64_t eos, bool& aborted) {
    const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, j = tid & 127;
    const uint32_t lane_sel = (uint32_t)(32 * (warp & 3)) << 16;
    uint8_t* misc = sm + C_MISC;
    uint64_t* bar_x = reinterpret_cast<uint64_t*>(misc + M_BAR_X);
    uint64_t* bar_s = reinterpret_cast<uint64_t*>(misc + M_BAR_S);
    uint64_t* bar_o = reinterpret_cast<uint64_t*>(misc + M_BAR_O);
    uint64_t* bar_lfull = reinterpret_cast<uint64_t*>(misc + M_LFULL);
    uint64_t* bar_gfull = reinterpret_cast<uint64_t*>(misc + M_GFULL);
    uint64_t* bar_v = reinterpret_cast<uint64_t*>(misc + M_BAR_V);
    const uint32_t tm = *reinterpret_cast<uint32_t*>(misc + M_TMEM);
    const int H = p.H;
    const int nchunks = (int)((eos - bos + kC - 1) / kC);
    uint32_t ph_x = 0, ph_s = 0, ph_lfull = 0, ph_gfull = 0, ph_v = 0;   // bit i: barrier i
    const uint8_t* ring = p.ring + (size_t)smid() * (kRing * kSlotBytes);
    const int64_t sbase = ((int64_t)n_seq * H + h) * kD * kD;

    float sreg[32];                     // S[32*wg + cc][j]
#pragma unroll
    for (int cc = 0; cc < 32; ++cc)
        sreg[cc] = p.h0 ? p.h0[sbase + (int64_t)(32 * wg + cc) * kD + j] : 0.f;

    // V tile of chunk nn into ring entry nn % 3 by TMA: two (64 channels x 64 tokens) boxes,
    // 128B-swizzled. Rows past the sequence do not matter (the matching rows of Lk, Yh and Wh
    // are zero). Thread kLoader (warp 2) issues every V and ring load, beside warp 0's MMA issue.
    constexpr int kLoader = 64;
    auto issue_v = [&](int nn) {
        if (tid == kLoader) {
            const int e = nn % 3;
            const uint32_t base = sb + C_V + (uint32_t)e * 16384;
            const int c0 = (int)(bos + (int64_t)nn * kC);
            mbar_arrive_expect_tx(bar_v + e, 16384u);
            tma_load_3d(base, &p.tv, 0, h, c0, bar_v + e);
            tma_load_3d(base + 8192, &p.tv, 64, h, c0, bar_v + e);
        }
    };
    // Factors of chunk nn from its global ring slot into shared slot nn % 2 (the shared slot
    // must be free): waits for the producer's announcement, then one bulk load.
    auto issue_load = [&](int nn) -> bool {
        bool ok = true;
        if (tid == kLoader) {
            const int rs = nn % kRing;
            ok = mbar_wait_cluster_bounded(bar_gfull + rs, (ph_gfull >> rs) & 1u, kWaitCycles);
            ph_gfull ^= 1u << rs;
            if (ok) {
                fence_proxy_async_global();
                uint64_t* bl = bar_lfull + (nn & 1);
                const uint32_t dst = sb + C_SLOT0 + (uint32_t)(nn & 1) * kSlotBytes;
                mbar_arrive_expect_tx(bl, kSlotBytes);
                bulk_load(dst, ring + (size_t)rs * kSlotBytes, kSlotBytes, bl);
            } else {
                atomicOr(p.err, kErrTimeout);
            }
        }
        return ok;
    };
    // Factors and V tile of chunk nn both in (one polling thread, one block barrier); then
    // its ring slot may take chunk nn + kRing.
    auto wait_next = [&](int nn) -> bool {
        const int sl = nn & 1, e = nn % 3;
        int fail = 0;
        if (tid == kPoller) {
            const bool ok = mbar_wait_bounded(bar_lfull + sl, (ph_lfull >> sl) & 1u, kWaitCycles) &&
                            mbar_wait_bounded(bar_v + e, (ph_v >> e) & 1u, kWaitCycles);
            if (!ok) {
                atomicOr(p.err, kErrTimeout);
                fail = 1;
            }
        }
        ph_lfull ^= 1u << sl;
        ph_v ^= 1u << e;
        if (__syncthreads_or(fail)) return false;
        if (tid == 0 && nn + kRing < nchunks)
            mbar_arrive_remote_relaxed(map_to_rank(sb + P_MISC + M_GFREE + 8u * (uint32_t)(nn % kRing),
                                                   1 + (nn + kRing) % kProducers));
        return true;
    };
    // [X | O](nn) = Sm(nn) [Lk^T | Lq^T] (one converged warp; A operand Sm in tensor memory)
    auto issue_xo = [&](int nn) {
        const uint32_t so = C_SLOT0 + (uint32_t)(nn & 1) * kSlotBytes;
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 128, false, true);
        const uint64_t b0 = make_desc(sb + so + S_LK, S_LQ - S_LK, 1024);
        const uint32_t d = tm + ((nn & 1) ? TXO1 : TXO0);
        if (elect_one()) {
#pragma unroll
            for (int s = 0; s < 8; ++s) mma_bf16_ts(d, tm + TC_SM + 8 * s, desc_add(b0, s * 2048), id, s > 0);
            mma_commit(bar_x);
        }
        __syncwarp();
    };
    // state delta U Yh (commit S), then O(nn) += U Wh (commit O); A operand U in tensor memory
    auto issue_u = [&](int nn) {
        const uint32_t so = C_SLOT0 + (uint32_t)(nn & 1) * kSlotBytes;
        tc_fence_after();
        const uint32_t idS = idesc_bf16(128, 128, false, false);
        const uint32_t idO = idesc_bf16(128, 64, false, false);
        const uint64_t bY = make_desc(sb + so + S_YW, 16, 1024);
        const uint64_t bW = make_desc(sb + so + S_YW + 128 * 128, 16, 1024);
        const uint32_t dO = tm + ((nn & 1) ? TXO1 : TXO0) + 64;
        if (elect_one()) {
#pragma unroll
            for (int s = 0; s < 4; ++s) mma_bf16_ts(tm + TC_DS, tm + TC_U + 8 * s, desc_add(bY, s * 32), idS, s > 0);
            mma_commit(bar_s);
#pragma unroll
            for (int s = 0; s < 4; ++s) mma_bf16_ts(dO, tm + TC_U + 8 * s, desc_add(bW, s * 32), idO, 1);
            mma_commit(bar_o);
        }
        __syncwarp();
    };
    // Sm(nn) = (S^T diag(e^{gamma_ref(nn)})) as bf16 pairs along the key channel
    auto pack_sm = [&](int nn, uint32_t* w) {
        const float* fac = reinterpret_cast<const float*>(sm + C_SLOT0 + (uint32_t)(nn & 1) * kSlotBytes + S_FAC);
        const float4* e4 = reinterpret_cast<const float4*>(fac + 32 * wg);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
            const float4 e = e4[q4];
            w[2 * q4] = pack_bf16(sreg[4 * q4] * e.x, sreg[4 * q4 + 1] * e.y);
            w[2 * q4 + 1] = pack_bf16(sreg[4 * q4 + 2] * e.z, sreg[4 * q4 + 3] * e.w);
        }
    };
    // U(nn) = V(nn)^T - X(nn) for value channel j and tokens [16 wg, 16 wg + 16), as bf16
    // pairs along the token into tensor memory. V[t][j] sits in box j / 64, row t, 16-byte
    // chunk ((j % 64) / 8) ^ (t % 8) of the 128B-swizzled tile.
    auto make_u = [&](int nn) {
        tc_fence_after();
        float xv[16];
        tmem_ld16(tm + lane_sel + ((nn & 1) ? TXO1 : TXO0) + 16 * wg, xv);
        const uint8_t* vt = sm + C_V + (uint32_t)(nn % 3) * 16384 + 8192 * (j >> 6) + (j & 7) * 2;
        const int jc = (j & 63) >> 3;
        uint32_t w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t0 = 16 * wg + 2 * u;
            const float v0 = bf(reinterpret_cast<const __nv_bfloat16*>(vt + t0 * 128 + ((jc ^ (t0 & 7)) << 4)));
            const float v1 = bf(reinterpret_cast<const __nv_bfloat16*>(vt + (t0 + 1) * 128 + ((jc ^ ((t0 + 1) & 7)) << 4)));
            w[u] = pack_bf16(v0 - xv[2 * u], v1 - xv[2 * u + 1]);
        }
        tmem_st8(tm + lane_sel + TC_U + 8 * wg, w);
        tmem_wait_st();
    };
    // O of chunk nn, by warps 1..15 (warp 4 also takes warp 0's share): TMEM -> bf16
    // [token][channel] staging -> one TMA tile store (a ragged last chunk: one bulk copy per
    // valid token, so rows of the next sequence are never touched)
    auto epilogue_o = [&](int nn) -> bool {
        if (warp == 1) bulk_wait_read0();       // the previous O tile has left the staging
        const bool ok = group_wait(bar_o, (uint32_t)(nn & 1), nullptr, 0, p.err);   // once per chunk
        tc_fence_after();
        const uint32_t to = tm + lane_sel + ((nn & 1) ? TXO1 : TXO0) + 64;
        __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(sm + C_OST);
        for (int part = (warp == 4 ? 0 : 1); part < 2; ++part) {
            const int t0 = part ? 16 * wg : 0;
            float ov[16];
            tmem_ld16(to + t0, ov);
#pragma unroll
            for (int t = 0; t < 16; ++t) st[(t0 + t) * kD + j] = __float2bfloat16_rn(p.scale * ov[t]);
        }
        fence_async_smem();
        tc_fence_before();
        group_sync();
        if (warp == 1) {
            const int64_t c0 = bos + (int64_t)nn * kC;
            const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
            const int lane = tid & 31;
            if (L == kC) {
                if (lane == 0) tma_store_3d(&p.to, 0, h, (int)c0, sb + C_OST);
            } else {
                for (int r = lane; r < L; r += 32)
                    bulk_store(p.o + ((c0 + r) * H + h) * kD, sb + C_OST + r * 256, 256);
            }
            bulk_commit();
        }
        return ok;
    };

    // prologue: V tiles of chunks 0..2, factors of chunks 0 and 1, Sm(0), then [X | O](0)
    if (nchunks > 0) {
        issue_v(0);
        if (nchunks > 1) issue_v(1);
        if (nchunks > 2) issue_v(2);
        // chunk 0 must have arrived (which frees ring slot 0 for chunk kRing) before the loader
        // waits for chunk 1: a producer announces a chunk only during its next task
        if (__syncthreads_or(!issue_load(0))) aborted = true;   // (seen by every thread)
        if (!aborted && !wait_next(0)) aborted = true;
        if (!aborted && nchunks > 1 && __syncthreads_or(!issue_load(1))) aborted = true;
        if (!aborted) {
            uint32_t w[16];
            pack_sm(0, w);
            tmem_st16(tm + lane_sel + TC_SM + 16 * wg, w);
            tmem_wait_st();
            tc_fence_before();
            __syncthreads();
            if (warp == 0) issue_xo(0);
        }
    }

    // Warp 0 issues the MMAs and blocks for about their execution time, so after each issue
    // warps 1..15 go on alone (named barrier 1) and warp 0 catches up at the next block-wide
    // barrier. A failed wait only raises `fail`; the block leaves the loop together at the
    // next block-wide barrier.
    int fail = 0;
    for (int n = 0; n < nchunks && !aborted; ++n) {
        const float* fac = reinterpret_cast<const float*>(sm + C_SLOT0 + (uint32_t)(n & 1) * kSlotBytes + S_FAC);
        const bool more = n + 1 < nchunks;
        const int n1 = n + 1, sl1 = n1 & 1, e1 = n1 % 3;
        trace_mark(0, n, 0);
        // (1) U(n) = V(n)^T - X(n), then U [Yh | Wh]
        if (!block_wait_or(bar_x, ph_x & 1u, fail, p.err)) { aborted = true; break; }
        ph_x ^= 1u;
        trace_mark(0, n, 1);
        make_u(n);
        tc_fence_before();
        __syncthreads();
        trace_mark(0, n, 2);
        // (2) the next chunk's operands and this chunk's state delta
        if (warp == 0) {
            issue_u(n);
            trace_mark(0, n, 3);
            if (more && !warp_wait(bar_lfull + sl1, (ph_lfull >> sl1) & 1u, p.err)) fail = 1;
            if (!warp_wait(bar_s, ph_s & 1u, p.err)) fail = 1;
        } else {
            if (more && !group_wait(bar_lfull + sl1, (ph_lfull >> sl1) & 1u, bar_v + e1, (ph_v >> e1) & 1u, p.err))
                fail = 1;
            if (more && tid == 32 && n1 + kRing < nchunks)    // ring slot of n + 1 may take n + 1 + kRing
                mbar_arrive_remote_relaxed(map_to_rank(sb + P_MISC + M_GFREE + 8u * (uint32_t)(n1 % kRing),
                                                       1 + (n1 + kRing) % kProducers));
            if (!group_wait(bar_s, ph_s & 1u, nullptr, 0, p.err)) fail = 1;
        }
        if (more) {
            ph_lfull ^= 1u << sl1;
            ph_v ^= 1u << e1;
        }
        ph_s ^= 1u;
        trace_mark(0, n, 4);
        // (3) state update S' = e^{gamma_C} S + U Yh, then Sm(n + 1)
        tc_fence_after();
        {
            float v32[32];
            tmem_ld32(tm + lane_sel + TC_DS + 32 * wg, v32);
            const float4* eC4 = reinterpret_cast<const float4*>(fac + 128 + 32 * wg);
#pragma unroll
            for (int t4 = 0; t4 < 8; ++t4) {
                const float4 ec = eC4[t4];
                const float* v = v32 + 4 * t4;
                const int cc = 4 * t4;
                sreg[cc] = fmaf(ec.x, sreg[cc], v[0]);
                sreg[cc + 1] = fmaf(ec.y, sreg[cc + 1], v[1]);
                sreg[cc + 2] = fmaf(ec.z, sreg[cc + 2], v[2]);
                sreg[cc + 3] = fmaf(ec.w, sreg[cc + 3], v[3]);
            }
        }
        if (more) {
            uint32_t w[16];
            pack_sm(n1, w);
            tmem_st16(tm + lane_sel + TC_SM + 16 * wg, w);
            tmem_wait_st();
        }
        trace_mark(0, n, 5);
        tc_fence_before();
        if (__syncthreads_or(fail)) { aborted = true; break; }
        trace_mark(0, n, 6);
        if (warp == 0) {
            // (4) the next chunk's [X | O]
            if (more) issue_xo(n1);
            trace_mark(0, n, 7);
        } else {
            // (4') output of chunk n, then the loads that the completed chunk n made possible:
            // shared slot n % 2 takes chunk n + 2, V ring entry n % 3 takes V(n + 3)
            if (!epilogue_o(n)) fail = 1;
            trace_mark(0, n, 8, 32);
            if (n + 2 < nchunks) issue_load(n + 2);   // a failed wait flags the error word; the
                                                      // consumer then gives up at the next wait
            if (n + 3 < nchunks) issue_v(n + 3);
            trace_mark(0, n, 9, 32);
        }
    }
    if (warp == 1) bulk_wait0();
    if (p.ht && !aborted) {
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) p.ht[sbase + (int64_t)(32 * wg + cc) * kD + j] = sreg[cc];
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
        // every barrier completes once per use: one arrival (plus transaction bytes where a TMA
        // or bulk copy feeds it)
        for (uint32_t b = 0; b < kBars; ++b) mbar_init(reinterpret_cast<uint64_t*>(misc + 8 * b), 1);
        if (is_consumer) {
            const uint32_t id = smid();
            *reinterpret_cast<uint32_t*>(misc + M_SMID) = id;
            if ((int)id >= p.ring_sms) atomicOr(p.err, kErrTimeout);
        }
    }
    tc_fence_before();
    cluster_sync();                     // barriers of every CTA exist before any remote arrive
    tc_fence_after();

    // a consumer SM outside the workspace's ring table (flagged above): nobody touches the ring
    bool aborted = (int)ld_cluster_u32(map_to_rank(sb + C_MISC + M_SMID, 0)) >= p.ring_sms;
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

// Ring tables for SM ids 0 .. kRingSms - 1 (a B200 has 148 SMs).
constexpr int kRingSms = 160;
size_t chunk_tcx_workspace_bytes() { return (size_t)kRingSms * kRing * kSlotBytes; }

cudaError_t launch_chunk_tcx(const ChunkArgs& a, void* workspace, size_t workspace_bytes,
                             unsigned int* err, cudaStream_t stream) {
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
    p.ring = static_cast<uint8_t*>(workspace);
    p.ring_sms = (int)(workspace_bytes / ((size_t)kRing * kSlotBytes));
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
