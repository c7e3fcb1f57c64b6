// chunk_tcx.cu -- chunked KDA prefill, bf16 I/O, dk = dv = 128, chunk 64, as a producer /
// consumer pipeline inside one thread-block cluster per (sequence, head).
//
// The recurrence (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...", section
// "Что именно изменилось"; m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...") is
// linear in the state, so one chunk maps the state at its start, S (dk x dv, row = key
// channel), to the state at its end by S' = M S + N with M, N built from the chunk's inputs
// alone. This kernel splits along that line: producers build the chunk's factors, which do not
// depend on S; the consumer applies them. With gamma the within-chunk cumulative log-decay,
// gamma_C its last row and gamma_ref a per-chunk reference (token 31, or 0 when a half chunk
// decays by more than e^-80 in some channel), per chunk (rows = tokens):
//   Lk = k e^{gamma - gamma_ref},  Lq = q e^{gamma - gamma_ref},  R = k e^{gamma_s - gamma}
//   [A ; P] = [Lk ; Lq] R^T        (strictly / inclusively lower triangular parts)
//   T' = (I + diag(beta) A)^-1 diag(beta)
//   Yh^T = diag(e^{gamma_C - gamma_s}) R^T T',   Wh^T = P T'
// (gamma_s = gamma_ref, or gamma_C on the exact path) and with Sm = diag(e^{gamma_ref}) S:
//   X = Lk Sm,  U = V - X                      (the part of V the decayed state misses)
//   S' = diag(e^{gamma_C}) S + Yh^T U          (fp32 state, fp32 decay term)
//   O  = scale (Lq Sm + Wh^T U)
// A chunk that fails the range test forms A and P exactly on CUDA cores (gamma_ref = 0, so
// every factor is <= 1).
//
// Cluster of 4 CTAs of 17 warps: rank 0 is the consumer, ranks 1..3 are producers, each
// preparing every third chunk. A chunk's factors (57 KB) travel through L2, not DSMEM: the
// producer's I/O lane bulk-stores them into a ring in global memory owned by the consumer's SM
// and announces them on a cluster barrier ("gfull"); the consumer's loader warp bulk-loads them
// into shared memory and hands the ring slot back ("gfree").
//
// The consumer runs the value columns as two independent halves of 64 (state columns do not
// interact), each on its own 8 warps with its own MMA issuer, so that one half's tensor-core
// products overlap the other half's CUDA-core work. Per half and chunk: [X ; Lq Sm] = [Lk ; Lq]
// Sm (M = 128 token rows, N = 64), U = V - X, then the state delta Yh^T U and the output term
// Wh^T U; the fp32 state stays in registers (thread = key channel x 32 value columns).
//
// Compile-time variants serve kda_chunk_fwd_fused. kGate: the producers form g from raw
// gate logits, g = -exp(A_log[h]) softplus(x + dt_bias) (m.lqnn.cn/news/205170: the gate comes
// from a_log_bias and dt_bias), in the fold, and beta = sigmoid(b) from raw logits. kNorm: the
// consumer's output warps apply the gated RMSNorm o / sqrt(mean(o^2) + eps) * w * sigmoid(z)
// (sarnas.ru, section "Отвергнутые решения") before the store, the two value halves exchanging
// their per-token sums of squares through shared memory. kConv: q, k, v arrive raw; the
// producers load them with a 3-token halo and apply the causal depthwise conv (kernel 4), SiLU
// and the L2 norm of q, k in shared memory before the fold (m.lqnn.cn/news/205170: q/k/v pass a
// kernel-4 causal conv), and send v after the conv with the chunk's factors.
//
// Every wait is bounded (a launch parameter); a wait that gives up sets the error word, and the
// CTA leaves its loop, waits for its own copies and products in flight, and frees its tensor
// memory.
#include <atomic>

#include "common.cuh"
#include "launchers.h"
#include "tc.cuh"
#include "tma_host.h"

namespace kda {

long long g_chunk_wait_cycles = 0;   // 0: the default bound

namespace {

using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kWarps = 17;
constexpr int kThreads = 32 * kWarps;     // 16 compute warps + 1 I/O (producer) or loader warp
constexpr int kCompute = 512;
constexpr int kIoWarp = 16;
constexpr int kProducers = 3;
constexpr int kCluster = 1 + kProducers;
constexpr float kHalfRange = 80.f;       // largest natural-log decay allowed per half chunk
constexpr float kLog2e = 1.4426950408889634f;
constexpr long long kDefaultWaitCycles = 4000000000LL;   // ~2 s at 1.9 GHz
constexpr int kGate = 1, kNorm = 2, kConv = 4;   // variant bits
constexpr int kStates = 8;    // stretch launch: the second half of the clusters forms
                              // transitions; outputs optional
constexpr int kHalo = 3;                 // kConv: the conv's three earlier tokens
constexpr float kLn2 = 0.6931471805599453f;

// ---- one chunk's hand-off (identical image in a global ring slot and the consumer's slots) ----
constexpr uint32_t S_LKQ = 0;            // [Lk ; Lq]: K-major, 2 atom columns (channels) x 128 rows
constexpr uint32_t S_FAC = 32768;        // e^{gamma_ref}[128], e^{gamma_C}[128] (fp32)
constexpr uint32_t kAPart = 33792;       // [Lk ; Lq | factors]
constexpr uint32_t S_YW = kAPart;        // [Yh^T (rows key ch 0..127) ; Wh^T (rows token)]: K-major
constexpr uint32_t kBPart = 24576;
constexpr uint32_t S_V = kAPart + kBPart;   // kConv: V after the conv, [half][token][64 ch] SW128
constexpr uint32_t kVPart = 16384;
constexpr uint32_t kSlotBytes = kAPart + kBPart + kVPart;
constexpr int kRing = kTcxRingSlots;
static_assert(kSlotBytes == kTcxSlotBytes, "slot size");
static_assert(kAPart % 1024 == 0 && kBPart % 1024 == 0, "slot parts stay swizzle-atom aligned");

// ---- producer shared memory ----
constexpr uint32_t kRawTile = 17408;     // 68 token rows of 256 B: 64, after 3 halo rows with kConv
constexpr uint32_t P_Q = 0;              // q tile [rows][128] bf16 (TMA, unswizzled); with kConv
                                         //   raw, then overwritten by the conv's output
constexpr uint32_t P_K = kRawTile;       // k tile, the same
constexpr uint32_t P_V = 2 * kRawTile;   // kConv: raw v tile
constexpr uint32_t P_G = 3 * kRawTile;   // g tile [64][128] fp32 (kGate: bf16 logits); with kConv
                                         //   v after the conv (the slot's V part) once g is read
constexpr uint32_t P_LKQ = P_G + 32768;  // [Lk ; Lq | factors]: the slot's A part image
constexpr uint32_t P_R = P_LKQ + kAPart; // R: K-major, 2 atom columns x 64 token rows
constexpr uint32_t P_PO = P_R + 16384;   // P': K-major, 64 token rows x 64 (A of Wh^T; its M = 128
                                         //     padding rows read T' and give unused rows)
constexpr uint32_t P_TP = P_PO + 8192;   // T': rows r (K), 64 columns i (N): MN-major B
constexpr int kLd = 68;                  // fp32 row stride of the 64 x 64 inverse scratch
constexpr int kLdY = 24;                 // row stride of the per-warp 16 x 16 products
constexpr uint32_t P_NM = P_TP + 8192;   // N = diag(beta) A (fp32 [64][kLd]); during the fold the
                                         //   per-warp decay sums [16][128]
constexpr uint32_t P_TM = P_NM + 64 * kLd * 4;   // T (fp32 [64][kLd])
constexpr uint32_t P_Y = P_TM + 64 * kLd * 4;    // [4][16][kLdY] fp32
constexpr uint32_t P_ST = ((P_Y + 4 * 16 * kLdY * 4 + 1023) / 1024) * 1024;   // [Yh^T ; Wh^T] staging
constexpr uint32_t P_GX = P_TM;          // exact path: natural-log gamma fp32 [64][128] (32 KB over
                                         //   T, Y and the staging, all idle at that point)
constexpr uint32_t P_MISC = P_ST + kBPart;
static_assert(P_LKQ % 1024 == 0 && P_R % 1024 == 0 && P_PO % 1024 == 0 && P_TP % 1024 == 0 &&
              P_ST % 1024 == 0, "operand tiles are swizzle-atom aligned");
static_assert((kC + kHalo) * 256 <= kRawTile && 2 * kVPart / 2 <= 32768 && 16 * 128 * 4 <= 64 * kLd * 4,
              "tile and scratch sizes");
static_assert(P_GX + 64 * 128 * 4 <= P_MISC, "exact-path scratch");

// ---- consumer shared memory ----
constexpr uint32_t C_A = 0;                        // A parts of chunks n % 2
constexpr uint32_t C_B = 2 * kAPart;               // B parts of chunks n % 2
constexpr uint32_t C_V = C_B + 2 * kBPart;         // V tiles [half][n % 2] (64 ch x 64 tokens, SW128)
constexpr uint32_t C_SM = C_V + 4 * 8192;          // Sm per half: MN-major B (K = key ch, N = 64)
constexpr uint32_t C_U = C_SM + 2 * 16384;         // U per half: MN-major B (K = token, N = 64)
constexpr uint32_t C_OST = C_U + 2 * 8192;         // O staging per half (64 ch x 64 tokens, SW128)
constexpr uint32_t C_MISC = C_OST + 2 * 8192;
static_assert(C_V % 1024 == 0 && C_SM % 1024 == 0 && C_U % 1024 == 0 && C_OST % 1024 == 0,
              "consumer tiles are swizzle-atom aligned");

// ---- misc areas: mbarriers (8 bytes each) from offset 0, scalars from 256 ----
constexpr uint32_t M_TMEM = 256;      // TMEM base address (both roles)
constexpr uint32_t M_TMP = 260;       // unit_of scratch
constexpr uint32_t M_SMID = 264;      // consumer: its SM id (selects the global ring)
// producer barriers
constexpr uint32_t M_QK_FULL = 0, M_G_FULL = 8, M_RAW_FREE = 16, M_LKQ_READY = 24, M_LKQ_FREE = 32,
                   M_ST_READY = 40, M_ST_FREE = 48, M_AP = 56, M_YW = 64, M_GFREE = 72;
constexpr int kBarsP = 9 + kRing;
constexpr uint32_t M_BETA = 512;      // beta[64]
constexpr uint32_t M_GA = 768;        // gamma at token 31, per channel (log2 units)
constexpr uint32_t M_GC = 1280;       // gamma at token 63 (log2 units)
constexpr uint32_t M_RHF = 1792;      // e^{gamma_C - gamma_s} per channel
constexpr uint32_t M_DT = 2304;       // kGate: dt_bias of this head [128]
constexpr uint32_t M_WCV = 2816;      // kConv: this head's conv weights, halved, as float4 (4 taps)
                                      //   [q, k, v][channel % 8][channel / 8] (a warp's 16
                                      //   channel groups read 16 consecutive float4)
constexpr uint32_t kMiscP = M_WCV + 3 * 128 * 16;
// consumer barriers ([X ; O] and delta per half; A, B parts per slot; V per half and slot;
// kNorm: the halves' sums of squares per chunk parity, each half's output gate tile; 224..239
// spare)
constexpr uint32_t M_XO = 0, M_DS = 16, M_AFULL = 32, M_BFULL = 48, M_AFREE = 64, M_BFREE = 80,
                   M_VFULL = 96, M_VFREE = 128, M_GFULL = 160, M_NRM = 208, M_ZFULL = 240;
constexpr int kBarsC = 32;
constexpr uint32_t M_WN = 512;        // kNorm: the norm weight [128]
constexpr uint32_t M_SS = 1024;       // kNorm: sums of squares [chunk % 3][half][column part][64]
constexpr uint32_t kMiscC = M_SS + 3 * 2 * 2 * 64 * 4;
static_assert(M_GFREE + 8 * kRing <= M_TMEM && M_ZFULL + 16 <= M_TMEM && M_GFULL + 8 * kRing <= M_NRM &&
              8 * kBarsC == M_ZFULL + 16, "barrier area");

constexpr uint32_t kSmemBytes =
    ((P_MISC + kMiscP) > (C_MISC + kMiscC) ? (P_MISC + kMiscP) : (C_MISC + kMiscC)) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// producer TMEM columns: A|P (M = 128: rows 0..63 A, 64..127 P; N = 64), Yh^T, Wh^T
constexpr uint32_t TP_AP = 0, TP_Y = 64, TP_W = 128, kTmemP = 256;
// consumer TMEM columns: per half h, [X ; Lq Sm] for even / odd chunks at 128 h + 64 b, the
// state delta at 256 + 64 h
constexpr uint32_t kTmemC = 512;

// named barriers: 1 = producer compute warps, 5 = its inverse warps; 1 + h = consumer half h,
// 3 + h = that half's output warps
constexpr int kBarCompute = 1, kBarInverse = 5;

struct Params {
    CUtensorMap tq, tk, tg;           // q, k [T,H,128] bf16, g [T,H,128] f32: (128, 1, 64) boxes
    CUtensorMap tv, to;               // v, o [T,H,128] bf16: (64, 1, 64) boxes, 128B swizzle
    CUtensorMap tz;                   // kNorm: the output gate z [T,H,128] bf16, as o
    const __nv_bfloat16* q;           // the exact path reads q, k, g directly
    const __nv_bfloat16* k;
    const float* g;
    const float* beta;
    float scale;
    const float* h0;
    float* ht;
    __nv_bfloat16* o;                 // kStates: may be null (no output)
    // kStates: clusters units .. 2 units - 1 form each unit's transition instead (the state
    // started from the identity, v taken as zero), written to mt [N,H,128,128] (or null: none);
    // their output, scale M_t^T q_t (the query carried back to the unit's start), goes to o2
    // through the to2 map (or nowhere when o2 is null)
    CUtensorMap to2;
    __nv_bfloat16* o2;
    float* mt;
    int units;                        // N * H
    const int32_t* cu;
    uint8_t* ring;                    // workspace: ring_sms x kRing x kSlotBytes
    int ring_sms;
    int T_pad;
    int N, H;
    unsigned int* err;
    long long wait_cycles;            // bound of every wait in the main loops
    // kGate: raw gate logits (the tg map covers them, bf16), raw beta logits, A_log [H],
    // dt_bias [H*128]
    const __nv_bfloat16* g_raw;
    const __nv_bfloat16* beta_raw;
    const float* A_log;
    const float* dt_bias;
    // kNorm: the output norm's gate z [T,H,128] bf16, weight [128], epsilon
    const __nv_bfloat16* z;
    const float* w_norm;
    float norm_eps;
    // kConv: q, k, v are raw (tq, tk, tv map them in 67-token boxes from 3 tokens back); conv
    // weights [H*128, 4] of q, k, v; the conv history [N, H*384, 3] (or null: zero); L2 epsilon
    const float* wconv[3];
    const __nv_bfloat16* conv_state;
    float l2_eps;
};

// softplus(x) = log(1 + e^x) = max(x, 0) + log(1 + e^-|x|), one ex2 and one lg2 on the SFU
// (for e^-|x| below fp32 resolution next to 1 the second term is lost, an absolute error
// below 1e-7).
__device__ __forceinline__ float softplus_fast(float x) {
    float l;
    const float e = ex2_approx(-fabsf(x) * kLog2e);
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.f + e));
    return fmaxf(x, 0.f) + l * kLn2;
}
// sigmoid with the fast divide (two ulp, far below the bf16 rounding of what it scales; the
// correctly rounded divide's software sequence cost the normed prefill half its time)
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// sigmoid(x) = (1 + tanh(x / 2)) / 2 with one SFU operation (tanh.approx: absolute error below
// 2.5e-4 in the sigmoid; the output gate it feeds is stored as bf16, relative error 2^-9)
__device__ __forceinline__ float sigmoid_tanh(float x) {
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(0.5f * x));
    return fmaf(0.5f, th, 0.5f);
}
// Prefetch of a 3-D tiled box into L2 (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2_3d(const void* tmap, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];"
                 ::"l"(tmap), "r"(c0), "r"(c1), "r"(c2) : "memory");
}
// silu(z) from h = z / 2: h + h tanh(h) (the conv prologue sums with halved weights).
__device__ __forceinline__ float silu_half(float hz) {
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(hz));
    return fmaf(hz, th, hz);
}

__device__ __forceinline__ void st16(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ uint4 ld16(const uint8_t* base, uint32_t off) {
    return *reinterpret_cast<const uint4*>(base + off);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                      pack_bf16(v[6], v[7]));
}
__device__ __forceinline__ void unpack8(uint4 w, float* v) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = unpack_bf16(a[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ uint64_t* bar_at(uint8_t* misc, uint32_t off) {
    return reinterpret_cast<uint64_t*>(misc + off);
}
// A bounded wait whose result every lane of the warp agrees on; a failure sets the error word.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const Params& p) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, parity, p.wait_cycles));
    if (!ok && (threadIdx.x & 31) == 0) atomicOr(p.err, kErrTimeout);
    return ok;
}
// The same for one thread.
__device__ __forceinline__ bool wait_one(uint64_t* bar, uint32_t parity, const Params& p,
                                         bool cluster_scope = false) {
    const bool ok = cluster_scope ? mbar_wait_cluster(bar, parity, p.wait_cycles)
                                  : mbar_wait(bar, parity, p.wait_cycles);
    if (!ok) atomicOr(p.err, kErrTimeout);
    return ok;
}

// Sequence / head of this cluster. Packed batches with at most kThreads sequences are processed
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

// Exact A and P on CUDA cores for a chunk whose decay fails the range test: natural-log gamma
// from the global g (thread = channel), then one warp per (r, i) pair with lanes over channels,
// reading q and k from the chunk's shared tiles (kept until the exact path is done). Writes N = diag(beta) A into the inverse's scratch and P
// into its operand. Rare, so kept out of line. Every compute thread calls it.
template <int MODE>
__device__ __noinline__ void exact_ap(const Params& p, uint8_t* sm, const float* s_beta, int h,
                                      int64_t c0, int L) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* Gx = reinterpret_cast<float*>(sm + P_GX);
    float* Nm = reinterpret_cast<float*>(sm + P_NM);
    __nv_bfloat16* Po = reinterpret_cast<__nv_bfloat16*>(sm + P_PO);
    const int64_t rs = (int64_t)p.H * kD;
    if (tid < kD) {
        float a = 0.f;
        for (int t = 0; t < kC; ++t) {
            if (t < L) {
                if constexpr ((MODE & kGate) != 0) {
                    const float x = __bfloat162float(p.g_raw[(c0 + t) * rs + (int64_t)h * kD + tid]) +
                                    p.dt_bias[h * kD + tid];
                    a -= expf(p.A_log[h]) * (x > 20.f ? x : log1pf(expf(x)));
                } else {
                    a += p.g[(c0 + t) * rs + (int64_t)h * kD + tid];
                }
            }
            Gx[t * kD + tid] = a;
        }
    }
    bar_sync(kBarCompute, kCompute);
    for (int pidx = warp; pidx < kC * (kC + 1) / 2; pidx += kCompute / 32) {
        int r = (int)((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
        while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
        while (r * (r + 1) / 2 > pidx) --r;
        const int i = pidx - r * (r + 1) / 2;
        float a = 0.f, pp = 0.f;
        if (r < L) {
            constexpr int halo = (MODE & kConv) != 0 ? kHalo : 0;
            const __nv_bfloat16* kr = reinterpret_cast<const __nv_bfloat16*>(sm + P_K) + (r + halo) * kD;
            const __nv_bfloat16* qr = reinterpret_cast<const __nv_bfloat16*>(sm + P_Q) + (r + halo) * kD;
            const __nv_bfloat16* ki = reinterpret_cast<const __nv_bfloat16*>(sm + P_K) + (i + halo) * kD;
            for (int cc = lane; cc < kD; cc += 32) {
                const float kd = __bfloat162float(ki[cc]) * expf(Gx[r * kD + cc] - Gx[i * kD + cc]);
                a = fmaf(__bfloat162float(kr[cc]), kd, a);
                pp = fmaf(__bfloat162float(qr[cc]), kd, pp);
            }
        }
        a = warp_sum(a);
        pp = warp_sum(pp);
        if (lane == 0) {
            Nm[r * kLd + i] = (i < r) ? s_beta[r] * a : 0.f;
            if (i < r) Nm[i * kLd + r] = 0.f;
            Po[(sw128(r, i >> 3, 0, 0) + (i & 7) * 2) / 2] = __float2bfloat16_rn(pp);
            if (i < r) Po[(sw128(i, r >> 3, 0, 0) + (r & 7) * 2) / 2] = __float2bfloat16_rn(0.f);
        }
    }
}

// T' = T diag(beta) of one 16 x 16 block held as an mma accumulator (rows R0.., cols C0..),
// times `sign`, written as bf16 into the T' operand.
__device__ __forceinline__ void store_tp16(uint8_t* sm, int R0, int C0, const float (*acc)[4],
                                           float sign, const float* s_beta) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int col = C0 + 8 * nt + 2 * t;
        const float b0 = sign * s_beta[col], b1 = sign * s_beta[col + 1];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = R0 + g + 8 * hh;
            *reinterpret_cast<uint32_t*>(sm + P_TP + sw128(row, col >> 3, 0, 0) + (col & 7) * 2) =
                pack_bf16(acc[nt][2 * hh] * b0, acc[nt][2 * hh + 1] * b1);
        }
    }
}
// scale * (a 16 x 16 mma accumulator) into an fp32 block with row stride ld.
__device__ __forceinline__ void store_f16(float* C, int ld, const float (*acc)[4], float scale) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        C[g * ld + 8 * nt + 2 * t] = scale * acc[nt][0];
        C[g * ld + 8 * nt + 2 * t + 1] = scale * acc[nt][1];
        C[(g + 8) * ld + 8 * nt + 2 * t] = scale * acc[nt][2];
        C[(g + 8) * ld + 8 * nt + 2 * t + 1] = scale * acc[nt][3];
    }
}

// T' = (I + N)^-1 diag(beta) for the strictly lower triangular N in the scratch, by block
// recursion on the unit lower triangular matrix (the inverse of [[A, 0], [B, C]] is
// [[A^-1, 0], [-C^-1 B A^-1, C^-1]]): 8 x 8 diagonal blocks by substitution and their 16 x 16
// merges in fp32 inside one warp per 16-block, then 16 -> 32 -> 64 as warp-level tensor-core
// products (TF32 inputs, fp32 sums). Run by warps 0..3; T' is written as bf16 as each block
// becomes final (its blocks above the diagonal stay zero from the kernel start).
__device__ void inverse(uint8_t* sm, const float* s_beta) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* Nm = reinterpret_cast<float*>(sm + P_NM);
    float* Tm = reinterpret_cast<float*>(sm + P_TM);
    float* Y = reinterpret_cast<float*>(sm + P_Y);
    float* Yw = Y + warp * 16 * kLdY;
    const int o16 = 16 * warp;
    // level 0: the two 8 x 8 diagonal blocks of this warp's 16-block, one column per lane
    if (lane < 16) {
        const int o = o16 + 8 * (lane >> 3), i = lane & 7;
        const float* Nb = Nm + o * kLd + o;
        float x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float s0 = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) s0 = fmaf(Nb[r * kLd + m], x[m], s0);
            x[r] = (r < i) ? 0.f : (r == i ? 1.f : -s0);
            Tm[(o + r) * kLd + o + i] = x[r];
        }
    }
    __syncwarp();
    // level 1: Y = N21 T11 (8 x 8), then T21 = -T22 Y; the upper-right 8 x 8 is zero
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
        const int e = lane + 32 * e2, r = e >> 3, j = e & 7;
        float y = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) y = fmaf(Nm[(o16 + 8 + r) * kLd + o16 + m], Tm[(o16 + m) * kLd + o16 + j], y);
        Yw[r * 8 + j] = y;
        Tm[(o16 + r) * kLd + o16 + 8 + j] = 0.f;
    }
    __syncwarp();
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
        const int e = lane + 32 * e2, r = e >> 3, j = e & 7;
        float t = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) t = fmaf(Tm[(o16 + 8 + r) * kLd + o16 + 8 + m], Yw[m * 8 + j], t);
        Tm[(o16 + 8 + r) * kLd + o16 + j] = -t;
    }
    __syncwarp();
    {   // T' of the diagonal 16-block: lane = (row, 8-column half)
        const int rr = o16 + (lane >> 1), c8 = o16 + 8 * (lane & 1);
        float w8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            w8[u] = (c8 + u <= rr) ? Tm[rr * kLd + c8 + u] * s_beta[c8 + u] : 0.f;
        st16(sm, P_TP + sw128(rr, c8 >> 3, 0, 0), pack8(w8));
    }
    bar_sync(kBarInverse, 128);
    // level 2: 16 -> 32 on warps 0, 1 (32-block = warp)
    if (warp < 2) {
        const int o = 32 * warp;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        warp_block_mma16(acc, Nm + (o + 16) * kLd + o, kLd, Tm + o * kLd + o, kLd);
        store_f16(Yw, kLdY, acc, 1.f);
        __syncwarp();
        float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        warp_block_mma16(acc2, Tm + (o + 16) * kLd + o + 16, kLd, Yw, kLdY);
        store_f16(Tm + (o + 16) * kLd + o, kLd, acc2, -1.f);
        store_tp16(sm, o + 16, o, acc2, -1.f, s_beta);
    }
    bar_sync(kBarInverse, 128);
    // level 3: the lower-left 32 x 32 as 2 x 2 blocks of 16, warp = (a, b)
    const int a = warp >> 1, b = warp & 1;
    {
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        for (int k2 = b; k2 < 2; ++k2)            // Y_ab = sum_k N21_ak T11_kb
            warp_block_mma16(acc, Nm + (32 + 16 * a) * kLd + 16 * k2, kLd, Tm + (16 * k2) * kLd + 16 * b, kLd);
        store_f16(Yw, kLdY, acc, 1.f);
    }
    bar_sync(kBarInverse, 128);
    {
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        for (int k2 = 0; k2 <= a; ++k2)           // T21_ab = -sum_k T22_ak Y_kb
            warp_block_mma16(acc, Tm + (32 + 16 * a) * kLd + 32 + 16 * k2, kLd, Y + (2 * k2 + b) * 16 * kLdY, kLdY);
        store_tp16(sm, 32 + 16 * a, 16 * b, acc, -1.f, s_beta);
    }
}

template <int MODE>
__device__ void producer(const Params& p, uint8_t* sm, uint32_t sb, int prank, int n_seq, int h,
                         int64_t bos, int64_t eos, bool aborted) {
    constexpr bool kG = (MODE & kGate) != 0;
    constexpr bool kCv = (MODE & kConv) != 0;
    constexpr uint32_t kGBytes = kG ? 16384u : 32768u;   // raw logits bf16, or g fp32
    constexpr int halo = kCv ? kHalo : 0;
    constexpr uint32_t kTileBytes = (kC + halo) * 256;   // one q / k / v tile
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* misc = sm + P_MISC;
    const uint32_t tm = *reinterpret_cast<uint32_t*>(misc + M_TMEM);
    const int H = p.H;
    const int nchunks = (int)((eos - bos + kC - 1) / kC);
    const int ntasks = nchunks >= prank ? (nchunks - prank) / kProducers + 1 : 0;
    const uint32_t c_misc = map_to_rank(sb + C_MISC, 0);
    auto chunk_of = [&](int task) { return prank - 1 + kProducers * task; };

    if (warp == kIoWarp) {
        // ---------------- I/O warp: lane 0 loads tiles, lane 1 stores and announces ----------
        if (lane == 0 && !aborted && ntasks > 0) {
            auto issue_qkv = [&](int task) {
                const int c0 = (int)(bos + (int64_t)chunk_of(task) * kC) - halo;
                mbar_arrive_expect_tx(bar_at(misc, M_QK_FULL), (kCv ? 3u : 2u) * kTileBytes);
                tma_load_3d(sb + P_Q, &p.tq, 0, h, c0, bar_at(misc, M_QK_FULL));
                tma_load_3d(sb + P_K, &p.tk, 0, h, c0, bar_at(misc, M_QK_FULL));
                if constexpr (kCv) tma_load_3d(sb + P_V, &p.tv, 0, h, c0, bar_at(misc, M_QK_FULL));
            };
            auto issue_g = [&](int task) {
                const int c0 = (int)(bos + (int64_t)chunk_of(task) * kC);
                mbar_arrive_expect_tx(bar_at(misc, M_G_FULL), kGBytes);
                tma_load_3d(sb + P_G, &p.tg, 0, h, c0, bar_at(misc, M_G_FULL));
            };
            issue_qkv(0);
            issue_g(0);
            int last_qkv = 0, last_g = 0;
            for (int task = 0; task + 1 < ntasks; ++task) {
                if (!wait_one(bar_at(misc, M_RAW_FREE), task & 1, p)) break;
                issue_qkv(task + 1);
                last_qkv = task + 1;
                // with kConv the g tile holds the conv's v until that leaves with the A part
                if (kCv && !wait_one(bar_at(misc, M_LKQ_FREE), task & 1, p)) break;
                issue_g(task + 1);
                last_g = task + 1;
            }
            // the tiles of the last loads must land before the CTA may leave
            mbar_wait(bar_at(misc, M_QK_FULL), last_qkv & 1, kDefaultWaitCycles);
            mbar_wait(bar_at(misc, M_G_FULL), last_g & 1, kDefaultWaitCycles);
        } else if (lane == 1 && !aborted && ntasks > 0) {
            uint8_t* ring = p.ring + (size_t)ld_cluster_u32(c_misc + M_SMID) * ((size_t)kRing * kSlotBytes);
            uint32_t ph_gfree = 0;
            for (int task = 0; task < ntasks; ++task) {
                const int n = chunk_of(task);
                const int rs = n % kRing;
                uint8_t* slot = ring + (size_t)rs * kSlotBytes;
                if (!wait_one(bar_at(misc, M_LKQ_READY), task & 1, p)) break;
                if (n >= kRing) {
                    const bool ok = wait_one(bar_at(misc, M_GFREE + 8u * rs), (ph_gfree >> rs) & 1u, p, true);
                    ph_gfree ^= 1u << rs;
                    if (!ok) break;
                }
                bulk_store(slot + S_LKQ, sb + P_LKQ, kAPart);
                if constexpr (kCv) bulk_store(slot + S_V, sb + P_G, kVPart);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(bar_at(misc, M_LKQ_FREE));
                if (!wait_one(bar_at(misc, M_ST_READY), task & 1, p)) break;
                bulk_store(slot + S_YW, sb + P_ST, kBPart);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(bar_at(misc, M_ST_FREE));
                bulk_wait0();
                fence_proxy_async_global();
                mbar_arrive_remote(c_misc + M_GFULL + 8u * (uint32_t)rs);
            }
            bulk_wait0();
        }
        __syncwarp();
        return;
    }

    // ---------------- compute warps ----------------
    float* s_beta = reinterpret_cast<float*>(misc + M_BETA);
    float* s_ga = reinterpret_cast<float*>(misc + M_GA);
    float* s_gc = reinterpret_cast<float*>(misc + M_GC);
    float* s_rhf = reinterpret_cast<float*>(misc + M_RHF);
    float* s_wsum = reinterpret_cast<float*>(sm + P_NM);   // (the inverse's scratch is idle)
    float* facs = reinterpret_cast<float*>(sm + P_LKQ + S_FAC);
    const int cg = lane & 15, tp = lane >> 4;           // fold: channel group of 8, token pair
    const int t0 = 4 * warp + 2 * tp;                   // fold: tokens t0, t0 + 1
    const int q4 = warp & 3, cb = warp >> 2;            // TMEM lane quarter, 16-column block
    const uint32_t lane_sel = (uint32_t)(32 * q4) << 16;
    int ap_issued = 0, ap_waited = 0, yw_issued = 0, yw_waited = 0;   // warp 0's products
    auto beta_at = [&](int64_t t) {
        if constexpr (kG) return sigmoid_f(__bfloat162float(p.beta_raw[t * H + h]));
        else return p.beta[t * H + h];
    };
    float cneg = 0.f;                                   // kGate: -exp(A_log[h]) log2(e)
    if constexpr (kG) {
        cneg = -expf(p.A_log[h]) * kLog2e;
        if (tid < kD) reinterpret_cast<float*>(misc + M_DT)[tid] = p.dt_bias[h * kD + tid];
        bar_sync(kBarCompute, kCompute);
    }
    float beta_nx = 0.f;                                // beta of the next task (threads < 64)
    if (ntasks > 0 && tid < kC) {
        const int64_t c0 = bos + (int64_t)chunk_of(0) * kC;
        if (c0 + tid < eos) beta_nx = beta_at(c0 + tid);
    }
    int fail = aborted ? 1 : 0;
    for (int task = 0; task < ntasks && !aborted; ++task) {
        const int n = chunk_of(task);
        const int64_t c0 = bos + (int64_t)n * kC;
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
        const uint32_t ph = (uint32_t)task & 1u;
        if (tid < kC) s_beta[tid] = beta_nx;
        beta_nx = 0.f;
        if (task + 1 < ntasks && tid < kC) {
            const int64_t c1 = bos + (int64_t)chunk_of(task + 1) * kC;
            if (c1 + tid < eos) beta_nx = beta_at(c1 + tid);
        }
        trace_mark(prank, n, 0);
        bool ok = wait_warp(bar_at(misc, M_QK_FULL), ph, p) && wait_warp(bar_at(misc, M_G_FULL), ph, p) &&
                  (task == 0 || wait_warp(bar_at(misc, M_LKQ_FREE), ph ^ 1u, p));
        trace_mark(prank, n, 1);
        // ---- fold, part 1: decay sums (log2 units) of the token pair, then of the warp's 4 tokens ----
        float s0[8], s1[8], xo[8];
        if (ok) {
            float ga[8], gb[8];                          // log-decay of tokens t0, t0 + 1 (log2)
            if constexpr (kG) {
                float xa[8], xb[8];
                unpack8(ld16(sm, P_G + t0 * 256 + cg * 16), xa);
                unpack8(ld16(sm, P_G + (t0 + 1) * 256 + cg * 16), xb);
                const float* dt = reinterpret_cast<const float*>(misc + M_DT) + 8 * cg;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    ga[c] = cneg * softplus_fast(xa[c] + dt[c]);
                    gb[c] = cneg * softplus_fast(xb[c] + dt[c]);
                }
            } else {
                const float4* G = reinterpret_cast<const float4*>(sm + P_G);
                const float4 a0 = G[t0 * 32 + 2 * cg], a1 = G[t0 * 32 + 2 * cg + 1];
                const float4 b0 = G[(t0 + 1) * 32 + 2 * cg], b1 = G[(t0 + 1) * 32 + 2 * cg + 1];
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    ga[c] = av[c] * kLog2e;
                    gb[c] = bv[c] * kLog2e;
                }
            }
            const float m0 = t0 < L ? 1.f : 0.f, m1 = t0 + 1 < L ? 1.f : 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                s0[c] = ga[c] * m0;
                s1[c] = fmaf(gb[c], m1, s0[c]);
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) s0[c] = s1[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) xo[c] = __shfl_xor_sync(0xffffffffu, s1[c], 16);
        if (ok && tp == 0) {
            float4* W = reinterpret_cast<float4*>(s_wsum + warp * kD + 8 * cg);
            W[0] = make_float4(s1[0] + xo[0], s1[1] + xo[1], s1[2] + xo[2], s1[3] + xo[3]);
            W[1] = make_float4(s1[4] + xo[4], s1[5] + xo[5], s1[6] + xo[6], s1[7] + xo[7]);
        }
        fail |= !ok;
        if (bar_sync_or(kBarCompute, kCompute, fail)) break;
        // ---- exclusive prefix over the 16 warps, per channel; range test ----
        int bad_c = 0;
        if (tid < kD) {
            float run = 0.f, ga = 0.f;
#pragma unroll
            for (int ww = 0; ww < 16; ++ww) {
                const float v = s_wsum[ww * kD + tid];
                s_wsum[ww * kD + tid] = run;
                run += v;
                if (ww == 7) ga = run;
            }
            s_ga[tid] = ga;
            s_gc[tid] = run;
            const float kHalf2 = kHalfRange * kLog2e;
            bad_c = (ga < -kHalf2) || (run - ga < -kHalf2);
        }
        const bool bad = bar_sync_or(kBarCompute, kCompute, bad_c) != 0;
        trace_mark(prank, n, 8);
        if constexpr (kCv) {
            // ---- conv prologue: q, k, v of tokens t0, t0 + 1 (8 channels each) from raw rows
            //      t0 - 3 .. t0 + 1 (history before the sequence: the conv cache or zero), SiLU,
            //      and the L2 norm of q and k over the 16 lanes that hold a token's 128 channels
            uint4 outv[2][2];                            // q, k after the conv (v is stored at once)
#pragma unroll
            for (int z = 2; z >= 0; --z) {
                const uint32_t tile = z == 0 ? P_Q : (z == 1 ? P_K : P_V);
                // the five raw rows t0 - 3 .. t0 + 1 of this thread's 8 channels, packed
                uint4 rows[5];
#pragma unroll
                for (int j = 0; j < 5; ++j) {
                    const int r = t0 - kHalo + j;                 // token row relative to c0
                    rows[j] = ld16(sm, tile + (r + kHalo) * 256 + cg * 16);
                    if (c0 + r < bos) {                           // before the sequence
                        float x[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            float hv = 0.f;
                            if (p.conv_state != nullptr) {
                                const int64_t ch = (int64_t)z * H * kD + (int64_t)h * kD + 8 * cg + c;
                                hv = __bfloat162float(p.conv_state[((int64_t)n_seq * H * 3 * kD + ch) * 3 +
                                                                   (kHalo - (int)(bos - (c0 + r)))]);
                            }
                            x[c] = hv;
                        }
                        rows[j] = pack8(x);
                    }
                }
                // y = (weights / 2) . x, so that SiLU is h + h tanh(h) straight from the sum
                float y0[8], y1[8];
                const float4* wz = reinterpret_cast<const float4*>(misc + M_WCV) + z * kD + cg;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 w = wz[16 * c];
                    float xc[5];
#pragma unroll
                    for (int j = 0; j < 5; ++j) {
                        const uint32_t wd = (&rows[j].x)[c >> 1];
                        xc[j] = __uint_as_float((c & 1) ? (wd & 0xffff0000u) : (wd << 16));
                    }
                    y0[c] = fmaf(w.w, xc[3], fmaf(w.z, xc[2], fmaf(w.y, xc[1], w.x * xc[0])));
                    y1[c] = fmaf(w.w, xc[4], fmaf(w.z, xc[3], fmaf(w.y, xc[2], w.x * xc[1])));
                }
                float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    y0[c] = silu_half(y0[c]);
                    y1[c] = silu_half(y1[c]);
                    ss0 = fmaf(y0[c], y0[c], ss0);
                    ss1 = fmaf(y1[c], y1[c], ss1);
                }
                if (z < 2) {
#pragma unroll
                    for (int o = 1; o < 16; o <<= 1) {
                        ss0 += __shfl_xor_sync(0xffffffffu, ss0, o);
                        ss1 += __shfl_xor_sync(0xffffffffu, ss1, o);
                    }
                    const float i0 = rsqrtf(ss0 + p.l2_eps), i1 = rsqrtf(ss1 + p.l2_eps);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        y0[c] *= i0;
                        y1[c] *= i1;
                    }
                }
                if (z == 2) {                            // the g tile is dead: v goes there now
                    st16(sm, P_G + (uint32_t)(cg >> 3) * 8192 + sw128(t0, cg & 7, 0, 0), pack8(y0));
                    st16(sm, P_G + (uint32_t)(cg >> 3) * 8192 + sw128(t0 + 1, cg & 7, 0, 0), pack8(y1));
                } else {
                    outv[z][0] = pack8(y0);
                    outv[z][1] = pack8(y1);
                }
            }
            bar_sync(kBarCompute, kCompute);             // every raw row has been read
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int t = t0 + u;
                st16(sm, P_Q + (t + kHalo) * 256 + cg * 16, outv[0][u]);
                st16(sm, P_K + (t + kHalo) * 256 + cg * 16, outv[1][u]);
            }
            bar_sync(kBarCompute, kCompute);
        }
        trace_mark(prank, n, 9);
        // ---- fold, part 2: folded operands Lk, Lq (A of A|P and of the consumer's X | O), R ----
        {
            const int ac = cg >> 3, ch = cg & 7;
            float gam0[8], gam1[8], gr[8], gs[8];
            {
                const float4* W = reinterpret_cast<const float4*>(s_wsum + warp * kD + 8 * cg);
                const float4 w0 = W[0], w1 = W[1];
                const float off[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float base = off[c] + (tp ? xo[c] : 0.f);
                    gam0[c] = base + s0[c];
                    gam1[c] = base + s1[c];
                }
                const float4* GA = reinterpret_cast<const float4*>(s_ga + 8 * cg);
                const float4* GC = reinterpret_cast<const float4*>(s_gc + 8 * cg);
                const float4 ga0 = GA[0], ga1 = GA[1], gc0 = GC[0], gc1 = GC[1];
                const float gav[8] = {ga0.x, ga0.y, ga0.z, ga0.w, ga1.x, ga1.y, ga1.z, ga1.w};
                const float gcv[8] = {gc0.x, gc0.y, gc0.z, gc0.w, gc1.x, gc1.y, gc1.z, gc1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    gr[c] = bad ? 0.f : gav[c];
                    gs[c] = bad ? gcv[c] : gav[c];
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int t = t0 + u;
                const bool valid = t < L;
                float qv[8], kv[8];
                unpack8(ld16(sm, P_Q + (t + halo) * 256 + cg * 16), qv);
                unpack8(ld16(sm, P_K + (t + halo) * 256 + cg * 16), kv);
                uint32_t lk[4], lq[4], rr[4];
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float gm0 = u ? gam1[c] : gam0[c], gm1 = u ? gam1[c + 1] : gam0[c + 1];
                    const float a0 = ex2_approx(gm0 - gr[c]), a1 = ex2_approx(gm1 - gr[c + 1]);
                    const float b0 = ex2_approx(gs[c] - gm0), b1 = ex2_approx(gs[c + 1] - gm1);
                    const float k0 = valid ? kv[c] : 0.f, k1 = valid ? kv[c + 1] : 0.f;
                    const float q0 = valid ? qv[c] : 0.f, q1 = valid ? qv[c + 1] : 0.f;
                    lk[c / 2] = pack_bf16(k0 * a0, k1 * a1);
                    lq[c / 2] = pack_bf16(q0 * a0, q1 * a1);
                    rr[c / 2] = pack_bf16(k0 * b0, k1 * b1);
                }
                st16(sm, P_LKQ + sw128(t, ch, ac, 128), make_uint4(lk[0], lk[1], lk[2], lk[3]));
                st16(sm, P_LKQ + sw128(64 + t, ch, ac, 128), make_uint4(lq[0], lq[1], lq[2], lq[3]));
                st16(sm, P_R + sw128(t, ch, ac, 64), make_uint4(rr[0], rr[1], rr[2], rr[3]));
            }
            if (tid < kD) {
                const float ga = s_ga[tid], gc = s_gc[tid];
                const float gra = bad ? 0.f : ga, gsa = bad ? gc : ga;
                facs[tid] = ex2_approx(gra);
                facs[kD + tid] = ex2_approx(gc);
                s_rhf[tid] = ex2_approx(gc - gsa);
            }
        }
        fence_async_smem();
        tc_fence_before();
        bar_sync(kBarCompute, kCompute);
        trace_mark(prank, n, 2);
        if (tid == 0) {
            if (!bad) mbar_arrive(bar_at(misc, M_RAW_FREE));   // the q, k (v) tiles are dead
            mbar_arrive(bar_at(misc, M_LKQ_READY));            // [Lk ; Lq | factors] may leave
        }
        if (warp == 0) {                               // [A ; P] = [Lk ; Lq] R^T
            tc_fence_after();
            if (elect_one()) {
                const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tm + TP_AP, make_desc(sb + P_LKQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                             make_desc(sb + P_R + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), id, s > 0);
                mma_commit(bar_at(misc, M_AP));
            }
            __syncwarp();
            ++ap_issued;
        }
        // ---- extraction: N = diag(beta) A (strictly lower, fp32), P' (inclusive, bf16) ----
        ok = wait_warp(bar_at(misc, M_AP), ph, p);
        trace_mark(prank, n, 3);
        if (warp == 0 && ok) ++ap_waited;
        tc_fence_after();
        if (ok && !bad) {
            float val[16];
            tmem_ld16(tm + lane_sel + TP_AP + 16 * cb, val);
            const int i0 = 16 * cb;
            if (q4 < 2) {
                const int r = 32 * q4 + lane;
                const float br = s_beta[r];
                float* Nr = reinterpret_cast<float*>(sm + P_NM) + r * kLd + i0;
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    float4 w;
                    w.x = (i0 + 4 * i4 + 0 < r) ? br * val[4 * i4 + 0] : 0.f;
                    w.y = (i0 + 4 * i4 + 1 < r) ? br * val[4 * i4 + 1] : 0.f;
                    w.z = (i0 + 4 * i4 + 2 < r) ? br * val[4 * i4 + 2] : 0.f;
                    w.w = (i0 + 4 * i4 + 3 < r) ? br * val[4 * i4 + 3] : 0.f;
                    reinterpret_cast<float4*>(Nr)[i4] = w;
                }
            } else {
                const int r = 32 * (q4 - 2) + lane;
#pragma unroll
                for (int k8 = 0; k8 < 2; ++k8) {
                    float pv[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) pv[u] = (i0 + 8 * k8 + u <= r) ? val[8 * k8 + u] : 0.f;
                    st16(sm, P_PO + sw128(r, 2 * cb + k8, 0, 0), pack8(pv));
                }
            }
        }
        fail |= !ok;
        if (bad) {
            // the exact path uses the staging as scratch: the previous chunk must have left it
            ok = task == 0 || wait_warp(bar_at(misc, M_ST_FREE), ph ^ 1u, p);
            fail |= !ok;
            if (bar_sync_or(kBarCompute, kCompute, fail)) break;
            exact_ap<MODE>(p, sm, s_beta, h, c0, L);
        }
        fence_async_smem();
        if (bar_sync_or(kBarCompute, kCompute, fail)) break;
        if (bad && tid == 0) mbar_arrive(bar_at(misc, M_RAW_FREE));   // the exact path is done
        trace_mark(prank, n, 4);
        // ---- T' = (I + N)^-1 diag(beta) on warps 0..3 ----
        if (warp < 4) inverse(sm, s_beta);
        fence_async_smem();
        bar_sync(kBarCompute, kCompute);
        trace_mark(prank, n, 5);
        // ---- Yh^T = R^T T' (M = key ch) and Wh^T = P' T' (M = token) ----
        if (warp == 0) {
            tc_fence_after();
            if (elect_one()) {
                const uint32_t idY = idesc_bf16(128, 64, true, true);
                const uint32_t idW = idesc_bf16(128, 64, false, true);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tm + TP_Y, make_desc(sb + P_R + s * 2048, 8192, 1024),
                             make_desc(sb + P_TP + s * 2048, 8192, 1024), idY, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tm + TP_W, make_desc(sb + P_PO + s * 32, 16, 1024),
                             make_desc(sb + P_TP + s * 2048, 8192, 1024), idW, s > 0);
                mma_commit(bar_at(misc, M_YW));
            }
            __syncwarp();
            ++yw_issued;
        }
        ok = wait_warp(bar_at(misc, M_YW), ph, p);
        trace_mark(prank, n, 6);
        if (warp == 0 && ok) ++yw_waited;
        if (ok && !bad && task > 0) ok = wait_warp(bar_at(misc, M_ST_FREE), ph ^ 1u, p);
        tc_fence_after();
        // ---- staging: Yh^T rows scaled by e^{gamma_C - gamma_s}, then Wh^T, as bf16 ----
        if (ok) {
            float val[16];
            const int c = 32 * q4 + lane;
            tmem_ld16(tm + lane_sel + TP_Y + 16 * cb, val);
            const float f = s_rhf[c];
#pragma unroll
            for (int u = 0; u < 16; ++u) val[u] *= f;
            st16(sm, P_ST + sw128(c, 2 * cb, 0, 0), pack8(val));
            st16(sm, P_ST + sw128(c, 2 * cb + 1, 0, 0), pack8(val + 8));
            if (q4 < 2) {
                tmem_ld16(tm + lane_sel + TP_W + 16 * cb, val);
                st16(sm, P_ST + sw128(128 + c, 2 * cb, 0, 0), pack8(val));
                st16(sm, P_ST + sw128(128 + c, 2 * cb + 1, 0, 0), pack8(val + 8));
            }
        }
        fail |= !ok;
        fence_async_smem();
        tc_fence_before();
        if (bar_sync_or(kBarCompute, kCompute, fail)) break;
        if (tid == 0) mbar_arrive(bar_at(misc, M_ST_READY));
        trace_mark(prank, n, 7);
    }
    // products still in flight must finish before the tensor memory is freed (the last commit
    // on each barrier covers every earlier product)
    if (warp == 0) {
        if (ap_issued > ap_waited)
            mbar_wait(bar_at(misc, M_AP), (uint32_t)(ap_issued - 1) & 1u, kDefaultWaitCycles);
        if (yw_issued > yw_waited)
            mbar_wait(bar_at(misc, M_YW), (uint32_t)(yw_issued - 1) & 1u, kDefaultWaitCycles);
    }
}

// ============================== consumer ==============================

template <int MODE>
__device__ void consumer(const Params& p, uint8_t* sm, uint32_t sb, int n_seq, int h,
                         int64_t bos, int64_t eos, bool aborted, bool trans_unit) {
    constexpr bool kN = (MODE & kNorm) != 0;
    constexpr bool kSt = (MODE & kStates) != 0;
    const bool trans = kSt && trans_unit;
    // this unit's output (a transition's goes to o2 through to2), or none
    const bool has_out = !kSt || (trans ? p.o2 : p.o) != nullptr;
    constexpr bool kCv = (MODE & kConv) != 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* misc = sm + C_MISC;
    const uint32_t tm = *reinterpret_cast<uint32_t*>(misc + M_TMEM);
    const int H = p.H;
    const int nchunks = (int)((eos - bos + kC - 1) / kC);

    if (warp == kIoWarp) {
        // ---------------- loader: V tiles, each chunk's factors, ring slots back ----------------
        if (lane == 0 && !aborted && nchunks > 0) {
            const uint8_t* ring = p.ring + (size_t)smid() * ((size_t)kRing * kSlotBytes);
            uint32_t ph_gfull = 0;
            int loaded = 0;          // chunks whose A and B loads were issued
            int v_issued = 0;        // chunks whose V tiles were issued
            bool ok = true;
            // the ring slot of chunk mm goes back to the producer that writes chunk mm + kRing
            // once both of its loads have landed
            auto release = [&](int mm) -> bool {
                const uint32_t par = (uint32_t)(mm >> 1) & 1u;
                if (!wait_one(bar_at(misc, M_AFULL + 8 * (mm & 1)), par, p) ||
                    !wait_one(bar_at(misc, M_BFULL + 8 * (mm & 1)), par, p))
                    return false;
                if constexpr (kCv) {        // the V tiles were read from the slot too
                    if (!wait_one(bar_at(misc, M_VFULL + 8 * (mm & 1)), par, p) ||
                        !wait_one(bar_at(misc, M_VFULL + 8 * (2 + (mm & 1))), par, p))
                        return false;
                }
                if (mm + kRing < nchunks)
                    mbar_arrive_remote(map_to_rank(sb + P_MISC + M_GFREE + 8u * (uint32_t)(mm % kRing),
                                                   1 + (mm + kRing) % kProducers));
                return true;
            };
            for (int m = 0; m < nchunks && ok; ++m) {
                const int sl = m & 1;
                const uint32_t pfree = (uint32_t)((m - 2) >> 1) & 1u;
                const int c0 = (int)(bos + (int64_t)m * kC);
                const int rs = m % kRing;
                const uint8_t* slot = ring + (size_t)rs * kSlotBytes;
                // V tiles: by TMA from v, or (kConv) the conv's output from the ring slot. A
                // transition takes v as zero: its tiles come from token rows before the tensor,
                // which the copy fills with zeros (the column coordinate stays aligned)
                if constexpr (!kCv) {
                    const int vrow = trans ? -2 * kC : c0;
                    for (int hh = 0; hh < 2; ++hh) {
                        uint64_t* vf = bar_at(misc, M_VFULL + 8 * (2 * hh + sl));
                        if (m >= 2 && !(ok = wait_one(bar_at(misc, M_VFREE + 8 * (2 * hh + sl)), pfree, p))) break;
                        mbar_arrive_expect_tx(vf, 8192u);
                        tma_load_3d(sb + C_V + (uint32_t)(2 * hh + sl) * 8192, &p.tv, 64 * hh, h, vrow, vf);
                        v_issued = m + 1;
                    }
                    if (!ok) break;
                }
                ok = wait_one(bar_at(misc, M_GFULL + 8 * rs), (ph_gfull >> rs) & 1u, p, true);
                ph_gfull ^= 1u << rs;
                if (!ok) break;
                fence_proxy_async_global();
                if constexpr (kCv) {
                    for (int hh = 0; hh < 2; ++hh) {
                        uint64_t* vf = bar_at(misc, M_VFULL + 8 * (2 * hh + sl));
                        if (m >= 2 && !(ok = wait_one(bar_at(misc, M_VFREE + 8 * (2 * hh + sl)), pfree, p))) break;
                        mbar_arrive_expect_tx(vf, 8192u);
                        bulk_load(sb + C_V + (uint32_t)(2 * hh + sl) * 8192, slot + S_V + hh * 8192, 8192u, vf);
                        v_issued = m + 1;
                    }
                    if (!ok) break;
                }
                if (m >= 2 && !(ok = wait_one(bar_at(misc, M_AFREE + 8 * sl), pfree, p))) break;
                mbar_arrive_expect_tx(bar_at(misc, M_AFULL + 8 * sl), kAPart);
                bulk_load(sb + C_A + (uint32_t)sl * kAPart, slot + S_LKQ, kAPart, bar_at(misc, M_AFULL + 8 * sl));
                if (m >= 2 && !(ok = wait_one(bar_at(misc, M_BFREE + 8 * sl), pfree, p))) {
                    // the A load of this chunk is in flight: it must land before the CTA leaves
                    mbar_wait(bar_at(misc, M_AFULL + 8 * sl), (uint32_t)(m >> 1) & 1u, kDefaultWaitCycles);
                    break;
                }
                mbar_arrive_expect_tx(bar_at(misc, M_BFULL + 8 * sl), kBPart);
                bulk_load(sb + C_B + (uint32_t)sl * kBPart, slot + S_YW, kBPart, bar_at(misc, M_BFULL + 8 * sl));
                loaded = m + 1;
                if (m >= 1) ok = release(m - 1);
            }
            if (ok && loaded == nchunks) release(nchunks - 1);
            // every copy issued into this CTA's shared memory must land before it leaves
            for (int mm = (loaded > 2 ? loaded - 2 : 0); mm < loaded; ++mm) {
                const uint32_t par = (uint32_t)(mm >> 1) & 1u;
                mbar_wait(bar_at(misc, M_AFULL + 8 * (mm & 1)), par, kDefaultWaitCycles);
                mbar_wait(bar_at(misc, M_BFULL + 8 * (mm & 1)), par, kDefaultWaitCycles);
            }
            for (int mm = (v_issued > 2 ? v_issued - 2 : 0); mm < v_issued; ++mm)
                for (int hh = 0; hh < 2; ++hh)
                    mbar_wait(bar_at(misc, M_VFULL + 8 * (2 * hh + (mm & 1))), (uint32_t)(mm >> 1) & 1u,
                              kDefaultWaitCycles);
        }
        __syncwarp();
        return;
    }

    // ---------------- the two halves of the value columns ----------------
    const int half = warp >> 3, lw = warp & 7, q = lw & 3, cp = lw >> 2;
    const int tid_h = tid & 255;
    const uint32_t lane_sel = (uint32_t)(32 * q) << 16;
    const int bar_half = 1 + half, bar_out = 3 + half;
    const uint32_t t_xo = tm + 128 * half, t_ds = tm + 256 + 64 * half;
    uint64_t* bar_xo = bar_at(misc, M_XO + 8 * half);
    uint64_t* bar_ds = bar_at(misc, M_DS + 8 * half);
    const uint32_t sm_h = C_SM + 16384u * half, u_h = C_U + 8192u * half, ost_h = C_OST + 8192u * half;
    const int i_row = 32 * q + lane;                 // state row (key channel) of this thread
    const int jg0 = 64 * half + 32 * cp;             // its first value column
    const int64_t sbase = ((int64_t)n_seq * H + h) * kD * kD;
    const bool issuer = (lw == 0);
    int xo_issued = 0, xo_waited = 0, ds_issued = 0, ds_waited = 0;   // issuer's bookkeeping

    float S[32];
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (trans) {                             // the identity
            const int d = i_row - (jg0 + 4 * c4);
            v = make_float4(d == 0, d == 1, d == 2, d == 3);
        } else if (p.h0) {
            v = reinterpret_cast<const float4*>(p.h0 + sbase + (int64_t)i_row * kD + jg0)[c4];
        }
        S[4 * c4] = v.x; S[4 * c4 + 1] = v.y; S[4 * c4 + 2] = v.z; S[4 * c4 + 3] = v.w;
    }
    auto fac = [&](int nn) {
        return reinterpret_cast<const float*>(sm + C_A + (uint32_t)(nn & 1) * kAPart + S_FAC);
    };
    // Sm(nn) = diag(e^{gamma_ref(nn)}) S as bf16, MN-major (K = key channel, N = value column)
    auto write_sm = [&](int nn) {
        const float e = fac(nn)[i_row];
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
            float w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) w[u] = S[8 * k8 + u] * e;
            st16(sm, sm_h + sw128(i_row, 4 * cp + k8, 0, 0), pack8(w));
        }
    };
    auto issue_xo = [&](int nn) {
        tc_fence_after();
        if (elect_one()) {
            const uint32_t id = idesc_bf16(128, 64, false, true);
            const uint32_t a = sb + C_A + (uint32_t)(nn & 1) * kAPart + S_LKQ;
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(t_xo + 64 * (nn & 1), make_desc(a + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                         make_desc(sb + sm_h + s * 2048, 8192, 1024), id, s > 0);
            mma_commit(bar_xo);
        }
        __syncwarp();
        ++xo_issued;
    };
    // O of chunk nn (rows 64..127 of its [X ; O] accumulator) by the output warps: bf16 through
    // the swizzled staging and one TMA store, or straight to global for a ragged last chunk
    // (rows past the sequence belong to the next one). The named barriers run whether or not
    // `ok` holds, so the four warps always meet.
    // kNorm, by the output warps once O(nn) is complete in tensor memory (the wait for the
    // [X ; O] products of chunk nn + 1 covers it), while the other warps form U: the per-token
    // sums of squares over this half's 64 columns, published for both halves' epilogues, and
    // the gate tile of chunk nn (landed in the staging buffer) turned into sigmoid(z) w_norm in
    // place. Returns false if a wait gave up; the named barrier runs either way.
    auto norm_prep = [&](int nn, bool ok) -> bool {
        const int t = 32 * (q - 2) + lane;
        float ss = 0.f;
        if (ok) {
#pragma unroll
            for (int hx = 0; hx < 2; ++hx) {
                float ov[16];
                tmem_ld16(t_xo + 64 * (nn & 1) + lane_sel + 32 * cp + 16 * hx, ov);
#pragma unroll
                for (int u = 0; u < 16; ++u) ss = fmaf(ov[u], ov[u], ss);
            }
        }
        float* s_ss = reinterpret_cast<float*>(misc + M_SS) + (nn % 3) * 256;
        s_ss[(2 * half + cp) * 64 + t] = ss * p.scale * p.scale;
        bar_sync(bar_out, 128);
        if (ok && lw == 2 && lane == 0) mbar_arrive(bar_at(misc, M_NRM + 8 * (nn & 1)));
        ok = ok && wait_warp(bar_at(misc, M_ZFULL + 8 * half), (uint32_t)nn & 1u, p);
        if (ok) {
            const float* wn = reinterpret_cast<const float*>(misc + M_WN) + jg0;
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                const uint32_t off = ost_h + sw128(t, 4 * cp + k8, 0, 0);
                float zv[8];
                unpack8(ld16(sm, off), zv);
#pragma unroll
                for (int u = 0; u < 8; ++u) zv[u] = sigmoid_tanh(zv[u]) * wn[8 * k8 + u];
                st16(sm, off, pack8(zv));
            }
        }
        return ok;
    };
    auto epilogue_o = [&](int nn, bool ok) {
        const int64_t c0 = bos + (int64_t)nn * kC;
        const int L = (int)(eos - c0 < kC ? eos - c0 : kC);
        const int t = 32 * (q - 2) + lane;
        const uint32_t src = t_xo + 64 * (nn & 1) + lane_sel + 32 * cp;
        float inv = 0.f;                            // kNorm: 1 / rms of token t over 128 columns
        uint4 zr[4];
        if constexpr (kN) {
            // sigmoid(z) w_norm for this thread's 32 outputs, formed in the staging tile by
            // norm_prep (the same thread, the same 16-byte chunks, which it overwrites below)
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8)
                zr[k8] = ok ? ld16(sm, ost_h + sw128(t, 4 * cp + k8, 0, 0)) : make_uint4(0, 0, 0, 0);
            // both halves' sums of squares of chunk nn, published by norm_prep
            const float* s_ss = reinterpret_cast<const float*>(misc + M_SS) + (nn % 3) * 256;
            ok = ok && wait_warp(bar_at(misc, M_NRM + 8 * (nn & 1)), (uint32_t)(nn >> 1) & 1u, p);
            if (ok) {
                const float tot = s_ss[t] + s_ss[64 + t] + s_ss[128 + t] + s_ss[192 + t];
                inv = rsqrtf(tot * (1.f / kD) + p.norm_eps);
            }
        }
        // this thread's 16 output values hx (scaled, and normed with kNorm), as bf16
        auto finish = [&](int hx, float* ov) {
#pragma unroll
            for (int u = 0; u < 16; ++u) ov[u] *= p.scale;
            if constexpr (kN) {
                float zv[16];
                unpack8(zr[2 * hx], zv);
                unpack8(zr[2 * hx + 1], zv + 8);
#pragma unroll
                for (int u = 0; u < 16; ++u) ov[u] = ov[u] * inv * zv[u];
            }
        };
        if (L == kC) {
            const bool storer = (lw == 2 && lane == 0);
            if (storer) bulk_wait_read0();          // the previous tile has left the staging
            bar_sync(bar_out, 128);
            if (ok) {
#pragma unroll
                for (int hx = 0; hx < 2; ++hx) {
                    float ov[16];
                    tmem_ld16(src + 16 * hx, ov);
                    finish(hx, ov);
                    st16(sm, ost_h + sw128(t, 4 * cp + 2 * hx, 0, 0), pack8(ov));
                    st16(sm, ost_h + sw128(t, 4 * cp + 2 * hx + 1, 0, 0), pack8(ov + 8));
                }
            }
            fence_async_smem();
            bar_sync(bar_out, 128);
            if (storer && ok) {
                if constexpr (kSt)
                    tma_store_3d(trans ? &p.to2 : &p.to, 64 * half, h, (int)c0, sb + ost_h);
                else
                    tma_store_3d(&p.to, 64 * half, h, (int)c0, sb + ost_h);
                bulk_commit();
            }
        } else if (ok) {
            uint4* dst = reinterpret_cast<uint4*>((trans ? p.o2 : p.o) + ((c0 + t) * H + h) * kD + jg0);
#pragma unroll
            for (int hx = 0; hx < 2; ++hx) {
                float ov[16];
                tmem_ld16(src + 16 * hx, ov);       // (warp-collective: every lane loads)
                finish(hx, ov);
                if (t < L) {
                    dst[2 * hx] = pack8(ov);
                    dst[2 * hx + 1] = pack8(ov + 8);
                }
            }
        }
    };

    bool stop = aborted;
    int fail = aborted ? 1 : 0;
    // kNorm: the storer of each half loads chunk n's output gate into its staging tile in step (4)
    // of chunk n, well after chunk n - 1's output has been read from it; the epilogue of chunk n
    // reads it a step later
    int z_issued = 0;
    if (kN && lw == 2 && lane == 0 && !stop) {       // the first two gate tiles into L2
        for (int nn = 0; nn < 2 && nn < nchunks; ++nn)
            tma_prefetch_l2_3d(&p.tz, 64 * half, h, (int)(bos + (int64_t)nn * kC));
    }
    // prologue: Sm(0), then [X ; O](0)
    if (!stop && nchunks > 0) {
        const bool ok = wait_warp(bar_at(misc, M_AFULL), 0, p);
        if (ok) write_sm(0);
        fail |= !ok;
        fence_async_smem();
        stop = bar_sync_or(bar_half, 256, fail) != 0;
        if (!stop && issuer) issue_xo(0);
    }
    for (int n = 0; n < nchunks && !stop; ++n) {
        const int b = n & 1;
        // (1) [X ; O](n) is in tensor memory: U(n) = V(n) - X(n) from rows 0..63, and the output
        //     of chunk n - 1 from rows 64..127 of the other accumulator
        bool ok = wait_warp(bar_xo, (uint32_t)b, p);
        trace_mark(0, n, 8 * half + 0, 256 * half);
        if (issuer && ok) ++xo_waited;
        tc_fence_after();
        if (ok && n > 0 && tid_h == 0) mbar_arrive(bar_at(misc, M_BFREE + 8 * ((n - 1) & 1)));
        if constexpr (kN) {
            if (q >= 2 && n > 0) ok = norm_prep(n - 1, ok);
        }
        if (q < 2) {
            if (ok) ok = wait_warp(bar_at(misc, M_VFULL + 8 * (2 * half + b)), (uint32_t)(n >> 1) & 1u, p);
            if (ok) {
                const int t = 32 * q + lane;
                const uint8_t* vt = sm + C_V + (uint32_t)(2 * half + b) * 8192;
#pragma unroll
                for (int hx = 0; hx < 2; ++hx) {
                    float xv[16];
                    tmem_ld16(t_xo + 64 * b + lane_sel + 32 * cp + 16 * hx, xv);
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const int ck = 4 * cp + 2 * hx + k2;
                        float vv[8];
                        unpack8(ld16(vt, t * 128 + ((ck ^ (t & 7)) << 4)), vv);
#pragma unroll
                        for (int u = 0; u < 8; ++u) vv[u] -= xv[8 * k2 + u];
                        st16(sm, u_h + sw128(t, ck, 0, 0), pack8(vv));
                    }
                }
            }
        }
        fail |= !ok;
        fence_async_smem();
        tc_fence_before();
        if (bar_sync_or(bar_half, 256, fail)) { stop = true; break; }
        trace_mark(0, n, 8 * half + 1, 256 * half);
        if (tid_h == 0) mbar_arrive(bar_at(misc, M_VFREE + 8 * (2 * half + b)));
        // the output of chunk n - 1, by the output warps, while the delta product runs (this
        // keeps it off the path from X(n) to the delta)
        trace_mark(0, n, 8 * half + 4, 256 * half + 64);
        if (has_out && q >= 2 && n > 0) epilogue_o(n - 1, ok);
        trace_mark(0, n, 8 * half + 6, 256 * half + 64);
        // (2) state delta Yh^T U (commit), then O(n) += Wh^T U
        if (issuer) {
            if (wait_warp(bar_at(misc, M_BFULL + 8 * b), (uint32_t)(n >> 1) & 1u, p)) {
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t id = idesc_bf16(128, 64, false, true);
                    const uint32_t bp = sb + C_B + (uint32_t)b * kBPart;
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(t_ds, make_desc(bp + s * 32, 16, 1024), make_desc(sb + u_h + s * 2048, 8192, 1024),
                                 id, s > 0);
                    mma_commit(bar_ds);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16(t_xo + 64 * b, make_desc(bp + 8192 + s * 32, 16, 1024),
                                 make_desc(sb + u_h + s * 2048, 8192, 1024), id, 1);
                }
                __syncwarp();
                ++ds_issued;
            } else {
                fail = 1;
            }
        }
        // (3) S' = e^{gamma_C} S + delta, then Sm(n + 1)
        ok = wait_warp(bar_ds, (uint32_t)b, p);
        trace_mark(0, n, 8 * half + 2, 256 * half);
        if (issuer && ok) ++ds_waited;
        tc_fence_after();
        if (ok) {
            const float eC = fac(n)[kD + i_row];
#pragma unroll
            for (int hx = 0; hx < 2; ++hx) {
                float dv[16];
                tmem_ld16(t_ds + lane_sel + 32 * cp + 16 * hx, dv);
#pragma unroll
                for (int u = 0; u < 16; ++u) S[16 * hx + u] = fmaf(eC, S[16 * hx + u], dv[u]);
            }
        }
        if (ok) {
            if (n + 1 < nchunks) {
                ok = wait_warp(bar_at(misc, M_AFULL + 8 * ((n + 1) & 1)), (uint32_t)((n + 1) >> 1) & 1u, p);
                if (ok) write_sm(n + 1);
            }
        }
        fail |= !ok;
        fence_async_smem();
        tc_fence_before();
        if (bar_sync_or(bar_half, 256, fail)) { stop = true; break; }
        trace_mark(0, n, 8 * half + 3, 256 * half);
        if (tid_h == 0) mbar_arrive(bar_at(misc, M_AFREE + 8 * b));
        if (kN && lw == 2 && lane == 0) {
            bulk_wait_read0();
            uint64_t* zf = bar_at(misc, M_ZFULL + 8 * half);
            mbar_arrive_expect_tx(zf, 8192u);
            tma_load_3d(sb + ost_h, &p.tz, 64 * half, h, (int)(bos + (int64_t)n * kC), zf);
            z_issued = n + 1;
            // the gate tile two chunks on, into L2, so that its load then hits L2
            if (n + 2 < nchunks) tma_prefetch_l2_3d(&p.tz, 64 * half, h, (int)(bos + (int64_t)(n + 2) * kC));
        }
        // (4) the next chunk's [X ; O], or a commit that covers O(n) after the last chunk
        if (issuer) {
            if (n + 1 < nchunks) {
                issue_xo(n + 1);
            } else {
                tc_fence_after();
                if (elect_one()) mma_commit(bar_xo);
                __syncwarp();
                ++xo_issued;
            }
        }
    }
    if (!stop && nchunks > 0) {
        const bool ok = wait_warp(bar_xo, (uint32_t)(nchunks & 1), p);
        if (issuer && ok) ++xo_waited;
        tc_fence_after();
        bool oke = ok;
        if constexpr (kN) {
            if (q >= 2) oke = norm_prep(nchunks - 1, oke);
        }
        if (has_out && q >= 2) epilogue_o(nchunks - 1, oke);
        stop = bar_sync_or(bar_half, 256, !ok) != 0;
    }
    float* const hdst = trans ? p.mt : p.ht;
    if (!stop && hdst != nullptr) {
        float4* dst = reinterpret_cast<float4*>(hdst + sbase + (int64_t)i_row * kD + jg0);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) dst[c4] = make_float4(S[4 * c4], S[4 * c4 + 1], S[4 * c4 + 2], S[4 * c4 + 3]);
    }
    if (lw == 2 && lane == 0) {
        bulk_wait0();
        if (kN && z_issued > 0)                 // the last gate tile has landed
            mbar_wait(bar_at(misc, M_ZFULL + 8 * half), (uint32_t)(z_issued - 1) & 1u, kDefaultWaitCycles);
    }
    // products still in flight must finish before the tensor memory is freed
    if (issuer) {
        if (xo_issued > xo_waited) mbar_wait(bar_xo, (uint32_t)((xo_issued - 1) & 1), kDefaultWaitCycles);
        if (ds_issued > ds_waited) mbar_wait(bar_ds, (uint32_t)((ds_issued - 1) & 1), kDefaultWaitCycles);
    }
}

template <int MODE>
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
    const int cid = (int)(blockIdx.x / kCluster);
    const bool trans = (MODE & kStates) != 0 && cid >= p.units;
    unit_of(p, trans ? cid - p.units : cid, reinterpret_cast<int*>(misc + M_TMP), n_seq, h, bos, eos);

    const uint32_t ncols = is_consumer ? kTmemC : kTmemP;
    if (warp == 0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), ncols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        // every barrier completes once per use: one arrival (plus transaction bytes where a TMA
        // or bulk copy feeds it), except the consumer's slot-free barriers: one per half
        if (is_consumer) {
            for (int b = 0; b < kBarsC; ++b) {
                const uint32_t off = 8u * b;
                const bool two = (off >= M_AFREE && off < M_VFULL) || (off >= M_NRM && off < M_NRM + 16);
                mbar_init(bar_at(misc, off), two ? 2 : 1);
            }
            const uint32_t id = smid();
            *reinterpret_cast<uint32_t*>(misc + M_SMID) = id;
            if ((int)id >= p.ring_sms) atomicOr(p.err, kErrTimeout);
        } else {
            for (int b = 0; b < kBarsP; ++b) mbar_init(bar_at(misc, 8u * b), 1);
        }
        fence_mbar_init();
    }
    if (is_consumer && (MODE & kNorm) != 0)          // the output norm's weight
        for (int i = threadIdx.x; i < kD; i += kThreads) reinterpret_cast<float*>(misc + M_WN)[i] = p.w_norm[i];
    if (!is_consumer && (MODE & kConv) != 0) {       // this head's conv weights, halved
        for (int i = threadIdx.x; i < 3 * kD; i += kThreads) {
            const int zz = i / kD, ch = i % kD;
            const float4 w = reinterpret_cast<const float4*>(p.wconv[zz])[(size_t)h * kD + ch];
            reinterpret_cast<float4*>(misc + M_WCV)[zz * kD + (ch % 8) * 16 + ch / 8] =
                make_float4(0.5f * w.x, 0.5f * w.y, 0.5f * w.z, 0.5f * w.w);
        }
    }
    if (!is_consumer) {     // T' blocks above the diagonal are never written: zero them once
        for (int e = threadIdx.x; e < 8192 / 16; e += kThreads) st16(sm, P_TP + 16 * e, make_uint4(0, 0, 0, 0));
        fence_async_smem();
    }
    tc_fence_before();
    cluster_sync();                     // barriers of every CTA exist before any remote arrive
    tc_fence_after();

    // a consumer SM outside the workspace's ring table (flagged above): nobody touches the ring
    const bool aborted = (int)ld_cluster_u32(map_to_rank(sb + C_MISC + M_SMID, 0)) >= p.ring_sms;
    if (is_consumer) consumer<MODE>(p, sm, sb, n_seq, h, bos, eos, aborted, trans);
    else producer<MODE>(p, sm, sb, (int)crank, n_seq, h, bos, eos, aborted);

    tc_fence_before();
    __syncthreads();
    cluster_sync();                     // no CTA leaves while a peer may still write to it
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*reinterpret_cast<uint32_t*>(misc + M_TMEM), ncols);
    }
}

}  // namespace

size_t chunk_tcx_workspace_bytes() { return kTcxWorkspaceBytes; }

int chunk_tcx_cluster_slots() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    static std::atomic<int> cached[64];
    if (dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    const auto kernel = chunk_tcx_kernel<0>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCluster * 64, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return 0;
    if (dev < 64 && n > 0) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

cudaError_t launch_chunk_tcx(const ChunkArgs& a, void* workspace, size_t workspace_bytes,
                             unsigned int* err, cudaStream_t stream) {
    const int64_t units = (int64_t)a.N * a.H;
    if (units == 0) return cudaSuccess;
    const int mode = (a.g_raw != nullptr ? kGate : 0) | (a.z != nullptr ? kNorm : 0) |
                     (a.wconv[0] != nullptr ? kConv : 0);
    const bool transitions = (a.mt != nullptr || a.o_trans != nullptr);
    const bool states = (a.o == nullptr || transitions);
    if (states && mode != 0) return cudaErrorInvalidValue;    // stretch launches: plain inputs
    using KernelFn = void (*)(Params);
    static const KernelFn kernels[8] = {
        chunk_tcx_kernel<0>, chunk_tcx_kernel<1>, chunk_tcx_kernel<2>, chunk_tcx_kernel<3>,
        chunk_tcx_kernel<4>, chunk_tcx_kernel<5>, chunk_tcx_kernel<6>, chunk_tcx_kernel<7>};
    const KernelFn kernel = states ? chunk_tcx_kernel<kStates> : kernels[mode];
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    Params p;
    const bool gate = (mode & kGate) != 0, conv = (mode & kConv) != 0;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int tile_rows = conv ? kC + kHalo : kC;
    const bool maps_ok =
        make_tmap_thd(&p.tq, a.q, BF, 2, a.T_tot, a.H, kD, kD, tile_rows, false) &&
        make_tmap_thd(&p.tk, a.k, BF, 2, a.T_tot, a.H, kD, kD, tile_rows, false) &&
        (gate ? make_tmap_thd(&p.tg, a.g_raw, BF, 2, a.T_tot, a.H, kD, kD, kC, false)
              : make_tmap_thd(&p.tg, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.T_tot, a.H, kD, kD, kC, false)) &&
        (conv ? make_tmap_thd(&p.tv, a.v, BF, 2, a.T_tot, a.H, kD, kD, tile_rows, false)
              : make_tmap_thd(&p.tv, a.v, BF, 2, a.T_tot, a.H, kD, 64, kC, true)) &&
        (a.o == nullptr || make_tmap_thd(&p.to, a.o, BF, 2, a.T_tot, a.H, kD, 64, kC, true)) &&
        (a.o_trans == nullptr || make_tmap_thd(&p.to2, a.o_trans, BF, 2, a.T_tot, a.H, kD, 64, kC, true)) &&
        (a.z == nullptr || make_tmap_thd(&p.tz, a.z, BF, 2, a.T_tot, a.H, kD, 64, kC, true));
    if (!maps_ok) return cudaErrorInvalidValue;
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.g = a.g;
    p.beta = a.beta;
    p.scale = a.scale;
    p.h0 = a.h0;
    p.ht = a.ht;
    p.o = static_cast<__nv_bfloat16*>(a.o);
    p.mt = a.mt;
    p.o2 = static_cast<__nv_bfloat16*>(a.o_trans);
    p.units = (int)units;
    p.cu = a.cu;
    p.T_pad = a.T_pad;
    p.N = a.N;
    p.H = a.H;
    p.err = err;
    p.wait_cycles = g_chunk_wait_cycles > 0 ? g_chunk_wait_cycles : kDefaultWaitCycles;
    p.ring = static_cast<uint8_t*>(workspace);
    p.ring_sms = (int)(workspace_bytes / ((size_t)kRing * kSlotBytes));
    p.g_raw = static_cast<const __nv_bfloat16*>(a.g_raw);
    p.beta_raw = static_cast<const __nv_bfloat16*>(a.beta_raw);
    p.A_log = a.A_log;
    p.dt_bias = a.dt_bias;
    p.z = static_cast<const __nv_bfloat16*>(a.z);
    p.w_norm = a.w_norm;
    p.norm_eps = a.norm_eps;
    for (int i = 0; i < 3; ++i) p.wconv[i] = a.wconv[i];
    p.conv_state = static_cast<const __nv_bfloat16*>(a.conv_state);
    p.l2_eps = a.l2_eps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * (transitions ? 2 : 1) * kCluster), 1, 1);
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
    e = cudaLaunchKernelEx(&cfg, kernel, p);
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
