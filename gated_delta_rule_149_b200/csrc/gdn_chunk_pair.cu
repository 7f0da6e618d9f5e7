// Chunkwise GDN recurrence on sm_100a, split across the two CTAs of a cluster:
// one CTA prepares every chunk's state-independent operands, the other runs
// only the serial state chain.
//
// The recurrence (librediffusion PR #21 page, "What's added": the GDN
// linear-attention recurrence; the causal-streaming and bidirectional forms
// of the flashdreams SANA-WM page), per head, with H = S^T (dk x dv):
//     H_t = a_t (I - b_t k_t k_t^T) H_{t-1} + b_t k_t v_t^T,   o_t = H_t^T q_t
// is evaluated 64 tokens at a time in its WY/UT form.  Per chunk, in scan
// order, with g = log2 a, G_i = sum of g up to and including token i,
// gamma_i = 2^G_i, e_i = 2^(G_end - G_i):
//     A  = strict-lower [ b_i 2^(G_i - G_j) k_i.k_j ],  P = lower [ 2^(G_i - G_j) q_i.k_j ]
//     T  = (I + A)^-1,  T1 = T diag(b gamma),  T2 = T diag(b)
//     U  = T2 V - T1 K H_prev                      (the delta-rule values)
//     O  = diag(gamma) Q H_prev + P U              (the outputs)
//     H  = gamma_end H_prev + K^T diag(e) U        (the next state)
// Substituting U into O gives both from one product with the previous state:
//     [O; U] = [P T2; T2] V + [Q'; -W] H_prev,   Q' = diag(gamma) Q - P T1 K,  W = T1 K,
// so everything except that product and the state update is independent of
// the state, and a chunk's operands A1 = [P T2; T2] (128 x 64) and
// A2 = [Q'; -W] (128 x dk) can be formed ahead of the chain.
//
// One 2-CTA cluster per (direction, batch*head):
//   rank 0, prep:  gates, the masks of [Q;K] K^T, the 64 x 64 solve, the
//                  products P [T1 | T2] and [P T1; T1] K and their epilogues
//                  (tcgen05 MMAs, fp32 accumulators in TMEM); writes A1, A2,
//                  e and gamma_end of each chunk into a small ring of slots in
//                  global memory (it stays in L2: a few chunks per scan);
//   rank 1, chain: loads V, K and the ring slot of each chunk, and runs
//                  D = V^T A1^T + H^T A2^T   (M = dv = 128, N = 128: O^T and U^T)
//                  S = Ubar^T K              (Ubar = diag(e) U; M = dv, N = dk)
//                  H^T <- gamma_end H^T + S  (fp32 in registers)
//                  with H^T and Ubar^T as bf16 A operands in TMEM, and writes O.
// The two CTAs hand slots over with mbarrier arrivals across the cluster; the
// data itself travels through L2 because the shared-memory path between the
// SMs of a cluster is several times slower than L2 for this volume (48 KB per
// chunk).  Bidirectional: both scans run in the same launch; for each output
// tile the first writer stores its bf16 partial and the second adds its fp32
// partial to it and rounds once, after an arrival counter shows the first is
// visible.  With a cooperative launch every cluster is resident and the first
// writer of each tile is known in advance; otherwise a claim on the counter
// decides it at run time.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"
#include "gdn_chunk_common.cuh"

namespace gdn {

extern float *g_debug_dump;
extern long long *g_prof_buf;
void *g_debug_ring = nullptr;
int g_kernel_select = 0;

namespace {

// 14 warps: TMA, MMA, group A (8 warps: two per TMEM lane quarter), group B
// (4 warps: one per quarter).  At most four warps per SM sub-partition leave
// 128 registers a thread (the chain's state threads hold 64 fp32 values).
constexpr int kPThreads = 448;
constexpr int kGroup = 256, kGroupB = 128;
// named barriers: solver groups (2), finisher / output group, gate threads of each
// solver group; the chain's state group uses kBarA
constexpr int kBarA = 1, kBarB = 2, kBarGate = 3, kBarA2 = 4, kBarGate2 = 5;
constexpr int kNG = 4;                    // gate buffers (each solver group computes its next chunk's)
constexpr uint32_t kGateFloats = 9 * 64;
constexpr int kNSlot = 4;                 // ring slots per scan

// ring slot: A1 [128 rows x 64] bf16, A2 [kb][128 rows x 64] bf16 (both 128B-swizzled
// images), then e[64] and gamma_end (fp32)
constexpr uint32_t kSlotA1 = 0, kSlotA2 = 16384, kSlotGates = 49152, kSlotBytes = 49664;

// shared memory (from a 1024-aligned base); the barrier block sits at the same
// offset in both CTAs so that remote arrivals can address it
constexpr uint32_t kOffBar = 0;
// prep
constexpr uint32_t kPStage = 1024;                        // 2 x [kb0: Q|K][kb1: Q|K]
constexpr uint32_t kPStageBytes = 32768;
constexpr uint32_t kPP = kPStage + 2 * kPStageBytes;      // 2 x 8 KB P
constexpr uint32_t kPTB = kPP + 16384;                    // 2 x [PT1 | T1 | PT2 | T2], 8 KB each
constexpr uint32_t kPA2 = kPTB + 65536;                   // A2 staging [kb][128 rows]
constexpr uint32_t kPA = kPA2 + 32768;                    // 2 x fp32 [64][kLDA] solve buffers
constexpr uint32_t kPAStride = 64 * kLDA * 4;
constexpr uint32_t kPGates = kPA + 2 * kPAStride;
constexpr uint32_t kPGst = kPGates + kNG * kGateFloats * 4;   // 512 B: e, gamma_end of the slot
constexpr uint32_t kPEnd = kPGst + 512;
// chain
constexpr int kNVK = 2;                                   // V/K stages
constexpr uint32_t kCStage = 1024;                        // kNVK x [V0 | V1 | K0 | K1]
constexpr uint32_t kCA = kCStage + kNVK * 32768;          // 2 ring-slot images
constexpr uint32_t kCABytes = 50176;
constexpr uint32_t kCO = kCA + 2 * kCABytes;              // 2 output tiles [dv block][64 tokens][64]
constexpr uint32_t kCEnd = kCO + 2 * 16384;
constexpr uint32_t kSmemBytes = (kPEnd > kCEnd ? kPEnd : kCEnd);
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kPP % 1024 == 0 && kPTB % 1024 == 0 && kPA2 % 1024 == 0 && kCA % 1024 == 0 &&
              kCABytes % 1024 == 0 && kCO % 1024 == 0 && kPGst % 16 == 0, "tile alignment");

// TMEM columns
constexpr uint32_t kTD1 = 0, kTD2 = 128, kTD3 = 256;                 // prep
constexpr uint32_t kTD = 0, kTS = 256, kTH = 384, kTUb = 448;         // chain
constexpr uint32_t kTmemCols = 512;

// Chunk-0 products of scan (0, 0) can be dumped for debugging in builds with
// GDN_DEBUG_DUMP; production builds compile the dump code out.
#ifdef GDN_DEBUG_DUMP
constexpr bool kDbgOn = true;
#else
constexpr bool kDbgOn = false;
#endif

constexpr uint32_t kIdM1 = idesc_bf16(128, 64, false, false);   // [Q;K] K^T
constexpr uint32_t kIdM2 = idesc_bf16(64, 128, false, true);    // P [T1 | T2]
constexpr uint32_t kIdM3 = idesc_bf16(128, 128, false, true);   // [P T1; T1] K
constexpr uint32_t kIdA = idesc_bf16(128, 128, true, false);    // V^T A1^T
constexpr uint32_t kIdB = idesc_bf16(128, 128, false, false);   // H^T A2^T (A in TMEM)
constexpr uint32_t kIdC = idesc_bf16(128, 128, false, true);    // Ubar^T K (A in TMEM)

struct PairParams {
    const float *beta, *decay, *state_in;
    float *state_out;
    __nv_bfloat16 *o;
    uint8_t *ring;       // [dirs][BH][kNSlot] slots
    int *counters;       // bidi arrival counters [BH][n_chunks], zeroed
    int *err;            // device error word
    float *debug;        // optional: chunk-0 D and S of scan (0, 0)
    long long *trace;    // tracing builds: clock64 marks of scan (0, 0)
    int BH, T, n_chunks;
    int predict;         // bidi: every cluster resident, first writer known in advance
};

struct Bars {
    // prep
    uint64_t st_full[2], st_empty[2], d1_full[2], d1_empty[2], tp_full[2], p_free[2], t_free[2];
    uint64_t d2_full, d2_empty, e2_done, d3_full, d3_empty;
    uint64_t g_full[kNG], g_empty[kNG];
    uint64_t slot_empty[kNSlot];
    // chain
    uint64_t vk_full[kNVK], vk_empty[kNVK], a_full[2], a_empty[2], d_full[2], d_empty[2], o_full[2];
    uint64_t u_full, s_full, h_full;
    uint64_t slot_full[kNSlot];
    uint64_t drain;
    float gscal[kNG][2];   // per gate buffer: G_end, factorised (1) or not (0)
    uint32_t tmem_slot;
    int abort_flag;
    int s_old;
    float s_wsum[2];
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

struct Ctx {
    uint8_t *smem;
    uint32_t sbase;
    Bars *bars;
    volatile int *abort_flag;
    uint32_t tmem;
    int dir, bh, NC, T;
    uint8_t *ring;   // this scan's kNSlot slots
};

template <int DIR>
__device__ __forceinline__ int chunk_of(const Ctx &x, int i) { return DIR ? (x.NC - 1 - i) : i; }
__device__ __forceinline__ float *gates_buf(const Ctx &x, int g)
{
    return reinterpret_cast<float *>(x.smem + kPGates) + g * kGateFloats;
}

// Tracing builds (-DGDN_TRACE): clock64() at role marks of scan (0, 0) for chunks
// kTr0 .. kTr0 + 7, stored at trace[(rank * 32 + mark) * 8 + chunk - kTr0].
constexpr int kTr0 = 100;
__device__ __forceinline__ void tr(const PairParams &p, const Ctx &x, int rank, int mark, int i)
{
#ifdef GDN_TRACE
    if (p.trace && x.dir == 0 && x.bh == 0 && i >= kTr0 && i < kTr0 + 8)
        p.trace[(rank * 32 + mark) * 8 + i - kTr0] = (long long)clock64();
#endif
}

// Bounded wait on a phase completed by arrivals from the other CTA of the cluster.
__device__ __noinline__ bool wait_cluster_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                               int *err, int code)
{
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 255) == 255 && globaltimer() - t0 > kWaitLimitNs) break;
    }
    atomicOr(err, code);
    *abort_flag = 1;
    return false;
}

__device__ __forceinline__ bool wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             int *err, int code)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    return wait_cluster_slow(bar, parity, abort_flag, err, code);
}

// Lets every MMA this thread issued complete (bounded) before TMEM is released.
__device__ __forceinline__ void drain_mmas(Bars &B)
{
    mma_commit(&B.drain);
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&B.drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
}

// Waits (bounded) for copies still in flight on a transaction barrier after an abort.
__device__ __forceinline__ void drain_copies(uint64_t *bar, uint32_t parity)
{
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < 200000000ull) {}
}

// ================================================================== prep CTA

template <int DIR>
__device__ __forceinline__ void prep_tma(const Ctx &x, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                                         const PairParams &p)
{
    Bars &B = *x.bars;
    int issued = 0;
    for (int i = 0; i < x.NC; ++i) {
        const int s = i & 1;
        if (i >= 2 && !wait_bar(&B.st_empty[s], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 1)) break;
        const int c = chunk_of<DIR>(x, i);
        uint8_t *st = x.smem + kPStage + s * kPStageBytes;
        mbar_arrive_expect_tx(&B.st_full[s], 32768);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(st + kb * 16384, tmQ, &B.st_full[s], kb * 64, c * kC, x.bh);
            tma_load_3d(st + kb * 16384 + 8192, tmK, &B.st_full[s], kb * 64, c * kC, x.bh);
        }
        issued = i + 1;
    }
    if (*x.abort_flag)
        for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i) drain_copies(&B.st_full[i & 1], (i >> 1) & 1);
}

// MMA issue: [Q;K] K^T of chunk i, then P [T1 | T2] and [P T1; T1] K of chunk i - 1.
__device__ __forceinline__ void prep_mma(const Ctx &x, const PairParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    for (int i = 0; i <= x.NC; ++i) {
        if (i < x.NC) {
            const int s = i & 1;
            if (!wait_bar(&B.st_full[s], (i >> 1) & 1, x.abort_flag, p.err, 2)) break;
            if (i >= 2 && !wait_bar(&B.d1_empty[s], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 3)) break;
            const uint32_t sQK = x.sbase + kPStage + s * kPStageBytes;
            const uint64_t a = sw128_desc(sQK, 16, 1024), b = sw128_desc(sQK + 8192, 16, 1024);
            tc_fence_after();
            mma_run<4, 2, 2>(tm + kTD1 + 64 * s, a, b, kIdM1, false);
            mma_run<4, 2, 2>(tm + kTD1 + 64 * s, a + 1024, b + 1024, kIdM1, true);
            mma_commit(&B.d1_full[s]);
            tr(p, x, 0, 16, i);
        }
        if (i == 0) continue;
        const int j = i - 1, bj = j & 1;
        if (!wait_bar(&B.tp_full[bj], (j >> 1) & 1, x.abort_flag, p.err, 4)) break;
        if (j >= 1 && !wait_bar(&B.d2_empty, (j - 1) & 1, x.abort_flag, p.err, 5)) break;
        const uint32_t tb = x.sbase + kPTB + bj * 32768;
        tc_fence_after();
        // P [T1 | T2]: B is MN-major, the T1 and T2 tiles are its two 64-column groups
        mma_run<4, 2, 128>(tm + kTD2, sw128_desc(x.sbase + kPP + bj * 8192, 16, 1024),
                           sw128_desc(tb + 8192, 16384, 1024), kIdM2, false);
        mma_commit(&B.d2_full);
        mma_commit(&B.p_free[bj]);
        tr(p, x, 0, 17, j);
        if (!wait_bar(&B.e2_done, j & 1, x.abort_flag, p.err, 6)) break;
        if (j >= 1 && !wait_bar(&B.d3_empty, (j - 1) & 1, x.abort_flag, p.err, 7)) break;
        tc_fence_after();
        // [P T1; T1] K: B = K [token][dk] MN-major, dk groups 16 KB apart in the stage
        mma_run<4, 2, 128>(tm + kTD3, sw128_desc(tb, 16, 1024),
                           sw128_desc(x.sbase + kPStage + bj * kPStageBytes + 8192, 16384, 1024), kIdM3, false);
        mma_commit(&B.d3_full);
        mma_commit(&B.t_free[bj]);
        tr(p, x, 0, 18, j);
    }
    drain_mmas(B);
}

// Mask epilogue of this warp's 32 physical columns [32 hf, +32) of one row of
// [Q;K] K^T, in four groups of 8 (a loop: this code runs once per chunk, so its
// size costs more than its instruction count).  Rows 0-63 (TMEM quarters 0-1)
// give P row r: j kept at or before r in scan order; rows 64-127 give A row r,
// written in scan order: j strictly before r, times b_r.  The decay ratio
// 2^(G_r - G_j) is a product of a row and a column factor when the chunk's
// factors are all normal floats (`fact`), else one exp2 of the difference.
template <int DIR>
__device__ __forceinline__ void mask_rows(uint32_t taddr, const float *gt, float *As, uint8_t *sP, int qd,
                                          int lane, int hf, bool fact)
{
    const int r = (qd & 1) * 32 + lane;                  // physical token row
    const int lr = DIR ? 63 - r : r;                     // its scan position
    const bool pm = qd < 2;                              // P (else A)
    const bool useB = lr >= 32 && (DIR ? (hf == 1) : (hf == 0));   // cross-half pairs
    const float *cf = gt + (useB ? gCB : gCA) * 64 + 32 * hf;
    const float br = pm ? 1.f : gt[gBet * 64 + r];
    const float rf = br * gt[(useB ? gRB : gRA) * 64 + r];
    const float Gr = gt[gG * 64 + r];
#pragma unroll 1
    for (int g8 = 0; g8 < 4; ++g8) {
        float xv[8];
        tmem_ld8(taddr + 8 * g8, xv);
        tmem_wait_ld();
        const int j0 = 32 * hf + 8 * g8;   // physical column of xv[0]
        if (fact) {
#pragma unroll
            for (int u = 0; u < 8; ++u) xv[u] *= rf * cf[8 * g8 + u];
        } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) xv[u] *= br * exp2f(Gr - gt[gG * 64 + j0 + u]);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = j0 + u;
            const bool keep = pm ? (DIR ? (j >= r) : (j <= r)) : (DIR ? (j > r) : (j < r));
            if (!keep) xv[u] = 0.f;
        }
        if (pm) {
            st_tile_v4(sP, sw128_off(r, j0), pack_bf16(xv[0], xv[1]), pack_bf16(xv[2], xv[3]),
                       pack_bf16(xv[4], xv[5]), pack_bf16(xv[6], xv[7]));
        } else if (DIR) {   // scan-order columns 63 - j run backwards
            float4 *dst = reinterpret_cast<float4 *>(As + lr * kLDA + 56 - j0);
            dst[0] = make_float4(xv[7], xv[6], xv[5], xv[4]);
            dst[1] = make_float4(xv[3], xv[2], xv[1], xv[0]);
        } else {
            float4 *dst = reinterpret_cast<float4 *>(As + lr * kLDA + j0);
            dst[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
            dst[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
        }
    }
}

// Solver groups (two groups of 4 warps, warp w reading TMEM lane quarter
// qd = w % 4): group g takes the chunks i with i % 2 == g, so that two chunks'
// solves, each a long chain of dependent steps, run at once.  Per chunk: the
// masks of [Q;K] K^T, then T = (I + A)^-1 written as T1 = T diag(b gamma) and
// T2 = T diag(b); meanwhile the group's gate threads prepare the gates of its
// next chunk.  pt is the thread's index in its group (0..127).
template <int DIR>
__device__ __forceinline__ void prep_solver(const Ctx &x, const PairParams &p, int pt, int qd, int g)
{
    Bars &B = *x.bars;
    const int lane = pt & 31;
    const int bar = g ? kBarA2 : kBarA, gbar = g ? kBarGate2 : kBarGate;
    float *As = reinterpret_cast<float *>(x.smem + kPA + g * kPAStride);
    const uint32_t tm_lane = (uint32_t)(qd * 32) << 16;
    const float *beta_h = p.beta + (size_t)x.bh * x.T;
    const float *decay_h = p.decay + (size_t)x.bh * x.T;

    // gate threads: pt 64..127 (scan position gpt), on their own 64-thread barrier
    const bool gate_thr = pt >= 64;
    const int gpt = pt - 64;
    float ra = 1.f, rb = 0.f;
    auto load_raw = [&](int j) {
        ra = 1.f;
        rb = 0.f;
        if (gate_thr && j < x.NC) {
            const int pp = DIR ? (63 - gpt) : gpt;
            const int t = chunk_of<DIR>(x, j) * kC + pp;
            if (t < x.T) {   // padded tokens: identity (b = 0, log decay = 0)
                ra = __ldg(decay_h + t);
                rb = __ldg(beta_h + t);
            }
        }
    };
    auto compute_gates = [&](int j) {
        const int gj = j % kNG;
        float *gt = gates_buf(x, gj);
        if (j >= kNG) wait_bar(&B.g_empty[gj], ((j / kNG) + 1) & 1, x.abort_flag, p.err, 8);
        float v = fmaxf(log2f(ra), -120.f);   // decay below 2^-120 acts as 2^-120
        const float bcur = rb;
        load_raw(j + 2);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        if (gpt == 31) x.bars->s_wsum[g] = v;
        named_bar(gbar, 64);
        {
            const float G = (gpt >= 32) ? v + x.bars->s_wsum[g] : v;
            const int pp = DIR ? (63 - gpt) : gpt;
            gt[gG * 64 + pp] = G;
            const float gam = exp2f(G);
            gt[gGam * 64 + pp] = gam;
            gt[gBet * 64 + pp] = bcur;
            gt[gBG * 64 + pp] = bcur * gam;
        }
        named_bar(gbar, 64);
        // references: scan positions 15 (first half), 47 (second half), 31 (boundary)
        const float R1 = gt[gG * 64 + (DIR ? 48 : 15)];
        const float R2 = gt[gG * 64 + (DIR ? 16 : 47)];
        const float Rm = gt[gG * 64 + (DIR ? 32 : 31)];
        const float G0 = gt[gG * 64 + (DIR ? 63 : 0)];
        const float G32 = gt[gG * 64 + (DIR ? 31 : 32)];
        const float Gend = gt[gG * 64 + (DIR ? 0 : 63)];
        // factorised decay products are exact while every factor is a normal float
        const bool fact = (G0 - R1) <= 120.f && (R1 - Rm) <= 120.f && (G32 - R2) <= 120.f &&
                          (R2 - Gend) <= 120.f;
        {
            const float G = gt[gG * 64 + gpt];
            const int lp = DIR ? 63 - gpt : gpt;
            const float Rh = (lp >= 32) ? R2 : R1;
            gt[gEb * 64 + gpt] = exp2f(Gend - G);
            gt[gRA * 64 + gpt] = exp2f(G - Rh);
            gt[gCA * 64 + gpt] = exp2f(Rh - G);
            gt[gRB * 64 + gpt] = exp2f(G - Rm);
            gt[gCB * 64 + gpt] = exp2f(Rm - G);
            if (gpt == 0) {
                x.bars->gscal[gj][0] = Gend;
                x.bars->gscal[gj][1] = fact ? 1.f : 0.f;
            }
        }
        named_bar(gbar, 64);
        if (gpt == 0) mbar_arrive(&B.g_full[gj]);
    };
    load_raw(g);

    // the first step only computes the gates of the group's first chunk
#pragma unroll 1
    for (int i = g - 2; i < x.NC; i += 2) {
        const int b = g;   // = i & 1: this group's P, T and D1 buffers
        const int gi = (i + 2 * kNG) % kNG;
        float *gt = gates_buf(x, gi);
        uint8_t *tb = x.smem + kPTB + b * 32768;
        if (i >= 0) {
            const bool fact = x.bars->gscal[gi][1] != 0.f;
            if (pt == 0) tr(p, x, 0, 0, i);
            wait_bar(&B.d1_full[b], (i >> 1) & 1, x.abort_flag, p.err, 9);
            if (i >= 2) wait_bar(&B.p_free[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 10);
            if (pt == 0) tr(p, x, 0, 1, i);
            tc_fence_after();
            uint8_t *sP = x.smem + kPP + b * 8192;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf)
                mask_rows<DIR>(x.tmem + tm_lane + kTD1 + 64 * b + 32 * hf, gt, As, sP, qd, lane, hf, fact);
            if (pt == 0) tr(p, x, 0, 7, i);
            tc_fence_before();
            fence_proxy_async_smem();
            if (named_bar_any(bar, 128, *x.abort_flag)) return;
            if (pt == 0) mbar_arrive(&B.d1_empty[b]);
            if (pt == 0) tr(p, x, 0, 2, i);
        }

        // T = (I + A)^-1; meanwhile the gate threads prepare the group's next chunk's gates
        if (gate_thr && i + 2 < x.NC) compute_gates(i + 2);
        if (i < 0) {
            named_bar(bar, 128);
            continue;
        }
        // T1 / T2 of this buffer must be done with (chunk i - 2: its products and its ring copy)
        if (i >= 2) wait_bar(&B.t_free[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 11);
        if (pt == 0) tr(p, x, 0, 3, i);
        solve_diag_blocks<0, 0>(As, gt, tb + 8192, tb + 24576, nullptr, DIR, pt, bar, 128);
        if (pt == 0) tr(p, x, 0, 4, i);
        // the six strips below the diagonal blocks and the diagonal blocks' T1, T2:
        // eight pieces of work, two for each of the group's warps
        solve_off_diag_compact(As, gt, tb + 8192, tb + 24576, DIR, pt);
        solve_off_diag_compact(As, gt, tb + 8192, tb + 24576, DIR, pt + 128);
        if ((pt & 31) == 0) tr(p, x, 0, 20 + (pt >> 5) + 4 * g, i);
        fence_proxy_async_smem();
        if (named_bar_any(bar, 128, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.tp_full[b]);
        if (pt == 0) tr(p, x, 0, 5, i);
    }
}

// Finisher group (4 warps, warp w reads TMEM lane quarter qd = w % 4): P T1 and
// P T2 into the operand tiles, Q' = gamma Q - P T1 K and -W = -T1 K into A2,
// then the chunk's ring slot.
template <int DIR>
__device__ __forceinline__ void prep_finisher(const Ctx &x, const PairParams &p, int ft, int qd)
{
    Bars &B = *x.bars;
    const int lane = ft & 31;
    const uint32_t tm_lane = (uint32_t)(qd * 32) << 16;
    const uint32_t slot_full_remote = mapa_shared(smem_u32(&B.slot_full[0]), 1);
    int issued = 0;   // leader: chunks whose ring copies were issued
    // leader, once chunk j's copies have completed: publish the slot to the chain
    auto publish = [&](int j) {
        fence_proxy_async_global();
        mbar_arrive_remote(slot_full_remote + 8u * (j % kNSlot));
    };
#pragma unroll 1
    for (int i = 0; i < x.NC; ++i) {
        const int b = i & 1, gi = i % kNG;
        uint8_t *tb = x.smem + kPTB + b * 32768;
        const float *gt = gates_buf(x, gi);

        // ---- P [T1 | T2] (M = 64: lanes 0-15 of quarter qd hold rows 16 qd ..)
        if (ft == 0) tr(p, x, 0, 8, i);
        wait_bar(&B.d2_full, i & 1, x.abort_flag, p.err, 12);
        if (ft == 0) tr(p, x, 0, 9, i);
        tc_fence_after();
        {
            float v[32];
            const int r = 16 * qd + lane;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {   // PT1 above T1, PT2 above T2
#pragma unroll 1
                for (int h2 = 0; h2 < 2; ++h2) {
                    tmem_ld32(x.tmem + tm_lane + kTD2 + 64 * part + 32 * h2, v);
                    tmem_wait_ld();
                    if (lane < 16) store_half_row_bf16(tb + 16384 * part, r, h2, v);
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        // the previous chunk's ring copies have completed: its slot can be published
        if (ft == 0 && i > 0) bulk_wait0();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (ft == 0) {
            mbar_arrive(&B.e2_done);
            mbar_arrive(&B.d2_empty);
            if (i > 0) publish(i - 1);
        }
        if (ft == 0) tr(p, x, 0, 10, i);

        // ---- A2 = [gamma Q - P T1 K; -T1 K]
        // (the waits below also order this group's reads of the gates, of the Q tile
        // and of the solver's T2 rows after the writes that published them)
        wait_bar(&B.g_full[gi], (i / kNG) & 1, x.abort_flag, p.err, 13);
        wait_bar(&B.st_full[b], (i >> 1) & 1, x.abort_flag, p.err, 16);
        wait_bar(&B.tp_full[b], (i >> 1) & 1, x.abort_flag, p.err, 17);
        wait_bar(&B.d3_full, i & 1, x.abort_flag, p.err, 14);
        if (ft == 0) tr(p, x, 0, 11, i);
        tc_fence_after();
        {
            const int n = 32 * qd + lane;   // row of [P T1; T1] K
            const float gq = (n < 64) ? gt[gGam * 64 + n] : 0.f;
            float v[32];
#pragma unroll 1
            for (int kb = 0; kb < 2; ++kb) {
                const uint8_t *qrow = x.smem + kPStage + b * kPStageBytes + kb * 16384;   // Q, key block kb
                uint8_t *a2 = x.smem + kPA2 + kb * 16384;
#pragma unroll 1
                for (int h2 = 0; h2 < 2; ++h2) {
                    tmem_ld32(x.tmem + tm_lane + kTD3 + 64 * kb + 32 * h2, v);
                    tmem_wait_ld();
                    if (n < 64) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint4 w = *reinterpret_cast<const uint4 *>(qrow + sw128_off(n, 32 * h2 + 8 * q4));
                            const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float2 f = __bfloat1622float2(w2[u]);
                                v[8 * q4 + 2 * u] = fmaf(gq, f.x, -v[8 * q4 + 2 * u]);
                                v[8 * q4 + 2 * u + 1] = fmaf(gq, f.y, -v[8 * q4 + 2 * u + 1]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = -v[e];
                    }
                    store_half_row_bf16(a2, n, h2, v);
                }
            }
        }
        if (ft < 16) {
            *reinterpret_cast<float4 *>(x.smem + kPGst + 16 * ft) =
                *reinterpret_cast<const float4 *>(gt + gEb * 64 + 4 * ft);
        } else if (ft == 16) {
            *reinterpret_cast<float4 *>(x.smem + kPGst + 256) =
                make_float4(exp2f(x.bars->gscal[gi][0]), 0.f, 0.f, 0.f);
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (ft == 0) {
            mbar_arrive(&B.d3_empty);
            mbar_arrive(&B.st_empty[b]);
            mbar_arrive(&B.g_empty[gi]);
        }
        if (ft == 0) tr(p, x, 0, 12, i);

        // ---- ring slot: A1, A2, e, gamma_end (bulk copies, published a chunk later)
        if (ft == 0) {
            tr(p, x, 0, 13, i);
            const int s = i % kNSlot;
            if (i < kNSlot || wait_cluster(&B.slot_empty[s], ((i / kNSlot) + 1) & 1, x.abort_flag, p.err, 15)) {
                uint8_t *slot = x.ring + (size_t)s * kSlotBytes;
                bulk_store(slot + kSlotA1, tb + 16384, 16384);
                bulk_store(slot + kSlotA2, x.smem + kPA2, 32768);
                bulk_store(slot + kSlotGates, x.smem + kPGst, 512);
                bulk_commit();
                issued = i + 1;
                // once the copies have read them, the A1 tile goes back to the solver
                // and A2 staging may be rewritten
                bulk_wait_read0();
                mbar_arrive(&B.t_free[b]);
            }
            tr(p, x, 0, 14, i);
        }
    }
    if (ft == 0) {
        bulk_wait0();
        if (!*x.abort_flag && issued == x.NC) publish(x.NC - 1);
    }
}

// ================================================================== chain CTA

template <int DIR>
__device__ __forceinline__ void chain_tma(const Ctx &x, const CUtensorMap *tmK, const CUtensorMap *tmV,
                                          const PairParams &p)
{
    Bars &B = *x.bars;
    int vk_issued = 0, a_issued = 0;
    for (int i = 0; i < x.NC; ++i) {
        const int st = i % kNVK, ab = i & 1, s = i % kNSlot;
        if (i >= kNVK && !wait_bar(&B.vk_empty[st], ((i / kNVK) + 1) & 1, x.abort_flag, p.err, 21)) break;
        const int c = chunk_of<DIR>(x, i);
        uint8_t *sv = x.smem + kCStage + st * 32768;
        mbar_arrive_expect_tx(&B.vk_full[st], 32768);
        tma_load_3d(sv, tmV, &B.vk_full[st], 0, c * kC, x.bh);
        tma_load_3d(sv + 8192, tmV, &B.vk_full[st], 64, c * kC, x.bh);
        tma_load_3d(sv + 16384, tmK, &B.vk_full[st], 0, c * kC, x.bh);
        tma_load_3d(sv + 24576, tmK, &B.vk_full[st], 64, c * kC, x.bh);
        vk_issued = i + 1;
        if (i >= 2 && !wait_bar(&B.a_empty[ab], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 22)) break;
        tr(p, x, 1, 0, i);
        if (!wait_cluster(&B.slot_full[s], (i / kNSlot) & 1, x.abort_flag, p.err, 23)) break;
        tr(p, x, 1, 1, i);
        fence_proxy_async_global();
        const uint8_t *slot = x.ring + (size_t)s * kSlotBytes;
        uint8_t *dst = x.smem + kCA + ab * kCABytes;
        mbar_arrive_expect_tx(&B.a_full[ab], kSlotBytes);
        bulk_load(dst, slot, 16384, &B.a_full[ab]);
        bulk_load(dst + 16384, slot + 16384, 16384, &B.a_full[ab]);
        bulk_load(dst + 32768, slot + 32768, 16384, &B.a_full[ab]);
        bulk_load(dst + 49152, slot + 49152, 512, &B.a_full[ab]);
        a_issued = i + 1;
    }
    if (*x.abort_flag) {
        for (int i = (vk_issued > kNVK ? vk_issued - kNVK : 0); i < vk_issued; ++i)
            drain_copies(&B.vk_full[i % kNVK], (i / kNVK) & 1);
        for (int i = (a_issued > 2 ? a_issued - 2 : 0); i < a_issued; ++i) drain_copies(&B.a_full[i & 1], (i >> 1) & 1);
    }
}

__device__ __forceinline__ void chain_mma(const Ctx &x, const PairParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    const uint32_t slot_empty_remote = mapa_shared(smem_u32(&B.slot_empty[0]), 0);
    for (int i = 0; i < x.NC; ++i) {
        const int st = i % kNVK, ab = i & 1, db = i & 1;
        if (!wait_bar(&B.vk_full[st], (i / kNVK) & 1, x.abort_flag, p.err, 24)) break;
        if (!wait_bar(&B.a_full[ab], (i >> 1) & 1, x.abort_flag, p.err, 25)) break;
        mbar_arrive_remote(slot_empty_remote + 8u * (i % kNSlot));   // the slot's data has landed
        tr(p, x, 1, 2, i);
        if (i >= 2 && !wait_bar(&B.d_empty[db], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 26)) break;
        tr(p, x, 1, 3, i);
        const uint32_t sv = x.sbase + kCStage + st * 32768;
        const uint32_t sa = x.sbase + kCA + ab * kCABytes;
        const uint32_t dD = tm + kTD + 128 * db;
        tc_fence_after();
        // D = V^T A1^T: A = V (MN-major, dv groups 8 KB apart), B = A1 (K-major)
        mma_run<4, 128, 2>(dD, sw128_desc(sv, 8192, 1024), sw128_desc(sa + kSlotA1, 16, 1024), kIdA, false);
        if (!wait_bar(&B.h_full, i & 1, x.abort_flag, p.err, 27)) break;
        tr(p, x, 1, 4, i);
        tc_fence_after();
        // D += H^T A2^T: A = H^T (bf16 in TMEM), B = A2 (K-major, key blocks 16 KB apart)
        {
            const uint64_t dA2 = sw128_desc(sa + kSlotA2, 16, 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ta(dD, tm + kTH + 8 * k, dA2 + (uint64_t)((k >> 2) * 1024 + (k & 3) * 2), kIdB, 1u);
        }
        mma_commit(&B.d_full[db]);
        mma_commit(&B.a_empty[ab]);
        if (!wait_bar(&B.u_full, i & 1, x.abort_flag, p.err, 28)) break;
        tr(p, x, 1, 5, i);
        tc_fence_after();
        // S = Ubar^T K: A = Ubar^T (bf16 in TMEM), B = K (MN-major, dk groups 8 KB apart)
        {
            const uint64_t dK = sw128_desc(sv + 16384, 8192, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16_ta(tm + kTS, tm + kTUb + 8 * k, dK + (uint64_t)(k * 128), kIdC, k > 0 ? 1u : 0u);
        }
        mma_commit(&B.s_full);
        mma_commit(&B.vk_empty[st]);
    }
    drain_mmas(B);
}

// State group (8 warps): H^T in fp32 registers, thread (quarter q, half h) holds
// row d = 32 q + lane, key columns [64 h, +64).  U epilogue: tokens [32 h, +32)
// of U^T, scaled by e, into Ubar^T (bf16, TMEM); state epilogue: H^T <-
// gamma_end H^T + S into registers and its bf16 copy into TMEM.
template <int DIR>
__device__ __forceinline__ void chain_state(const Ctx &x, const PairParams &p, int ct, int q, int h)
{
    Bars &B = *x.bars;
    const int lane = ct & 31, d = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const bool dbg = kDbgOn && p.debug != nullptr && x.dir == 0 && x.bh == 0;
    float hs[64];
    {
        const float *s0 = (DIR == 0 && p.state_in) ? p.state_in + (size_t)x.bh * kDK * 128 + (size_t)(64 * h) * 128 + d
                                                   : nullptr;
#pragma unroll
        for (int j = 0; j < 64; ++j) hs[j] = s0 ? s0[(size_t)j * 128] : 0.f;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16(hs[32 * h2 + 2 * j], hs[32 * h2 + 2 * j + 1]);
            tmem_st16(x.tmem + tl + kTH + 32 * h + 16 * h2, w);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    named_bar(kBarA, kGroup);
    if (ct == 0) mbar_arrive(&B.h_full);

#pragma unroll 1
    for (int i = 0; i < x.NC; ++i) {
        const int db = i & 1, ab = i & 1;
        const float *eg = reinterpret_cast<const float *>(x.smem + kCA + ab * kCABytes + kSlotGates);
        // ---- Ubar^T (e and gamma_end come with the chunk's ring slot)
        wait_bar(&B.a_full[ab], (i >> 1) & 1, x.abort_flag, p.err, 34);
        wait_bar(&B.d_full[db], (i >> 1) & 1, x.abort_flag, p.err, 31);
        if (ct == 0) tr(p, x, 1, 8, i);
        tc_fence_after();
        {
            uint32_t w[16];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float u[16];
                tmem_ld16(x.tmem + tl + kTD + 128 * db + 64 + 32 * h + 16 * h2, u);
                tmem_wait_ld();
                if (dbg && i == 0)
                    for (int j = 0; j < 16; ++j) p.debug[d * 128 + 64 + 32 * h + 16 * h2 + j] = u[j];
                const float4 *e4 = reinterpret_cast<const float4 *>(eg + 32 * h + 16 * h2);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 ev = e4[m];
                    w[8 * h2 + 2 * m] = pack_bf16(u[4 * m] * ev.x, u[4 * m + 1] * ev.y);
                    w[8 * h2 + 2 * m + 1] = pack_bf16(u[4 * m + 2] * ev.z, u[4 * m + 3] * ev.w);
                }
            }
            tmem_st16(x.tmem + tl + kTUb + 16 * h, w);
            tmem_wait_st();
        }
        tc_fence_before();
        if (named_bar_any(kBarA, kGroup, *x.abort_flag)) return;
        if (ct == 0) {
            mbar_arrive(&B.u_full);
            mbar_arrive(&B.d_empty[db]);
        }
        if (ct == 0) tr(p, x, 1, 9, i);
        // ---- H^T <- gamma_end H^T + S
        wait_bar(&B.s_full, i & 1, x.abort_flag, p.err, 32);
        if (ct == 0) tr(p, x, 1, 10, i);
        tc_fence_after();
        {
            const float ge = eg[64];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t w[16];
#pragma unroll
                for (int h4 = 0; h4 < 2; ++h4) {
                    float sv[16];
                    const int c0 = 32 * h2 + 16 * h4;
                    tmem_ld16(x.tmem + tl + kTS + 64 * h + c0, sv);
                    tmem_wait_ld();
                    if (dbg && i == 0)
                        for (int j = 0; j < 16; ++j) p.debug[16384 + d * 128 + 64 * h + c0 + j] = sv[j];
#pragma unroll
                    for (int j = 0; j < 16; ++j) hs[c0 + j] = fmaf(ge, hs[c0 + j], sv[j]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) w[8 * h4 + j] = pack_bf16(hs[c0 + 2 * j], hs[c0 + 2 * j + 1]);
                }
                tmem_st16(x.tmem + tl + kTH + 32 * h + 16 * h2, w);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        if (named_bar_any(kBarA, kGroup, *x.abort_flag)) return;
        if (ct == 0) {
            mbar_arrive(&B.h_full);
            mbar_arrive(&B.a_empty[ab]);
        }
        if (ct == 0) tr(p, x, 1, 11, i);
    }
    if (p.state_out) {
        float *so = p.state_out + ((size_t)DIR * p.BH + x.bh) * kDK * 128 + (size_t)(64 * h) * 128 + d;
#pragma unroll
        for (int j = 0; j < 64; ++j) so[(size_t)j * 128] = hs[j];
    }
}

// Output group (4 warps): thread (quarter q) owns column d = 32 q + lane of each
// chunk's O tile.  The tile is assembled in shared memory as [dv block][token]
// rows (the TMA layout of o) and written with one TMA store.  Bidirectional:
// the first writer of a tile stores its bf16 partial and then publishes it on
// the tile's counter; the second loads that partial by TMA (requested a chunk
// ahead when the first writer is known in advance), adds its fp32 partial and
// rounds once.
template <int DIR>
__device__ __forceinline__ void chain_out(const Ctx &x, const PairParams &p, const CUtensorMap *tmO, int ot, int q)
{
    Bars &B = *x.bars;
    const int lane = ot & 31, d = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const bool lead = ot == 0;
    const bool dbg = kDbgOn && p.debug != nullptr && x.dir == 0 && x.bh == 0;
    // this thread's column in a staging tile: dv block d / 64, column d % 64
    const uint32_t dblk = (uint32_t)(d >> 6) * 8192u;
    int nload[2] = {0, 0};   // partial loads issued into each staging tile so far
    int loaded_ahead = -1;   // leader: the chunk whose partial load is already in flight
    int nissued[2] = {0, 0}; // leader: partial loads issued into each staging tile
    auto pred_first = [&](int c) { return DIR == ((2 * c < x.NC) ? 0 : 1); };
    auto counter = [&](int c) { return p.counters + (size_t)x.bh * x.NC + c; };
    auto load_partial = [&](int c, int ob) {
        uint8_t *stg = x.smem + kCO + ob * 16384;
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&B.o_full[ob], 16384);
        ++nissued[ob];
        tma_load_3d(stg, tmO, &B.o_full[ob], 0, c * kC, x.bh);
        tma_load_3d(stg + 8192, tmO, &B.o_full[ob], 64, c * kC, x.bh);
    };
#pragma unroll 1
    for (int i = 0; i < x.NC; ++i) {
        const int db = i & 1, ob = i & 1, c = chunk_of<DIR>(x, i);
        uint8_t *stg = x.smem + kCO + ob * 16384;
        const bool bidi = p.counters != nullptr;
        bool first = true;
        if (bidi) {
            if (p.predict) {
                // every cluster resident: the forward scan reaches the first half of the
                // chunks first, the reverse scan the second half
                first = pred_first(c);
            } else {
                // arrival order decided at run time by a claim on the counter
                // (0 -> 1 -> 2); the first writer's published partial brings it to 3
                if (lead) x.bars->s_old = atomicAdd(counter(c), 1);
                named_bar(kBarB, kGroupB);
                first = x.bars->s_old == 0;
            }
            if (!first && lead && loaded_ahead != i) {
                bool ok = spin_global_at_least(counter(c), p.predict ? 1 : 3, x.abort_flag);
                if (!ok) {
                    if (!*x.abort_flag) atomicOr(p.err, 32);
                    *x.abort_flag = 1;
                } else {
                    bulk_wait_read1();   // the staging tile's previous store has read it
                    load_partial(c, ob);
                }
            }
        }
        wait_bar(&B.d_full[db], (i >> 1) & 1, x.abort_flag, p.err, 33);
        // the staging tile's store of two chunks ago must have read it before it is rewritten
        if (lead) bulk_wait_read1();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (!first) {
            wait_bar(&B.o_full[ob], nload[ob] & 1, x.abort_flag, p.err, 35);
            ++nload[ob];
        }
        tc_fence_after();
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
            float v[32];
            tmem_ld32(x.tmem + tl + kTD + 128 * db + 32 * h2, v);
            tmem_wait_ld();
            if (dbg && i == 0)
                for (int j = 0; j < 32; ++j) p.debug[d * 128 + 32 * h2 + j] = v[j];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                __nv_bfloat16 *e = reinterpret_cast<__nv_bfloat16 *>(stg + dblk + sw128_off(32 * h2 + j, d & 63));
                float y = v[j];
                if (!first) y += __bfloat162float(*e);
                *e = __float2bfloat16_rn(y);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (lead) {
            mbar_arrive(&B.d_empty[db]);
            tma_store_3d(tmO, stg, 0, c * kC, x.bh);
            tma_store_3d(tmO, stg + 8192, 64, c * kC, x.bh);
            bulk_commit();
            if (bidi && first) {
                // publish the partial once its writes are performed
                bulk_wait0();
                fence_proxy_async_global();
                __threadfence();
                atomicAdd(counter(c), 1);
            }
            // request the next tile's partial now if its first writer is known and done
            if (bidi && p.predict && i + 1 < x.NC) {
                const int cn = chunk_of<DIR>(x, i + 1);
                if (!pred_first(cn)) {
                    int seen;
                    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(seen) : "l"(counter(cn)) : "memory");
                    if (seen >= 1) {
                        bulk_wait_read1();   // tile (i + 1) & 1: its store of chunk i - 1 has read it
                        load_partial(cn, (i + 1) & 1);
                        loaded_ahead = i + 1;
                    }
                }
            }
        }
    }
    if (lead) {
        bulk_wait0();   // every store performed before the CTA exits
        for (int ob = 0; ob < 2; ++ob)   // partial loads still in flight after an abort
            for (int k = nload[ob]; k < nissued[ob]; ++k) drain_copies(&B.o_full[ob], k & 1);
    }
}

// ================================================================== kernel

__global__ void __launch_bounds__(kPThreads, 1)
gdn_chunk_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      const PairParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();

    Ctx x;
    x.smem = smem;
    x.sbase = smem_u32(smem);
    x.bars = reinterpret_cast<Bars *>(smem + kOffBar);
    x.abort_flag = &x.bars->abort_flag;
    x.dir = blockIdx.y;
    x.bh = blockIdx.z;
    x.T = p.T;
    x.NC = p.n_chunks;
    x.ring = p.ring + ((size_t)x.dir * p.BH + x.bh) * kNSlot * kSlotBytes;
    Bars &B = *x.bars;

    if (tid == 0) {
        uint64_t *all = reinterpret_cast<uint64_t *>(&B);
        const int nbar = (int)(offsetof(Bars, gscal) / sizeof(uint64_t));
        for (int k = 0; k < nbar; ++k) mbar_init(&all[k], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&B.t_free[b], 2);    // [P T1; T1] K done, ring copy done
            mbar_init(&B.a_empty[b], 2);   // D += H^T A2^T done, state epilogue done
            mbar_init(&B.d_empty[b], 2);   // output epilogue, U epilogue
        }
        B.abort_flag = 0;
        fence_mbar_init();
        if (rank == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
        } else {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmO);
        }
    }
    if (warp == 0) {
        tmem_alloc(&B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (rank == 0) {
        float *As0 = reinterpret_cast<float *>(smem + kPA);
        for (int i = tid; i < 2 * 64 * kLDA; i += kPThreads) As0[i] = 0.f;
        // T1, T2: the triangle the solve never writes stays zero for the whole scan
        for (int b = 0; b < 2; ++b) {
            uint32_t *t1 = reinterpret_cast<uint32_t *>(smem + kPTB + b * 32768 + 8192);
            uint32_t *t2 = reinterpret_cast<uint32_t *>(smem + kPTB + b * 32768 + 24576);
            for (int i = tid; i < 8192 / 4; i += kPThreads) t1[i] = t2[i] = 0u;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = B.tmem_slot;
    cluster_sync_all();   // both CTAs' barriers are initialised before any remote arrival

    if (rank == 0) {
        if (warp == 0) {
            if (lane == 0) {
                if (x.dir) prep_tma<1>(x, &tmQ, &tmK, p);
                else prep_tma<0>(x, &tmQ, &tmK, p);
            }
        } else if (warp == 1) {
            if (lane == 0) prep_mma(x, p);
        } else if (warp < 10) {
            const int g = (warp - 2) >> 2, pt = tid - 64 - 128 * g, qd = warp & 3;
            if (x.dir) prep_solver<1>(x, p, pt, qd, g);
            else prep_solver<0>(x, p, pt, qd, g);
        } else {
            const int ft = tid - 320, qd = warp & 3;
            if (x.dir) prep_finisher<1>(x, p, ft, qd);
            else prep_finisher<0>(x, p, ft, qd);
        }
    } else {
        if (warp == 0) {
            if (lane == 0) {
                if (x.dir) chain_tma<1>(x, &tmK, &tmV, p);
                else chain_tma<0>(x, &tmK, &tmV, p);
            }
        } else if (warp == 1) {
            if (lane == 0) chain_mma(x, p);
        } else if (warp < 10) {
            const int ct = tid - 64, q = warp & 3, h = (warp - 2) >> 2;
            if (x.dir) chain_state<1>(x, p, ct, q, h);
            else chain_state<0>(x, p, ct, q, h);
        } else {
            const int ot = tid - 320, q = warp & 3;
            if (x.dir) chain_out<1>(x, p, &tmO, ot, q);
            else chain_out<0>(x, p, &tmO, ot, q);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(x.tmem, kTmemCols);
    cluster_sync_all();   // the partner may address this CTA's barriers until it is done
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 3D map over a [BH, T, 128] bf16 tensor; box = 64 (inner) x 64 (tokens) x 1, 128B swizzle.
bool make_map(CUtensorMap *m, const void *base, int T, int BH)
{
    EncodeTiledFn enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {256, (cuuint64_t)T * 256};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct DevInfo {
    bool init = false;
    int max_clusters = 0;   // 2-CTA clusters resident at once
};

// Per device: the kernel's shared-memory attribute and how many of its
// clusters fit on the GPU at once.
cudaError_t device_info(DevInfo **out)
{
    static std::mutex mu;
    static DevInfo info[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    DevInfo &d = info[dev];
    if (!d.init) {
        err = cudaFuncSetAttribute(gdn_chunk_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kSmemAlloc);
        if (err != cudaSuccess) return err;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kPThreads);
        cfg.dynamicSmemBytes = kSmemAlloc;
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 2;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, gdn_chunk_pair_kernel, &cfg);
        if (err != cudaSuccess) return err;
        d.max_clusters = n;
        d.init = true;
    }
    *out = &d;
    return cudaSuccess;
}

}  // namespace

bool chunk_pair_supported(const FwdArgs &a)
{
    // chosen on request only (g_kernel_select == 2): on the measured workloads the
    // single-CTA kernel is still the faster one
    return g_kernel_select == 2 && !a.fp32 && a.dk == kDK && a.dv == 128 && a.n_seg == 1 &&
           a.seg0 == 0 && a.seg_chunks == 0;
}

cudaError_t launch_chunk_pair(const FwdArgs &a, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv, mo;
    const int BH = a.B * a.H;
    if (!make_map(&mq, a.q, a.T, BH) || !make_map(&mk, a.k, a.T, BH) || !make_map(&mv, a.v, a.T, BH) ||
        !make_map(&mo, a.o, a.T, BH))
        return cudaErrorInvalidValue;
    DevInfo *info = nullptr;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;

    PairParams p;
    p.beta = a.beta; p.decay = a.decay; p.state_in = a.state_in; p.state_out = a.state_out;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.BH = BH; p.T = a.T;
    p.n_chunks = (a.T + kC - 1) / kC;
    p.debug = g_debug_dump;
    p.trace = g_prof_buf;
    err = device_error_word(&p.err);
    if (err != cudaSuccess) return err;

    const int dirs = a.bidi ? 2 : 1;
    const size_t ring_bytes = (size_t)dirs * BH * kNSlot * kSlotBytes;
    const size_t cnt_bytes = a.bidi ? (size_t)BH * p.n_chunks * sizeof(int) : 0;
    uint8_t *ws = nullptr;
    err = ws_alloc(reinterpret_cast<void **>(&ws), ring_bytes + cnt_bytes, stream);
    if (err != cudaSuccess) return err;
    p.ring = g_debug_ring ? static_cast<uint8_t *>(g_debug_ring) : ws;
    p.counters = a.bidi ? reinterpret_cast<int *>(ws + ring_bytes) : nullptr;
    if (a.bidi) err = cudaMemsetAsync(p.counters, 0, cnt_bytes, stream);

    if (err == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[2];
        cfg.gridDim = dim3(2, dirs, BH);
        cfg.blockDim = dim3(kPThreads);
        cfg.dynamicSmemBytes = kSmemAlloc;
        cfg.stream = stream;
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 2;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        at[1].id = cudaLaunchAttributeCooperative;
        at[1].val.cooperative = 1;
        cfg.attrs = at;
        // bidirectional: a cooperative launch makes every cluster resident (or is
        // refused), so the first writer of each output tile can be fixed in advance
        const bool coop = a.bidi && dirs * BH <= info->max_clusters;
        cfg.numAttrs = coop ? 2 : 1;
        p.predict = coop ? 1 : 0;
        err = cudaLaunchKernelEx(&cfg, gdn_chunk_pair_kernel, mq, mk, mv, mo, p);
        if (err != cudaSuccess && coop) {
            (void)cudaGetLastError();
            cfg.numAttrs = 1;
            p.predict = 0;
            err = cudaLaunchKernelEx(&cfg, gdn_chunk_pair_kernel, mq, mk, mv, mo, p);
        }
        if (err == cudaSuccess) err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    cudaError_t e2 = ws_free(ws, stream);
    if (err == cudaSuccess) err = e2;
    return err;
}

}  // namespace gdn

// Test hooks (not part of the documented ABI).
// gdn_debug_ring: a device buffer of at least dirs*B*H*4*49664 bytes that the
// paired kernel uses as its operand ring instead of workspace (NULL: off), so
// a test can read the prepared operands of each chunk back.
// gdn_debug_kernel_select: 0 picks the kernel by shape, 1 forces the
// single-CTA chunkwise kernel for every bf16 call, 2 asks for the paired-SM
// kernel wherever it applies (dk = dv = 128, whole sequences).
extern "C" void gdn_debug_ring(void *device_buffer) { gdn::g_debug_ring = device_buffer; }
extern "C" void gdn_debug_kernel_select(int which) { gdn::g_kernel_select = which; }
