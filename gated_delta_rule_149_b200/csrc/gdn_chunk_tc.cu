// Chunkwise GDN recurrence on sm_100a tensor cores (tcgen05 + TMEM + TMA),
// warp-specialised so that the work of chunk i+1 that does not depend on the
// state overlaps the serial state update of chunk i.
//
// The recurrence (librediffusion PR #21 page, "What's added": the GDN
// linear-attention recurrence; the causal-streaming and bidirectional forms
// of the flashdreams SANA-WM page), per head, with H = S^T (dk x dv):
//     H_t = a_t (I - b_t k_t k_t^T) H_{t-1} + b_t k_t v_t^T,   o_t = H_t^T q_t
// is evaluated 64 tokens at a time in its WY/UT form.  Per chunk, in scan
// order (forward: ascending t; reverse: descending t), with g = log2 a,
// G_i = sum of g up to and including token i, gamma_i = 2^G_i:
//     A    = strict-lower [ b_i 2^(G_i - G_j) k_i.k_j ]          (64 x 64)
//     P    = lower        [ 2^(G_i - G_j) q_i.k_j ]               (64 x 64)
//     T    = (I + A)^-1                                          (fp32/tf32 solve)
//     W    = T diag(b gamma) K,     U~ = T diag(b) V
//     U    = U~ - W H_prev                                       (serial step)
//     O    = diag(gamma) Q H_prev + P U
//     H    = gamma_end H_prev + K^T diag(2^(G_end - G)) U          (serial step)
// Only 2^(G_i - G_j) with j at or before i is used.  It is formed as a product
// of a row and a column factor: around the middle of the half-chunk when i and
// j lie in the same 32-token half, around the boundary between the halves
// when they do not (both factors are then <= 1); when a half-chunk decays by
// more than 2^-240 (a factor could leave the normal range) it is formed
// directly, so nothing overflows however strong the decay.
//
// One CTA per (64-wide dv slice, direction, batch*head), 20 warps:
//   warps 0-7   chain: fp32 state in registers (each thread owns 32 columns
//                      of one row of the dk x 64 slice); W and gamma*Q
//                      operands, U, state and output epilogues;
//   warps 8-15  prep:  gates, masks, the triangular solve (16x16 diagonal
//                      blocks by substitution, the blocks below by strip-wise
//                      block substitution with tf32 mma.sync), written straight
//                      into T1 = T diag(b gamma) and T2 = T diag(b);
//   warp 16     TMA:   q, k and the v slice of each chunk, three stages ahead;
//   warp 17     MMA:   issues the state-independent products ([Q;K]K^T, W, U~);
//   warp 18     MMA:   issues the serial-chain products (W H, Q H, K^T Ubar, P U);
//   warp 19     combine: the grid-wide handshake of the bidirectional tiles.
// Tensor-core products (bf16 operands, fp32 accumulation in TMEM):
//     [Q;K] K^T        M=128 N=64  K=dk     -> QK^T, KK^T
//     W^T = K^T T1^T   M=128 N=64  K=64
//     U~  = T2 V       M=64  N=64  K=64
//     U  -= W H        M=64  N=64  K=dk     (A negated in the descriptor)
//     O   = (gamma Q) H, O += P U           M=64 N=64
//     D_S = K^T Ubar   M=128 N=64  K=64     (Ubar = diag(2^(G_end-G)) U)
// Bidirectional: both scans run in the same launch; for each (head, chunk,
// slice) output tile the first writer stores its partial and the second adds
// its own in L2 once an arrival counter shows the first is visible.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"
#include "gdn_chunk_common.cuh"
#include "../../include/gdn_debug.h"

namespace gdn {

extern float *g_debug_dump;
extern long long *g_prof_buf;

namespace {

using namespace ptx;

constexpr int kDVS = 64;         // dv columns per CTA
constexpr int kThreads = 640;    // 8 chain + 8 prep + TMA + 2 MMA-issue + combine warps
constexpr int kChainThreads = 256, kPrepThreads = 256;
constexpr int kNS = 3;           // input stages
constexpr int kBarPrep = 1, kBarChain = 2, kBarGates = 3;   // named barriers (prep, chain, gate warps)

// TMEM columns (fp32 accumulators)
constexpr uint32_t kColD1 = 0;     // [Q;K] K^T   (M=128)
constexpr uint32_t kColW = 64;     // W^T         (M=128)
constexpr uint32_t kColU0 = 128;   // U~ then U   (M=64), 2 buffers
constexpr uint32_t kColO0 = 256;   // O           (M=64), 2 buffers
constexpr uint32_t kColS = 384;    // K^T Ubar    (M=128)
constexpr uint32_t kTmemCols = 512;

// Shared memory (bytes from a 1024-aligned base)
constexpr uint32_t kStageBytes = 40 * 1024;            // [kb0: Q|K][kb1: Q|K] 32 KB + V 8 KB
constexpr uint32_t kOffStage = 0;
constexpr uint32_t kOffP = kNS * kStageBytes;          // 2 x 8 KB  bf16 [i][j]
constexpr uint32_t kOffW = kOffP + 16384;              // 16 KB bf16 [d][i]  (W, MN-major)
constexpr uint32_t kOffU = kOffW + 16384;              // 8 KB  bf16 [i][e]
constexpr uint32_t kOffUb = kOffU + 8192;              // 8 KB
constexpr uint32_t kOffH = kOffUb + 8192;              // 16 KB bf16 [d][e]
constexpr uint32_t kOffA = kOffH + 16384;              // fp32 [64][68], scan order: A, then T in place
constexpr uint32_t kOffT1 = kOffA + 64 * kLDA * 4;     // 8 KB bf16 [i][j]
constexpr uint32_t kOffT2 = kOffT1 + 8192;             // 8 KB bf16 [i][j]
constexpr int kNG = 3;                                 // gate buffers (prep runs ahead)
constexpr uint32_t kGateFloats = 9 * 64;               // per buffer, see GateIdx
constexpr uint32_t kOffGates = kOffT2 + 8192;
constexpr uint32_t kOffBar = kOffGates + kNG * kGateFloats * 4;
constexpr uint32_t kOffProf = kOffBar + 512;            // 32 x 8 B (profiling builds)
constexpr uint32_t kSmemBytes = kOffProf + 256;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;     // alignment slack
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kOffT1 % 1024 == 0 && kOffT2 % 1024 == 0 && kOffP % 1024 == 0, "tile alignment");


constexpr uint32_t kIdM1 = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdW = idesc_bf16(128, 64, true, false);
constexpr uint32_t kIdUt = idesc_bf16(64, 64, false, true);
constexpr uint32_t kIdUc = idesc_bf16(64, 64, true, true, true);   // -W H
constexpr uint32_t kIdOq = idesc_bf16(64, 64, false, true);
constexpr uint32_t kIdS = idesc_bf16(128, 64, true, true);
constexpr uint32_t kIdPU = idesc_bf16(64, 64, false, true);


struct TcParams {
    const float *beta, *decay, *state_in;
    float *state_out;
    __nv_bfloat16 *o;
    int *counters;       // bidi arrival counters [BH][n_chunks][n_slices], zeroed
    int *err;            // device error word
    float *debug;        // optional: first-chunk intermediates of CTA (0,0,0)
    long long *prof;     // optional (profiling builds): per-phase cycle counts of CTA (0,0,0)
    int BH, T, dv, n_chunks, n_slices;
    int n_seg, seg0, seg_chunks;   // segments of each head in this launch (1, 0, n_chunks: whole)
    int predict;         // bidi: all CTAs resident, first writer of each tile known in advance
};

// Phase timers for profiling builds (-DGDN_PROFILE): each role's leader
// thread in CTA (0,0,0) adds the cycles since its previous mark to a slot.
#ifdef GDN_PROFILE
// Per-slot cycle accumulators live in shared memory (kOffProf); the leader
// thread of each role adds the cycles since its previous mark.
#define PROF_DECL(lead)                                                                     \
    const bool prof_on = p.prof != nullptr && (lead) && blockIdx.x == 0 && blockIdx.y == 0 && \
                         blockIdx.z == 0;                                                   \
    long long prof_t = clock64();                                                           \
    long long *prof_s = reinterpret_cast<long long *>(x.smem + kOffProf);
#define PROF_MARK(slot)                                \
    do {                                               \
        if (prof_on) {                                 \
            const long long prof_n = clock64();        \
            prof_s[slot] += prof_n - prof_t;           \
            prof_t = prof_n;                           \
        }                                              \
    } while (0)
#define PROF_FLUSH() \
    do {             \
    } while (0)
#define PROF_SETC(c) \
    do {             \
    } while (0)
#elif defined(GDN_TRACE)
// Event trace for tracing builds (-DGDN_TRACE): the leader thread of each role
// in CTA (0,0,0) stores clock64() at each mark for the chunks of a short window
// (role-local chunk index), to read the critical path off the timestamps.
constexpr int kTrace0 = 200, kTraceN = 4, kTraceBase = 4096;
#define PROF_DECL(lead)                                                                     \
    const bool prof_on = p.prof != nullptr && (lead) && blockIdx.x == 0 && blockIdx.y == 0 && \
                         blockIdx.z == 0;                                                   \
    int prof_c = 0;
#define PROF_SETC(c) prof_c = (c)
#define PROF_MARK(slot)                                                                    \
    do {                                                                                   \
        if (prof_on && prof_c >= kTrace0 && prof_c < kTrace0 + kTraceN)                    \
            p.prof[kTraceBase + (prof_c - kTrace0) * 32 + (slot)] = (long long)clock64(); \
    } while (0)
#define PROF_FLUSH() \
    do {             \
    } while (0)
#else
#define PROF_DECL(lead)
#define PROF_MARK(slot) \
    do {                \
    } while (0)
#define PROF_FLUSH() \
    do {             \
    } while (0)
#define PROF_SETC(c) \
    do {             \
    } while (0)
#endif

// First-chunk intermediates can be dumped for debugging in builds with
// GDN_DEBUG_DUMP; production builds compile the dump code out.
#ifdef GDN_DEBUG_DUMP
constexpr bool kDbgOn = true;
#else
constexpr bool kDbgOn = false;
#endif
// Debug dump layout (floats): 6 TMEM snapshots of 128 lanes x 64 columns
// (D1, W^T, U~, U, O, D_S) then the 64 x 64 solve result in scan order.
constexpr int kDbgD1 = 0, kDbgW = 8192, kDbgUt = 16384, kDbgU = 24576, kDbgO = 32768,
              kDbgS = 40960, kDbgT = 49152;

// mbarriers
struct Bars {
    uint64_t stage_full[kNS], stage_empty[kNS];
    uint64_t d1_full, d1_empty, tp_full, wu_full, wmn_full, dw_empty;
    uint64_t chain_full, u_full, s_full, h_full, drain, drain2;
    uint64_t o_full[2], do_empty[2], du_empty[2], p_empty[2], g_full[kNG], g_empty[kNG];
    float gscal[kNG][2];   // per gate buffer: G_end, factorised (1) or not (0)
    uint32_t tmem_slot;
    int abort_flag;
    int s_old;
    float s_wsum;
    int stored_upto;   // last output tile the chain warps stored as first writer
    int ready_upto;    // last output tile whose other-direction partial is visible
};
static_assert(sizeof(Bars) <= 512, "barrier block");

__device__ __forceinline__ void dbg_half(float *dst, int row, int h, const float *x)
{
#pragma unroll
    for (int e = 0; e < 32; ++e) dst[row * 64 + 32 * h + e] = x[e];
}


struct Ctx {
    uint8_t *smem;
    uint32_t sbase;
    Bars *bars;
    volatile int *abort_flag;
    uint32_t tmem;
    int slice, dir, bh, NC, T, dv;
    int row;   // state row (head, segment): blockIdx.z
    int c0;    // first (global) chunk of this CTA's segment
};

__device__ __forceinline__ uint32_t stage_addr(const Ctx &x, int i) { return x.sbase + kOffStage + (uint32_t)(i % kNS) * kStageBytes; }
template <int DIR>
__device__ __forceinline__ int chunk_of(const Ctx &x, int i) { return x.c0 + (DIR ? (x.NC - 1 - i) : i); }
__device__ __forceinline__ float *gates_buf(const Ctx &x, int g) { return reinterpret_cast<float *>(x.smem + kOffGates) + g * kGateFloats; }

// ------------------------------------------------------------------ TMA warp
template <int DIR>
__device__ __forceinline__ void tma_role(const Ctx &x, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                         const CUtensorMap *tmV, const TcParams &p)
{
    Bars &B = *x.bars;
    int issued = 0;
    PROF_DECL(true);
    for (int i = 0; i < x.NC; ++i) {
        const int s = i % kNS;
        PROF_SETC(i);
        PROF_MARK(1);
        if (i >= kNS && !wait_bar(&B.stage_empty[s], ((i / kNS) + 1) & 1, x.abort_flag, p.err, 1)) break;
        PROF_MARK(0);
        const int c = chunk_of<DIR>(x, i);
        uint8_t *st = x.smem + (stage_addr(x, i) - x.sbase);
        mbar_arrive_expect_tx(&B.stage_full[s], 5 * 8192);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(st + kb * 16384, tmQ, &B.stage_full[s], kb * 64, c * kC, x.bh);
            tma_load_3d(st + kb * 16384 + 8192, tmK, &B.stage_full[s], kb * 64, c * kC, x.bh);
        }
        tma_load_3d(st + 32768, tmV, &B.stage_full[s], x.slice * kDVS, c * kC, x.bh);
        PROF_MARK(18);
        issued = i + 1;
    }
    PROF_FLUSH();
    if (*x.abort_flag) {   // let copies in flight land before the CTA exits
        for (int i = (issued > kNS ? issued - kNS : 0); i < issued; ++i) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(&B.stage_full[i % kNS], (i / kNS) & 1) &&
                   globaltimer() - t0 < 200000000ull) {}
        }
    }
}

// ------------------------------------------------------------------ MMA warps
// An issuing thread shares its SM sub-partition's issue slots with four busy
// epilogue warps, so every instruction between two MMAs stretches the MMA
// stream: each product is one unrolled run of MMAs whose operand descriptors
// are a base descriptor plus an immediate (the 14-bit start-address field,
// in 16-byte units, holds any shared-memory address, so adding to the
// descriptor never carries out of it); loop-invariant bases are built once.
// Two issuing threads, each waiting (suspended) on its next products' inputs in
// a fixed order: one for the state-independent products of the prep pipeline,
// one for the serial-chain products.  tcgen05.commit tracks the MMAs of the
// issuing thread only; the mbarrier protocol orders the two streams.


// [Q;K] K^T, then W^T = K^T T1^T and U~ = T2 V, chunk after chunk.
__device__ __forceinline__ void mma_prep_role(const Ctx &x, const TcParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    const uint64_t dT1 = sw128_desc(x.sbase + kOffT1, 16, 1024), dT2 = sw128_desc(x.sbase + kOffT2, 16, 1024);
    PROF_DECL(true);
    // [Q;K] K^T of chunk j (needs its stage loaded and D1 read out for chunk j-1)
    auto issue_m1 = [&](int j) -> bool {
        PROF_SETC(j);
        if (!wait_bar(&B.stage_full[j % kNS], (j / kNS) & 1, x.abort_flag, p.err, 11)) return false;
        if (j > 0 && !wait_bar(&B.d1_empty, (j - 1) & 1, x.abort_flag, p.err, 12)) return false;
        PROF_MARK(2);
        const uint32_t sQK = stage_addr(x, j);
        const uint64_t a = sw128_desc(sQK, 16, 1024), b = sw128_desc(sQK + 8192, 16, 1024);
        tc_fence_after();
        mma_run<4, 2, 2>(tm + kColD1, a, b, kIdM1, false);                  // K block 0
        mma_run<4, 2, 2>(tm + kColD1, a + 1024, b + 1024, kIdM1, true);     // K block 1 (+16 KB)
        mma_commit(&B.d1_full);
        PROF_MARK(6);
        return true;
    };
    // step j: [Q;K] K^T of chunk j first (its inputs are usually ready long
    // before the T1/T2 of chunk j - 1), then W^T = K^T T1^T, U~ = T2 V of
    // chunk i = j - 1
#pragma unroll 1
    for (int j = 0; j <= x.NC; ++j) {
        if (j < x.NC && !issue_m1(j)) break;
        if (j == 0) continue;
        const int i = j - 1, b = i & 1;
        PROF_SETC(i);
        if (!wait_bar(&B.tp_full, i & 1, x.abort_flag, p.err, 13)) break;
        PROF_MARK(12);
        if (i >= 2 && !wait_bar(&B.du_empty[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 14)) break;
        if (i >= 1 && !wait_bar(&B.dw_empty, (i - 1) & 1, x.abort_flag, p.err, 19)) break;
        PROF_MARK(7);
        const uint32_t sQK = stage_addr(x, i);
        const uint64_t dKmn = sw128_desc(sQK + 8192, 16384, 1024), dVmn = sw128_desc(sQK + 32768, 8192, 1024);
        tc_fence_after();
        mma_run<4, 128, 2>(tm + kColW, dKmn, dT1, kIdW, false);
        mma_run<4, 2, 128>(tm + kColU0 + 64 * b, dT2, dVmn, kIdUt, false);
        mma_commit(&B.wu_full);
        PROF_MARK(5);
    }
    PROF_FLUSH();
    // every issued MMA completes before the CTA releases its TMEM
    mma_commit(&B.drain);
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&B.drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
}

// U -= W H and O = (gamma Q) H, then D_S = K^T Ubar and O += P U.
__device__ __forceinline__ void mma_chain_role(const Ctx &x, const TcParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    const uint64_t dP = sw128_desc(x.sbase + kOffP, 16, 1024), dW = sw128_desc(x.sbase + kOffW, 8192, 1024);
    const uint64_t dU = sw128_desc(x.sbase + kOffU, 8192, 1024), dUb = sw128_desc(x.sbase + kOffUb, 8192, 1024);
    const uint64_t dH = sw128_desc(x.sbase + kOffH, 8192, 1024);
    PROF_DECL(true);
    for (int i = 0; i < x.NC; ++i) {
        const int b = i & 1;
        const uint32_t sQK = stage_addr(x, i);
        PROF_SETC(i);
        PROF_MARK(28);
        if (!wait_bar(&B.wmn_full, i & 1, x.abort_flag, p.err, 15)) break;
        if (!wait_bar(&B.h_full, i & 1, x.abort_flag, p.err, 16)) break;
        if (i >= 2 && !wait_bar(&B.do_empty[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 17)) break;
        PROF_MARK(29);
        const uint64_t dQ = sw128_desc(sQK, 16, 1024);
        tc_fence_after();
        mma_run<8, 128, 128>(tm + kColU0 + 64 * b, dW, dH, kIdUc, true);
        mma_commit(&B.chain_full);
        mma_run<4, 2, 128>(tm + kColO0 + 64 * b, dQ, dH, kIdOq, false);               // K block 0
        mma_run<4, 2, 128>(tm + kColO0 + 64 * b, dQ + 1024, dH + 512, kIdOq, true);   // K block 1
        PROF_MARK(4);
        if (!wait_bar(&B.u_full, i & 1, x.abort_flag, p.err, 18)) break;
        PROF_MARK(30);
        tc_fence_after();
        mma_run<4, 128, 128>(tm + kColS, sw128_desc(sQK + 8192, 16384, 1024), dUb, kIdS, false);
        mma_commit(&B.s_full);
        mma_run<4, 2, 128>(tm + kColO0 + 64 * b, dP + (uint64_t)(b * 512), dU, kIdPU, true);
        mma_commit(&B.o_full[b]);
        mma_commit(&B.p_empty[b]);
        mma_commit(&B.stage_empty[i % kNS]);
        PROF_MARK(3);
    }
    PROF_FLUSH();
    mma_commit(&B.drain2);
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&B.drain2, 0) && globaltimer() - t0 < kWaitLimitNs) {}
}

// ------------------------------------------------------------------ prep warps
// 8 warps (256 threads).  Warp pw reads TMEM lane quarter pw & 3 and handles
// columns [32 * (pw >> 2), +32) of each row it owns.
// Mask epilogue of one half row of [Q;K] K^T with every decay ratio taken as
// one exp2 of a difference (the factorised form would leave the normal float
// range: some half-chunk decays by more than 2^-120).  Rare, so it is kept out
// of line; it reads its TMEM half row itself.
template <int DIR>
__device__ __noinline__ void m1_epi_direct(uint32_t taddr, const float *gt, float *As, uint8_t *sP,
                                           int qd, int lane, int hf)
{
    float xv[32];
    tmem_ld32(taddr, xv);
    tmem_wait_ld();
    const int r = (qd & 1) * 32 + lane;
    const int lr = DIR ? 63 - r : r;
    const float Gr = gt[gG * 64 + r];
    const float *Gj = gt + gG * 64 + 32 * hf;
    if (qd < 2) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int j = 32 * hf + e;
            const bool keep = DIR ? (j >= r) : (j <= r);
            xv[e] = keep ? exp2f(Gr - Gj[e]) * xv[e] : 0.f;
        }
        store_half_row_bf16(sP, r, hf, xv);
    } else {
        const float br = gt[gBet * 64 + r];
        float4 *Arow = reinterpret_cast<float4 *>(As + lr * kLDA + (DIR ? 32 * (1 - hf) : 32 * hf));
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            float o4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = DIR ? 31 - (4 * m + u) : 4 * m + u;
                const int lj = DIR ? 63 - (32 * hf + e) : 32 * hf + e;
                o4[u] = (lj < lr) ? br * exp2f(Gr - Gj[e]) * xv[e] : 0.f;
            }
            Arow[m] = make_float4(o4[0], o4[1], o4[2], o4[3]);
        }
    }
}

template <int DIR>
__device__ __forceinline__ void prep_role(const Ctx &x, const TcParams &p, int pt)
{
    Bars &B = *x.bars;
    const int pw = pt >> 5, lane = pt & 31, qd = pw & 3, hf = pw >> 2;
    float *As = reinterpret_cast<float *>(x.smem + kOffA);
    const uint32_t tm_lane = (uint32_t)(qd * 32) << 16;
    const float *beta_h = p.beta + (size_t)x.bh * x.T;
    const float *decay_h = p.decay + (size_t)x.bh * x.T;
    // the logical (scan-order) half that this warp's 32 physical columns fall in
    const bool col_h1 = DIR ? (hf == 1) : (hf == 0);

    // Gates are computed one chunk ahead by prep warps 2-3 (gate thread
    // gpt = pt - 64 handles scan position gpt), on their own 64-thread
    // barrier, while warps 0-1 run the diagonal blocks of the previous solve.
    const bool gate_thr = pt >= 64 && pt < 128;
    const int gpt = pt - 64;
    float ra = 1.f, rb = 0.f;
    auto load_raw = [&](int j) {
        ra = 1.f;
        rb = 0.f;
        if (gate_thr && j < x.NC) {
            const int pp = DIR ? (63 - gpt) : gpt;
            const int t = chunk_of<DIR>(x, j) * kC + pp;
            if (t < x.T) {
                ra = __ldg(decay_h + t);
                rb = __ldg(beta_h + t);
            }
        }
    };
    // gates (log2 domain) of chunk j into buffer j & 1; gate threads only
    auto compute_gates = [&](int j) {
        const int gj = j % kNG;
        float *gt = gates_buf(x, gj);
#ifdef GDN_TRACE
        const bool trg = p.prof && gpt == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 &&
                         j >= kTrace0 && j < kTrace0 + kTraceN;
        if (trg) p.prof[kTraceBase + (j - kTrace0) * 32 + 8] = (long long)clock64();
#endif
        if (j >= kNG) wait_bar(&B.g_empty[gj], ((j / kNG) + 1) & 1, x.abort_flag, p.err, 2);
        float v = fmaxf(log2f(ra), -120.f);   // decay below 2^-120 acts as 2^-120
        const float bcur = rb;
        load_raw(j + 1);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        if (gpt == 31) x.bars->s_wsum = v;
        named_bar(kBarGates, 64);
        {
            const float G = (gpt >= 32) ? v + x.bars->s_wsum : v;
            const int pp = DIR ? (63 - gpt) : gpt;
            gt[gG * 64 + pp] = G;
            const float gam = exp2f(G);
            gt[gGam * 64 + pp] = gam;
            gt[gBet * 64 + pp] = bcur;
            gt[gBG * 64 + pp] = bcur * gam;
        }
        named_bar(kBarGates, 64);
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
        named_bar(kBarGates, 64);
        if (gpt == 0) mbar_arrive(&B.g_full[gj]);
#ifdef GDN_TRACE
        if (trg) p.prof[kTraceBase + (j - kTrace0) * 32 + 9] = (long long)clock64();
#endif
    };
    load_raw(0);
    PROF_DECL(pt == 0);

    // step i = -1 only computes the gates of chunk 0
#pragma unroll 1
    for (int i = -1; i < x.NC; ++i) {
        const int b = i & 1;
        const int gi = (i + kNG) % kNG;
        float *gt = gates_buf(x, gi);
        const bool dbg = kDbgOn && p.debug != nullptr && i == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&
                         blockIdx.z == 0;
        if (i >= 0) {
            const bool fact = x.bars->gscal[gi][1] != 0.f;
            PROF_SETC(i);
            PROF_MARK(16);

            // ---- masks: P (rows of QK^T) and A (rows of KK^T, scan order)
            wait_bar(&B.d1_full, i & 1, x.abort_flag, p.err, 3);
            if (i >= 2) wait_bar(&B.p_empty[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 4);
            PROF_MARK(10);
            tc_fence_after();
            if (!fact) {
                m1_epi_direct<DIR>(x.tmem + tm_lane + kColD1 + 32 * hf, gt, As, x.smem + kOffP + b * 8192, qd,
                                   lane, hf);
            } else {
                float xv[32];
                tmem_ld32(x.tmem + tm_lane + kColD1 + 32 * hf, xv);
                tmem_wait_ld();
                if (dbg) dbg_half(p.debug + kDbgD1, qd * 32 + lane, hf, xv);
                const int r = (qd & 1) * 32 + lane;            // physical token row
                const int lr = DIR ? 63 - r : r;
                const bool useB = lr >= 32 && col_h1;           // cross-half pairs
                const float *cf = gt + (useB ? gCB : gCA) * 64 + 32 * hf;
                if (qd < 2) {
                    // P row r: keep j at or before r in scan order
                    const float rf = gt[(useB ? gRB : gRA) * 64 + r];
    #pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * hf + e;
                        const bool keep = DIR ? (j >= r) : (j <= r);
                        xv[e] = keep ? rf * cf[e] * xv[e] : 0.f;
                    }
                    store_half_row_bf16(x.smem + kOffP + b * 8192, r, hf, xv);
                } else {
                    // A row r, written in scan order: row lr, columns lj
                    const float rf = gt[gBet * 64 + r] * gt[(useB ? gRB : gRA) * 64 + r];
                    float4 *Arow = reinterpret_cast<float4 *>(As + lr * kLDA + (DIR ? 32 * (1 - hf) : 32 * hf));
    #pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        float o4[4];
    #pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int e = DIR ? 31 - (4 * m + u) : 4 * m + u;   // physical column 32 hf + e
                            const int lj = DIR ? 63 - (32 * hf + e) : 32 * hf + e;
                            o4[u] = (lj < lr) ? rf * cf[e] * xv[e] : 0.f;
                        }
                        Arow[m] = make_float4(o4[0], o4[1], o4[2], o4[3]);
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            PROF_MARK(11);
            if (named_bar_any(kBarPrep, kPrepThreads, *x.abort_flag)) return;
            if (pt == 0) mbar_arrive(&B.d1_empty);
        }

        // ---- T = (I + A)^-1 ; meanwhile warps 2-3 prepare the next chunk's gates
        if (gate_thr && i + 1 < x.NC) compute_gates(i + 1);
        if (i < 0) {
            named_bar(kBarPrep, kPrepThreads);
            continue;
        }
        // the products of chunk i-1 must be done with the previous T1, T2
        if (i >= 1) wait_bar(&B.wu_full, (i - 1) & 1, x.abort_flag, p.err, 6);
        tc_fence_after();
        float *dbgT = dbg ? p.debug + kDbgT : nullptr;
        solve_diag_blocks<kBarPrep, kPrepThreads>(As, gt, x.smem + kOffT1, x.smem + kOffT2, dbgT, DIR, pt);
        PROF_MARK(13);
        solve_off_diag(As, gt, x.smem + kOffT1, x.smem + kOffT2, dbgT, DIR, pt);
        PROF_MARK(17);
        fence_proxy_async_smem();
        PROF_MARK(14);
        if (named_bar_any(kBarPrep, kPrepThreads, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.tp_full);

    }
    PROF_FLUSH();
}

// ------------------------------------------------------------------ chain warps
// 8 warps (256 threads).  Thread (warp cw, lane) owns state row
// d = 32 * (cw & 3) + lane, columns [32 * (cw >> 2), +32) of the slice.
// Per chunk i, in this order, so that only the U and state epilogues sit on
// the serial chain:
//   U of chunk i  ->  W and gamma*Q of chunk i+1 (while K^T Ubar runs, when
//   its inputs are ready; else before U of chunk i+1)  ->  state update of
//   chunk i  ->  output tile of chunk i (while W H of chunk i+1 runs).
template <int DIR>
__device__ __forceinline__ void chain_role(const Ctx &x, const TcParams &p, int ct)
{
    Bars &B = *x.bars;
    const int cw = ct >> 5, lane = ct & 31, cq = cw & 3, chf = cw >> 2;
    const uint32_t tm_lane = (uint32_t)(cq * 32) << 16;
    const int d = cq * 32 + lane;
    const int r = cq * 16 + lane;   // M=64 accumulators: lanes 0-15 of quarter cq hold rows 16 cq ..
    const bool dbg0 = kDbgOn && p.debug != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
    int w_done = -1;   // last chunk whose W epilogue is done

    float h[32];
    {
        const float *s0 = (DIR == 0 && p.state_in)
                              ? p.state_in + ((size_t)x.row * kDK + d) * x.dv + x.slice * kDVS + 32 * chf
                              : nullptr;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 v4 = s0 ? *reinterpret_cast<const float4 *>(s0 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            h[e] = v4.x; h[e + 1] = v4.y; h[e + 2] = v4.z; h[e + 3] = v4.w;
        }
        store_half_row_bf16(x.smem + kOffH, d, chf, h);
    }
    fence_proxy_async_smem();
    named_bar(kBarChain, kChainThreads);
    if (ct == 0) mbar_arrive(&B.h_full);
    PROF_DECL(ct == 0);

    // W (MN-major, row d = key index) and gamma-scaled Q of chunk j
    auto w_epi = [&](int j) -> bool {
        const int gj = j % kNG;
        PROF_SETC(j);
        wait_bar(&B.g_full[gj], (j / kNG) & 1, x.abort_flag, p.err, 7);
        wait_bar(&B.wu_full, j & 1, x.abort_flag, p.err, 5);
        PROF_MARK(26);
        tc_fence_after();
        {
            float xv[32];
            tmem_ld32(x.tmem + tm_lane + kColW + 32 * chf, xv);
            tmem_wait_ld();
            if (dbg0 && j == 0) {
                dbg_half(p.debug + kDbgW, d, chf, xv);
                float yv[32];
                tmem_ld32(x.tmem + tm_lane + kColU0 + 32 * chf, yv);
                tmem_wait_ld();
                dbg_half(p.debug + kDbgUt, d, chf, yv);
            }
            store_half_row_bf16(x.smem + kOffW, d, chf, xv);
        }
        {
            // gamma-scale Q in place (Q is no longer needed unscaled); bf16x2
            // products: gamma is rounded to bf16 first, one more bf16 rounding
            const int rq = ct >> 2, kb = (ct >> 1) & 1, part = ct & 1;
            const __nv_bfloat162 g2 = __float2bfloat162_rn(gates_buf(x, gj)[gGam * 64 + rq]);
            uint8_t *rowbase = x.smem + kOffStage + (uint32_t)(j % kNS) * kStageBytes + kb * 16384;
            uint4 w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) w[q] = *reinterpret_cast<const uint4 *>(rowbase + sw128_off(rq, 8 * (4 * part + q)));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 *v = reinterpret_cast<__nv_bfloat162 *>(&w[q]);
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = __hmul2(v[u], g2);
                *reinterpret_cast<uint4 *>(rowbase + sw128_off(rq, 8 * (4 * part + q))) = w[q];
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        PROF_MARK(27);
        if (named_bar_any(kBarChain, kChainThreads, *x.abort_flag)) return false;
        if (ct == 0) {
            mbar_arrive(&B.wmn_full);
            mbar_arrive(&B.dw_empty);
        }
        return true;
    };

    // output tile of chunk j: O = (gamma Q) H_prev + P U, from TMEM to o
    // (bidirectional: combined with the other direction's partial)
    auto out_tile = [&](int j) -> bool {
        const int bj = j & 1, c = chunk_of<DIR>(x, j);
        wait_bar(&B.o_full[bj], (j >> 1) & 1, x.abort_flag, p.err, 10);
        PROF_MARK(24);
        tc_fence_after();
        float xv[32];
        tmem_ld32(x.tmem + tm_lane + kColO0 + 64 * bj + 32 * chf, xv);
        tmem_wait_ld();
        if (dbg0 && j == 0) dbg_half(p.debug + kDbgO, d, chf, xv);
        const int t = c * kC + r;
        const bool mine = lane < 16 && t < x.T;
        __nv_bfloat16 *orow = p.o + ((size_t)x.bh * x.T + (mine ? t : 0)) * x.dv + x.slice * kDVS + 32 * chf;
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16(xv[2 * e], xv[2 * e + 1]);
        // causal: this CTA writes the tile.  Bidirectional: the direction that
        // reaches the tile first writes its partial, the second adds its own.
        bool first = true, add = false;
        if (p.counters != nullptr) {
            int *cnt = p.counters + ((size_t)x.bh * x.NC + c) * p.n_slices + x.slice;
            if (p.predict) {
                // every CTA is resident: the forward scan reaches the first
                // half of the chunks first, the reverse scan the second half.
                // The combine warp counts and checks the partials; here the
                // second writer only waits (in shared memory) for its word.
                first = DIR == ((2 * c < x.NC) ? 0 : 1);
                if (!first) add = wait_smem_at_least(&B.ready_upto, j, x.abort_flag, p.err, 33);
            } else {
                // arrival order decided at run time by a claim on the counter
                // (0 -> 1 -> 2); the partial's arrival brings it to 3
                if (ct == 0) x.bars->s_old = atomicAdd(cnt, 1);
                named_bar(kBarChain, kChainThreads);
                first = x.bars->s_old == 0;
                if (first) {
                    if (mine)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4 *>(orow + 8 * q) =
                                make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    named_bar(kBarChain, kChainThreads);
                    if (ct == 0) {
                        __threadfence();
                        atomicAdd(cnt, 1);
                    }
                } else {
                    if (ct == 0 && !spin_global_at_least(cnt, 3, x.abort_flag)) {
                        atomicOr(p.err, 32);
                        *x.abort_flag = 1;
                    }
                    named_bar(kBarChain, kChainThreads);
                    add = !*x.abort_flag;
                }
                first = false;   // stored above, or added below
            }
        }
        // second writer: the fp32 partial is read from TMEM again (the tile is
        // released only after this step), so that it need not stay in registers
        // across the waits above; the load is warp-wide (every lane takes part).
        // It adds the first writer's stored partial (read past L1: written by
        // another SM) and rounds to bf16 once.
        if (__any_sync(0xffffffffu, add)) {
            float xa[32];
            tc_fence_after();
            tmem_ld32(x.tmem + tm_lane + kColO0 + 64 * bj + 32 * chf, xa);
            tmem_wait_ld();
            if (mine && add) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(orow + 8 * q));
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
                    uint32_t r4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 f = __bfloat1622float2(h2[u]);
                        r4[u] = pack_bf16(f.x + xa[8 * q + 2 * u], f.y + xa[8 * q + 2 * u + 1]);
                    }
                    *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(r4[0], r4[1], r4[2], r4[3]);
                }
            }
        } else if (mine && first) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
        tc_fence_before();
        PROF_MARK(25);
        if (named_bar_any(kBarChain, kChainThreads, *x.abort_flag)) return false;
        if (ct == 0) {
            mbar_arrive(&B.do_empty[bj]);
            // predicted first writer: the tile is stored; the combine warp
            // makes it visible to the other direction and counts it
            if (p.counters != nullptr && p.predict && first) st_release_cta(&B.stored_upto, j);
        }
        return true;
    };

#pragma unroll 1
    for (int i = 0; i < x.NC; ++i) {
        const int b = i & 1, gi = i % kNG;
        const float *gt = gates_buf(x, gi);
        const bool dbg = dbg0 && i == 0;
        PROF_SETC(i);
        PROF_MARK(19);

        // s = 0: the W epilogue of chunk i unless it ran early, then U of i;
        // s = 1: the W epilogue of chunk i+1 if its inputs are ready now
#pragma unroll 1
        for (int s = 0; s < 2; ++s) {
            const int j = i + s;
            bool run_w = j < x.NC && w_done < j;
            if (s == 1 && run_w) {
                const bool ready = mbar_test_wait(&B.g_full[j % kNG], (j / kNG) & 1) &&
                                   mbar_test_wait(&B.wu_full, j & 1);
                run_w = !named_bar_any(kBarChain, kChainThreads, !ready);
            }
            if (run_w) {
                if (!w_epi(j)) return;
                w_done = j;
                PROF_SETC(i);
            }
            if (s == 1) break;

            // ---- U and Ubar rows of chunk i
            wait_bar(&B.chain_full, i & 1, x.abort_flag, p.err, 8);
            PROF_MARK(20);
            tc_fence_after();
            {
                float xv[32];
                tmem_ld32(x.tmem + tm_lane + kColU0 + 64 * b + 32 * chf, xv);
                tmem_wait_ld();
                if (dbg) dbg_half(p.debug + kDbgU, d, chf, xv);
                if (lane < 16) {
                    store_half_row_bf16(x.smem + kOffU, r, chf, xv);
                    const float eb = gt[gEb * 64 + r];
#pragma unroll
                    for (int e = 0; e < 32; ++e) xv[e] *= eb;
                    store_half_row_bf16(x.smem + kOffUb, r, chf, xv);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            PROF_MARK(21);
            if (named_bar_any(kBarChain, kChainThreads, *x.abort_flag)) return;
            if (ct == 0) {
                mbar_arrive(&B.u_full);
                mbar_arrive(&B.du_empty[b]);
            }
        }

        // ---- state update (fp32 registers) and its bf16 copy
        wait_bar(&B.s_full, i & 1, x.abort_flag, p.err, 9);
        PROF_MARK(22);
        tc_fence_after();
        {
            float xv[32];
            tmem_ld32(x.tmem + tm_lane + kColS + 32 * chf, xv);
            tmem_wait_ld();
            if (dbg) dbg_half(p.debug + kDbgS, d, chf, xv);
            const float ge = exp2f(x.bars->gscal[gi][0]);
#pragma unroll
            for (int e = 0; e < 32; ++e) h[e] = fmaf(ge, h[e], xv[e]);
            store_half_row_bf16(x.smem + kOffH, d, chf, h);
        }
        tc_fence_before();
        fence_proxy_async_smem();
        PROF_MARK(23);
        if (named_bar_any(kBarChain, kChainThreads, *x.abort_flag)) return;
        if (ct == 0) {
            mbar_arrive(&B.h_full);
            mbar_arrive(&B.g_empty[gi]);
        }

        // ---- output tile of chunk i (overlaps the next chunk's W H)
        if (!out_tile(i)) return;
    }
    PROF_FLUSH();

    if (p.state_out) {
        float *so = p.state_out + (((size_t)DIR * gridDim.z + x.row) * kDK + d) * x.dv + x.slice * kDVS + 32 * chf;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4 *>(so + e) = make_float4(h[e], h[e + 1], h[e + 2], h[e + 3]);
    }
}

// ------------------------------------------------------------------ combine warp
// Bidirectional launches whose CTAs are all resident (the first writer of each
// output tile is known in advance): one thread takes the grid-wide handshake
// of each tile off the chain warps.  For a tile this CTA writes first it waits
// until the chain warps have stored it, then makes the stores visible device-
// wide and bumps the tile's counter; for a tile it writes second it waits for
// the other direction's count and then releases the chain warps to add.
template <int DIR>
__device__ __forceinline__ void combine_role(const Ctx &x, const TcParams &p)
{
    if (p.counters == nullptr || !p.predict) return;
    Bars &B = *x.bars;
    for (int i = 0; i < x.NC; ++i) {
        const int c = chunk_of<DIR>(x, i);
        int *cnt = p.counters + ((size_t)x.bh * x.NC + c) * p.n_slices + x.slice;
        if (DIR == ((2 * c < x.NC) ? 0 : 1)) {
            if (!wait_smem_at_least(&B.stored_upto, i, x.abort_flag, p.err, 34)) return;
            __threadfence();
            atomicAdd(cnt, 1);
        } else {
            if (!spin_global_at_least(cnt, 1, x.abort_flag)) {
                if (!*x.abort_flag) atomicOr(p.err, 32);
                *x.abort_flag = 1;
                return;
            }
            st_release_cta(&B.ready_upto, i);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const TcParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Align by offsetting the shared array itself (not through an integer
    // cast), so that every access below stays a shared-memory access.
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    Ctx x;
    x.smem = smem;
    x.sbase = smem_u32(smem);
    x.bars = reinterpret_cast<Bars *>(smem + kOffBar);
    x.abort_flag = &x.bars->abort_flag;
    x.slice = blockIdx.x;
    x.dir = blockIdx.y;
    x.row = blockIdx.z;
    x.bh = blockIdx.z / p.n_seg;
    x.c0 = (p.seg0 + blockIdx.z % p.n_seg) * p.seg_chunks;
    x.T = p.T;
    x.NC = min(p.seg_chunks, p.n_chunks - x.c0);   // >= 1: the host launches no empty segment
    x.dv = p.dv;
    Bars &B = *x.bars;

    if (tid == 0) {
        uint64_t *all = reinterpret_cast<uint64_t *>(&B);
        const int nbar = (int)(offsetof(Bars, gscal) / sizeof(uint64_t));
        for (int k = 0; k < nbar; ++k) mbar_init(&all[k], 1);
        B.abort_flag = 0;
        B.stored_upto = -1;
        B.ready_upto = -1;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 0) {
        tmem_alloc(&B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    float *As0 = reinterpret_cast<float *>(smem + kOffA);
    for (int i = tid; i < 64 * kLDA; i += kThreads) As0[i] = 0.f;
    // T1, T2: the upper triangle stays zero for the whole scan
    uint32_t *T12 = reinterpret_cast<uint32_t *>(smem + kOffT1);
    for (int i = tid; i < 16384 / 4; i += kThreads) T12[i] = 0u;
    if (tid < 32) reinterpret_cast<long long *>(smem + kOffProf)[tid] = 0;
#ifdef GDN_PROFILE
    const unsigned long long prof_start = globaltimer();
#endif
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = B.tmem_slot;

    if (warp < 8) {
        if (x.dir) chain_role<1>(x, p, tid);
        else chain_role<0>(x, p, tid);
    } else if (warp < 16) {
        if (x.dir) prep_role<1>(x, p, tid - kChainThreads);
        else prep_role<0>(x, p, tid - kChainThreads);
    } else if (warp == 16) {
        if (lane == 0) {
            if (x.dir) tma_role<1>(x, &tmQ, &tmK, &tmV, p);
            else tma_role<0>(x, &tmQ, &tmK, &tmV, p);
        }
    } else if (warp == 17) {
        if (lane == 0) mma_prep_role(x, p);
    } else if (warp == 18) {
        if (lane == 0) mma_chain_role(x, p);
    } else {
        if (lane == 0) {
            if (x.dir) combine_role<1>(x, p);
            else combine_role<0>(x, p);
        }
    }

    tc_fence_before();
    __syncthreads();
#ifdef GDN_PROFILE
    if (p.prof && tid < 32 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
        p.prof[tid] += reinterpret_cast<long long *>(smem + kOffProf)[tid];
    if (p.prof && tid == 0) {
        const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
        p.prof[32 + 2 * cta] = (long long)prof_start;
        p.prof[33 + 2 * cta] = (long long)globaltimer();
    }
#endif
    if (warp == 0) tmem_dealloc(x.tmem, kTmemCols);
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

// 3D map over a [BH, T, inner] bf16 tensor; box = 64 (inner) x 64 (tokens) x 1.
bool make_map(CUtensorMap *m, const void *base, int inner, int T, int BH)
{
    EncodeTiledFn enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)T * inner * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The kernel's dynamic shared-memory size, set once per device.
cudaError_t set_smem_attribute()
{
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    err = cudaFuncSetAttribute(gdn_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemAlloc);
    if (err == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return err;
}

// Whether every CTA of the grid fits on the GPU at once (one CTA per SM, as
// the shared-memory footprint forces), so that each bidirectional output
// tile's first writer can be fixed in advance; such grids are launched
// cooperatively, which makes every CTA resident together.
cudaError_t all_resident(int n_ctas, int *out)
{
    int dev = 0, sms = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    *out = (err == cudaSuccess && n_ctas <= sms) ? 1 : 0;
    return err;
}

// Launches the kernel; cooperatively when its CTAs count on one another being
// resident (a bidirectional grid with the writer order fixed in advance).
cudaError_t launch_tc_kernel(dim3 grid, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                             const TcParams &p, bool cooperative, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = cooperative ? 1 : 0;
    cudaError_t err = cudaLaunchKernelEx(&cfg, gdn_chunk_tc_kernel, mq, mk, mv, p);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err == cudaSuccess) count_launches(1);
    return err;
}

}  // namespace

float *g_debug_dump = nullptr;
long long *g_prof_buf = nullptr;

bool chunk_tc_supported(const FwdArgs &a)
{
    return !a.fp32 && a.dk == kDK && (a.dv == 64 || a.dv == 128);
}

cudaError_t launch_chunk_tc(const FwdArgs &a, cudaStream_t stream)
{
    if (chunk_pool_supported(a)) return launch_chunk_pool(a, stream);
    CUtensorMap mq, mk, mv;
    const int BH = a.B * a.H;
    if (!make_map(&mq, a.q, a.dk, a.T, BH) || !make_map(&mk, a.k, a.dk, a.T, BH) ||
        !make_map(&mv, a.v, a.dv, a.T, BH))
        return cudaErrorInvalidValue;

    TcParams p;
    p.beta = a.beta; p.decay = a.decay; p.state_in = a.state_in; p.state_out = a.state_out;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.BH = BH; p.T = a.T; p.dv = a.dv;
    p.n_chunks = (a.T + kC - 1) / kC;
    p.n_slices = a.dv / kDVS;
    p.n_seg = a.n_seg;
    p.seg0 = a.seg0;
    p.seg_chunks = a.seg_chunks > 0 ? a.seg_chunks : p.n_chunks;
    p.counters = nullptr;
    p.debug = g_debug_dump;
    p.prof = g_prof_buf;
    cudaError_t err = device_error_word(&p.err);
    if (err != cudaSuccess) return err;
    if (a.bidi && (a.n_seg != 1 || p.seg_chunks != p.n_chunks)) return cudaErrorInvalidValue;
    if (a.n_seg < 1 || (size_t)BH * a.n_seg > 65535 ||
        (a.seg0 + a.n_seg - 1) * (size_t)p.seg_chunks >= (size_t)p.n_chunks)
        return cudaErrorInvalidValue;   // every launched segment holds at least one chunk
    err = all_resident(BH * (a.bidi ? 2 : 1) * p.n_slices, &p.predict);
    if (err != cudaSuccess) return err;

    err = set_smem_attribute();
    if (err != cudaSuccess) return err;
    const size_t n_cnt = (size_t)BH * p.n_chunks * p.n_slices;
    if (a.bidi) {
        err = ws_alloc(reinterpret_cast<void **>(&p.counters), n_cnt * sizeof(int), stream);
        if (err != cudaSuccess) return err;
        err = cudaMemsetAsync(p.counters, 0, n_cnt * sizeof(int), stream);
    }
    if (err == cudaSuccess)
        err = launch_tc_kernel(dim3(p.n_slices, a.bidi ? 2 : 1, BH * a.n_seg), mq, mk, mv, p,
                               a.bidi && p.predict, stream);
    if (p.counters) {
        cudaError_t e2 = ws_free(p.counters, stream);
        if (err == cudaSuccess) err = e2;
    }
    return err;
}

// ------------------------------------------------------ allocation-free variant
//
// Some callers cannot allocate device memory while they run this library:
// plugins hosted by a framework that owns every byte of device memory (media
// and real-time video pipelines, inference engines with a fixed memory plan),
// and streaming loops that must not touch an allocator mid-run because a pool
// allocation can block or grow the footprint at an unpredictable moment.  For
// them the bidirectional arrival counters (the only scratch this kernel needs)
// live in a fixed file-scope device array instead of a stream-ordered
// allocation.  Every device that loads this library holds the array (1 MiB)
// until the process exits.

constexpr size_t kNoAllocCounters = (size_t)1 << 18;   // 262,144 counters = 1 MiB
static __device__ __align__(256) int g_noalloc_counters[kNoAllocCounters];

size_t noalloc_capacity() { return kNoAllocCounters; }

cudaError_t launch_chunk_tc_noalloc(const FwdArgs &a, cudaStream_t stream)
{
    CUtensorMap mq, mk, mv;
    const int BH = a.B * a.H;
    if (!make_map(&mq, a.q, a.dk, a.T, BH) || !make_map(&mk, a.k, a.dk, a.T, BH) ||
        !make_map(&mv, a.v, a.dv, a.T, BH))
        return cudaErrorInvalidValue;

    TcParams p;
    p.beta = a.beta; p.decay = a.decay; p.state_in = a.state_in; p.state_out = a.state_out;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.BH = BH; p.T = a.T; p.dv = a.dv;
    p.n_chunks = (a.T + kC - 1) / kC;
    p.n_slices = a.dv / kDVS;
    p.n_seg = 1;
    p.seg0 = 0;
    p.seg_chunks = p.n_chunks;
    p.counters = nullptr;
    p.debug = nullptr;
    p.prof = nullptr;
    cudaError_t err = device_error_word(&p.err);
    if (err != cudaSuccess) return err;
    err = all_resident(BH * (a.bidi ? 2 : 1) * p.n_slices, &p.predict);
    if (err != cudaSuccess) return err;
    err = set_smem_attribute();
    if (err != cudaSuccess) return err;

    if (a.bidi) {
        const size_t n_cnt = (size_t)BH * p.n_chunks * p.n_slices;
        if (n_cnt > kNoAllocCounters) return cudaErrorInvalidValue;   // checked by the caller too
        // Host code cannot use the array's name as a device address: look the
        // address up on every call (cheap), with the caller's device current.
        void *ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_noalloc_counters);
        if (err != cudaSuccess) return err;
        p.counters = static_cast<int *>(ptr);
        // the array keeps the previous call's contents: the counters must start at zero
        err = cudaMemsetAsync(p.counters, 0, n_cnt * sizeof(int), stream);
        if (err != cudaSuccess) return err;
    }
    return launch_tc_kernel(dim3(p.n_slices, a.bidi ? 2 : 1, BH), mq, mk, mv, p, a.bidi && p.predict, stream);
}

}  // namespace gdn

// Test hook (declared in gdn_debug.h): when set to a device buffer of
// 53248 floats, the next chunkwise launches dump the first chunk's
// intermediates of CTA (0,0,0) there.  NULL turns it off.
extern "C" void gdn_debug_dump(float *device_buffer) { gdn::g_debug_dump = device_buffer; }

// Test hook for profiling builds: per-phase cycle counters of CTA (0,0,0),
// 32 long longs (zeroed by the caller).  Ignored unless built with GDN_PROFILE.
extern "C" void gdn_debug_profile(long long *device_buffer) { gdn::g_prof_buf = device_buffer; }

cudaError_t gdn::set_wait_limit_tc(unsigned long long ns) { return set_module_wait_limit(ns); }
