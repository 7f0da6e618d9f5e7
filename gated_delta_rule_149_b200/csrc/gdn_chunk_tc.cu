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
// Only 2^(G_i - G_j) with j at or before i is used.  It is formed as
// 2^(G_i - G_m) * 2^(G_m - G_j) around the chunk's mid-range G_m when the
// chunk's total decay is at most 2^-240 (each factor then stays a normal
// float), and directly otherwise, so nothing overflows however strong the decay.
//
// One CTA per (64-wide dv slice, direction, batch*head), 10 warps:
//   warps 0-3  chain:  fp32 state in registers (thread d owns row d of the
//                      dk x 64 slice); U, state and output epilogues;
//   warps 4-7  prep:   gates, masks, the triangular solve (16x16 diagonal
//                      blocks by substitution, the rest with tf32 mma.sync),
//                      T1 = T diag(b gamma), T2 = T diag(b), gamma*Q, W;
//   warp 8     TMA:    q, k and the v slice of each chunk, three stages ahead;
//   warp 9     MMA:    issues every tcgen05.mma from one thread, in whatever
//                      order the mbarriers allow (serial-chain products first).
// Tensor-core products (bf16 operands, fp32 accumulation in TMEM):
//     [Q;K] K^T        M=128 N=64  K=dk     -> QK^T, KK^T
//     W^T = K^T T1^T   M=128 N=64  K=64
//     U~  = T2 V       M=64  N=64  K=64
//     U  -= W H        M=64  N=64  K=dk     (A negated in the descriptor)
//     O   = (gamma Q) H, O += P U           M=64 N=64
//     D_S = K^T Ubar   M=128 N=64  K=64     (Ubar = diag(2^(G_end-G)) U)
// Bidirectional: both scans run in the same launch; for each (head, chunk,
// slice) output tile the first finisher writes its partial and the second
// adds its own and writes the sum (an arrival counter decides who is who).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"

namespace gdn {

extern float *g_debug_dump;

namespace {

using namespace ptx;

constexpr int kC = 64;           // chunk length
constexpr int kDK = 128;         // key dim served by this kernel
constexpr int kDVS = 64;         // dv columns per CTA
constexpr int kThreads = 320;    // 4 chain + 4 prep + TMA + MMA warps
constexpr int kNS = 3;           // input stages
constexpr int kLDA = 68;         // fp32 row stride of the solve buffers
constexpr int kBarPrep = 1, kBarChain = 2;   // named barriers, 128 threads each

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
constexpr uint32_t kOffA = kOffH + 16384;              // fp32 [64][68], scan order
constexpr uint32_t kOffT1 = kOffA;                     // T1, T2 (bf16) reuse A after the solve
constexpr uint32_t kOffT2 = kOffA + 8192;
constexpr uint32_t kOffT = kOffA + 64 * kLDA * 4;      // fp32 [64][68], scan order
constexpr uint32_t kOffY = kOffT + 64 * kLDA * 4;      // 4 warps x 16 x 8 fp32
constexpr uint32_t kGateFloats = 9 * 64;               // per buffer, see GateIdx
constexpr uint32_t kOffGates = kOffY + 4 * 512;        // 2 buffers
constexpr uint32_t kOffBar = kOffGates + 2 * kGateFloats * 4;
constexpr uint32_t kSmemBytes = kOffBar + 512;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;     // alignment slack
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kOffA % 1024 == 0 && kOffT2 % 1024 == 0 && kOffP % 1024 == 0, "tile alignment");

// gate arrays (64 floats each, physical token order unless noted)
enum GateIdx { gG = 0, gGam, gBet, gBG, gEb, gRf, gCf, gCfl /* scan order */, gScal };

constexpr uint32_t kIdM1 = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdW = idesc_bf16(128, 64, true, false);
constexpr uint32_t kIdUt = idesc_bf16(64, 64, false, true);
constexpr uint32_t kIdUc = idesc_bf16(64, 64, true, true, true);   // -W H
constexpr uint32_t kIdOq = idesc_bf16(64, 64, false, true);
constexpr uint32_t kIdS = idesc_bf16(128, 64, true, true);
constexpr uint32_t kIdPU = idesc_bf16(64, 64, false, true);

constexpr unsigned long long kWaitLimitNs = 4000000000ull;   // 4 s per wait

struct TcParams {
    const float *beta, *decay, *state_in;
    float *state_out;
    __nv_bfloat16 *o;
    int *counters;       // bidi arrival counters [BH][n_chunks][n_slices], zeroed
    int *err;            // device error word
    float *debug;        // optional: first-chunk intermediates of CTA (0,0,0)
    int BH, T, dv, n_chunks, n_slices;
};

// Debug dump layout (floats): 6 TMEM snapshots of 128 lanes x 64 columns
// (D1, W^T, U~, U, O, D_S) then the 64 x 64 solve result in scan order.
constexpr int kDbgD1 = 0, kDbgW = 8192, kDbgUt = 16384, kDbgU = 24576, kDbgO = 32768,
              kDbgS = 40960, kDbgT = 49152;

// mbarriers
struct Bars {
    uint64_t stage_full[kNS], stage_empty[kNS];
    uint64_t d1_full, d1_empty, tp_full, wu_full, wmn_full, wmn_empty;
    uint64_t chain_full, u_full, s_full, h_full, drain;
    uint64_t o_full[2], do_empty[2], du_empty[2], p_empty[2], g_full[2], g_empty[2];
    uint32_t tmem_slot;
    int abort_flag;
    int s_old;
    float s_wsum;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase; on timeout records the error and raises
// the CTA's abort flag (callers then reach their group's next barrier and
// leave together).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int *err, int code)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 255) == 255 && globaltimer() - t0 > kWaitLimitNs) break;
    }
    atomicOr(err, code);
    *abort_flag = 1;
    return false;
}

__device__ __forceinline__ void named_bar(int id)
{
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// Named barrier over a 128-thread group that also ORs a predicate across it,
// so that every thread of the group takes the same abort decision.
__device__ __forceinline__ bool named_bar_any(int id, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, %2, 128, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)pred), "r"(id) : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d) : "memory");
}

// Writes 64 fp32 values as one 128-byte bf16 row of a 128B-swizzled tile.
__device__ __forceinline__ void store_row_bf16(uint32_t tile, uint32_t row, const float *x)
{
#pragma unroll
    for (int q = 0; q < 8; ++q)
        st_shared_v4(tile + sw128_off(row, 8 * q), pack_bf16(x[8 * q + 0], x[8 * q + 1]),
                     pack_bf16(x[8 * q + 2], x[8 * q + 3]), pack_bf16(x[8 * q + 4], x[8 * q + 5]),
                     pack_bf16(x[8 * q + 6], x[8 * q + 7]));
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float *x)
{
    tmem_ld32(taddr, x);
    tmem_ld32(taddr + 32, x + 32);
    tmem_wait_ld();
}

__device__ __forceinline__ void dbg_rows(float *dst, int row, const float *x)
{
#pragma unroll
    for (int e = 0; e < 64; ++e) dst[row * 64 + e] = x[e];
}

__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D += A * B, m16n8k8, tf32 inputs, fp32 accumulation (warp-wide).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// T = (I + A)^-1 for a strictly lower-triangular 64 x 64 fp32 A (scan order),
// by the 128 prep threads.  16 x 16 diagonal blocks by forward substitution
// (one column per thread), then the off-diagonal blocks by distance from the
// diagonal, T_ab = -T_aa sum_{m=b}^{a-1} A_am T_mb, on tf32 tensor cores
// (one 16 x 8 column strip per warp and step).  The upper triangle of Ts is
// zero on entry and stays zero.
__device__ void solve_unit_lower(const float *As, float *Ts, float *Yall, int pt)
{
    if (pt < 64) {
        const int a = pt >> 4, c = pt & 15;
        const float *Ab = As + (16 * a) * kLDA + 16 * a;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) s = fmaf(Ab[r * kLDA + m], x[m], s);
            if (r > c) x[r] = -s;
        }
        float *Tb = Ts + (16 * a) * kLDA + 16 * a;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * kLDA + c] = x[r];
    }
    named_bar(kBarPrep);
    const int pw = pt >> 5, lane = pt & 31, g = lane >> 2, q = lane & 3;
    float *Y = Yall + pw * 128;   // 16 x 8, row-major
    for (int dist = 1; dist <= 3; ++dist) {
        const int items = (4 - dist) * 2;
        for (int it = pw; it < items; it += 4) {
            const int blk = it >> 1, nt = it & 1, a = dist + blk, b = blk;
            const int col0 = 16 * b + 8 * nt;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            for (int kk = 16 * b; kk < 16 * a; kk += 8) {
                uint32_t af[4], bf[2];
                const float *Ar = As + (16 * a + g) * kLDA + kk + q;
                af[0] = to_tf32(Ar[0]);
                af[1] = to_tf32(Ar[8 * kLDA]);
                af[2] = to_tf32(Ar[4]);
                af[3] = to_tf32(Ar[8 * kLDA + 4]);
                const float *Br = Ts + (kk + q) * kLDA + col0 + g;
                bf[0] = to_tf32(Br[0]);
                bf[1] = to_tf32(Br[4 * kLDA]);
                mma_tf32(d, af, bf);
            }
            Y[g * 8 + 2 * q] = d[0];
            Y[g * 8 + 2 * q + 1] = d[1];
            Y[(g + 8) * 8 + 2 * q] = d[2];
            Y[(g + 8) * 8 + 2 * q + 1] = d[3];
            __syncwarp();
            float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < 16; kk += 8) {
                uint32_t af[4], bf[2];
                const float *Dr = Ts + (16 * a + g) * kLDA + 16 * a + kk + q;
                af[0] = to_tf32(Dr[0]);
                af[1] = to_tf32(Dr[8 * kLDA]);
                af[2] = to_tf32(Dr[4]);
                af[3] = to_tf32(Dr[8 * kLDA + 4]);
                bf[0] = to_tf32(Y[(kk + q) * 8 + g]);
                bf[1] = to_tf32(Y[(kk + q + 4) * 8 + g]);
                mma_tf32(e, af, bf);
            }
            float *Tr = Ts + (16 * a + g) * kLDA + col0 + 2 * q;
            Tr[0] = -e[0];
            Tr[1] = -e[1];
            Tr[8 * kLDA] = -e[2];
            Tr[8 * kLDA + 1] = -e[3];
            __syncwarp();
        }
        named_bar(kBarPrep);
    }
}

struct Ctx {
    uint8_t *smem;
    uint32_t sbase;
    Bars *bars;
    volatile int *abort_flag;
    uint32_t tmem;
    int slice, dir, bh, NC, T, dv;
};

__device__ __forceinline__ uint32_t stage_addr(const Ctx &x, int i) { return x.sbase + kOffStage + (uint32_t)(i % kNS) * kStageBytes; }
__device__ __forceinline__ int chunk_of(const Ctx &x, int i) { return x.dir ? (x.NC - 1 - i) : i; }
__device__ __forceinline__ float *gates_buf(const Ctx &x, int b) { return reinterpret_cast<float *>(x.smem + kOffGates) + b * kGateFloats; }

// ------------------------------------------------------------------ TMA warp
__device__ void tma_role(const Ctx &x, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                         const CUtensorMap *tmV, const TcParams &p)
{
    Bars &B = *x.bars;
    int issued = 0;
    for (int i = 0; i < x.NC; ++i) {
        const int s = i % kNS;
        if (i >= kNS && !wait_bar(&B.stage_empty[s], ((i / kNS) + 1) & 1, x.abort_flag, p.err, 1)) break;
        const int c = chunk_of(x, i);
        uint8_t *st = x.smem + (stage_addr(x, i) - x.sbase);
        mbar_arrive_expect_tx(&B.stage_full[s], 5 * 8192);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(st + kb * 16384, tmQ, &B.stage_full[s], kb * 64, c * kC, x.bh);
            tma_load_3d(st + kb * 16384 + 8192, tmK, &B.stage_full[s], kb * 64, c * kC, x.bh);
        }
        tma_load_3d(st + 32768, tmV, &B.stage_full[s], x.slice * kDVS, c * kC, x.bh);
        issued = i + 1;
    }
    if (*x.abort_flag) {   // let copies in flight land before the CTA exits
        for (int i = (issued > kNS ? issued - kNS : 0); i < issued; ++i) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(&B.stage_full[i % kNS], (i / kNS) & 1) &&
                   globaltimer() - t0 < 200000000ull) {}
        }
    }
}

// ------------------------------------------------------------------ MMA warp
__device__ void mma_role(const Ctx &x, const TcParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    const uint32_t sP = x.sbase + kOffP, sW = x.sbase + kOffW, sU = x.sbase + kOffU;
    const uint32_t sUb = x.sbase + kOffUb, sH = x.sbase + kOffH;
    const uint32_t sT1 = x.sbase + kOffT1, sT2 = x.sbase + kOffT2;
    int nm1 = 0, nwu = 0, nch = 0, nst = 0;
    unsigned long long t_last = globaltimer();
    while (nst < x.NC) {
        if (*x.abort_flag) break;
        bool did = false;
        if (nst < nch && mbar_test(&B.u_full, nst & 1)) {
            // ---- state products of chunk nst: D_S = K^T Ubar, then O += P U
            const int i = nst, b = i & 1;
            const uint32_t sQK = stage_addr(x, i);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + kColS, sw128_desc(sQK + 8192 + ks * 2048, 16384, 1024),
                         sw128_desc(sUb + ks * 2048, 8192, 1024), kIdS, ks != 0);
            mma_commit(&B.s_full);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + kColO0 + 64 * b, sw128_desc(sP + b * 8192 + ks * 32, 16, 1024),
                         sw128_desc(sU + ks * 2048, 8192, 1024), kIdPU, 1);
            mma_commit(&B.o_full[b]);
            mma_commit(&B.p_empty[b]);
            mma_commit(&B.stage_empty[i % kNS]);
            ++nst;
            did = true;
        } else if (nch < nwu && mbar_test(&B.wmn_full, nch & 1) && mbar_test(&B.h_full, nch & 1) &&
                   (nch < 2 || mbar_test(&B.do_empty[nch & 1], ((nch >> 1) + 1) & 1))) {
            // ---- serial-chain products of chunk nch: U -= W H ; O = (gamma Q) H
            const int i = nch, b = i & 1;
            const uint32_t sQK = stage_addr(x, i);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + kColU0 + 64 * b, sw128_desc(sW + ks * 2048, 8192, 1024),
                         sw128_desc(sH + ks * 2048, 8192, 1024), kIdUc, 1);
            mma_commit(&B.chain_full);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tm + kColO0 + 64 * b, sw128_desc(sQK + kb * 16384 + ks * 32, 16, 1024),
                             sw128_desc(sH + (kb * 4 + ks) * 2048, 8192, 1024), kIdOq, (kb | ks) != 0);
            mma_commit(&B.wmn_empty);
            ++nch;
            did = true;
        } else if (nwu < nm1 && mbar_test(&B.tp_full, nwu & 1) &&
                   (nwu < 2 || mbar_test(&B.du_empty[nwu & 1], ((nwu >> 1) + 1) & 1))) {
            // ---- W^T = K^T T1^T ; U~ = T2 V
            const int i = nwu, b = i & 1;
            const uint32_t sQK = stage_addr(x, i), sV = sQK + 32768;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + kColW, sw128_desc(sQK + 8192 + ks * 2048, 16384, 1024),
                         sw128_desc(sT1 + ks * 32, 16, 1024), kIdW, ks != 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + kColU0 + 64 * b, sw128_desc(sT2 + ks * 32, 16, 1024),
                         sw128_desc(sV + ks * 2048, 8192, 1024), kIdUt, ks != 0);
            mma_commit(&B.wu_full);
            ++nwu;
            did = true;
        } else if (nm1 < x.NC && mbar_test(&B.stage_full[nm1 % kNS], (nm1 / kNS) & 1) &&
                   (nm1 == 0 || mbar_test(&B.d1_empty, (nm1 - 1) & 1))) {
            // ---- [Q;K] K^T
            const uint32_t sQK = stage_addr(x, nm1);
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tm + kColD1, sw128_desc(sQK + kb * 16384 + ks * 32, 16, 1024),
                             sw128_desc(sQK + kb * 16384 + 8192 + ks * 32, 16, 1024), kIdM1, (kb | ks) != 0);
            mma_commit(&B.d1_full);
            ++nm1;
            did = true;
        }
        if (did) {
            t_last = globaltimer();
        } else if (globaltimer() - t_last > kWaitLimitNs) {
            atomicOr(p.err, 16);
            *x.abort_flag = 1;
            break;
        }
    }
    // every issued MMA completes before the CTA releases its TMEM
    mma_commit(&B.drain);
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(&B.drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
}

// ------------------------------------------------------------------ prep warps
__device__ void prep_role(const Ctx &x, const TcParams &p, int pt)
{
    Bars &B = *x.bars;
    const int pw = pt >> 5, lane = pt & 31;
    float *As = reinterpret_cast<float *>(x.smem + kOffA);
    float *Ts = reinterpret_cast<float *>(x.smem + kOffT);
    float *Yall = reinterpret_cast<float *>(x.smem + kOffY);
    const uint32_t tm_lane = (uint32_t)(pw * 32) << 16;
    const float *beta_h = p.beta + (size_t)x.bh * x.T;
    const float *decay_h = p.decay + (size_t)x.bh * x.T;

    // raw gates of the next chunk, fetched one chunk ahead (thread pt < 64
    // handles scan position pt)
    float ra = 1.f, rb = 0.f;
    auto load_raw = [&](int i) {
        ra = 1.f;
        rb = 0.f;
        if (pt < 64 && i < x.NC) {
            const int pp = x.dir ? (63 - pt) : pt;
            const int t = chunk_of(x, i) * kC + pp;
            if (t < x.T) {
                ra = __ldg(decay_h + t);
                rb = __ldg(beta_h + t);
            }
        }
    };
    load_raw(0);

    for (int i = 0; i < x.NC; ++i) {
        const int b = i & 1;
        float *gt = gates_buf(x, b);
        const bool dbg = p.debug != nullptr && i == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&
                         blockIdx.z == 0;

        // ---- gates (log2 domain) for chunk i
        if (i >= 2) wait_bar(&B.g_empty[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 2);
        float gsum = 0.f, bcur = rb;
        if (pt < 64) {
            float v = fmaxf(log2f(ra), -120.f);   // decay below 2^-120 acts as 2^-120
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += y;
            }
            if (pt == 31) x.bars->s_wsum = v;
            gsum = v;
        }
        load_raw(i + 1);
        if (named_bar_any(kBarPrep, *x.abort_flag)) return;
        if (pt < 64) {
            const float G = (pt >= 32) ? gsum + x.bars->s_wsum : gsum;
            const int pp = x.dir ? (63 - pt) : pt;
            gt[gG * 64 + pp] = G;
            const float gam = exp2f(G);
            gt[gGam * 64 + pp] = gam;
            gt[gBet * 64 + pp] = bcur;
            gt[gBG * 64 + pp] = bcur * gam;
            if (pt == 63) gt[gScal * 64] = G;   // G_end
        }
        named_bar(kBarPrep);
        const float Gend = gt[gScal * 64];
        const float Gm = 0.5f * Gend;
        const bool fact = Gend >= -240.f;
        if (pt < 64) {
            const float G = gt[gG * 64 + pt];
            gt[gEb * 64 + pt] = exp2f(Gend - G);
            gt[gRf * 64 + pt] = exp2f(G - Gm);
            const float cf = exp2f(Gm - G);
            gt[gCf * 64 + pt] = cf;
            gt[gCfl * 64 + (x.dir ? 63 - pt : pt)] = cf;
        }
        named_bar(kBarPrep);
        if (pt == 0) mbar_arrive(&B.g_full[b]);

        // ---- masks: P (rows of QK^T) and A (rows of KK^T, scan order)
        wait_bar(&B.d1_full, i & 1, x.abort_flag, p.err, 3);
        if (i >= 2) wait_bar(&B.p_empty[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 4);
        tc_fence_after();
        {
            float xv[64];
            tmem_ld64(x.tmem + tm_lane + kColD1, xv);
            if (dbg) dbg_rows(p.debug + kDbgD1, pt, xv);
            if (pw < 2) {
                const int r = pt;                        // physical row of P
                const int lr = x.dir ? 63 - r : r;
                if (fact) {
                    const float rf = gt[gRf * 64 + r];
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const int lj = x.dir ? 63 - j : j;
                        xv[j] = (lj <= lr) ? rf * gt[gCf * 64 + j] * xv[j] : 0.f;
                    }
                } else {
                    const float Gr = gt[gG * 64 + r];
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const int lj = x.dir ? 63 - j : j;
                        xv[j] = (lj <= lr) ? exp2f(Gr - gt[gG * 64 + j]) * xv[j] : 0.f;
                    }
                }
                store_row_bf16(x.sbase + kOffP + b * 8192, r, xv);
            } else {
                const int r = pt - 64;
                const int lr = x.dir ? 63 - r : r;
                const float br = gt[gBet * 64 + r];
                float *Arow = As + lr * kLDA;
                if (fact) {
                    const float rf = br * gt[gRf * 64 + r];
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        float o4[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int lj = 4 * m + u;
                            const float xj = x.dir ? xv[63 - lj] : xv[lj];
                            o4[u] = (lj < lr) ? rf * gt[gCfl * 64 + lj] * xj : 0.f;
                        }
                        *reinterpret_cast<float4 *>(Arow + 4 * m) = make_float4(o4[0], o4[1], o4[2], o4[3]);
                    }
                } else {
                    const float Gr = gt[gG * 64 + r];
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        float o4[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int lj = 4 * m + u;
                            const int j = x.dir ? 63 - lj : lj;
                            const float xj = x.dir ? xv[63 - lj] : xv[lj];
                            o4[u] = (lj < lr) ? br * exp2f(Gr - gt[gG * 64 + j]) * xj : 0.f;
                        }
                        *reinterpret_cast<float4 *>(Arow + 4 * m) = make_float4(o4[0], o4[1], o4[2], o4[3]);
                    }
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarPrep, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.d1_empty);

        // ---- gamma-scale Q in place (the unscaled Q is no longer needed)
        {
            const int r = pt >> 1, kb = pt & 1;
            const float gr = gt[gGam * 64 + r];
            const uint32_t rowbase = stage_addr(x, i) + kb * 16384;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t addr = rowbase + sw128_off(r, 8 * q);
                uint32_t w[4];
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w[u]));
                    w[u] = pack_bf16(f.x * gr, f.y * gr);
                }
                st_shared_v4(addr, w[0], w[1], w[2], w[3]);
            }
        }

        // ---- T = (I + A)^-1
        solve_unit_lower(As, Ts, Yall, pt);
        if (dbg)
            for (int e = pt; e < 64 * 64; e += 128) p.debug[kDbgT + e] = Ts[(e >> 6) * kLDA + (e & 63)];

        // ---- T1 = T diag(b gamma), T2 = T diag(b), physical order, into A's space
        {
            const int r = pt & 63;
            const bool second = pt >= 64;
            const int lr = x.dir ? 63 - r : r;
            const float *Trow = Ts + lr * kLDA;
            const float *scale = gt + (second ? gBet : gBG) * 64;
            float xv[64];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float4 t4 = *reinterpret_cast<const float4 *>(Trow + 4 * m);   // scan cols 4m..4m+3
                const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int lj = 4 * m + u;
                    if (x.dir) xv[63 - lj] = tv[u];
                    else xv[lj] = tv[u];
                }
            }
#pragma unroll
            for (int j = 0; j < 64; ++j) xv[j] *= scale[j];
            store_row_bf16(x.sbase + (second ? kOffT2 : kOffT1), r, xv);
        }
        fence_proxy_async_smem();
        if (named_bar_any(kBarPrep, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.tp_full);

        // ---- W (MN-major, row d = key index) to shared memory
        wait_bar(&B.wu_full, i & 1, x.abort_flag, p.err, 5);
        if (i >= 1) wait_bar(&B.wmn_empty, (i - 1) & 1, x.abort_flag, p.err, 6);
        tc_fence_after();
        {
            float xv[64];
            tmem_ld64(x.tmem + tm_lane + kColW, xv);
            if (dbg) {
                dbg_rows(p.debug + kDbgW, pt, xv);
                float yv[64];
                tmem_ld64(x.tmem + tm_lane + kColU0 + 64 * b, yv);
                dbg_rows(p.debug + kDbgUt, pt, yv);
            }
            store_row_bf16(x.sbase + kOffW, pt, xv);
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarPrep, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.wmn_full);
    }
}

// ------------------------------------------------------------------ chain warps
__device__ void chain_role(const Ctx &x, const TcParams &p, int ct)
{
    Bars &B = *x.bars;
    const int warp = ct >> 5, lane = ct & 31;
    const uint32_t tm_lane = (uint32_t)(warp * 32) << 16;

    float h[kDVS];
    {
        const float *s0 = (x.dir == 0 && p.state_in)
                              ? p.state_in + ((size_t)x.bh * kDK + ct) * x.dv + x.slice * kDVS
                              : nullptr;
#pragma unroll
        for (int e = 0; e < kDVS; e += 4) {
            const float4 v4 = s0 ? *reinterpret_cast<const float4 *>(s0 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            h[e] = v4.x; h[e + 1] = v4.y; h[e + 2] = v4.z; h[e + 3] = v4.w;
        }
        store_row_bf16(x.sbase + kOffH, ct, h);
    }
    fence_proxy_async_smem();
    named_bar(kBarChain);
    if (ct == 0) mbar_arrive(&B.h_full);

    for (int i = 0; i < x.NC; ++i) {
        const int b = i & 1, c = chunk_of(x, i);
        const float *gt = gates_buf(x, b);
        const bool dbg = p.debug != nullptr && i == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&
                         blockIdx.z == 0;

        // ---- U and Ubar rows (M=64 layout: warp w, lanes 0-15 hold rows 16w..16w+15)
        wait_bar(&B.g_full[b], (i >> 1) & 1, x.abort_flag, p.err, 7);
        wait_bar(&B.chain_full, i & 1, x.abort_flag, p.err, 8);
        tc_fence_after();
        {
            float xv[64];
            tmem_ld64(x.tmem + tm_lane + kColU0 + 64 * b, xv);
            if (dbg) dbg_rows(p.debug + kDbgU, ct, xv);
            if (lane < 16) {
                const int r = warp * 16 + lane;
                store_row_bf16(x.sbase + kOffU, r, xv);
                const float eb = gt[gEb * 64 + r];
#pragma unroll
                for (int e = 0; e < 64; ++e) xv[e] *= eb;
                store_row_bf16(x.sbase + kOffUb, r, xv);
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarChain, *x.abort_flag)) return;
        if (ct == 0) {
            mbar_arrive(&B.u_full);
            mbar_arrive(&B.du_empty[b]);
        }

        // ---- state update (fp32 registers) and its bf16 copy
        wait_bar(&B.s_full, i & 1, x.abort_flag, p.err, 9);
        tc_fence_after();
        {
            float xv[64];
            tmem_ld64(x.tmem + tm_lane + kColS, xv);
            if (dbg) dbg_rows(p.debug + kDbgS, ct, xv);
            const float ge = exp2f(gt[gScal * 64]);
#pragma unroll
            for (int e = 0; e < 64; ++e) h[e] = fmaf(ge, h[e], xv[e]);
            store_row_bf16(x.sbase + kOffH, ct, h);
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarChain, *x.abort_flag)) return;
        if (ct == 0) {
            mbar_arrive(&B.h_full);
            mbar_arrive(&B.g_empty[b]);
        }

        // ---- output tile
        wait_bar(&B.o_full[b], (i >> 1) & 1, x.abort_flag, p.err, 10);
        tc_fence_after();
        {
            float xv[64];
            tmem_ld64(x.tmem + tm_lane + kColO0 + 64 * b, xv);
            if (dbg) dbg_rows(p.debug + kDbgO, ct, xv);
            const int r = warp * 16 + lane;
            const int t = c * kC + r;
            const bool mine = lane < 16 && t < x.T;
            __nv_bfloat16 *orow = p.o + ((size_t)x.bh * x.T + (mine ? t : 0)) * x.dv + x.slice * kDVS;
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = pack_bf16(xv[2 * e], xv[2 * e + 1]);
            if (p.counters == nullptr) {
                if (mine)
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            } else {
                int *cnt = p.counters + ((size_t)x.bh * x.NC + c) * p.n_slices + x.slice;
                if (ct == 0) x.bars->s_old = atomicAdd(cnt, 1);
                named_bar(kBarChain);
                if (x.bars->s_old == 0) {
                    if (mine)
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    named_bar(kBarChain);
                    if (ct == 0) {
                        __threadfence();
                        atomicAdd(cnt, 1);
                    }
                } else {
                    if (ct == 0) {
                        const unsigned long long t0 = globaltimer();
                        int seen = 0;
                        for (uint32_t it = 0; it < (1u << 30); ++it) {
                            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(seen) : "l"(cnt) : "memory");
                            if (seen >= 3) break;
                            if ((it & 255) == 255 && globaltimer() - t0 > kWaitLimitNs) break;
                        }
                        if (seen < 3) {
                            atomicOr(p.err, 32);
                            *x.abort_flag = 1;
                        }
                        __threadfence();
                    }
                    named_bar(kBarChain);
                    if (mine && !*x.abort_flag) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 o4 = __ldcg(reinterpret_cast<const uint4 *>(orow + 8 * q));
                            const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
                            uint32_t sw[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ow[u]));
                                sw[u] = pack_bf16(f.x + xv[8 * q + 2 * u], f.y + xv[8 * q + 2 * u + 1]);
                            }
                            *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
                        }
                    }
                }
            }
        }
        tc_fence_before();
        if (named_bar_any(kBarChain, *x.abort_flag)) return;
        if (ct == 0) mbar_arrive(&B.do_empty[b]);
    }

    if (p.state_out) {
        float *so = p.state_out + (((size_t)x.dir * p.BH + x.bh) * kDK + ct) * x.dv + x.slice * kDVS;
#pragma unroll
        for (int e = 0; e < kDVS; e += 4)
            *reinterpret_cast<float4 *>(so + e) = make_float4(h[e], h[e + 1], h[e + 2], h[e + 3]);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    Ctx x;
    x.smem = smem;
    x.sbase = smem_u32(smem);
    x.bars = reinterpret_cast<Bars *>(smem + kOffBar);
    x.abort_flag = &x.bars->abort_flag;
    x.slice = blockIdx.x;
    x.dir = blockIdx.y;
    x.bh = blockIdx.z;
    x.T = p.T;
    x.NC = p.n_chunks;
    x.dv = p.dv;
    Bars &B = *x.bars;

    if (tid == 0) {
        uint64_t *all = reinterpret_cast<uint64_t *>(&B);
        const int nbar = (int)(offsetof(Bars, tmem_slot) / sizeof(uint64_t));
        for (int k = 0; k < nbar; ++k) mbar_init(&all[k], 1);
        B.abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 0) {
        tmem_alloc(&B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    float *Ts = reinterpret_cast<float *>(smem + kOffT);
    for (int i = tid; i < 64 * kLDA; i += kThreads) Ts[i] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = B.tmem_slot;

    if (warp < 4) {
        chain_role(x, p, tid);
    } else if (warp < 8) {
        prep_role(x, p, tid - 128);
    } else if (warp == 8) {
        if (lane == 0) tma_role(x, &tmQ, &tmK, &tmV, p);
    } else {
        if (lane == 0) mma_role(x, p);
    }

    tc_fence_before();
    __syncthreads();
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

}  // namespace

float *g_debug_dump = nullptr;

bool chunk_tc_supported(const FwdArgs &a)
{
    return !a.fp32 && a.dk == kDK && (a.dv == 64 || a.dv == 128);
}

cudaError_t launch_chunk_tc(const FwdArgs &a, cudaStream_t stream)
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
    p.counters = nullptr;
    p.debug = g_debug_dump;
    cudaError_t err = device_error_word(&p.err);
    if (err != cudaSuccess) return err;

    err = cudaFuncSetAttribute(gdn_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemAlloc);
    if (err != cudaSuccess) return err;
    const size_t n_cnt = (size_t)BH * p.n_chunks * p.n_slices;
    if (a.bidi) {
        err = cudaMallocAsync(reinterpret_cast<void **>(&p.counters), n_cnt * sizeof(int), stream);
        if (err != cudaSuccess) return err;
        err = cudaMemsetAsync(p.counters, 0, n_cnt * sizeof(int), stream);
    }
    if (err == cudaSuccess) {
        dim3 grid(p.n_slices, a.bidi ? 2 : 1, BH);
        gdn_chunk_tc_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, p);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (p.counters) {
        cudaError_t e2 = cudaFreeAsync(p.counters, stream);
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

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
int *g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

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
    p.counters = nullptr;
    p.debug = nullptr;
    cudaError_t err = device_error_word(&p.err);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(gdn_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemAlloc);
    if (err != cudaSuccess) return err;

    if (a.bidi) {
        const size_t n_cnt = (size_t)BH * p.n_chunks * p.n_slices;
        if (n_cnt > kNoAllocCounters) return cudaErrorInvalidValue;   // checked by the caller too
        int dev = 0;
        err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        {
            // Host code cannot use the array's name as a device address: look the
            // address up once per device, with that device current.
            std::lock_guard<std::mutex> lock(g_noalloc_mu);
            if (!g_noalloc_ptr[dev]) {
                void *ptr = nullptr;
                err = cudaGetSymbolAddress(&ptr, g_noalloc_counters);
                if (err != cudaSuccess) return err;
                g_noalloc_ptr[dev] = static_cast<int *>(ptr);
            }
            p.counters = g_noalloc_ptr[dev];
        }
        // the array keeps the previous call's contents: the counters must start at zero
        err = cudaMemsetAsync(p.counters, 0, n_cnt * sizeof(int), stream);
        if (err != cudaSuccess) return err;
    }
    dim3 grid(p.n_slices, a.bidi ? 2 : 1, BH);
    gdn_chunk_tc_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(mq, mk, mv, p);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launches(1);
    return err;
}

}  // namespace gdn

// Test hook (not part of the documented ABI): when set to a device buffer of
// 53248 floats, the next chunkwise launches dump the first chunk's
// intermediates of CTA (0,0,0) there.  NULL turns it off.
extern "C" void gdn_debug_dump(float *device_buffer) { gdn::g_debug_dump = device_buffer; }
