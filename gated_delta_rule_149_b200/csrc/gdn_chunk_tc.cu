// Chunkwise GDN recurrence on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The recurrence (librediffusion PR #21 page, "What's added": the GDN
// linear-attention recurrence; the causal-streaming and bidirectional forms
// of the flashdreams SANA-WM page), per head, with H = S^T (dk x dv):
//     H_t = a_t (I - b_t k_t k_t^T) H_{t-1} + b_t k_t v_t^T,   o_t = H_t^T q_t
// is evaluated 64 tokens at a time in its WY/UT form.  Per chunk, in scan
// order (forward: ascending t; reverse: descending t), with g = log a,
// G_i = sum of g up to and including token i, gamma_i = exp(G_i):
//     A    = strict-lower [ b_i exp(G_i - G_j) k_i.k_j ]        (64 x 64)
//     P    = lower        [ exp(G_i - G_j) q_i.k_j ]             (64 x 64)
//     T    = (I + A)^-1                                          (fp32 solve)
//     W    = T diag(b gamma) K,     U~ = T diag(b) V
//     U    = U~ - W H_prev                                       (serial step)
//     O    = diag(gamma) Q H_prev + P U
//     H    = gamma_end H_prev + K^T diag(exp(G_end - G)) U         (serial step)
// Only exp(G_i - G_j) with j at or before i is ever formed, so every exponent
// is <= 0 and nothing overflows however strong the decay.
//
// One CTA per (64-wide dv slice, direction, batch*head).  The fp32 state lives
// in registers (thread d owns row d of the dk x 64 slice) and a bf16 copy in
// shared memory feeds the tensor cores.  Tensor-core products (bf16 operands,
// fp32 accumulation in TMEM):
//     [Q;K] K^T        M=128 N=64  K=dk     -> QK^T, KK^T
//     W^T = K^T T1^T   M=128 N=64  K=64     (T1 = T diag(b gamma))
//     U~  = T2 V       M=64  N=64  K=64     (T2 = T diag(b))
//     U  -= W H        M=64  N=64  K=dk     (A negated in the descriptor)
//     O   = (gamma Q) H, O += P U           M=64 N=64
//     D_S = K^T Ubar   M=128 N=64  K=64     (Ubar = diag(exp(G_end-G)) U)
// Bidirectional: both scans run in the same launch; for each (head, chunk,
// slice) output tile the first finisher writes its partial and the second
// adds its own and writes the sum (an arrival counter decides who is who).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"

namespace gdn {

extern float *g_debug_dump;

namespace {

using namespace ptx;

constexpr int kC = 64;          // chunk length
constexpr int kDK = 128;        // key dim served by this kernel
constexpr int kDVS = 64;        // dv columns per CTA
constexpr int kThreads = 128;
constexpr int kLDA = 68;        // fp32 row stride of the solve buffers

// TMEM columns (fp32 accumulators)
constexpr uint32_t kColD1 = 0;     // [Q;K] K^T   (M=128)
constexpr uint32_t kColW = 64;     // W^T         (M=128)
constexpr uint32_t kColU = 128;    // U~ then U   (M=64)
constexpr uint32_t kColO = 192;    // O           (M=64)
constexpr uint32_t kColS = 256;    // K^T Ubar    (M=128)
constexpr uint32_t kTmemCols = 512;

// Shared-memory carve-up (bytes from a 1024-aligned base)
constexpr uint32_t kStageBytes = 40 * 1024;          // [kb0: Q|K][kb1: Q|K] 32 KB + V 8 KB
constexpr uint32_t kOffStage = 0;                    // 2 stages
constexpr uint32_t kOffT1 = 2 * kStageBytes;         // 8 KB  bf16 [i][j]
constexpr uint32_t kOffT2 = kOffT1 + 8192;           // 8 KB
constexpr uint32_t kOffP = kOffT2 + 8192;            // 8 KB
constexpr uint32_t kOffW = kOffP + 8192;             // 16 KB bf16 [d][i]  (W, MN-major)
constexpr uint32_t kOffU = kOffW + 16384;            // 8 KB  bf16 [i][e]
constexpr uint32_t kOffUb = kOffU + 8192;            // 8 KB
constexpr uint32_t kOffH = kOffUb + 8192;            // 16 KB bf16 [d][e]
constexpr uint32_t kOffA = kOffH + 16384;            // fp32 [64][68] (logical order)
constexpr uint32_t kOffT = kOffA + 64 * kLDA * 4;    // fp32 [64][68] (logical order)
constexpr uint32_t kOffY = kOffT + 64 * kLDA * 4;    // fp32 [3][256]
constexpr uint32_t kOffGates = kOffY + 3 * 256 * 4;  // G, gamma, beta, b*gamma, ebar: 5 x 64 fp32
constexpr uint32_t kOffMisc = kOffGates + 5 * 64 * 4;
constexpr uint32_t kSmemBytes = kOffMisc + 128;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // alignment slack

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
              kDbgS = 40960, kDbgT = 49152, kDbgFloats = 53248;

__device__ __forceinline__ void dbg_rows(float *dst, int tid, const float *x)
{
#pragma unroll
    for (int e = 0; e < 64; ++e) dst[tid * 64 + e] = x[e];
}

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase; on timeout records the error and raises
// the CTA's abort flag.
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

// T = (I + A)^-1 for a strictly lower-triangular 64 x 64 fp32 A (logical
// order), blocked: 16 x 16 diagonal blocks by forward substitution, then the
// off-diagonal blocks by distance, T_ab = -T_aa sum_{m=b}^{a-1} A_am T_mb.
// The upper triangle of Ts must be zero on entry and stays zero.
__device__ void solve_unit_lower(const float *As, float *Ts, float *Y, int tid)
{
    if (tid < 64) {
        const int a = tid >> 4, c = tid & 15;
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
    __syncthreads();
    for (int dist = 1; dist <= 3; ++dist) {
        const int nel = (4 - dist) * 256;
        for (int e = tid; e < nel; e += kThreads) {
            const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
            const int a = dist + blk, b = blk;
            const float *Arow = As + (16 * a + r) * kLDA;
            float s = 0.f;
            for (int m = 16 * b + c; m < 16 * a; ++m) s = fmaf(Arow[m], Ts[m * kLDA + 16 * b + c], s);
            Y[e] = s;
        }
        __syncthreads();
        for (int e = tid; e < nel; e += kThreads) {
            const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
            const int a = dist + blk, b = blk;
            const float *Drow = Ts + (16 * a + r) * kLDA + 16 * a;
            float s = 0.f;
            for (int m = 0; m <= r; ++m) s = fmaf(Drow[m], Y[(blk << 8) + m * 16 + c], s);
            Ts[(16 * a + r) * kLDA + 16 * b + c] = -s;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);

    const int slice = blockIdx.x, dir = blockIdx.y, bh = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, NC = p.n_chunks, dv = p.dv;

    float *As = reinterpret_cast<float *>(smem + kOffA);
    float *Ts = reinterpret_cast<float *>(smem + kOffT);
    float *Yb = reinterpret_cast<float *>(smem + kOffY);
    float *sG = reinterpret_cast<float *>(smem + kOffGates);
    float *sGam = sG + 64, *sBet = sG + 128, *sBG = sG + 192, *sEb = sG + 256;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(smem + kOffMisc);       // [2]
    uint64_t *bar_mma = bar_tma + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 3);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_old = reinterpret_cast<int *>(tmem_slot + 2);
    float *s_gend = reinterpret_cast<float *>(tmem_slot + 3);
    float *s_wsum = reinterpret_cast<float *>(tmem_slot + 4);

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    for (int i = tid; i < 64 * kLDA; i += kThreads) Ts[i] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tm_lane = (uint32_t)(warp * 32) << 16;   // this warp's TMEM lane quarter

    // ---- initial state: thread d owns row d of the dk x 64 slice
    float h[kDVS];
    {
        const float *s0 = (dir == 0 && p.state_in)
                              ? p.state_in + ((size_t)bh * kDK + tid) * dv + slice * kDVS
                              : nullptr;
#pragma unroll
        for (int e = 0; e < kDVS; e += 4) {
            float4 v4 = s0 ? *reinterpret_cast<const float4 *>(s0 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            h[e] = v4.x; h[e + 1] = v4.y; h[e + 2] = v4.z; h[e + 3] = v4.w;
        }
        store_row_bf16(sbase + kOffH, tid, h);
    }

    auto stage_addr = [&](int s) { return sbase + kOffStage + (uint32_t)s * kStageBytes; };
    auto issue_tma = [&](int step, int s) {
        const int c = dir ? (NC - 1 - step) : step;
        const uint32_t st = stage_addr(s);
        mbar_arrive_expect_tx(&bar_tma[s], 5 * 8192);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(smem + (st - sbase) + kb * 16384, &tmQ, &bar_tma[s], kb * 64, c * kC, bh);
            tma_load_3d(smem + (st - sbase) + kb * 16384 + 8192, &tmK, &bar_tma[s], kb * 64, c * kC, bh);
        }
        tma_load_3d(smem + (st - sbase) + 32768, &tmV, &bar_tma[s], slice * kDVS, c * kC, bh);
    };

    if (tid == 0) issue_tma(0, 0);
    uint32_t ph_tma[2] = {0u, 0u};
    uint32_t ph_mma = 0u;
    bool ok = true;

    const float *beta_h = p.beta + (size_t)bh * T;
    const float *decay_h = p.decay + (size_t)bh * T;

    for (int step = 0; step < NC && ok; ++step) {
        const int c = dir ? (NC - 1 - step) : step;
        const int s = step & 1;
        const uint32_t st = stage_addr(s);
        const uint32_t sQK = st, sV = st + 32768;
        const bool dbg = p.debug != nullptr && step == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&
                         blockIdx.z == 0;
        if (tid == 0 && step + 1 < NC) issue_tma(step + 1, s ^ 1);

        // ---- gates: thread l < 64 handles scan position l (physical p)
        {
            float g = 0.f, b = 0.f;
            int pp = 0;
            if (tid < 64) {
                pp = dir ? (63 - tid) : tid;
                const int t = c * kC + pp;
                if (t < T) {
                    g = fmaxf(log2f(decay_h[t]), -120.f);   // decay < 2^-120 acts as 2^-120
                    b = beta_h[t];
                }
                float x = g;   // inclusive scan within the warp
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                if (tid == 31) *s_wsum = x;
                g = x;
            }
            __syncthreads();
            if (tid < 64) {
                const float G = (tid >= 32) ? g + *s_wsum : g;
                sG[pp] = G;
                const float gam = exp2f(G);
                sGam[pp] = gam;
                sBet[pp] = b;
                sBG[pp] = b * gam;
                if (tid == 63) *s_gend = G;
            }
            __syncthreads();
            if (tid < 64) sEb[tid] = exp2f(*s_gend - sG[tid]);
        }

        // ---- [Q;K] K^T
        wait_bar(&bar_tma[s], ph_tma[s], abort_flag, p.err, 1);
        __syncthreads();                      // every thread then takes the same branch
        if (*abort_flag) { ok = false; break; }
        ph_tma[s] ^= 1u;
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = sw128_desc(sQK + kb * 16384 + ks * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(sQK + kb * 16384 + 8192 + ks * 32, 16, 1024);
                    mma_bf16(tmem + kColD1, ad, bd, kIdM1, (kb | ks) != 0);
                }
            mma_commit(bar_mma);
        }
        __syncthreads();   // gates visible to all
        wait_bar(bar_mma, ph_mma, abort_flag, p.err, 2);
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        ph_mma ^= 1u;
        tc_fence_after();

        // ---- P (rows 0-63 of D1) and A (rows 64-127) in scan order
        {
            float x[64];
            tmem_ld32(tmem + tm_lane + kColD1, x);
            tmem_ld32(tmem + tm_lane + kColD1 + 32, x + 32);
            tmem_wait_ld();
            if (dbg) dbg_rows(p.debug + kDbgD1, tid, x);
            if (tid < 64) {
                const int i = tid;
                const float Gi = sG[i];
                const int li = dir ? 63 - i : i;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const int lj = dir ? 63 - j : j;
                    x[j] = (lj <= li) ? exp2f(Gi - sG[j]) * x[j] : 0.f;
                }
                store_row_bf16(sbase + kOffP, i, x);
            } else {
                const int i = tid - 64;
                const float Gi = sG[i], bi = sBet[i];
                const int li = dir ? 63 - i : i;
                float *Arow = As + li * kLDA;
#pragma unroll
                for (int lj = 0; lj < 64; ++lj) {
                    const int j = dir ? 63 - lj : lj;
                    const float xv = dir ? x[63 - lj] : x[lj];
                    Arow[lj] = (lj < li) ? bi * exp2f(Gi - sG[j]) * xv : 0.f;
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- gamma-scale Q in place (Q is no longer needed unscaled)
        {
            const int i = tid >> 1, kb = tid & 1;
            const float gi = sGam[i];
            const uint32_t rowbase = sQK + kb * 16384;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t addr = rowbase + sw128_off(i, 8 * q);
                uint32_t w[4];
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&w[u]);
                    float2 f = __bfloat1622float2(v);
                    w[u] = pack_bf16(f.x * gi, f.y * gi);
                }
                st_shared_v4(addr, w[0], w[1], w[2], w[3]);
            }
        }

        // ---- T = (I + A)^-1 ; T1 = T diag(b gamma), T2 = T diag(b) (physical order)
        solve_unit_lower(As, Ts, Yb, tid);
        {
            const int i = tid & 63;
            const bool second = tid >= 64;
            const int li = dir ? 63 - i : i;
            const float *Trow = Ts + li * kLDA;
            const float *scale = second ? sBet : sBG;
            float x[64];
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const int lj = dir ? 63 - j : j;
                x[j] = Trow[lj] * scale[j];
            }
            store_row_bf16(sbase + (second ? kOffT2 : kOffT1), i, x);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- W^T = K^T T1^T (M=128) and U~ = T2 V (M=64)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sw128_desc(sQK + 8192 + ks * 2048, 16384, 1024);
                const uint64_t bd = sw128_desc(sbase + kOffT1 + ks * 32, 16, 1024);
                mma_bf16(tmem + kColW, ad, bd, kIdW, ks != 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sw128_desc(sbase + kOffT2 + ks * 32, 16, 1024);
                const uint64_t bd = sw128_desc(sV + ks * 2048, 8192, 1024);
                mma_bf16(tmem + kColU, ad, bd, kIdUt, ks != 0);
            }
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma, abort_flag, p.err, 3);
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        ph_mma ^= 1u;
        tc_fence_after();

        // ---- W (MN-major, row d = key index) to shared memory
        {
            float x[64];
            tmem_ld32(tmem + tm_lane + kColW, x);
            tmem_ld32(tmem + tm_lane + kColW + 32, x + 32);
            tmem_wait_ld();
            if (dbg) {
                dbg_rows(p.debug + kDbgW, tid, x);
                float y[64];
                tmem_ld32(tmem + tm_lane + kColU, y);
                tmem_ld32(tmem + tm_lane + kColU + 32, y + 32);
                tmem_wait_ld();
                dbg_rows(p.debug + kDbgUt, tid, y);
                for (int e = tid; e < 64 * 64; e += kThreads) p.debug[kDbgT + e] = Ts[(e >> 6) * kLDA + (e & 63)];
            }
            store_row_bf16(sbase + kOffW, tid, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- U = U~ - W H ;  O = (gamma Q) H
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = sw128_desc(sbase + kOffW + ks * 2048, 8192, 1024);
                const uint64_t bd = sw128_desc(sbase + kOffH + ks * 2048, 8192, 1024);
                mma_bf16(tmem + kColU, ad, bd, kIdUc, 1);
            }
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = sw128_desc(sQK + kb * 16384 + ks * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(sbase + kOffH + (kb * 4 + ks) * 2048, 8192, 1024);
                    mma_bf16(tmem + kColO, ad, bd, kIdOq, (kb | ks) != 0);
                }
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma, abort_flag, p.err, 4);
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        ph_mma ^= 1u;
        tc_fence_after();

        // ---- U and Ubar rows (M=64 layout: warp w, lanes 0-15 hold rows 16w..16w+15)
        {
            float x[64];
            tmem_ld32(tmem + tm_lane + kColU, x);
            tmem_ld32(tmem + tm_lane + kColU + 32, x + 32);
            tmem_wait_ld();
            if (dbg) dbg_rows(p.debug + kDbgU, tid, x);
            if (lane < 16) {
                const int r = warp * 16 + lane;
                store_row_bf16(sbase + kOffU, r, x);
                const float eb = sEb[r];
#pragma unroll
                for (int e = 0; e < 64; ++e) x[e] *= eb;
                store_row_bf16(sbase + kOffUb, r, x);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- D_S = K^T Ubar (M=128) ;  O += P U (M=64)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sw128_desc(sQK + 8192 + ks * 2048, 16384, 1024);
                const uint64_t bd = sw128_desc(sbase + kOffUb + ks * 2048, 8192, 1024);
                mma_bf16(tmem + kColS, ad, bd, kIdS, ks != 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sw128_desc(sbase + kOffP + ks * 32, 16, 1024);
                const uint64_t bd = sw128_desc(sbase + kOffU + ks * 2048, 8192, 1024);
                mma_bf16(tmem + kColO, ad, bd, kIdPU, 1);
            }
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma, abort_flag, p.err, 5);
        __syncthreads();
        if (*abort_flag) { ok = false; break; }
        ph_mma ^= 1u;
        tc_fence_after();

        // ---- state update (fp32 registers) and its bf16 copy
        {
            float x[64];
            tmem_ld32(tmem + tm_lane + kColS, x);
            tmem_ld32(tmem + tm_lane + kColS + 32, x + 32);
            tmem_wait_ld();
            if (dbg) dbg_rows(p.debug + kDbgS, tid, x);
            const float ge = exp2f(*s_gend);
#pragma unroll
            for (int e = 0; e < 64; ++e) h[e] = fmaf(ge, h[e], x[e]);
            store_row_bf16(sbase + kOffH, tid, h);
        }

        // ---- output tile
        {
            float x[64];
            tmem_ld32(tmem + tm_lane + kColO, x);
            tmem_ld32(tmem + tm_lane + kColO + 32, x + 32);
            tmem_wait_ld();
            if (dbg) dbg_rows(p.debug + kDbgO, tid, x);
            const int r = warp * 16 + lane;
            const int t = c * kC + r;
            const bool mine = lane < 16 && t < T;
            __nv_bfloat16 *orow = p.o + ((size_t)bh * T + t) * dv + slice * kDVS;
            if (p.counters == nullptr) {
                if (mine) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint4 w = make_uint4(pack_bf16(x[8 * q], x[8 * q + 1]), pack_bf16(x[8 * q + 2], x[8 * q + 3]),
                                             pack_bf16(x[8 * q + 4], x[8 * q + 5]), pack_bf16(x[8 * q + 6], x[8 * q + 7]));
                        *reinterpret_cast<uint4 *>(orow + 8 * q) = w;
                    }
                }
            } else {
                int *cnt = p.counters + ((size_t)bh * NC + c) * p.n_slices + slice;
                if (tid == 0) *s_old = atomicAdd(cnt, 1);
                __syncthreads();
                const int old = *s_old;
                if (old == 0) {
                    if (mine) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            uint4 w = make_uint4(pack_bf16(x[8 * q], x[8 * q + 1]), pack_bf16(x[8 * q + 2], x[8 * q + 3]),
                                                 pack_bf16(x[8 * q + 4], x[8 * q + 5]), pack_bf16(x[8 * q + 6], x[8 * q + 7]));
                            *reinterpret_cast<uint4 *>(orow + 8 * q) = w;
                        }
                    }
                    __syncthreads();
                    if (tid == 0) {
                        __threadfence();
                        atomicAdd(cnt, 1);
                    }
                } else {
                    if (tid == 0) {
                        const unsigned long long t0 = globaltimer();
                        int seen = 0;
                        for (uint32_t it = 0; it < (1u << 30); ++it) {
                            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(seen) : "l"(cnt) : "memory");
                            if (seen >= 3) break;
                            if ((it & 255) == 255 && globaltimer() - t0 > kWaitLimitNs) break;
                        }
                        if (seen < 3) { atomicOr(p.err, 6); *abort_flag = 1; }
                        __threadfence();
                    }
                    __syncthreads();
                    if (mine && !*abort_flag) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            uint4 w = __ldcg(reinterpret_cast<const uint4 *>(orow + 8 * q));
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                            uint32_t outw[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&ww[u]);
                                float2 f = __bfloat1622float2(v);
                                outw[u] = pack_bf16(f.x + x[8 * q + 2 * u], f.y + x[8 * q + 2 * u + 1]);
                            }
                            *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
                        }
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) ok = false;
    }

    // ---- final state
    if (ok && p.state_out) {
        float *so = p.state_out + (((size_t)dir * p.BH + bh) * kDK + tid) * dv + slice * kDVS;
#pragma unroll
        for (int e = 0; e < kDVS; e += 4)
            *reinterpret_cast<float4 *>(so + e) = make_float4(h[e], h[e + 1], h[e + 2], h[e + 3]);
    }

    // ---- teardown: on an aborted run, give in-flight copies and MMAs a bounded
    // chance to land before the TMEM is released.
    if (!ok && tid == 0) {
        volatile int dummy = 0;
        for (int s = 0; s < 2; ++s) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(&bar_tma[s], ph_tma[s]) && globaltimer() - t0 < 100000000ull) dummy++;
        }
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(bar_mma, ph_mma) && globaltimer() - t0 < 100000000ull) dummy++;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
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
