// Device helpers shared by the chunkwise tensor-core kernels: bounded waits
// (mbarrier phases, shared-memory words, device-wide counters) that record an
// error and raise the CTA's abort flag instead of hanging, named barriers,
// bf16 packing into 128B-swizzled tiles, and the 64 x 64 unit lower-
// triangular solve T = (I + A)^-1 of the WY/UT chunk form (fp32 substitution
// on the 16 x 16 diagonal blocks, tf32 mma.sync block substitution below
// them).  Included inside each kernel file's translation unit.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace gdn {
namespace {

using namespace ptx;

constexpr int kC = 64;           // chunk length
constexpr int kDK = 128;         // key dim served by the chunkwise kernels
constexpr int kLDA = 68;         // fp32 row stride of the solve buffers

// gate arrays (64 floats each, physical token order unless noted)
// G (log2 cumulative decay), gamma = 2^G, beta, beta*gamma, 2^(G_end - G), row/column
// factors of the decay products (A: same half of the chunk, B: across halves)
enum GateIdx { gG = 0, gGam, gBet, gBG, gEb, gRA, gRB, gCA, gCB };

constexpr unsigned long long kWaitLimitNs = 4000000000ull;   // 4 s per wait

// The limit the bounded waits below apply (one copy per module that includes
// this header; kWaitLimitNs unless a test lowers it to make a wait run out).
static __device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

// Sets this module's wait limit on the current device (synchronous).
static inline cudaError_t set_module_wait_limit(unsigned long long ns)
{
    return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase; on timeout records the error and raises
// the CTA's abort flag (callers then reach their group's next barrier and
// leave together).
__device__ __noinline__ bool wait_bar_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int *err, int code)
{
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 255) == 255 && globaltimer() - t0 > g_wait_limit_ns) break;
    }
    atomicOr(err, code);
    *abort_flag = 1;
    return false;
}

// The first try covers almost every wait; the loop with its timer and error
// path is kept out of line so that it does not crowd the instruction cache.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int *err, int code)
{
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, abort_flag, err, code);
}

__device__ __forceinline__ void st_release_cta(int *addr, int v)
{
    asm volatile("st.release.cta.shared.b32 [%0], %1;" ::"r"(smem_u32(addr)), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_cta(const int *addr)
{
    int v;
    asm volatile("ld.acquire.cta.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(addr)) : "memory");
    return v;
}

// Bounded wait until a shared-memory word written by another warp of the CTA
// reaches `target`; false on timeout (error recorded, abort raised) or abort.
__device__ __noinline__ bool wait_smem_slow(const int *addr, int target, volatile int *abort_flag, int *err,
                                            int code)
{
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (ld_acquire_cta(addr) >= target) return true;
        if (*abort_flag) return false;
        if ((it & 255) == 255 && globaltimer() - t0 > g_wait_limit_ns) break;
    }
    atomicOr(err, code);
    *abort_flag = 1;
    return false;
}

__device__ __forceinline__ bool wait_smem_at_least(const int *addr, int target, volatile int *abort_flag,
                                                   int *err, int code)
{
    if (ld_acquire_cta(addr) >= target) return true;
    return wait_smem_slow(addr, target, abort_flag, err, code);
}

// Bounded wait (one thread) until a device-wide counter reaches `target`,
// with acquire semantics at GPU scope; false on timeout or abort.
__device__ __noinline__ bool spin_global_at_least(const int *cnt, int target, volatile int *abort_flag)
{
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        int seen;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(seen) : "l"(cnt) : "memory");
        if (seen >= target) return true;
        if (*abort_flag) return false;
        if ((it & 63) == 63) {
            if (globaltimer() - t0 > g_wait_limit_ns) return false;
            __nanosleep(64);
        }
    }
    return false;
}

__device__ __forceinline__ void named_bar(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier over a 128-thread group that also ORs a predicate across it,
// so that every thread of the group takes the same abort decision.
__device__ __forceinline__ bool named_bar_any(int id, int count, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, %2, %3, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(count) : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Shared-memory tiles are written with plain stores through pointers derived
// from the dynamic shared array, so that the compiler can schedule them freely
// (the fences and barriers that publish them carry the ordering).
__device__ __forceinline__ void st_tile_v4(uint8_t *tile, uint32_t off, uint32_t a, uint32_t b, uint32_t c,
                                           uint32_t d)
{
    *reinterpret_cast<uint4 *>(tile + off) = make_uint4(a, b, c, d);
}

// Writes 32 fp32 values as half (64 bytes, 16-byte chunks 4h..4h+3) of a
// 128-byte bf16 row of a 128B-swizzled tile.
__device__ __forceinline__ void store_half_row_bf16(uint8_t *tile, uint32_t row, int h, const float *x)
{
#pragma unroll
    for (int q = 0; q < 4; ++q)
        st_tile_v4(tile, sw128_off(row, 32 * h + 8 * q), pack_bf16(x[8 * q + 0], x[8 * q + 1]),
                     pack_bf16(x[8 * q + 2], x[8 * q + 3]), pack_bf16(x[8 * q + 4], x[8 * q + 5]),
                     pack_bf16(x[8 * q + 6], x[8 * q + 7]));
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


// T = (I + A)^-1 for a strictly lower-triangular 64 x 64 fp32 A (scan order)
// in 16 x 16 blocks, written straight into the bf16 operands
// T1 = T diag(b gamma) and T2 = T diag(b) (physical order, 128B-swizzled):
//   1. the diagonal blocks D_a = (I + A_aa)^-1 by forward substitution, one
//      column per thread (right-looking, so one FMA per step is serial); D_a
//      replaces A_aa in place;
//   2. the blocks below them by block-forward substitution,
//      T_ab = -D_a sum_{b <= k < a} A_ak T_kb, each prep warp walking one
//      8-column strip of T down the block rows with tf32 mma.sync, its
//      earlier blocks kept in registers (no barrier between the steps),
//      while the two remaining warps write the diagonal blocks' T1, T2.
// The upper triangle of T1/T2 is never written: it is zeroed once.

// bf16 pair (scan-order row lr, columns lj and lj + 1) into a physical-order
// tile (dir 1: rows and columns reversed)
__device__ __forceinline__ void st_tpair(uint8_t *tile, int dir, int lr, int lj, float v0, float v1)
{
    const int pr = dir ? 63 - lr : lr;
    const int pc = dir ? 62 - lj : lj;   // the pair's lower physical column (even)
    *reinterpret_cast<uint32_t *>(tile + sw128_off(pr, pc)) = dir ? pack_bf16(v1, v0) : pack_bf16(v0, v1);
}

// BAR / NTHREADS: the named barrier that ends the step (or, with NTHREADS = 0,
// the run-time bar_id / bar_threads).
template <int BAR, int NTHREADS>
__device__ __forceinline__ void solve_diag_blocks(float *As, const float *gt, uint8_t *sT1, uint8_t *sT2,
                                               float *dbgT, int dir, int pt, int bar_id = 0, int bar_threads = 0)
{
    if (pt < 64) {
        const int a = pt >> 4, c = pt & 15;
        float *Ab = As + (16 * a) * kLDA + 16 * a;
        float x[16], acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            x[m] = (m == c) ? 1.f : ((m > c) ? -acc[m] : 0.f);
#pragma unroll
            for (int r = m + 1; r < 16; ++r) acc[r] = fmaf(Ab[r * kLDA + m], x[m], acc[r]);
        }
        __syncwarp();   // the block's 16 columns are one half warp: all reads done
#pragma unroll
        for (int r = 0; r < 16; ++r) Ab[r * kLDA + c] = x[r];
        if (dbgT)
            for (int r = 0; r < 16; ++r) dbgT[(16 * a + r) * 64 + 16 * a + c] = x[r];
    }
    if (NTHREADS) named_bar(BAR, NTHREADS);
    else named_bar(bar_id, bar_threads);
}

// T1, T2 of the four diagonal blocks, from D_a in place in A (64 threads: each
// writes 16 column pairs of one block row band; a compact loop, run by warps
// that have no off-diagonal strip).
__device__ __forceinline__ void store_diag_t12(const float *As, const float *gt, uint8_t *sT1, uint8_t *sT2,
                                               int dir, int t)
{
    const int a = t >> 4, cp = (t & 7) * 2, rh = (t >> 3) & 1;   // block, column pair, row half
    const int lj = 16 * a + cp;
    const int pc0 = dir ? 63 - lj : lj, pc1 = dir ? 62 - lj : lj + 1;
    const float sg0 = gt[gBG * 64 + pc0], sg1 = gt[gBG * 64 + pc1];
    const float sb0 = gt[gBet * 64 + pc0], sb1 = gt[gBet * 64 + pc1];
#pragma unroll 1
    for (int r = 8 * rh; r < 8 * rh + 8; ++r) {
        const int lr = 16 * a + r;
        const float2 v = *reinterpret_cast<const float2 *>(As + lr * kLDA + lj);
        st_tpair(sT1, dir, lr, lj, v.x * sg0, v.y * sg1);
        st_tpair(sT2, dir, lr, lj, v.x * sb0, v.y * sb1);
    }
}

// tf32 A fragment (rows r0.., columns k0..) of an fp32 [64][kLDA] matrix
__device__ __forceinline__ void ld_afrag(uint32_t (&a)[4], const float *M, int r0, int k0, int g, int q)
{
    const float *p = M + (r0 + g) * kLDA + k0 + q;
    a[0] = to_tf32(p[0]);
    a[1] = to_tf32(p[8 * kLDA]);
    a[2] = to_tf32(p[4]);
    a[3] = to_tf32(p[8 * kLDA + 4]);
}

// A 16 x 8 accumulator tile (C layout) rearranged, through shuffles, into the
// B operand of a following m16n8k8 product (two k-steps of 8 rows), as tf32
__device__ __forceinline__ void c_to_b(const float (&c)[4], uint32_t (&b)[2][2], int g, int q)
{
    const int src0 = q * 4 + (g >> 1), src1 = (q + 4) * 4 + (g >> 1);
    const bool odd = (g & 1) != 0;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const float lo0 = __shfl_sync(0xffffffffu, c[2 * ks], src0);
        const float hi0 = __shfl_sync(0xffffffffu, c[2 * ks + 1], src0);
        const float lo1 = __shfl_sync(0xffffffffu, c[2 * ks], src1);
        const float hi1 = __shfl_sync(0xffffffffu, c[2 * ks + 1], src1);
        b[ks][0] = to_tf32(odd ? hi0 : lo0);
        b[ks][1] = to_tf32(odd ? hi1 : lo1);
    }
}

// Prep warp pw: the strip of columns [16 jb + 8 hs, +8) of T below its
// diagonal block jb = pw / 2; the two warps of block column 3 (no block below
// it) write the diagonal blocks' T1, T2 instead.
__device__ __forceinline__ void solve_off_diag(const float *As, const float *gt, uint8_t *sT1, uint8_t *sT2,
                                            float *dbgT, int dir, int pt)
{
    const int pw = pt >> 5, lane = pt & 31, g = lane >> 2, q = lane & 3, hs = pw & 1, jb = pw >> 1;
    if (jb == 3) {   // no strip below block column 3: write the diagonal blocks' T1, T2
        store_diag_t12(As, gt, sT1, sT2, dir, pt - 192);
        return;
    }
    const int c0 = 16 * jb + 8 * hs;
    uint32_t tb[3][2][2];   // B fragments of the strip's blocks in block rows jb, jb+1, jb+2
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        tb[0][ks][0] = to_tf32(As[(16 * jb + 8 * ks + q) * kLDA + c0 + g]);
        tb[0][ks][1] = to_tf32(As[(16 * jb + 8 * ks + q + 4) * kLDA + c0 + g]);
    }
    const int lj = c0 + 2 * q;
    const int pc0 = dir ? 63 - lj : lj, pc1 = dir ? 62 - lj : lj + 1;
    const float sg0 = gt[gBG * 64 + pc0], sg1 = gt[gBG * 64 + pc1];
    const float sb0 = gt[gBet * 64 + pc0], sb1 = gt[gBet * 64 + pc1];
#pragma unroll
    for (int io = 1; io < 4; ++io) {
        const int ib = jb + io;   // block row
        if (ib > 3) break;
        // S = sum_k A_{ib,k} T_{k,jb}, two accumulators to halve the chain
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ko = 0; ko < 3; ++ko) {
            if (ko >= io) break;
            const int kb = jb + ko;
            uint32_t a[4];
            if (ko != 0 || hs == 0) {   // D_jb is zero above the strip's diagonal
                ld_afrag(a, As, 16 * ib, 16 * kb, g, q);
                mma_tf32(s0, a, tb[ko][0]);
            }
            ld_afrag(a, As, 16 * ib, 16 * kb + 8, g, q);
            mma_tf32(s1, a, tb[ko][1]);
        }
        float sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) sv[u] = s0[u] + s1[u];
        uint32_t sbf[2][2];
        c_to_b(sv, sbf, g, q);
        // T_{ib,jb} = -D_ib S
        float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t a[4];
            ld_afrag(a, As, 16 * ib, 16 * ib + 8 * ks, g, q);
            mma_tf32(t, a, sbf[ks]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) t[u] = -t[u];
        const int lr = 16 * ib + g;
        st_tpair(sT1, dir, lr, lj, t[0] * sg0, t[1] * sg1);
        st_tpair(sT1, dir, lr + 8, lj, t[2] * sg0, t[3] * sg1);
        st_tpair(sT2, dir, lr, lj, t[0] * sb0, t[1] * sb1);
        st_tpair(sT2, dir, lr + 8, lj, t[2] * sb0, t[3] * sb1);
        if (dbgT) {
            dbgT[lr * 64 + lj] = t[0];
            dbgT[lr * 64 + lj + 1] = t[1];
            dbgT[(lr + 8) * 64 + lj] = t[2];
            dbgT[(lr + 8) * 64 + lj + 1] = t[3];
        }
        if (io < 3) c_to_b(t, tb[io], g, q);
    }
}

// N MMAs of one product into d: the operand descriptors advance by A_STEP and
// B_STEP (16-byte units) per K step; the first MMA overwrites D unless acc.
template <int N, uint32_t A_STEP, uint32_t B_STEP>
__device__ __forceinline__ void mma_run(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc)
{
#pragma unroll
    for (int k = 0; k < N; ++k)
        mma_bf16(d, a + (uint64_t)(k * A_STEP), b + (uint64_t)(k * B_STEP), idesc, (k > 0 || acc) ? 1u : 0u);
}

// The off-diagonal blocks of T for 8 warps: warp pw walks the strip of block
// column jb = pw / 2, columns [16 jb + 8 (pw % 2), +8), down the block rows
// below it; the two warps of block column 3 (no block below it) write the
// diagonal blocks' T1, T2 instead.  One block row per loop step (compact code:
// the prep shares its SM's instruction caches with the other roles): every A
// fragment of the row is loaded before its products start, and the block
// products go to independent accumulators, so that a step waits on one round
// of shared loads and on the tensor products of its own chain.
__device__ __forceinline__ void solve_off_diag_strips(const float *As, const float *gt, uint8_t *sT1,
                                                      uint8_t *sT2, int dir, int pt)
{
    const int pw = pt >> 5, lane = pt & 31, g = lane >> 2, q = lane & 3, hs = pw & 1, jb = pw >> 1;
    if (jb == 3) {   // no strip below block column 3: write the diagonal blocks' T1, T2
        store_diag_t12(As, gt, sT1, sT2, dir, pt - 192);
        return;
    }
    const int c0 = 16 * jb + 8 * hs;
    uint32_t tb[3][2][2];   // B fragments of the strip's blocks in block rows jb, jb+1, jb+2
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        tb[0][ks][0] = to_tf32(As[(16 * jb + 8 * ks + q) * kLDA + c0 + g]);
        tb[0][ks][1] = to_tf32(As[(16 * jb + 8 * ks + q + 4) * kLDA + c0 + g]);
    }
#pragma unroll
    for (int kb = 1; kb < 3; ++kb)
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) tb[kb][ks][0] = tb[kb][ks][1] = 0u;
    const int lj = c0 + 2 * q;
    const int pc0 = dir ? 63 - lj : lj, pc1 = dir ? 62 - lj : lj + 1;
    const float sg0 = gt[gBG * 64 + pc0], sg1 = gt[gBG * 64 + pc1];
    const float sb0 = gt[gBet * 64 + pc0], sb1 = gt[gBet * 64 + pc1];
#pragma unroll 1
    for (int io = 1; io <= 3 - jb; ++io) {
        const int ib = jb + io;   // block row
        // the row's fragments: A_{ib, jb + kb} for kb < io, and D_ib
        uint32_t a[3][2][4], d[2][4];
#pragma unroll
        for (int kb = 0; kb < 3; ++kb)
            if (kb < io) {
                ld_afrag(a[kb][0], As, 16 * ib, 16 * (jb + kb), g, q);
                ld_afrag(a[kb][1], As, 16 * ib, 16 * (jb + kb) + 8, g, q);
            }
        ld_afrag(d[0], As, 16 * ib, 16 * ib, g, q);
        ld_afrag(d[1], As, 16 * ib, 16 * ib + 8, g, q);
        // S = sum_k A_{ib,k} T_{k,jb}, one accumulator per product
        float sp[3][2][4];
#pragma unroll
        for (int kb = 0; kb < 3; ++kb)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int u = 0; u < 4; ++u) sp[kb][ks][u] = 0.f;
        if (hs == 0) mma_tf32(sp[0][0], a[0][0], tb[0][0]);   // D_jb is zero above the strip's diagonal
        mma_tf32(sp[0][1], a[0][1], tb[0][1]);
#pragma unroll
        for (int kb = 1; kb < 3; ++kb)
            if (kb < io) {
                mma_tf32(sp[kb][0], a[kb][0], tb[kb][0]);
                mma_tf32(sp[kb][1], a[kb][1], tb[kb][1]);
            }
        float sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            sv[u] = (sp[0][0][u] + sp[0][1][u]) + (sp[1][0][u] + sp[1][1][u]) + (sp[2][0][u] + sp[2][1][u]);
        uint32_t sbf[2][2];
        c_to_b(sv, sbf, g, q);
        // T_{ib,jb} = -D_ib S
        float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
        mma_tf32(t0, d[0], sbf[0]);
        mma_tf32(t1, d[1], sbf[1]);
        float t[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) t[u] = -(t0[u] + t1[u]);
        const int lr = 16 * ib + g;
        st_tpair(sT1, dir, lr, lj, t[0] * sg0, t[1] * sg1);
        st_tpair(sT1, dir, lr + 8, lj, t[2] * sg0, t[3] * sg1);
        st_tpair(sT2, dir, lr, lj, t[0] * sb0, t[1] * sb1);
        st_tpair(sT2, dir, lr + 8, lj, t[2] * sb0, t[3] * sb1);
        if (io == 1) c_to_b(t, tb[1], g, q);
        else if (io == 2) c_to_b(t, tb[2], g, q);
    }
}

}  // namespace
}  // namespace gdn
