// Chunkwise GDN recurrence on sm_100a: one CTA per SM, split between the
// serial state chains (one CTA per scan) and a pool of preparation workers
// that serve every scan.
//
// The recurrence (the GDN linear-attention recurrence that the librediffusion
// PR #21 page names in "What's added", in the causal-streaming and
// bidirectional forms of the flashdreams SANA-WM page; the pages print no
// formula, this is the gated delta rule), per head, with H = S^T (dk x dv):
//     H_t = a_t (I - b_t k_t k_t^T) H_{t-1} + b_t k_t v_t^T,   o_t = H_t^T q_t
// is evaluated 64 tokens at a time in its WY/UT form.  Per chunk, in scan
// order, with g = log2 a, G_i = sum of g up to and including token i,
// gamma_i = 2^G_i, e_i = 2^(G_end - G_i):
//     A  = strict-lower [ b_i 2^(G_i - G_j) k_i.k_j ],  P = lower [ 2^(G_i - G_j) q_i.k_j ]
//     T  = (I + A)^-1,  T1 = T diag(b gamma),  T2 = T diag(b),  W = T1 K
//     U  = T2 V - W H_prev                          (the delta-rule values)
//     O  = diag(gamma) Q H_prev + P U               (the outputs)
//     H  = gamma_end H_prev + K^T diag(e) U         (the next state)
// P, T2 and W do not depend on the state: any SM can form them ahead of the
// chain, which is left with the products against the state.
//
// Roles (CTA = blockIdx.x):
//   CTA < n_scans, chain of scan CTA: loads V, K, Q and the scan's prepared
//       operands of each chunk, and runs
//           U^T = V^T T2^T - H^T W^T     (M = dv = 128, N = 64)
//           S = Ubar^T K                 (Ubar = diag(e) U; M = dv, N = dk)
//           H^T <- gamma_end H^T + S     (fp32 in registers)
//           O^T = H^T Q'^T + U^T P^T     (Q' = diag(gamma) Q; off the state's path)
//       with H^T, Ubar^T and U^T as bf16 A operands in TMEM, and writes O.
//   CTA >= n_scans, worker: takes (scan, chunk) items from a global counter in
//       chunk-major order and prepares them: gates, the masks of [Q;K] K^T
//       (P and A), the 64 x 64 solve, W^T = K^T T1^T and its epilogue
//       (tcgen05 MMAs, fp32 accumulators in TMEM); writes P, T2, -W^T, e, gamma
//       and gamma_end into the scan's ring of slots in global memory (a few
//       chunks per scan, so it stays in L2).
// A preparation is a long chain of dependent steps, independent from chunk to
// chunk; the chains are serial.  Giving the preparations their own pool of
// SMs lets as many run at once as the pool holds, whatever the number of
// scans.  Each slot carries a sequence word (chunk + 1 once filled) and each
// scan a count of chunks its chain has taken out, so a worker fills a slot
// only after its previous chunk was consumed; every wait is bounded.
// Bidirectional: both scans run in the same launch; for each output tile the
// first writer stores its bf16 partial and the second adds its fp32 partial
// to it and rounds once, after an arrival counter shows the first is visible
// (the forward scan writes first in the first half of the sequence).  The
// launch is cooperative: every CTA is resident, or the launch is refused.
// fp8 inputs (the FP8 instantiation): q, k, v arrive as E4M3 codes with one
// scale per head; workers form [Q;K] K^T on the codes (kind::f8f6f4) and widen
// only k to bf16, chains widen v, k and q; every other product is the bf16 one.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <climits>
#include <cstdint>
#include <mutex>

#include "gdn_internal.h"
#include "sm100_ptx.cuh"
#include "gdn_chunk_common.cuh"
#include "../../include/gdn_debug.h"

namespace gdn {

extern float *g_debug_dump;
extern long long *g_prof_buf;
void *g_debug_ring = nullptr;
int g_kernel_select = 0;
int g_stall_chunk = -1;
bool g_plain_launch = false;

namespace {

// 16 warps: TMA, MMA, group A (8 warps: two per TMEM lane quarter), group B
// (4 warps: one per quarter), 2 gate warps (workers) or converters (chains).
// Four warps per SM sub-partition leave 128 registers a thread (a chain's
// state threads hold 64 fp32 values).
constexpr int kThreads = 512;
constexpr int kGroup = 256, kGroupB = 128;
constexpr int kBarA = 1, kBarB = 2, kBarGate = 3, kBarConv = 4;   // named barriers
constexpr int kNG = 3;                    // gate buffers
constexpr int kNS = 3;                    // worker input stages
constexpr uint32_t kGateFloats = 9 * 64;
constexpr int kNSlot = 8;                 // ring slots per scan
// Flag words polled across SMs (a scan's slot sequence words, a scan's count
// of chunks taken out, the item counter) each get their own 128-byte line:
// sharing lines made the kernel up to 50 % slower depending on where the
// workspace landed.
constexpr int kFlagStride = 32;
static_assert(kNSlot <= kFlagStride, "a scan's slot words share its line");

// ring slot: P [64 x 64] and T2 [64 x 64] bf16 (128B-swizzled, token rows),
// -W^T [128 keys x 64 tokens] bf16 (128B-swizzled), then the gate block (fp32):
// e[64], gamma_end, 3 unused, gamma[64]
constexpr uint32_t kSlotP = 0, kSlotT2 = 8192, kSlotW = 16384, kSlotGates = 32768;
constexpr uint32_t kGateBlockBytes = 528, kSlotCopy = kSlotGates + kGateBlockBytes, kSlotBytes = 33792;
constexpr int kGamOff = 68;               // gamma's first float in the gate block

// shared memory (from a 1024-aligned base)
constexpr uint32_t kOffBar = 0;
// worker
constexpr uint32_t kWStage = 1024;                        // kNS x [kb0: Q|K][kb1: Q|K]
constexpr uint32_t kWStageBytes = 32768;
constexpr uint32_t kPTB = kWStage + kNS * kWStageBytes;   // 2 x [P | T1 | T2], 8 KB each
constexpr uint32_t kTBBytes = 24576;
constexpr uint32_t kPW = kPTB + 2 * kTBBytes;             // -W^T staging [128 keys][64 tokens]
constexpr uint32_t kPA = kPW + 16384;                     // fp32 [64][kLDA] solve buffer
constexpr uint32_t kPGates = kPA + 64 * kLDA * 4;
constexpr uint32_t kPGst = kPGates + kNG * kGateFloats * 4;   // the slot's gate block
constexpr uint32_t kPEnd = kPGst + 1024;
// chain
constexpr int kNVK = 2;                                   // V/K/Q stages
constexpr uint32_t kCStage = 1024;                        // kNVK x [V0 | V1 | K0 | K1 | Q0 | Q1]
constexpr uint32_t kCStageBytes = 49152;
constexpr uint32_t kCA = kCStage + kNVK * kCStageBytes;   // 2 ring-slot images
constexpr uint32_t kCABytes = kSlotBytes;
constexpr uint32_t kCO = kCA + 2 * kCABytes;              // 2 output tiles [dv block][64 tokens][64]
constexpr uint32_t kCEnd = kCO + 2 * 16384;
constexpr uint32_t kC8 = kCEnd;                           // fp8 inputs: staging of one chunk's v, k, q codes
constexpr uint32_t kCEnd8 = kC8 + 24576;
constexpr uint32_t kSmemBytes = (kPEnd > kCEnd8 ? kPEnd : kCEnd8);
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kPTB % 1024 == 0 && kTBBytes % 1024 == 0 && kPW % 1024 == 0 && kCA % 1024 == 0 &&
              kCABytes % 1024 == 0 && kCO % 1024 == 0 && kC8 % 1024 == 0 && kPGst % 16 == 0 &&
              kSlotCopy % 16 == 0 && kSlotCopy <= kSlotBytes,
              "tile alignment");

// TMEM columns
constexpr uint32_t kTD1 = 0, kTD3 = 256;                             // worker
constexpr uint32_t kTD = 0, kTS = 256, kTH = 384, kTUb = 448, kTUr = 480;   // chain: kTD = 2 x [O^T | U^T]
constexpr uint32_t kTmemCols = 512;

// Chunk-0 products of scan 0 can be dumped for debugging in builds with
// GDN_DEBUG_DUMP; production builds compile the dump code out.
#ifdef GDN_DEBUG_DUMP
constexpr bool kDbgOn = true;
#else
constexpr bool kDbgOn = false;
#endif

constexpr uint32_t kIdM1 = idesc_bf16(128, 64, false, false);   // [Q;K] K^T
constexpr uint32_t kIdM1f8 = idesc_e4m3(128, 64, false, false); // [Q;K] K^T on E4M3 codes
constexpr uint32_t kIdW = idesc_bf16(128, 64, true, false);     // K^T T1^T (A = K MN-major)
constexpr uint32_t kIdU1 = idesc_bf16(128, 64, true, false);    // V^T T2^T (A = V MN-major)
constexpr uint32_t kIdU2 = idesc_bf16(128, 64, false, true);    // H^T (-W^T) (A in TMEM, B MN-major)
constexpr uint32_t kIdO = idesc_bf16(128, 64, false, false);    // H^T Q'^T, U^T P^T (A in TMEM)
constexpr uint32_t kIdC = idesc_bf16(128, 128, false, true);    // Ubar^T K (A in TMEM)

struct PoolParams {
    const float *beta, *decay, *state_in;
    float *state_out;
    __nv_bfloat16 *o;
    uint8_t *ring;       // [n_scans][kNSlot] slots
    int *slot_seq;       // [n_scans][kFlagStride], first kNSlot used: chunk + 1 once the slot holds it, zeroed
    int *consumed;       // [n_scans][kFlagStride], first used: chunks the scan's chain has taken out, zeroed
    int *work;           // next item to hand out (own line), zeroed
    int *counters;       // bidi arrival counters [BH][n_chunks] of this launch's heads, zeroed
    int *err;            // device error word
    float *debug;        // optional: chunk-0 D and S of scan 0
    long long *trace;    // tracing builds: clock64 marks of scan 0 / worker 0
    int BH;              // heads in this launch
    int bh0;             // index of its first head in the tensors
    int BH_all;          // heads in the tensors (the reverse direction's state_out offset)
    int T, n_chunks, n_scans, n_items;
    int stall_chunk;     // testing: scan 0's chain waits for this chunk's slot without end (-1: never)
    // fp8 inputs (the FP8 kernel): q, k, v are E4M3 codes with one scale per head
    const float *q_scale, *k_scale, *v_scale;
};

struct Bars {
    // worker
    uint64_t it_full[kNS], st_full[kNS], st_empty[kNS], d1_full[2], d1_empty[2], tp_full[2], t_free[2];
    uint64_t d3_full, d3_empty;
    uint64_t g_full[kNG], g_empty[kNG];
    uint64_t cv_full[kNS];             // fp8: the stage's k tile widened to bf16
    // chain
    uint64_t vk_full[kNVK], vk_empty[kNVK], q_full[kNVK], a_full[2], a_empty[2];
    uint64_t du_full[2], do_full[2], d_empty[2], o_full[2];
    uint64_t u_full, s_full, h_full;
    uint64_t s8_full, s8_empty;        // fp8: the v, k code staging
    uint64_t q8_full, q8_empty;        // fp8: the q code staging
    uint64_t drain;
    float gscal[kNG][2];   // per gate buffer: G_end, factorised (1) or not (0)
    int gitem[kNG];        // per gate buffer: the item, or -1 after the last
    int sitem[kNS];        // per input stage: the item, or -1 after the last
    uint32_t tmem_slot;
    int abort_flag;
    int s_old;
    float s_wsum;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

struct Ctx {
    uint8_t *smem;
    uint32_t sbase;
    Bars *bars;
    volatile int *abort_flag;
    uint32_t tmem;
    int NC, T;
    // chain CTAs
    int scan, dir, bhl, bh;   // scan, its direction, head in this launch, head in the tensors
    uint8_t *ring;            // the scan's kNSlot slots
};

// An item's scan, direction, head (in the tensors), and chunk in scan order
// (items are handed out chunk-major: every scan's first chunk, then every
// scan's second, ...).
struct Item {
    int scan, dir, bh, ci, c;   // ci: scan-order position, c: chunk index in the sequence
};
__device__ __forceinline__ Item decode_item(const PoolParams &p, int k)
{
    Item it;
    it.ci = k / p.n_scans;
    it.scan = k - it.ci * p.n_scans;
    it.dir = it.scan >= p.BH ? 1 : 0;
    it.bh = p.bh0 + it.scan - it.dir * p.BH;
    it.c = it.dir ? p.n_chunks - 1 - it.ci : it.ci;
    return it;
}

template <int DIR>
__device__ __forceinline__ int chunk_of(const Ctx &x, int i) { return DIR ? (x.NC - 1 - i) : i; }
__device__ __forceinline__ float *gates_buf(const Ctx &x, int g)
{
    return reinterpret_cast<float *>(x.smem + kPGates) + g * kGateFloats;
}

// Tracing builds (-DGDN_TRACE): clock64() at role marks of scan 0's chain
// (rank 1) and of worker 0 (rank 0) for local steps kTr0 .. kTr0 + 7, stored at
// trace[(rank * 32 + mark) * 8 + step - kTr0].
__device__ __forceinline__ void tr(const PoolParams &p, int rank, int mark, int i)
{
#ifdef GDN_TRACE
    constexpr int kTr0 = 100;
    if (p.trace && blockIdx.x == (rank ? 0 : p.n_scans) && i >= kTr0 && i < kTr0 + 8)
        p.trace[(rank * 32 + mark) * 8 + i - kTr0] = (long long)clock64();
#else
    (void)p; (void)rank; (void)mark; (void)i;
#endif
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

__device__ __forceinline__ void st_release_gpu(int *addr, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_gpu(int *addr, int v)
{
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

// Bounded wait until a device-wide word reaches `target`; on timeout the error
// is recorded and the CTA's abort flag raised.  false on timeout or abort.
__device__ __forceinline__ bool wait_global(const int *word, int target, const Ctx &x, const PoolParams &p,
                                            int code)
{
    if (spin_global_at_least(word, target, x.abort_flag)) return true;
    if (!*x.abort_flag) atomicOr(p.err, code);
    *x.abort_flag = 1;
    return false;
}

// ------------------------------------------------------------------ fp8 inputs
// A chunk's q, k or v tile of E4M3 codes arrives by TMA as 64 token rows of
// 128 bytes (128B-swizzled, 8 KB); the tensor-core products take bf16, so 64
// threads widen it to scaled bf16 (x = scale * decode(code)) in the
// 128B-swizzled layout of the bf16 path: codes [0, 64) of each row into tile
// dst0, codes [64, 128) into dst1.

// 16 codes (one 16-byte chunk) times `scale`, as 8 packed bf16 pairs (the
// E4M3 to f16 widening is exact; one rounding, to bf16)
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 &c, float scale, uint32_t (&w)[8])
{
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __half2_raw hr =
                __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(words[i] >> (16 * h)), __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
            w[2 * i + h] = pack_bf16(f.x * scale, f.y * scale);
        }
}

// Thread t (of 64) takes the 16-code chunk t % 8 of rows t / 8 + 8 n.  Every
// thread reads its chunks before the group's barrier and writes after it, so
// a destination may overlap the source.  row_scale (optional): a factor per
// row, applied with scale.
__device__ __forceinline__ void e4m3_tile_to_bf16(const uint8_t *src, uint8_t *dst0, uint8_t *dst1, float scale,
                                                  int t, int bar_id, const float *row_scale = nullptr)
{
    const int j = t & 7, r0 = t >> 3, ph = r0 & 7;   // rows r0 + 8 n share the swizzle phase
    uint4 c[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) c[n] = *reinterpret_cast<const uint4 *>(src + (r0 + 8 * n) * 128 + ((j ^ ph) << 4));
    named_bar(bar_id, 64);
    uint8_t *d = (j >> 2) ? dst1 : dst0;
    const int m0 = 2 * (j & 3);   // the chunk's first 16-byte bf16 chunk in its 64-column tile
    const uint32_t o0 = (uint32_t)((m0 ^ ph) << 4), o1 = (uint32_t)(((m0 + 1) ^ ph) << 4);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        uint32_t w[8];
        e4m3x16_to_bf16(c[n], row_scale ? scale * row_scale[r0 + 8 * n] : scale, w);
        uint8_t *row = d + (r0 + 8 * n) * 128;
        *reinterpret_cast<uint4 *>(row + o0) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4 *>(row + o1) = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// Row r of a [64 tokens][128] bf16 tile held as two 128B-swizzled 64-column
// blocks 8 KB apart, times g, in place (one rounding).  The row's 16-byte
// chunks are visited in swizzle order, so 8 consecutive rows take 8 different
// bank groups.
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t w, float g)
{
    return pack_bf16(__uint_as_float(w << 16) * g, __uint_as_float(w & 0xffff0000u) * g);
}
__device__ __forceinline__ void scale_row_bf16(uint8_t *tile, int r, float g)
{
    uint4 w[16];   // every chunk loaded before the first store
#pragma unroll
    for (int m = 0; m < 16; ++m)
        w[m] = *reinterpret_cast<const uint4 *>(tile + (m >> 3) * 8192 + r * 128 + (((m & 7) ^ (r & 7)) << 4));
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        w[m].x = scale_bf16x2(w[m].x, g);
        w[m].y = scale_bf16x2(w[m].y, g);
        w[m].z = scale_bf16x2(w[m].z, g);
        w[m].w = scale_bf16x2(w[m].w, g);
        *reinterpret_cast<uint4 *>(tile + (m >> 3) * 8192 + r * 128 + (((m & 7) ^ (r & 7)) << 4)) = w[m];
    }
}

// ================================================================== workers

// TMA: hands out the items (one per input stage: published on it_full before
// its q, k tiles are loaded) and loads their q, k tiles; an item past the last
// one marks the end.
template <bool FP8>
__device__ __forceinline__ void worker_tma(const Ctx &x, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                                           const PoolParams &p)
{
    Bars &B = *x.bars;
    int issued = 0;
    for (int i = 0;; ++i) {
        const int s = i % kNS;
        if (i >= kNS && !wait_bar(&B.st_empty[s], ((i / kNS) + 1) & 1, x.abort_flag, p.err, 1)) break;
        const int k = atomicAdd(p.work, 1);
        if (k >= p.n_items) {
            B.sitem[s] = -1;
            mbar_arrive(&B.it_full[s]);
            mbar_arrive(&B.st_full[s]);
            break;
        }
        const Item it = decode_item(p, k);
        B.sitem[s] = k;
        mbar_arrive(&B.it_full[s]);
        uint8_t *st = x.smem + kWStage + s * kWStageBytes;
        if (FP8) {   // the E4M3 q, k tiles: [Q8; K8], the A operand of [Q;K] K^T on codes
            mbar_arrive_expect_tx(&B.st_full[s], 16384);
            tma_load_3d(st, tmQ, &B.st_full[s], 0, it.c * kC, it.bh);
            tma_load_3d(st + 8192, tmK, &B.st_full[s], 0, it.c * kC, it.bh);
        } else {
            mbar_arrive_expect_tx(&B.st_full[s], 32768);
            for (int kb = 0; kb < 2; ++kb) {
                tma_load_3d(st + kb * 16384, tmQ, &B.st_full[s], kb * 64, it.c * kC, it.bh);
                tma_load_3d(st + kb * 16384 + 8192, tmK, &B.st_full[s], kb * 64, it.c * kC, it.bh);
            }
        }
        issued = i + 1;
    }
    if (*x.abort_flag)
        for (int i = (issued > kNS ? issued - kNS : 0); i < issued; ++i) drain_copies(&B.st_full[i % kNS], (i / kNS) & 1);
}

// Gate warps (64 threads): the gates of each item in log2 form, as soon as the
// item is handed out: G (inclusive prefix sum of log2 a in scan order), gamma,
// b, b gamma, e = 2^(G_end - G), and the row/column factors of the decay ratios.
template <bool FP8>
__device__ __forceinline__ void worker_gates(const Ctx &x, const PoolParams &p, int gpt)
{
    Bars &B = *x.bars;
    const int lane = gpt & 31;
    for (int i = 0;; ++i) {
        const int s = i % kNS, gj = i % kNG;
        bool ok = wait_bar(&B.it_full[s], (i / kNS) & 1, x.abort_flag, p.err, 2);
        // both gate warps leave together: a thread whose wait gave up never
        // leaves the other waiting at the group's barrier
        if (named_bar_any(kBarGate, 64, !ok || *x.abort_flag)) break;
        const int k = B.sitem[s];
        if (FP8) {   // widen the stage's k codes to bf16 (for [P T1; T1] K) beside them
            if (k >= 0) {
                ok = wait_bar(&B.st_full[s], (i / kNS) & 1, x.abort_flag, p.err, 36);
                if (named_bar_any(kBarGate, 64, !ok || *x.abort_flag)) break;
                uint8_t *st = x.smem + kWStage + s * kWStageBytes;
                e4m3_tile_to_bf16(st + 8192, st + 16384, st + 24576, __ldg(p.k_scale + decode_item(p, k).bh), gpt,
                                  kBarGate);
                fence_proxy_async_smem();
                named_bar(kBarGate, 64);
            }
            if (gpt == 0) mbar_arrive(&B.cv_full[s]);   // (the end marker too)
        }
        if (i >= kNG) {
            ok = wait_bar(&B.g_empty[gj], ((i / kNG) + 1) & 1, x.abort_flag, p.err, 3);
            if (named_bar_any(kBarGate, 64, !ok || *x.abort_flag)) break;
        }
        if (k < 0) {   // past the last item: pass the end on
            if (gpt == 0) {
                B.gitem[gj] = -1;
                mbar_arrive(&B.g_full[gj]);
            }
            break;
        }
        const Item it = decode_item(p, k);
        const int dir = it.dir;
        float *gt = gates_buf(x, gj);
        // scan position gpt is token pp of the chunk; tokens past T are identity tokens
        const int pp = dir ? (63 - gpt) : gpt;
        const int t = it.c * kC + pp;
        float v = 0.f, bcur = 0.f;
        if (t < x.T) {
            v = fmaxf(log2f(__ldg(p.decay + (size_t)it.bh * x.T + t)), -120.f);   // decay below 2^-120 acts as 2^-120
            bcur = __ldg(p.beta + (size_t)it.bh * x.T + t);
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        if (gpt == 31) B.s_wsum = v;
        named_bar(kBarGate, 64);
        {
            const float G = (gpt >= 32) ? v + B.s_wsum : v;
            gt[gG * 64 + pp] = G;
            const float gam = exp2f(G);
            gt[gGam * 64 + pp] = gam;
            gt[gBet * 64 + pp] = bcur;
            gt[gBG * 64 + pp] = bcur * gam;
        }
        named_bar(kBarGate, 64);
        // references: scan positions 15 (first half), 47 (second half), 31 (boundary)
        const float R1 = gt[gG * 64 + (dir ? 48 : 15)];
        const float R2 = gt[gG * 64 + (dir ? 16 : 47)];
        const float Rm = gt[gG * 64 + (dir ? 32 : 31)];
        const float G0 = gt[gG * 64 + (dir ? 63 : 0)];
        const float G32 = gt[gG * 64 + (dir ? 31 : 32)];
        const float Gend = gt[gG * 64 + (dir ? 0 : 63)];
        // factorised decay products are exact while every factor is a normal float
        const bool fact = (G0 - R1) <= 120.f && (R1 - Rm) <= 120.f && (G32 - R2) <= 120.f &&
                          (R2 - Gend) <= 120.f;
        {
            const float G = gt[gG * 64 + gpt];
            const int lp = dir ? 63 - gpt : gpt;
            const float Rh = (lp >= 32) ? R2 : R1;
            gt[gEb * 64 + gpt] = exp2f(Gend - G);
            gt[gRA * 64 + gpt] = exp2f(G - Rh);
            gt[gCA * 64 + gpt] = exp2f(Rh - G);
            gt[gRB * 64 + gpt] = exp2f(G - Rm);
            gt[gCB * 64 + gpt] = exp2f(Rm - G);
            if (gpt == 0) {
                B.gscal[gj][0] = Gend;
                B.gscal[gj][1] = fact ? 1.f : 0.f;
                B.gitem[gj] = k;
            }
        }
        named_bar(kBarGate, 64);
        if (gpt == 0) mbar_arrive(&B.g_full[gj]);
    }
}

// MMA issue, per item j: W^T = K^T T1^T of item j once its solve is done,
// with [Q;K] K^T of item j + 2 beside it (its D1 buffer is free once item j's
// masks are read, which the solve follows).  The [Q;K] K^T products run two
// items ahead of the solver.
// [Q;K] K^T of item i (one thread; out of line, as it is issued from several
// places): 1 issued, 0 no such item (the end), -1 inputs not ready yet (only
// when !block), -2 abort.
__device__ __noinline__ int issue_qk(Bars *Bp, volatile int *abort_flag, int *err, uint32_t sbase, uint32_t tm,
                                     int i, bool block, bool fp8)
{
    Bars &B = *Bp;
    const int s = i % kNS, b1 = i & 1;
    if (!block && !(mbar_test_wait(&B.st_full[s], (i / kNS) & 1) &&
                    (i < 2 || mbar_test_wait(&B.d1_empty[b1], ((i >> 1) + 1) & 1))))
        return -1;
    if (!wait_bar(&B.st_full[s], (i / kNS) & 1, abort_flag, err, 4)) return -2;
    if (B.sitem[s] < 0) return 0;
    if (i >= 2 && !wait_bar(&B.d1_empty[b1], ((i >> 1) + 1) & 1, abort_flag, err, 5)) return -2;
    const uint32_t sQK = sbase + kWStage + s * kWStageBytes;
    const uint64_t a = sw128_desc(sQK, 16, 1024), b = sw128_desc(sQK + 8192, 16, 1024);
    tc_fence_after();
    if (fp8) {   // [Q8; K8] K8^T: one 128-byte row of codes per token, 32 codes per K step
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mma_f8(tm + kTD1 + 64 * b1, a + (uint64_t)(2 * k), b + (uint64_t)(2 * k), kIdM1f8, k > 0 ? 1u : 0u);
    } else {
        mma_run<4, 2, 2>(tm + kTD1 + 64 * b1, a, b, kIdM1, false);
        mma_run<4, 2, 2>(tm + kTD1 + 64 * b1, a + 1024, b + 1024, kIdM1, true);
    }
    mma_commit(&B.d1_full[b1]);
    return 1;
}

template <bool FP8>
__device__ __forceinline__ void worker_mma(const Ctx &x, const PoolParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    int last = -1;   // the number of items, once the end has been seen
    int next = 0;    // next item whose [Q;K] K^T is to be issued
    auto step_m1 = [&](bool block) -> bool {   // false on abort
        if (last >= 0) return true;
        const int r = issue_qk(x.bars, x.abort_flag, p.err, x.sbase, tm, next, block, FP8);
        if (r == -2) return false;
        if (r == 0) last = next;
        if (r == 1) {
            tr(p, 0, 16, next);
            ++next;
        }
        return true;
    };
    bool ok = step_m1(true) && step_m1(true);
    for (int j = 0; ok && (last < 0 || j < last); ++j) {
        const int bj = j & 1;
        if (!wait_bar(&B.tp_full[bj], (j >> 1) & 1, x.abort_flag, p.err, 6)) break;
        // item j + 2's [Q;K] K^T now if its tiles are in, else after W^T
        if (next == j + 2 && !step_m1(false)) break;
        if (j >= 1 && !wait_bar(&B.d3_empty, (j - 1) & 1, x.abort_flag, p.err, 9)) break;
        // fp8: K widened to bf16 by the gate warps
        if (FP8 && !wait_bar(&B.cv_full[j % kNS], (j / kNS) & 1, x.abort_flag, p.err, 41)) break;
        tc_fence_after();
        // W^T = K^T T1^T: A = K [token][dk] MN-major, dk groups 16 KB apart in the
        // stage (fp8: 8 KB apart, beside the codes); B = T1 (K-major)
        {
            const uint32_t st = x.sbase + kWStage + (j % kNS) * kWStageBytes;
            const uint32_t tb = x.sbase + kPTB + bj * kTBBytes;
            mma_run<4, 128, 2>(tm + kTD3,
                               FP8 ? sw128_desc(st + 16384, 8192, 1024) : sw128_desc(st + 8192, 16384, 1024),
                               sw128_desc(tb + 8192, 16, 1024), kIdW, false);
        }
        mma_commit(&B.d3_full);
        mma_commit(&B.t_free[bj]);
        tr(p, 0, 18, j);
        if (next == j + 2 && !step_m1(true)) break;
    }
    drain_mmas(B);
}

// Mask epilogue of this warp's 32 physical columns [32 hf, +32) of one row of
// [Q;K] K^T, read from TMEM in one load.  Rows 0-63 (TMEM quarters 0-1) give
// P row r: j kept at or before r in scan order; rows 64-127 give A row r,
// written in scan order: j strictly before r, times b_r.  The decay ratio
// 2^(G_r - G_j) is a product of a row and a column factor when the chunk's
// factors are all normal floats (`fact`), else one exp2 of the difference.
__device__ __forceinline__ void mask_rows(uint32_t taddr, const float *gt, float *As, uint8_t *sP, int qd,
                                          int lane, int hf, bool fact, int dir, float sc_p, float sc_a)
{
    const int r = (qd & 1) * 32 + lane;                  // physical token row
    const int lr = dir ? 63 - r : r;                     // its scan position
    const bool pm = qd < 2;                              // P (else A)
    const bool useB = lr >= 32 && (dir ? (hf == 1) : (hf == 0));   // cross-half pairs
    const float *cf = gt + (useB ? gCB : gCA) * 64 + 32 * hf;
    // sc_p, sc_a: the input scales of the [Q;K] K^T rows (fp8 codes), else 1
    const float br = pm ? sc_p : sc_a * gt[gBet * 64 + r];
    const float rf = br * gt[(useB ? gRB : gRA) * 64 + r];
    const int j0 = 32 * hf;                              // physical column of xv[0]
    float xv[32];
    tmem_ld32(taddr, xv);
    tmem_wait_ld();
    // kept columns: u in [lo, hi)
    const int rel = r - j0;
    const int lo = dir ? (pm ? rel : rel + 1) : 0;
    const int hi = dir ? 32 : (pm ? rel + 1 : rel);
    if (fact) {
#pragma unroll
        for (int u = 0; u < 32; ++u) xv[u] = (u >= lo && u < hi) ? xv[u] * (rf * cf[u]) : 0.f;
    } else {
        const float Gr = gt[gG * 64 + r];
#pragma unroll
        for (int u = 0; u < 32; ++u)
            xv[u] = (u >= lo && u < hi) ? xv[u] * (br * exp2f(Gr - gt[gG * 64 + j0 + u])) : 0.f;
    }
    if (pm) {
        store_half_row_bf16(sP, r, hf, xv);
    } else if (dir) {   // scan-order columns 63 - j run backwards
        float4 *dst = reinterpret_cast<float4 *>(As + lr * kLDA + 32 - j0);
#pragma unroll
        for (int m = 0; m < 8; ++m)
            dst[m] = make_float4(xv[31 - 4 * m], xv[30 - 4 * m], xv[29 - 4 * m], xv[28 - 4 * m]);
    } else {
        float4 *dst = reinterpret_cast<float4 *>(As + lr * kLDA + j0);
#pragma unroll
        for (int m = 0; m < 8; ++m) dst[m] = make_float4(xv[4 * m], xv[4 * m + 1], xv[4 * m + 2], xv[4 * m + 3]);
    }
}

// Solver group (8 warps; warp w reads TMEM lane quarter qd = w % 4 and columns
// [32 hf, +32) of each row it owns): per item, the masks of [Q;K] K^T, then
// T = (I + A)^-1 written as T1 = T diag(b gamma) and T2 = T diag(b).
template <bool FP8>
__device__ __forceinline__ void worker_solver(const Ctx &x, const PoolParams &p, int pt, int qd, int hf)
{
    Bars &B = *x.bars;
    const int lane = pt & 31;
    float *As = reinterpret_cast<float *>(x.smem + kPA);
    const uint32_t tm_lane = (uint32_t)(qd * 32) << 16;
#pragma unroll 1
    for (int i = 0;; ++i) {
        const int b = i & 1, gi = i % kNG;
        const float *gt = gates_buf(x, gi);
        uint8_t *tb = x.smem + kPTB + b * kTBBytes;   // [P | T1 | T2]
        if (pt == 0) tr(p, 0, 0, i);
        wait_bar(&B.g_full[gi], (i / kNG) & 1, x.abort_flag, p.err, 10);
        const int k = B.gitem[gi];
        if (named_bar_any(kBarA, kGroup, *x.abort_flag || k < 0)) return;
        const Item itk = decode_item(p, k);
        const int dir = itk.dir;
        float sc_p = 1.f, sc_a = 1.f;   // fp8: [Q;K] K^T was formed on the codes
        if (FP8) {
            const float sk = __ldg(p.k_scale + itk.bh);
            sc_p = __ldg(p.q_scale + itk.bh) * sk;
            sc_a = sk * sk;
        }
        const bool fact = B.gscal[gi][1] != 0.f;
        wait_bar(&B.d1_full[b], (i >> 1) & 1, x.abort_flag, p.err, 11);
        // this buffer's P, T1, T2 must be done with (item i - 2: its W^T product and its ring copies)
        if (i >= 2) wait_bar(&B.t_free[b], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 13);
        if (pt == 0) tr(p, 0, 1, i);
        tc_fence_after();
        mask_rows(x.tmem + tm_lane + kTD1 + 64 * b + 32 * hf, gt, As, tb, qd, lane, hf, fact, dir, sc_p, sc_a);
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarA, kGroup, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.d1_empty[b]);
        if (pt == 0) tr(p, 0, 2, i);
        solve_diag_blocks<kBarA, kGroup>(As, gt, tb + 8192, tb + 16384, nullptr, dir, pt);
        if (pt == 0) tr(p, 0, 4, i);
        solve_off_diag_strips(As, gt, tb + 8192, tb + 16384, dir, pt);
        fence_proxy_async_smem();
        if (named_bar_any(kBarA, kGroup, *x.abort_flag)) return;
        if (pt == 0) mbar_arrive(&B.tp_full[b]);
        if (pt == 0) tr(p, 0, 5, i);
    }
}

// Finisher group (4 warps, warp w reads TMEM lane quarter qd = w % 4): per item,
// -W^T into its staging tile and the gate block, then the item's slot in its
// scan's ring: P, T2, -W^T and the gate block by bulk copies, published to the
// chain once they have completed (at the start of the next item).
template <bool FP8>
__device__ __forceinline__ void worker_finisher(const Ctx &x, const PoolParams &p, int ft, int qd)
{
    Bars &B = *x.bars;
    const int lane = ft & 31;
    const uint32_t tm_lane = (uint32_t)(qd * 32) << 16;
    int pend_scan = -1, pend_c = 0, pend_b = -1;   // leader: the item whose ring copies are in flight
    // leader: once the copies have read their sources, the P / T2 buffer goes back
    // to the solver (the staging tiles are free); once they have completed, the
    // slot is published to the scan's chain
    auto publish = [&]() {
        if (pend_scan < 0) return;
        bulk_wait_read0();
        mbar_arrive(&B.t_free[pend_b]);
        bulk_wait0();
        fence_proxy_async_global();
        st_release_gpu(p.slot_seq + (size_t)pend_scan * kFlagStride + pend_c % kNSlot, pend_c + 1);
        pend_scan = -1;
    };
#pragma unroll 1
    for (int i = 0;; ++i) {
        const int b = i & 1, gi = i % kNG;
        const float *gt = gates_buf(x, gi);
        wait_bar(&B.g_full[gi], (i / kNG) & 1, x.abort_flag, p.err, 14);
        const int k = B.gitem[gi];
        // the previous item's copies complete before the staging tiles are rewritten
        if (ft == 0) publish();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag || k < 0)) break;
        const Item it = decode_item(p, k);

        // ---- -W^T: row n = key n, columns = the chunk's tokens
        if (ft == 0) tr(p, 0, 11, i);
        wait_bar(&B.d3_full, i & 1, x.abort_flag, p.err, 18);
        tc_fence_after();
        {
            const int n = 32 * qd + lane;
            float v[32];
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                tmem_ld32(x.tmem + tm_lane + kTD3 + 32 * h2, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = -v[e];
                store_half_row_bf16(x.smem + kPW, n, h2, v);
            }
        }
        // gate block: e, gamma_end, gamma
        if (ft < 16) {
            *reinterpret_cast<float4 *>(x.smem + kPGst + 16 * ft) =
                *reinterpret_cast<const float4 *>(gt + gEb * 64 + 4 * ft);
        } else if (ft == 16) {
            *reinterpret_cast<float4 *>(x.smem + kPGst + 256) =
                make_float4(exp2f(B.gscal[gi][0]), 0.f, 0.f, 0.f);
        } else if (ft < 33) {
            *reinterpret_cast<float4 *>(x.smem + kPGst + 4 * kGamOff + 16 * (ft - 17)) =
                *reinterpret_cast<const float4 *>(gt + gGam * 64 + 4 * (ft - 17));
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (ft == 0) {
            mbar_arrive(&B.d3_empty);
            mbar_arrive(&B.st_empty[i % kNS]);
            mbar_arrive(&B.g_empty[gi]);
        }
        if (ft == 0) tr(p, 0, 12, i);

        // ---- the item's slot (bulk copies, published at the start of the next item)
        if (ft == 0) {
            // the slot's previous chunk must have been taken out by the chain
            if (it.ci < kNSlot || wait_global(p.consumed + (size_t)it.scan * kFlagStride, it.ci - kNSlot + 1, x, p, 64)) {
                uint8_t *slot = p.ring + ((size_t)it.scan * kNSlot + it.ci % kNSlot) * kSlotBytes;
                const uint8_t *tb = x.smem + kPTB + b * kTBBytes;
                bulk_store(slot + kSlotP, tb, 8192);
                bulk_store(slot + kSlotT2, tb + 16384, 8192);
                bulk_store(slot + kSlotW, x.smem + kPW, 16384);
                bulk_store(slot + kSlotGates, x.smem + kPGst, kGateBlockBytes);
                bulk_commit();
                pend_scan = it.scan;
                pend_c = it.ci;
                pend_b = b;
            }
            tr(p, 0, 13, i);
        }
    }
    if (ft == 0) {
        if (!*x.abort_flag) publish();
        bulk_wait0();
    }
}

// ================================================================== chains

template <int DIR, bool FP8>
__device__ __forceinline__ void chain_tma(const Ctx &x, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                                          const CUtensorMap *tmV, const PoolParams &p)
{
    Bars &B = *x.bars;
    int vk_issued = 0, q_issued = 0, a_issued = 0;
    const int *seq = p.slot_seq + (size_t)x.scan * kFlagStride;
    for (int i = 0; i < x.NC; ++i) {
        const int st = i % kNVK, ab = i & 1, s = i % kNSlot;
        const int c = chunk_of<DIR>(x, i);
        if (FP8) {   // the E4M3 v, k tiles, and apart from them the q tile, into the staging
            // (widened into the stage by the converters; q waits for the slot's gamma)
            if (i >= 1 && !wait_bar(&B.s8_empty, (i - 1) & 1, x.abort_flag, p.err, 37)) break;
            mbar_arrive_expect_tx(&B.s8_full, 16384);
            tma_load_3d(x.smem + kC8, tmV, &B.s8_full, 0, c * kC, x.bh);
            tma_load_3d(x.smem + kC8 + 8192, tmK, &B.s8_full, 0, c * kC, x.bh);
            vk_issued = i + 1;
            if (i >= 1 && !wait_bar(&B.q8_empty, (i - 1) & 1, x.abort_flag, p.err, 43)) break;
            mbar_arrive_expect_tx(&B.q8_full, 8192);
            tma_load_3d(x.smem + kC8 + 16384, tmQ, &B.q8_full, 0, c * kC, x.bh);
            q_issued = i + 1;
        } else {
            if (i >= kNVK && !wait_bar(&B.vk_empty[st], ((i / kNVK) + 1) & 1, x.abort_flag, p.err, 21)) break;
            uint8_t *sv = x.smem + kCStage + st * kCStageBytes;
            mbar_arrive_expect_tx(&B.vk_full[st], 49152);
            tma_load_3d(sv, tmV, &B.vk_full[st], 0, c * kC, x.bh);
            tma_load_3d(sv + 8192, tmV, &B.vk_full[st], 64, c * kC, x.bh);
            tma_load_3d(sv + 16384, tmK, &B.vk_full[st], 0, c * kC, x.bh);
            tma_load_3d(sv + 24576, tmK, &B.vk_full[st], 64, c * kC, x.bh);
            tma_load_3d(sv + 32768, tmQ, &B.vk_full[st], 0, c * kC, x.bh);
            tma_load_3d(sv + 40960, tmQ, &B.vk_full[st], 64, c * kC, x.bh);
        }
        vk_issued = i + 1;
        if (i >= 2 && !wait_bar(&B.a_empty[ab], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 22)) break;
        tr(p, 1, 0, i);
        const int want = (x.scan == 0 && i == p.stall_chunk) ? INT_MAX : i + 1;
        if (!wait_global(seq + s, want, x, p, 65)) break;
        tr(p, 1, 1, i);
        fence_proxy_async_global();
        const uint8_t *slot = x.ring + (size_t)s * kSlotBytes;
        uint8_t *dst = x.smem + kCA + ab * kCABytes;
        mbar_arrive_expect_tx(&B.a_full[ab], kSlotCopy);
        bulk_load(dst, slot, 16384, &B.a_full[ab]);
        bulk_load(dst + 16384, slot + 16384, 16384, &B.a_full[ab]);
        bulk_load(dst + kSlotGates, slot + kSlotGates, kGateBlockBytes, &B.a_full[ab]);
        a_issued = i + 1;
    }
    if (*x.abort_flag) {
        if (FP8) {   // one load of each staging in flight at most
            if (vk_issued > 0) drain_copies(&B.s8_full, (vk_issued - 1) & 1);
            if (q_issued > 0) drain_copies(&B.q8_full, (q_issued - 1) & 1);
        } else {
            for (int i = (vk_issued > kNVK ? vk_issued - kNVK : 0); i < vk_issued; ++i)
                drain_copies(&B.vk_full[i % kNVK], (i / kNVK) & 1);
        }
        for (int i = (a_issued > 2 ? a_issued - 2 : 0); i < a_issued; ++i) drain_copies(&B.a_full[i & 1], (i >> 1) & 1);
    }
}

// Converters (2 warps): per chunk, Q' = diag(gamma) Q in the stage (the B
// operand of H^T Q'^T; gamma comes with the ring slot); with fp8 inputs, the
// staged E4M3 v, k tiles widened to scaled bf16 into the stage first (their
// staging then takes the next chunk's codes), and q widened with its scale
// times gamma.
template <bool FP8>
__device__ __forceinline__ void chain_convert(const Ctx &x, const PoolParams &p, int t)
{
    Bars &B = *x.bars;
    const float sv = FP8 ? __ldg(p.v_scale + x.bh) : 1.f, sk = FP8 ? __ldg(p.k_scale + x.bh) : 1.f;
    const float sq = FP8 ? __ldg(p.q_scale + x.bh) : 1.f;
#pragma unroll 1
    for (int i = 0; i < x.NC; ++i) {
        const int st = i % kNVK, ab = i & 1;
        uint8_t *stage = x.smem + kCStage + st * kCStageBytes;   // [V0 | V1 | K0 | K1 | Q0 | Q1]
        bool ok = true;
        if (FP8) {
            if (t == 0) {
                ok = wait_bar(&B.s8_full, i & 1, x.abort_flag, p.err, 38);
                if (ok && i >= kNVK) ok = wait_bar(&B.vk_empty[st], ((i / kNVK) + 1) & 1, x.abort_flag, p.err, 39);
            }
            if (named_bar_any(kBarConv, 64, !ok || *x.abort_flag)) break;
#pragma unroll 1
            for (int rd = 0; rd < 2; ++rd)
                e4m3_tile_to_bf16(x.smem + kC8 + 8192 * rd, stage + 16384 * rd, stage + 16384 * rd + 8192,
                                  rd ? sk : sv, t, kBarConv);
            fence_proxy_async_smem();
            named_bar(kBarConv, 64);
            if (t == 0) {
                mbar_arrive(&B.s8_empty);   // the staging may take the next chunk's v, k codes
                mbar_arrive(&B.vk_full[st]);
                ok = wait_bar(&B.q8_full, i & 1, x.abort_flag, p.err, 44);
            }
        } else if (t == 0) {
            ok = wait_bar(&B.vk_full[st], (i / kNVK) & 1, x.abort_flag, p.err, 39);
        }
        if (t == 0 && ok) ok = wait_bar(&B.a_full[ab], (i >> 1) & 1, x.abort_flag, p.err, 40);
        if (named_bar_any(kBarConv, 64, !ok || *x.abort_flag)) break;
        const float *gam = reinterpret_cast<const float *>(x.smem + kCA + ab * kCABytes + kSlotGates) + kGamOff;
        if (FP8) e4m3_tile_to_bf16(x.smem + kC8 + 16384, stage + 32768, stage + 40960, sq, t, kBarConv, gam);
        else scale_row_bf16(stage + 32768, t, gam[t]);
        fence_proxy_async_smem();
        named_bar(kBarConv, 64);
        if (t == 0) {
            if (FP8) mbar_arrive(&B.q8_empty);   // the q staging may take the next chunk's codes
            mbar_arrive(&B.q_full[st]);
        }
    }
}

// MMA issue, per chunk: U^T (its state-free part first, then the product with
// H^T), H^T Q'^T (while H^T is still the previous state), S = Ubar^T K once the
// state group has formed Ubar^T, then U^T P^T (off the state's path).
__device__ __forceinline__ void chain_mma(const Ctx &x, const PoolParams &p)
{
    Bars &B = *x.bars;
    const uint32_t tm = x.tmem;
    for (int i = 0; i < x.NC; ++i) {
        const int st = i % kNVK, ab = i & 1, db = i & 1;
        if (!wait_bar(&B.vk_full[st], (i / kNVK) & 1, x.abort_flag, p.err, 24)) break;
        if (!wait_bar(&B.a_full[ab], (i >> 1) & 1, x.abort_flag, p.err, 25)) break;
        // the slot's data has landed (the bulk copy that read it completed): it
        // may be refilled.  A relaxed store: no write of this thread needs
        // ordering before it, and a release here cost ~1k cycles a chunk.
        st_relaxed_gpu(p.consumed + (size_t)x.scan * kFlagStride, i + 1);
        tr(p, 1, 2, i);
        if (i >= 2 && !wait_bar(&B.d_empty[db], ((i >> 1) + 1) & 1, x.abort_flag, p.err, 26)) break;
        tr(p, 1, 3, i);
        const uint32_t sv = x.sbase + kCStage + st * kCStageBytes;
        const uint32_t sa = x.sbase + kCA + ab * kCABytes;
        const uint32_t dO = tm + kTD + 128 * db, dU = dO + 64;
        tc_fence_after();
        // U^T = V^T T2^T: A = V (MN-major, dv groups 8 KB apart), B = T2 (K-major)
        mma_run<4, 128, 2>(dU, sw128_desc(sv, 8192, 1024), sw128_desc(sa + kSlotT2, 16, 1024), kIdU1, false);
        if (!wait_bar(&B.h_full, i & 1, x.abort_flag, p.err, 27)) break;
        tr(p, 1, 4, i);
        tc_fence_after();
        // U^T += H^T (-W^T): A = H^T (bf16 in TMEM), B = -W^T [key][token] (MN-major)
        {
            const uint64_t dW = sw128_desc(sa + kSlotW, 8192, 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k) mma_bf16_ta(dU, tm + kTH + 8 * k, dW + (uint64_t)(k * 128), kIdU2, 1u);
        }
        mma_commit(&B.du_full[db]);
        // O^T = H^T Q'^T: B = Q' [token][dk] (K-major, key blocks 8 KB apart)
        if (!wait_bar(&B.q_full[st], (i / kNVK) & 1, x.abort_flag, p.err, 42)) break;
        tc_fence_after();
        {
            const uint64_t dQ = sw128_desc(sv + 32768, 16, 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ta(dO, tm + kTH + 8 * k, dQ + (uint64_t)((k >> 2) * 512 + (k & 3) * 2), kIdO,
                            k > 0 ? 1u : 0u);
        }
        if (!wait_bar(&B.u_full, i & 1, x.abort_flag, p.err, 28)) break;
        tr(p, 1, 5, i);
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
        // O^T += U^T P^T: A = U^T (bf16 in TMEM), B = P (K-major)
        {
            const uint64_t dP = sw128_desc(sa + kSlotP, 16, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_bf16_ta(dO, tm + kTUr + 8 * k, dP + (uint64_t)(2 * k), kIdO, 1u);
        }
        mma_commit(&B.do_full[db]);
        mma_commit(&B.a_empty[ab]);
    }
    drain_mmas(B);
}

// State group (8 warps): H^T in fp32 registers, thread (quarter q, half h) holds
// row d = 32 q + lane, key columns [64 h, +64).  U epilogue: tokens [32 h, +32)
// of U^T into U^T and, scaled by e, Ubar^T (both bf16, TMEM); state epilogue:
// H^T <- gamma_end H^T + S into registers and its bf16 copy into TMEM.
template <int DIR>
__device__ __forceinline__ void chain_state(const Ctx &x, const PoolParams &p, int ct, int q, int h)
{
    Bars &B = *x.bars;
    const int lane = ct & 31, d = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const bool dbg = kDbgOn && p.debug != nullptr && x.scan == 0;
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
        wait_bar(&B.du_full[db], (i >> 1) & 1, x.abort_flag, p.err, 31);
        if (ct == 0) tr(p, 1, 8, i);
        tc_fence_after();
        {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                float u[16];
                uint32_t we[8], wr[8];
                tmem_ld16(x.tmem + tl + kTD + 128 * db + 64 + 32 * h + 16 * h2, u);
                tmem_wait_ld();
                if (dbg && i == 0)
                    for (int j = 0; j < 16; ++j) p.debug[d * 128 + 64 + 32 * h + 16 * h2 + j] = u[j];
                const float4 *e4 = reinterpret_cast<const float4 *>(eg + 32 * h + 16 * h2);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 ev = e4[m];
                    we[2 * m] = pack_bf16(u[4 * m] * ev.x, u[4 * m + 1] * ev.y);
                    we[2 * m + 1] = pack_bf16(u[4 * m + 2] * ev.z, u[4 * m + 3] * ev.w);
                    wr[2 * m] = pack_bf16(u[4 * m], u[4 * m + 1]);
                    wr[2 * m + 1] = pack_bf16(u[4 * m + 2], u[4 * m + 3]);
                }
                tmem_st8(x.tmem + tl + kTUb + 16 * h + 8 * h2, we);
                tmem_st8(x.tmem + tl + kTUr + 16 * h + 8 * h2, wr);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        if (named_bar_any(kBarA, kGroup, *x.abort_flag)) return;
        if (ct == 0) {
            mbar_arrive(&B.u_full);
            mbar_arrive(&B.d_empty[db]);
        }
        if (ct == 0) tr(p, 1, 9, i);
        // ---- H^T <- gamma_end H^T + S
        wait_bar(&B.s_full, i & 1, x.abort_flag, p.err, 32);
        if (ct == 0) tr(p, 1, 10, i);
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
        if (ct == 0) tr(p, 1, 11, i);
    }
    if (p.state_out) {
        float *so = p.state_out + ((size_t)DIR * p.BH_all + x.bh) * kDK * 128 + (size_t)(64 * h) * 128 + d;
#pragma unroll
        for (int j = 0; j < 64; ++j) so[(size_t)j * 128] = hs[j];
    }
}

// Output group (4 warps): thread (quarter q) owns column d = 32 q + lane of each
// chunk's O tile.  A tile with no partial to add (causal calls, and a
// bidirectional tile's first writer) is written straight to o, one 2-byte
// store per token (a warp instruction covers 64 contiguous bytes of a row:
// two whole sectors); a first writer then publishes its bf16 partial on the
// tile's counter, after the group's barrier, with one thread's release
// (cumulative: it covers the stores the barrier ordered before it).  The
// second writer loads that partial by TMA (requested a chunk ahead) into a
// 128B-swizzled staging tile ([dv block][token] rows, the TMA layout of o),
// adds its fp32 partial, rounds once and stores the tile with TMA.
template <int DIR>
__device__ __forceinline__ void chain_out(const Ctx &x, const PoolParams &p, const CUtensorMap *tmO, int ot, int q)
{
    Bars &B = *x.bars;
    const int lane = ot & 31, d = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const bool lead = ot == 0;
    const bool dbg = kDbgOn && p.debug != nullptr && x.scan == 0;
    // this thread's column in a staging tile: dv block d / 64, column d % 64
    const uint32_t dblk = (uint32_t)(d >> 6) * 8192u;
    __nv_bfloat16 *col = p.o + (size_t)x.bh * x.T * 128 + d;   // o[bh][t][d] at col + 128 t
    int nload0 = 0, nload1 = 0;       // partial loads waited for, per staging tile
    int nissued0 = 0, nissued1 = 0;   // leader: partial loads issued, per staging tile
    int loaded_ahead = -1;            // leader: the chunk whose partial load is already in flight
    int pending = -1;                 // a first writer's tile published at the next chunk's first barrier
    const bool bidi = p.counters != nullptr;
    // every CTA is resident: the forward scan reaches the first half of the
    // chunks first, the reverse scan the second half
    auto first_of = [&](int c) { return DIR == ((2 * c < x.NC) ? 0 : 1); };
    auto counter = [&](int c) { return p.counters + (size_t)x.bhl * x.NC + c; };
    auto release_add = [&](int c) {
        asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(counter(c)) : "memory");
    };
    auto load_partial = [&](int c, int ob) {
        uint8_t *stg = x.smem + kCO + ob * 16384;
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&B.o_full[ob], 16384);
        if (ob) ++nissued1; else ++nissued0;
        tma_load_3d(stg, tmO, &B.o_full[ob], 0, c * kC, x.bh);
        tma_load_3d(stg + 8192, tmO, &B.o_full[ob], 64, c * kC, x.bh);
    };
#pragma unroll 1
    for (int i = 0; i < x.NC; ++i) {
        const int db = i & 1, ob = i & 1, c = chunk_of<DIR>(x, i);
        uint8_t *stg = x.smem + kCO + ob * 16384;
        const bool first = !bidi || first_of(c);
        if (!first && lead && loaded_ahead != i) {
            if (wait_global(counter(c), 1, x, p, 32)) {
                bulk_wait_read1();   // the staging tile's previous store has read it
                load_partial(c, ob);
            }
        }
        wait_bar(&B.do_full[db], (i >> 1) & 1, x.abort_flag, p.err, 33);
        // the staging tile's store of two chunks ago must have read it before it is rewritten
        if (lead && !first) bulk_wait_read1();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (pending >= 0) {   // the previous chunk's stores: every thread's were issued before the barrier
            if (lead) release_add(pending);
            pending = -1;
        }
        if (!first) {
            int &nl = ob ? nload1 : nload0;
            wait_bar(&B.o_full[ob], nl & 1, x.abort_flag, p.err, 35);
            ++nl;
        }
        tc_fence_after();
        __nv_bfloat16 *orow = col + (size_t)c * kC * 128;
        const int n = (x.T - c * kC) < kC ? (x.T - c * kC) : kC;   // the chunk's tokens (ragged tail)
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
            float v[32];
            tmem_ld32(x.tmem + tl + kTD + 128 * db + 32 * h2, v);
            tmem_wait_ld();
            if (dbg && i == 0)
                for (int j = 0; j < 32; ++j) p.debug[d * 128 + 32 * h2 + j] = v[j];
            if (first) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * h2 + j < n) orow[(size_t)(32 * h2 + j) * 128] = __float2bfloat16_rn(v[j]);
            } else {   // the first writer's partial: every load before the first store
                __nv_bfloat16 pv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    pv[j] = *reinterpret_cast<const __nv_bfloat16 *>(stg + dblk + sw128_off(32 * h2 + j, d & 63));
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    *reinterpret_cast<__nv_bfloat16 *>(stg + dblk + sw128_off(32 * h2 + j, d & 63)) =
                        __float2bfloat16_rn(v[j] + __bfloat162float(pv[j]));
            }
        }
        tc_fence_before();
        if (!first) fence_proxy_async_smem();
        if (named_bar_any(kBarB, kGroupB, *x.abort_flag)) break;
        if (lead) {
            mbar_arrive(&B.d_empty[db]);
            if (!first) {
                tma_store_3d(tmO, stg, 0, c * kC, x.bh);
                tma_store_3d(tmO, stg + 8192, 64, c * kC, x.bh);
                bulk_commit();
            }
        }
        if (bidi && first) {
            // published at the next chunk when that is a first-writer chunk too
            // (it does not wait for the other scan), else now
            if (i + 1 < x.NC && first_of(chunk_of<DIR>(x, i + 1))) pending = c;
            else if (lead) release_add(c);
        }
        // request the next tile's partial now if its first writer is done
        if (lead && bidi && i + 1 < x.NC) {
            const int cn = chunk_of<DIR>(x, i + 1);
            if (!first_of(cn)) {
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
    if (lead) {
        bulk_wait0();   // every store performed before the CTA exits
        for (int k = nload0; k < nissued0; ++k) drain_copies(&B.o_full[0], k & 1);   // after an abort
        for (int k = nload1; k < nissued1; ++k) drain_copies(&B.o_full[1], k & 1);
        if (pending >= 0 && !*x.abort_flag) release_add(pending);
    }
}

// ================================================================== kernel

// FP8: q, k, v are E4M3 codes, widened in shared memory (a separate
// instantiation, so that the bf16 kernel carries none of that code).
template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
gdn_chunk_pool_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      const PoolParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool chain = (int)blockIdx.x < p.n_scans;

    Ctx x;
    x.smem = smem;
    x.sbase = smem_u32(smem);
    x.bars = reinterpret_cast<Bars *>(smem + kOffBar);
    x.abort_flag = &x.bars->abort_flag;
    x.T = p.T;
    x.NC = p.n_chunks;
    x.scan = chain ? (int)blockIdx.x : 0;
    x.dir = x.scan >= p.BH ? 1 : 0;
    x.bhl = x.scan - x.dir * p.BH;
    x.bh = p.bh0 + x.bhl;
    x.ring = p.ring + (size_t)x.scan * kNSlot * kSlotBytes;
    Bars &B = *x.bars;

    if (tid == 0) {
        uint64_t *all = reinterpret_cast<uint64_t *>(&B);
        const int nbar = (int)(offsetof(Bars, gscal) / sizeof(uint64_t));
        for (int k = 0; k < nbar; ++k) mbar_init(&all[k], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&B.t_free[b], 2);    // W^T product done, ring copies read P and T2
            mbar_init(&B.a_empty[b], 2);   // the chunk's products done, state epilogue done
            mbar_init(&B.d_empty[b], 2);   // output epilogue, U epilogue
        }
        B.abort_flag = 0;
        fence_mbar_init();
        if (chain) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmO);
        } else {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
        }
    }
    if (warp == 0) {
        tmem_alloc(&B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (!chain) {
        float *As0 = reinterpret_cast<float *>(smem + kPA);
        for (int i = tid; i < 64 * kLDA; i += kThreads) As0[i] = 0.f;
        // T1, T2: the triangle the solve never writes stays zero throughout
        for (int b = 0; b < 2; ++b) {
            uint32_t *t1 = reinterpret_cast<uint32_t *>(smem + kPTB + b * kTBBytes + 8192);
            uint32_t *t2 = reinterpret_cast<uint32_t *>(smem + kPTB + b * kTBBytes + 16384);
            for (int i = tid; i < 8192 / 4; i += kThreads) t1[i] = t2[i] = 0u;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = B.tmem_slot;

    if (!chain) {
        if (warp == 0) {
            if (lane == 0) worker_tma<FP8>(x, &tmQ, &tmK, p);
        } else if (warp == 1) {
            if (lane == 0) worker_mma<FP8>(x, p);
        } else if (warp < 10) {
            worker_solver<FP8>(x, p, tid - 64, warp & 3, (warp - 2) >> 2);
        } else if (warp < 14) {
            worker_finisher<FP8>(x, p, tid - 320, warp & 3);
        } else {
            worker_gates<FP8>(x, p, tid - 448);
        }
    } else {
        if (warp == 0) {
            if (lane == 0) {
                if (x.dir) chain_tma<1, FP8>(x, &tmQ, &tmK, &tmV, p);
                else chain_tma<0, FP8>(x, &tmQ, &tmK, &tmV, p);
            }
        } else if (warp == 1) {
            if (lane == 0) chain_mma(x, p);
        } else if (warp < 10) {
            const int ct = tid - 64, q = warp & 3, h = (warp - 2) >> 2;
            if (x.dir) chain_state<1>(x, p, ct, q, h);
            else chain_state<0>(x, p, ct, q, h);
        } else if (warp < 14) {
            const int ot = tid - 320, q = warp & 3;
            if (x.dir) chain_out<1>(x, p, &tmO, ot, q);
            else chain_out<0>(x, p, &tmO, ot, q);
        } else {
            chain_convert<FP8>(x, p, tid - 448);
        }
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

// 3D map over a [BH, T, 128] bf16 tensor; box = 64 (inner) x 64 (tokens) x 1, 128B swizzle.
// 3D map over a [BH, T, 128] tensor of 2-byte (bf16) or 1-byte (E4M3 code)
// elements; box = 128 bytes (64 bf16 or 128 codes) x 64 tokens x 1, 128B swizzle.
bool make_map(CUtensorMap *m, const void *base, int T, int BH, bool bytes = false)
{
    EncodeTiledFn enc = get_encoder();
    if (!enc) return false;
    const cuuint64_t row = bytes ? 128 : 256;
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {row, (cuuint64_t)T * row};
    cuuint32_t box[3] = {bytes ? 128u : 64u, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct DevInfo {
    bool init = false;
    int sms = 0;
};

// Per device: the kernel's shared-memory attribute and the SM count.
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
        err = cudaFuncSetAttribute(gdn_chunk_pool_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kSmemAlloc);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(gdn_chunk_pool_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemAlloc);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        d.init = true;
    }
    *out = &d;
    return cudaSuccess;
}

// Workers kept beside the chains: a quarter of the SMs at least.
int min_workers(int sms) { return sms / 4 > 8 ? sms / 4 : 8; }

}  // namespace

bool chunk_pool_supported(const FwdArgs &a)
{
    return g_kernel_select != 1 && !a.fp32 && a.dk == kDK && a.dv == 128 && a.n_seg == 1 && a.seg0 == 0 &&
           a.seg_chunks == 0;
}

cudaError_t launch_chunk_pool(const FwdArgs &a, cudaStream_t stream, const float *q_scale, const float *k_scale,
                              const float *v_scale)
{
    CUtensorMap mq, mk, mv, mo;
    const int BH_all = a.B * a.H;
    const bool fp8 = q_scale != nullptr;
    if (!make_map(&mq, a.q, a.T, BH_all, fp8) || !make_map(&mk, a.k, a.T, BH_all, fp8) ||
        !make_map(&mv, a.v, a.T, BH_all, fp8) || !make_map(&mo, a.o, a.T, BH_all))
        return cudaErrorInvalidValue;
    DevInfo *info = nullptr;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const int dirs = a.bidi ? 2 : 1;
    const int n_chunks = (a.T + kC - 1) / kC;
    // heads per launch: every chain of a launch resident beside enough workers
    const int wave = (info->sms - min_workers(info->sms)) / dirs;
    if (wave < 1) return cudaErrorInvalidConfiguration;
    const int heads = BH_all < wave ? BH_all : wave;

    const size_t n_scans_max = (size_t)dirs * heads;
    const size_t ring_bytes = n_scans_max * kNSlot * kSlotBytes;
    const size_t flag_ints = (2 * n_scans_max + 1) * kFlagStride + (a.bidi ? (size_t)heads * n_chunks : 0);
    uint8_t *ws = nullptr;
    err = ws_alloc(reinterpret_cast<void **>(&ws), ring_bytes + flag_ints * sizeof(int), stream);
    if (err != cudaSuccess) return err;
    int *flags = reinterpret_cast<int *>(ws + ring_bytes);

    for (int h0 = 0; h0 < BH_all && err == cudaSuccess; h0 += heads) {
        PoolParams p;
        p.beta = a.beta; p.decay = a.decay; p.state_in = a.state_in; p.state_out = a.state_out;
        p.o = static_cast<__nv_bfloat16 *>(a.o);
        p.BH = BH_all - h0 < heads ? BH_all - h0 : heads;
        p.bh0 = h0;
        p.BH_all = BH_all;
        p.T = a.T;
        p.n_chunks = n_chunks;
        p.n_scans = dirs * p.BH;
        p.n_items = p.n_scans * n_chunks;
        p.debug = g_debug_dump;
        p.trace = g_prof_buf;
        p.ring = g_debug_ring ? static_cast<uint8_t *>(g_debug_ring) : ws;
        p.slot_seq = flags;
        p.consumed = flags + (size_t)p.n_scans * kFlagStride;
        p.work = p.consumed + (size_t)p.n_scans * kFlagStride;
        p.counters = a.bidi ? p.work + kFlagStride : nullptr;
        p.stall_chunk = h0 == 0 ? g_stall_chunk : -1;
        p.q_scale = q_scale;
        p.k_scale = k_scale;
        p.v_scale = v_scale;
        err = device_error_word(&p.err);
        if (err != cudaSuccess) break;
        err = cudaMemsetAsync(flags, 0, flag_ints * sizeof(int), stream);
        if (err != cudaSuccess) break;

        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        cfg.gridDim = dim3(info->sms);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemAlloc;
        cfg.stream = stream;
        // chains and workers wait for one another: every CTA must be resident
        at[0].id = cudaLaunchAttributeCooperative;
        at[0].val.cooperative = 1;
        cfg.attrs = at;
        cfg.numAttrs = g_plain_launch ? 0 : 1;
        err = fp8 ? cudaLaunchKernelEx(&cfg, gdn_chunk_pool_kernel<true>, mq, mk, mv, mo, p)
                  : cudaLaunchKernelEx(&cfg, gdn_chunk_pool_kernel<false>, mq, mk, mv, mo, p);
        if (err == cudaSuccess) err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    cudaError_t e2 = ws_free(ws, stream);
    if (err == cudaSuccess) err = e2;
    return err;
}

}  // namespace gdn

// Test hooks (declared in gdn_debug.h).
// gdn_debug_ring: a device buffer of at least dirs*B*H*8*33792 bytes that the
// pooled kernel uses as its operand ring instead of workspace (NULL: off), so a
// test can read back the prepared operands of each scan's last eight chunks.
// gdn_debug_kernel_select: 0 picks the kernel by shape (the pooled kernel for
// dk = dv = 128 whole sequences), 1 forces the single-CTA chunkwise kernel for
// every bf16 call.
// gdn_debug_stall: chunk c >= 0 makes scan 0's chain of the pooled kernel wait
// for chunk c's operands with a target nothing reaches, so the wait runs out
// (with a lowered limit, see gdn_debug_wait_limit) and the call ends with
// GDN_ERR_DEVICE_TIMEOUT; -1 (the default) turns it off.
// gdn_debug_plain_launch: 1 launches the pooled kernel without the cooperative
// attribute (same grid, one CTA per SM), for profilers that replay launches
// one at a time; 0 (the default) restores the cooperative launch.
extern "C" void gdn_debug_ring(void *device_buffer) { gdn::g_debug_ring = device_buffer; }
extern "C" void gdn_debug_kernel_select(int which) { gdn::g_kernel_select = which; }
extern "C" void gdn_debug_stall(int chunk) { gdn::g_stall_chunk = chunk; }
extern "C" void gdn_debug_plain_launch(int on) { gdn::g_plain_launch = on != 0; }

cudaError_t gdn::set_wait_limit_pool(unsigned long long ns) { return set_module_wait_limit(ns); }
