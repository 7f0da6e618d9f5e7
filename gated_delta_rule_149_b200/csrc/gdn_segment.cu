// Forms of the recurrence built from passes of the chunkwise kernel plus small
// kernels of their own: the segment-parallel causal scan, the frame-block
// read-out and the normalised read-out (sections below).
//
// Segment-parallel causal scan: a few long scans (few heads, many chunks) are
// split along time so that more SMs work at once.
//
// The recurrence is affine in the state.  For a segment p of a head, run from
// an initial state X, its final state is  P_p X + L_p  with
//     P_p = prod_t a_t (I - b_t k_t k_t^T)       (dk x dk, the segment's transition)
//     L_p = the final state of the segment run from zero,
// so the state entering segment p + 1 is  E_{p+1} = P_p E_p + L_p.  Three
// passes of the chunkwise kernel and one small combine give the same result as
// one sequential scan (the segment-parallel scan of the pages' streaming
// workloads: per-chunk latency is the product metric there):
//   1. segments 0 .. S-2 in parallel: segment 0 from the given state (its
//      output and its final state E_1 are final), the others from zero (L_p);
//   2. at the same time, on a second stream: segments 1 .. S-2 with v = 0
//      from the identity: their final states are the transitions P_p;
//   3. combine  E_{p+1} = P_p E_p + L_p  for p = 1 .. S-2 (serial over p,
//      parallel over heads and state columns; fp32);
//   4. segments 1 .. S-1 in parallel from E_p: their outputs, and the last
//      segment's final state.
// Segments are whole 64-token chunks; only the last may be shorter.

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kDKs = 128;   // the chunkwise kernel's key size

// SMs of the current device (grid-stride helper kernels launch one block per SM)
int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;   // a launch error, if any, surfaces at the launch itself
    return n;
}

__global__ void identity_fill_kernel(float *out, size_t n_mats)
{
    const size_t n = n_mats * kDKs * kDKs;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int i = (int)((e / kDKs) % kDKs), j = (int)(e % kDKs);
        out[e] = (i == j) ? 1.f : 0.f;
    }
}

__global__ void fill_kernel(float *out, size_t n, float value)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x)
        out[e] = value;
}

// Threads the state through consecutive pieces of one head (blockIdx.x), 16
// state columns (blockIdx.y) at a time:  E[0] = L[0],  E[j] = P[p0 + j - 1] E[j-1]
// + L[j]  for j = 1 .. steps.  L and E hold nrows [dk][dv] states per head, P
// holds prows [dk][dk] transitions per head.  128 threads, thread r owns row r
// of the 16-column block; the previous E block sits in shared memory and is
// read 4 columns at a time.
__global__ void __launch_bounds__(128) segment_combine_kernel(const float *L, const float *P, float *E,
                                                              int nrows, int prows, int p0, int steps,
                                                              int dv)
{
    __shared__ __align__(16) float Es[kDKs][16];
    const int bh = blockIdx.x, r = threadIdx.x;
    const int cg = 16 * blockIdx.y;          // first column of the block
    const size_t sz = (size_t)kDKs * dv;
    float acc[16];
    {
        const float *L0 = L + (size_t)bh * nrows * sz + (size_t)r * dv + cg;
        float *E1 = E + (size_t)bh * nrows * sz + (size_t)r * dv + cg;
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(L0 + c);
            acc[c] = v.x; acc[c + 1] = v.y; acc[c + 2] = v.z; acc[c + 3] = v.w;
            *reinterpret_cast<float4 *>(E1 + c) = v;
        }
    }
    for (int pp = 1; pp <= steps; ++pp) {
#pragma unroll
        for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4 *>(&Es[r][c]) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        __syncthreads();
        const float *Lp = L + ((size_t)bh * nrows + pp) * sz + (size_t)r * dv + cg;
        const float *Pr = P + ((size_t)bh * prows + p0 + pp - 1) * kDKs * kDKs + (size_t)r * kDKs;
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(Lp + c);
            acc[c] = v.x; acc[c + 1] = v.y; acc[c + 2] = v.z; acc[c + 3] = v.w;
        }
#pragma unroll 2
        for (int k = 0; k < kDKs; k += 4) {
            const float4 pk = *reinterpret_cast<const float4 *>(Pr + k);
            const float pv[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int c = 0; c < 16; c += 4) {
                    const float4 e = *reinterpret_cast<const float4 *>(&Es[k + u][c]);
                    acc[c] = fmaf(pv[u], e.x, acc[c]);
                    acc[c + 1] = fmaf(pv[u], e.y, acc[c + 1]);
                    acc[c + 2] = fmaf(pv[u], e.z, acc[c + 2]);
                    acc[c + 3] = fmaf(pv[u], e.w, acc[c + 3]);
                }
        }
        float *Ep = E + ((size_t)bh * nrows + pp) * sz + (size_t)r * dv + cg;
#pragma unroll
        for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4 *>(Ep + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        __syncthreads();
    }
}

size_t align_up(size_t n) { return (n + 255) & ~(size_t)255; }

// A second stream per device for the transition pass, with the two events that
// fork it from and join it to the caller's stream.  Created on first use and
// kept for the life of the process; calls hold the mutex while they enqueue,
// so concurrent callers never interleave on it.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDev = 64;
std::mutex g_side_mu;
SideStream g_side[kMaxDev];

cudaError_t side_stream(int dev, SideStream **out)
{
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    SideStream &x = g_side[dev];
    cudaError_t err = cudaSuccess;
    if (!x.s) err = cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking);
    if (err == cudaSuccess && !x.fork) err = cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming);
    if (err == cudaSuccess && !x.join) err = cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming);
    *out = &x;
    return err;
}

}  // namespace

int segment_count(int T, int n_segments, int *seg_chunks)
{
    const int nc = (T + 63) / 64;
    int s = n_segments < 1 ? 1 : n_segments;
    if (s > nc) s = nc;
    const int per = (nc + s - 1) / s;
    *seg_chunks = per;
    return (nc + per - 1) / per;
}

cudaError_t launch_segmented(const FwdArgs &a, int n_segments, cudaStream_t stream)
{
    int seg_chunks = 0;
    const int S = segment_count(a.T, n_segments, &seg_chunks);
    if (S <= 2) return launch_chunk_tc(a, stream);   // nothing runs in parallel

    const size_t BH = (size_t)a.B * a.H, sz = (size_t)a.dk * a.dv, pz = (size_t)a.dk * a.dk;
    const size_t nS = BH * (S - 1), nP = BH * (S - 2);
    const size_t b_sin = align_up(nS * sz * 4), b_l = b_sin, b_e = b_sin, b_f = b_sin;
    const size_t b_pin = align_up(nP * pz * 4), b_pout = b_pin;
    const size_t b_vz = align_up(BH * (size_t)a.T * a.dk * 2), b_ow = b_vz;
    uint8_t *ws = nullptr;
    cudaError_t err = ws_alloc(reinterpret_cast<void **>(&ws),
                                      b_sin + b_l + b_e + b_f + b_pin + b_pout + b_vz + b_ow, stream);
    if (err != cudaSuccess) return err;
    float *Sin = reinterpret_cast<float *>(ws);
    float *Lst = reinterpret_cast<float *>(ws + b_sin);
    float *Est = reinterpret_cast<float *>(ws + b_sin + b_l);
    float *Fst = reinterpret_cast<float *>(ws + b_sin + b_l + b_e);
    float *Pin = reinterpret_cast<float *>(ws + b_sin + b_l + b_e + b_f);
    float *Pst = reinterpret_cast<float *>(ws + b_sin + b_l + b_e + b_f + b_pin);
    void *Vz = ws + b_sin + b_l + b_e + b_f + b_pin + b_pout;
    void *Ow = ws + b_sin + b_l + b_e + b_f + b_pin + b_pout + b_vz;

    int dev = 0;
    err = cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream *side = nullptr;
    if (err == cudaSuccess) err = side_stream(dev, &side);

    // pass 2 (second stream, after the workspace exists): the transitions of
    // segments 1 .. S-2 (v = 0, identity state)
    if (err == cudaSuccess) err = cudaEventRecord(side->fork, stream);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(side->s, side->fork, 0);
    if (err == cudaSuccess) err = cudaMemsetAsync(Vz, 0, BH * (size_t)a.T * a.dk * 2, side->s);
    if (err == cudaSuccess) {
        identity_fill_kernel<<<sm_count(), 256, 0, side->s>>>(Pin, nP);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (err == cudaSuccess) {
        FwdArgs a2 = a;
        a2.v = Vz;
        a2.dv = a.dk;
        a2.o = Ow;
        a2.state_in = Pin;
        a2.state_out = Pst;
        a2.seg0 = 1;
        a2.n_seg = S - 2;
        a2.seg_chunks = seg_chunks;
        err = launch_chunk_tc(a2, side->s);
    }
    const bool forked = err == cudaSuccess;
    if (forked) err = cudaEventRecord(side->join, side->s);

    // pass 1 (caller's stream): segment 0 from the given state, segments
    // 1 .. S-2 from zero
    if (err == cudaSuccess) err = cudaMemsetAsync(Sin, 0, nS * sz * 4, stream);
    if (err == cudaSuccess && a.state_in)
        err = cudaMemcpy2DAsync(Sin, (S - 1) * sz * 4, a.state_in, sz * 4, sz * 4, BH,
                                cudaMemcpyDeviceToDevice, stream);
    if (err == cudaSuccess) {
        FwdArgs a1 = a;
        a1.state_in = Sin;
        a1.state_out = Lst;
        a1.seg0 = 0;
        a1.n_seg = S - 1;
        a1.seg_chunks = seg_chunks;
        err = launch_chunk_tc(a1, stream);
    }
    // join: whatever happened, the caller's stream waits for the second one
    // before anything (the workspace's release included) follows
    if (forked) {
        const cudaError_t ej = cudaStreamWaitEvent(stream, side->join, 0);
        if (err == cudaSuccess) err = ej;
    }
    // combine: the state entering each segment
    if (err == cudaSuccess) {
        segment_combine_kernel<<<dim3((unsigned)BH, a.dv / 16), 128, 0, stream>>>(Lst, Pst, Est, S - 1, S - 2, 0,
                                                                                   S - 2, a.dv);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    // pass 4: segments 1 .. S-1 from their entry states
    if (err == cudaSuccess) {
        FwdArgs a3 = a;
        a3.state_in = Est;
        a3.state_out = a.state_out ? Fst : nullptr;
        a3.seg0 = 1;
        a3.n_seg = S - 1;
        a3.seg_chunks = seg_chunks;
        err = launch_chunk_tc(a3, stream);
    }
    if (err == cudaSuccess && a.state_out)
        err = cudaMemcpy2DAsync(a.state_out, sz * 4, Fst + (size_t)(S - 2) * sz, (S - 1) * sz * 4, sz * 4, BH,
                                cudaMemcpyDeviceToDevice, stream);
    const cudaError_t e2 = ws_free(ws, stream);
    return err != cudaSuccess ? err : e2;
}


// ------------------------------------------------------------ frame-block read-out
//
// Every token of block f (tokens [f*Tb, (f+1)*Tb) of a head) is read out with
// the state after the whole block, o_t = H_{(f+1)Tb-1}^T q_t (the frame-block
// causal form of a linear-attention KV cache carried across video frames: a
// token sees its whole frame and every earlier one).  A head-major [B,H,T,d]
// tensor with T = F*Tb is also a [B*H*F, Tb, d] tensor, so every pass below is
// one chunkwise launch over B*H*F independent blocks:
//   1. the blocks from zero (block 0 of each head from the given state): L_f;
//   2. at the same time, on a second stream: the blocks' transitions P_f
//      (v = 0 from the identity);
//   3. combine: E_0 = L_0, E_f = P_f E_{f-1} + L_f, the state after block f;
//   4. read-out: every block from E_f with identity tokens (b = 0, a = 1), so
//      the state stays E_f and the kernel's output is o_t = E_f^T q_t.
cudaError_t launch_blockcausal(const FwdArgs &a, int block, cudaStream_t stream)
{
    const int F = a.T / block;
    const size_t BH = (size_t)a.B * a.H, BHF = BH * F, sz = (size_t)a.dk * a.dv, pz = (size_t)a.dk * a.dk;
    const size_t ntok = BH * (size_t)a.T;
    const size_t b_st = align_up(BHF * sz * 4), b_p = align_up(BHF * pz * 4);
    const size_t b_vz = align_up(ntok * a.dk * 2), b_g = align_up(ntok * 4);
    uint8_t *ws = nullptr;
    cudaError_t err = ws_alloc(reinterpret_cast<void **>(&ws), 3 * b_st + 2 * b_p + 2 * b_vz + 2 * b_g, stream);
    if (err != cudaSuccess) return err;
    float *Sin = reinterpret_cast<float *>(ws);
    float *Lst = reinterpret_cast<float *>(ws + b_st);
    float *Est = reinterpret_cast<float *>(ws + 2 * b_st);
    float *Pin = reinterpret_cast<float *>(ws + 3 * b_st);
    float *Pst = reinterpret_cast<float *>(ws + 3 * b_st + b_p);
    void *Vz = ws + 3 * b_st + 2 * b_p;
    void *Ow = ws + 3 * b_st + 2 * b_p + b_vz;
    float *Zb = reinterpret_cast<float *>(ws + 3 * b_st + 2 * b_p + 2 * b_vz);
    float *On = reinterpret_cast<float *>(ws + 3 * b_st + 2 * b_p + 2 * b_vz + b_g);

    FwdArgs blocks = a;   // the [B*H*F, Tb] view
    blocks.B = (int)BHF;
    blocks.H = 1;
    blocks.T = block;

    int dev = 0;
    err = cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream *side = nullptr;
    if (err == cudaSuccess) err = side_stream(dev, &side);

    // pass 2 (second stream): transitions of every block
    if (err == cudaSuccess) err = cudaEventRecord(side->fork, stream);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(side->s, side->fork, 0);
    if (err == cudaSuccess) err = cudaMemsetAsync(Vz, 0, ntok * a.dk * 2, side->s);
    if (err == cudaSuccess) {
        identity_fill_kernel<<<sm_count(), 256, 0, side->s>>>(Pin, BHF);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (err == cudaSuccess) {
        FwdArgs a2 = blocks;
        a2.v = Vz;
        a2.dv = a.dk;
        a2.o = Ow;
        a2.state_in = Pin;
        a2.state_out = Pst;
        err = launch_chunk_tc(a2, side->s);
    }
    const bool forked = err == cudaSuccess;
    if (forked) err = cudaEventRecord(side->join, side->s);

    // pass 1 (caller's stream): every block from zero, block 0 from the given
    // state; its outputs land in o and are overwritten by the read-out
    if (err == cudaSuccess) err = cudaMemsetAsync(Sin, 0, BHF * sz * 4, stream);
    if (err == cudaSuccess && a.state_in)
        err = cudaMemcpy2DAsync(Sin, F * sz * 4, a.state_in, sz * 4, sz * 4, BH, cudaMemcpyDeviceToDevice,
                                stream);
    if (err == cudaSuccess) {
        FwdArgs a1 = blocks;
        a1.state_in = Sin;
        a1.state_out = Lst;
        err = launch_chunk_tc(a1, stream);
    }
    if (forked) {
        const cudaError_t ej = cudaStreamWaitEvent(stream, side->join, 0);
        if (err == cudaSuccess) err = ej;
    }
    // combine: the state after every block
    if (err == cudaSuccess) {
        segment_combine_kernel<<<dim3((unsigned)BH, a.dv / 16), 128, 0, stream>>>(Lst, Pst, Est, F, F, 1, F - 1,
                                                                                   a.dv);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    // read-out with identity tokens
    if (err == cudaSuccess) err = cudaMemsetAsync(Zb, 0, ntok * 4, stream);
    if (err == cudaSuccess) {
        fill_kernel<<<sm_count(), 256, 0, stream>>>(On, ntok, 1.f);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (err == cudaSuccess) {
        FwdArgs a3 = blocks;
        a3.beta = Zb;
        a3.decay = On;
        a3.state_in = Est;
        a3.state_out = nullptr;
        err = launch_chunk_tc(a3, stream);
    }
    if (err == cudaSuccess && a.state_out)
        err = cudaMemcpy2DAsync(a.state_out, sz * 4, Est + (size_t)(F - 1) * sz, F * sz * 4, sz * 4, BH,
                                cudaMemcpyDeviceToDevice, stream);
    const cudaError_t e2 = ws_free(ws, stream);
    return err != cudaSuccess ? err : e2;
}

}  // namespace gdn

// ------------------------------------------------------------ normalised read-out
//
// o_t = (S_t q_t) / (z_t . q_t + eps), with z the same gated delta recurrence
// driven by a constant value of 1 (bidirectional: numerators and denominators
// summed over the two directions, then divided).  The numerator is the plain
// call; the denominator is a second call with a 64-wide value of ones (every
// column is the same z), on a second stream for causal calls; a last kernel
// divides.

namespace gdn {
namespace {

__global__ void fill_bf16_kernel(__nv_bfloat16 *out, size_t n, float value)
{
    const __nv_bfloat16 v = __float2bfloat16(value);
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x)
        out[e] = v;
}

// every column of the [rows][64] output is z_in[row]
__global__ void broadcast_cols_kernel(float *out, const float *z, size_t rows, int width)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < rows * width; e += (size_t)gridDim.x * blockDim.x)
        out[e] = z[e / width];
}

// o[row][c] /= (den[row][0] + eps), 8 bf16 values per thread step
__global__ void divide_rows_kernel(__nv_bfloat16 *o, const __nv_bfloat16 *den, size_t rows, int dv, int den_width,
                                   float eps)
{
    const int per = dv / 8;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < rows * per; e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / per;
        const float inv = 1.f / (__bfloat162float(den[row * den_width]) + eps);
        uint4 w = *reinterpret_cast<const uint4 *>(o + e * 8);
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&w);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 f = __bfloat1622float2(h[u]);
            h[u] = __floats2bfloat162_rn(f.x * inv, f.y * inv);
        }
        *reinterpret_cast<uint4 *>(o + e * 8) = w;
    }
}

}  // namespace

cudaError_t launch_normalized(const FwdArgs &a, const float *state_z_in, float *state_z_out, float eps,
                              cudaStream_t stream)
{
    const size_t BH = (size_t)a.B * a.H, ntok = BH * (size_t)a.T, ndir = a.bidi ? 2 : 1;
    // the value of ones: 128 wide when the pooled kernel can run the pass (it
    // serves dv = 128 only; every column then carries the same z), else 64
    FwdArgs az = a;
    az.dv = 128;
    const int zw = chunk_pool_supported(az) ? 128 : 64;
    const size_t b_ones = align_up(ntok * zw * 2), b_den = b_ones;
    const size_t b_zin = align_up(BH * a.dk * zw * 4), b_zout = align_up(ndir * BH * a.dk * zw * 4);
    uint8_t *ws = nullptr;
    cudaError_t err = ws_alloc(reinterpret_cast<void **>(&ws), b_ones + b_den + b_zin + b_zout, stream);
    if (err != cudaSuccess) return err;
    auto *ones = reinterpret_cast<__nv_bfloat16 *>(ws);
    auto *den = reinterpret_cast<__nv_bfloat16 *>(ws + b_ones);
    float *zin = reinterpret_cast<float *>(ws + b_ones + b_den);
    float *zout = reinterpret_cast<float *>(ws + b_ones + b_den + b_zin);

    // causal: the denominator pass is enqueued beside the numerator pass on a
    // second stream (they overlap as far as their grids leave SMs free; two
    // pooled launches each take every SM and run one after the other).
    // Bidirectional: after it, on the caller's stream.
    int dev = 0, sms = 0;
    err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream *side = nullptr;
    if (err == cudaSuccess && !a.bidi) err = side_stream(dev, &side);
    cudaStream_t ds = a.bidi ? stream : (side ? side->s : stream);
    bool forked = false;
    if (err == cudaSuccess && !a.bidi) {
        err = cudaEventRecord(side->fork, stream);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(side->s, side->fork, 0);
    }
    if (err == cudaSuccess && a.bidi) err = launch_chunk_tc(a, stream);   // numerator first
    if (err == cudaSuccess) {
        fill_bf16_kernel<<<sms, 256, 0, ds>>>(ones, ntok * zw, 1.f);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (err == cudaSuccess && state_z_in) {
        broadcast_cols_kernel<<<sms, 256, 0, ds>>>(zin, state_z_in, BH * a.dk, zw);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (err == cudaSuccess) {
        az.v = ones;
        az.dv = zw;
        az.o = den;
        az.state_in = state_z_in ? zin : nullptr;
        az.state_out = state_z_out ? zout : nullptr;
        err = launch_chunk_tc(az, ds);
    }
    if (!a.bidi && side) {
        forked = err == cudaSuccess;
        if (forked) err = cudaEventRecord(side->join, side->s);
        if (err == cudaSuccess) err = launch_chunk_tc(a, stream);            // numerator
        if (forked) {
            const cudaError_t ej = cudaStreamWaitEvent(stream, side->join, 0);
            if (err == cudaSuccess) err = ej;
        }
    }
    if (err == cudaSuccess) {
        divide_rows_kernel<<<sms * 4, 256, 0, stream>>>(static_cast<__nv_bfloat16 *>(a.o), den, ntok, a.dv, zw, eps);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    // z out: column 0 of every [dk][zw] state
    if (err == cudaSuccess && state_z_out)
        err = cudaMemcpy2DAsync(state_z_out, 4, zout, zw * 4, 4, ndir * BH * a.dk, cudaMemcpyDeviceToDevice, stream);
    const cudaError_t e2 = ws_free(ws, stream);
    return err != cudaSuccess ? err : e2;
}

}  // namespace gdn
