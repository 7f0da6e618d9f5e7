// Token-by-token GDN recurrence on CUDA cores, fp32 state and arithmetic.
//
// The fp32 path (and a slow cross-check for bf16 inputs).  One CTA per
// (batch*head, direction); thread j owns column j of the state H = S^T
// (dk fp32 registers).  Columns of H evolve independently under
//     u_j = b_t (v_tj - a_t sum_i H_ij k_ti),   H_ij <- a_t H_ij + k_ti u_j,
//     o_tj = sum_i H_ij q_ti,
// which is the GDN update S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T,
// o_t = S_t q_t (librediffusion PR #21 page, "What's added") written per column,
// so the scan needs no cross-thread reduction.  q, k, v and the gates of a
// group of tokens are staged once in shared memory and read as broadcasts.
//
// Bidirectional: the two directions run as separate CTAs and write fp32
// partial outputs to a stream-ordered workspace; a second kernel adds them
// and converts to the output dtype.
#include <cuda_bf16.h>

#include <algorithm>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kTok = 16;     // tokens staged per step
constexpr int kMaxD = 128;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

struct RecParams {
    const void *q, *k, *v;
    const float *beta, *decay, *state_in;
    float *state_out;
    void *o;          // final output (causal)
    float *part;      // bidi: [2][B*H*T*dv] fp32 partials
    int BH, T, dv;
};

template <int DK, typename TIn>
__global__ void __launch_bounds__(kMaxD)
gdn_recurrent_kernel(RecParams p)
{
    __shared__ float sk[kTok][DK];
    __shared__ float sq[kTok][DK];
    __shared__ float sv[kTok][kMaxD];
    __shared__ float sa[kTok];
    __shared__ float sb[kTok];

    const int bh = blockIdx.x;
    const int dir = blockIdx.y;           // 0 forward, 1 reverse
    const int T = p.T, dv = p.dv;
    const int col = threadIdx.x;          // blockDim.x == dv

    const TIn *q = static_cast<const TIn *>(p.q) + (size_t)bh * T * DK;
    const TIn *k = static_cast<const TIn *>(p.k) + (size_t)bh * T * DK;
    const TIn *v = static_cast<const TIn *>(p.v) + (size_t)bh * T * dv;
    const float *beta = p.beta + (size_t)bh * T;
    const float *decay = p.decay + (size_t)bh * T;

    float h[DK];
    if (dir == 0 && p.state_in) {
        const float *s0 = p.state_in + (size_t)bh * DK * dv;
#pragma unroll
        for (int i = 0; i < DK; ++i) h[i] = s0[(size_t)i * dv + col];
    } else {
#pragma unroll
        for (int i = 0; i < DK; ++i) h[i] = 0.f;
    }

    for (int s0 = 0; s0 < T; s0 += kTok) {
        const int ntok = min(kTok, T - s0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < ntok * DK; idx += blockDim.x) {
            const int s = idx / DK, i = idx % DK;
            const int t = dir ? (T - 1 - (s0 + s)) : (s0 + s);
            sk[s][i] = to_f32(k[(size_t)t * DK + i]);
            sq[s][i] = to_f32(q[(size_t)t * DK + i]);
        }
        for (int s = 0; s < ntok; ++s) {
            const int t = dir ? (T - 1 - (s0 + s)) : (s0 + s);
            sv[s][col] = to_f32(v[(size_t)t * dv + col]);
        }
        if (threadIdx.x < ntok) {
            const int s = threadIdx.x;
            const int t = dir ? (T - 1 - (s0 + s)) : (s0 + s);
            sa[s] = decay[t];
            sb[s] = beta[t];
        }
        __syncthreads();

        for (int s = 0; s < ntok; ++s) {
            const int t = dir ? (T - 1 - (s0 + s)) : (s0 + s);
            const float a = sa[s], b = sb[s];
            float d[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) d[r] = 0.f;
#pragma unroll
            for (int i = 0; i < DK; ++i) d[i & 7] = fmaf(h[i], sk[s][i], d[i & 7]);
            const float dot = ((d[0] + d[1]) + (d[2] + d[3])) + ((d[4] + d[5]) + (d[6] + d[7]));
            const float u = b * (sv[s][col] - a * dot);
            float e[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) e[r] = 0.f;
#pragma unroll
            for (int i = 0; i < DK; ++i) {
                h[i] = fmaf(a, h[i], sk[s][i] * u);
                e[i & 7] = fmaf(h[i], sq[s][i], e[i & 7]);
            }
            const float ot = ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
            if (p.part) {
                p.part[((size_t)dir * p.BH + bh) * T * dv + (size_t)t * dv + col] = ot;
            } else {
                static_cast<TIn *>(p.o)[(size_t)bh * T * dv + (size_t)t * dv + col] = from_f32<TIn>(ot);
            }
        }
    }

    if (p.state_out) {
        float *so = p.state_out + ((size_t)dir * p.BH + bh) * DK * dv;
#pragma unroll
        for (int i = 0; i < DK; ++i) so[(size_t)i * dv + col] = h[i];
    }
}

template <typename TIn>
__global__ void bidi_sum_kernel(const float *part, TIn *o, size_t n)
{
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        o[i] = from_f32<TIn>(part[i] + part[n + i]);
}

template <typename TIn>
cudaError_t launch_typed(const FwdArgs &a, cudaStream_t stream)
{
    RecParams p;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.beta = a.beta; p.decay = a.decay; p.state_in = a.state_in;
    p.state_out = a.state_out; p.o = a.o; p.part = nullptr;
    p.BH = a.B * a.H; p.T = a.T; p.dv = a.dv;

    const size_t n_out = (size_t)p.BH * a.T * a.dv;
    cudaError_t err = cudaSuccess;
    if (a.bidi) {
        err = ws_alloc(reinterpret_cast<void **>(&p.part), 2 * n_out * sizeof(float), stream);
        if (err != cudaSuccess) return err;
    }
    dim3 grid(p.BH, a.bidi ? 2 : 1);
    dim3 block(a.dv);
    switch (a.dk) {
        case 32:  gdn_recurrent_kernel<32, TIn><<<grid, block, 0, stream>>>(p); break;
        case 64:  gdn_recurrent_kernel<64, TIn><<<grid, block, 0, stream>>>(p); break;
        case 96:  gdn_recurrent_kernel<96, TIn><<<grid, block, 0, stream>>>(p); break;
        case 128: gdn_recurrent_kernel<128, TIn><<<grid, block, 0, stream>>>(p); break;
        default: err = cudaErrorInvalidValue;
    }
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err == cudaSuccess) count_launches(1);
    if (a.bidi) {
        if (err == cudaSuccess) {
            const int threads = 256;
            const int blocks = (int)std::min<size_t>((n_out + threads - 1) / threads, 148 * 16);
            bidi_sum_kernel<TIn><<<blocks, threads, 0, stream>>>(p.part, static_cast<TIn *>(a.o), n_out);
            err = cudaGetLastError();
            if (err == cudaSuccess) count_launches(1);
        }
        cudaError_t e2 = ws_free(p.part, stream);
        if (err == cudaSuccess) err = e2;
    }
    return err;
}

}  // namespace

cudaError_t launch_recurrent(const FwdArgs &a, cudaStream_t stream)
{
    return a.fp32 ? launch_typed<float>(a, stream) : launch_typed<__nv_bfloat16>(a, stream);
}

}  // namespace gdn
