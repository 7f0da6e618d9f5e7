// fp8 (E4M3) q, k, v with one fp32 scale per (batch, head): x = scale * x8.
//
// dk = dv = 128 (the pooled kernel): the kernel loads the codes by TMA, one
// byte per element, and widens each tile to scaled bf16 in shared memory
// before the tensor-core products (both operands of one product must have the
// same type, and the other operands are bf16).  Other shapes (dv = 64, or the
// single-CTA kernel forced): a pre-pass dequantises into bf16 workspace copies
// (16 codes per thread step, through the CUDA fp8 conversion) and the
// chunkwise kernel runs on them.

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "gdn_internal.h"

namespace gdn {
namespace {

// out[e] = bf16(scale[head of e] * decode(in[e])), 16 elements per step;
// per_head = T * d elements (a multiple of 16).
__global__ void dequant_e4m3_kernel(const uint8_t *in, const float *scale, __nv_bfloat16 *out, size_t n16,
                                    size_t per_head)
{
    for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < n16; g += (size_t)gridDim.x * blockDim.x) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(in + g * 16);
        const float s = scale[(g * 16) / per_head];
        const uint8_t *b = reinterpret_cast<const uint8_t *>(&raw);
        uint32_t w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            __nv_fp8_e4m3 lo, hi;
            lo.__x = b[2 * u];
            hi.__x = b[2 * u + 1];
            const __nv_bfloat162 v = __floats2bfloat162_rn(s * static_cast<float>(lo), s * static_cast<float>(hi));
            w[u] = *reinterpret_cast<const uint32_t *>(&v);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + g * 16);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

size_t align_up256(size_t n) { return (n + 255) & ~(size_t)255; }

}  // namespace

cudaError_t launch_fp8(const FwdArgs &a, const float *q_scale, const float *k_scale, const float *v_scale,
                       cudaStream_t stream)
{
    // dk = dv = 128: the pooled kernel loads the codes and widens them itself
    if (chunk_pool_supported(a)) return launch_chunk_pool(a, stream, q_scale, k_scale, v_scale);
    const size_t BH = (size_t)a.B * a.H, nk = BH * a.T * a.dk, nv = BH * a.T * a.dv;
    const size_t bq = align_up256(nk * 2), bv = align_up256(nv * 2);
    uint8_t *ws = nullptr;
    cudaError_t err = ws_alloc(reinterpret_cast<void **>(&ws), 2 * bq + bv, stream);
    if (err != cudaSuccess) return err;
    auto *q = reinterpret_cast<__nv_bfloat16 *>(ws);
    auto *k = reinterpret_cast<__nv_bfloat16 *>(ws + bq);
    auto *v = reinterpret_cast<__nv_bfloat16 *>(ws + 2 * bq);
    const struct { const void *in; const float *s; __nv_bfloat16 *out; size_t n, per; } job[3] = {
        {a.q, q_scale, q, nk, (size_t)a.T * a.dk}, {a.k, k_scale, k, nk, (size_t)a.T * a.dk},
        {a.v, v_scale, v, nv, (size_t)a.T * a.dv}};
    int dev = 0, sms = 0;
    if (err == cudaSuccess) err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    for (int j = 0; j < 3 && err == cudaSuccess; ++j) {
        // HBM-bound: enough blocks in flight on every SM (16 per SM)
        dequant_e4m3_kernel<<<sms * 16, 256, 0, stream>>>(static_cast<const uint8_t *>(job[j].in), job[j].s,
                                                          job[j].out, job[j].n / 16, job[j].per);
        err = cudaGetLastError();
        if (err == cudaSuccess) count_launches(1);
    }
    if (err == cudaSuccess) {
        FwdArgs b = a;
        b.q = q;
        b.k = k;
        b.v = v;
        err = launch_chunk_tc(b, stream);
    }
    const cudaError_t e2 = ws_free(ws, stream);
    return err != cudaSuccess ? err : e2;
}

}  // namespace gdn
