// libgdn C ABI: argument checks, dispatch, rollout threading, host-buffer
// entry point, device error word.  No C++ exception crosses this boundary
// (the catch-at-the-boundary convention of the librediffusion PR #21 C-API,
// and the reason-string prechecks of the SANA-WM camera-GDN backend error
// record), and every argument error is caught before anything is launched.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/gdn.h"
#include "../../include/gdn_debug.h"
#include "gdn_internal.h"

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return code;
}

int ok()
{
    g_msg[0] = '\0';
    return GDN_OK;
}

bool misaligned(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Shape / dtype / pointer checks shared by gdn_forward and gdn_rollout.
int check_common(const void *q, const void *k, const void *v, const float *beta,
                 const float *decay, const float *state_in, const float *state_out,
                 const void *o, int B, int H, int T, int dk, int dv, int mode,
                 const char *T_name)
{
    if (!q || !k || !v || !beta || !decay || !o)
        return fail(GDN_ERR_INVALID_ARG, "q, k, v, beta, decay and o must be non-NULL");
    if (B <= 0 || H <= 0 || T <= 0)
        return fail(GDN_ERR_INVALID_ARG, "B, H and %s must be positive (got %d, %d, %d)",
                    T_name, B, H, T);
    if (mode & ~(GDN_BIDI | GDN_FP32 | GDN_RECURRENT))
        return fail(GDN_ERR_INVALID_ARG, "unknown mode bits 0x%x", mode);
    if ((long long)B * H > 65535)
        return fail(GDN_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535", (long long)B * H);
    if (dk <= 0 || dv <= 0 || dk % 32 || dv % 32 || dk > 128 || dv > 128)
        return fail(GDN_ERR_UNSUPPORTED,
                    "dk and dv must be multiples of 32 in [32, 128] (got dk=%d, dv=%d)", dk, dv);
    const void *ptrs[] = {q, k, v, beta, decay, state_in, state_out, o};
    const char *names[] = {"q", "k", "v", "beta", "decay", "state_in", "state_out", "o"};
    for (int i = 0; i < 8; ++i)
        if (misaligned(ptrs[i]))
            return fail(GDN_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    return GDN_OK;
}

gdn::FwdArgs make_args(const void *q, const void *k, const void *v, const float *beta,
                       const float *decay, const float *state_in, float *state_out, void *o,
                       int B, int H, int T, int dk, int dv, int mode)
{
    gdn::FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.decay = decay;
    a.state_in = state_in; a.state_out = state_out; a.o = o;
    a.B = B; a.H = H; a.T = T; a.dk = dk; a.dv = dv;
    a.bidi = (mode & GDN_BIDI) != 0;
    a.fp32 = (mode & GDN_FP32) != 0;
    return a;
}

// Picks the kernel for validated arguments and launches it.
int dispatch(const gdn::FwdArgs &a, int mode, cudaStream_t stream)
{
    const bool recurrent = a.fp32 || (mode & GDN_RECURRENT);
    cudaError_t err;
    if (recurrent) {
        err = gdn::launch_recurrent(a, stream);
    } else if (gdn::chunk_tc_supported(a)) {
        err = gdn::launch_chunk_tc(a, stream);
    } else {
        return fail(GDN_ERR_UNSUPPORTED,
                    "bf16 chunkwise kernel needs dk = 128 and dv in {64, 128} (got dk=%d, dv=%d); "
                    "GDN_RECURRENT runs other sizes", a.dk, a.dv);
    }
    if (err != cudaSuccess)
        return fail(GDN_ERR_CUDA, "launch failed: %s", cudaGetErrorString(err));
    return ok();
}

size_t dtype_size(int mode) { return (mode & GDN_FP32) ? 4 : 2; }

// The kernels of host-buffer calls on one device run one after another
// whatever their streams: a chunkwise launch takes every SM (the pooled
// kernel's grid is one CTA per SM, launched cooperatively), so two side by side
// would only queue behind each other; in call order, each call's copies overlap
// the previous call's kernel.  Each call's kernels wait for the previous call's
// (an event per device) and record their own completion.
constexpr int kMaxOrderDev = 64;
std::mutex g_order_mu;
cudaEvent_t g_order_ev[kMaxOrderDev] = {};

int ordered_dispatch(const gdn::FwdArgs &a, int mode, cudaStream_t stream)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess && (dev < 0 || dev >= kMaxOrderDev)) e = cudaErrorInvalidDevice;
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "device: %s", cudaGetErrorString(e));
    std::lock_guard<std::mutex> lock(g_order_mu);
    if (!g_order_ev[dev]) e = cudaEventCreateWithFlags(&g_order_ev[dev], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, g_order_ev[dev], 0);   // no-op before the first record
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "call order: %s", cudaGetErrorString(e));
    const int rc = dispatch(a, mode, stream);
    if (rc != GDN_OK) return rc;
    e = cudaEventRecord(g_order_ev[dev], stream);
    return e == cudaSuccess ? GDN_OK : fail(GDN_ERR_CUDA, "call order: %s", cudaGetErrorString(e));
}

// gdn_forward on host buffers: stage the inputs in pool memory, run, copy the
// results back; `sync` waits for all of it before returning.
int host_call(const void *q, const void *k, const void *v, const float *beta, const float *decay,
              const float *state_in, float *state_out, void *o, int B, int H, int T, int dk, int dv,
              int mode, void *stream_, bool sync, const char *name)
{
    try {
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        cudaStream_t stream = static_cast<cudaStream_t>(stream_);
        const size_t BH = (size_t)B * H, es = dtype_size(mode);
        const size_t nqk = BH * T * dk * es, nv = BH * T * dv * es, ng = BH * T * sizeof(float);
        const size_t nst = BH * (size_t)dk * dv * sizeof(float);
        const size_t nso = nst * ((mode & GDN_BIDI) ? 2 : 1);
        // one device block, 256-byte aligned sub-buffers
        auto up = [](size_t n) { return (n + 255) & ~(size_t)255; };
        const size_t total = 2 * up(nqk) + 2 * up(nv) + 2 * up(ng) + (state_in ? up(nst) : 0) +
                             (state_out ? up(nso) : 0);
        char *base = nullptr;
        cudaError_t e = gdn::ws_alloc(reinterpret_cast<void **>(&base), total, stream);
        if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "device buffers: %s", cudaGetErrorString(e));
        char *p = base;
        auto take = [&p, &up](size_t n) { char *r = p; p += up(n); return r; };
        char *dq = take(nqk), *dk_ = take(nqk), *dv_ = take(nv), *dout = take(nv);
        float *db = reinterpret_cast<float *>(take(ng)), *da = reinterpret_cast<float *>(take(ng));
        float *dsi = state_in ? reinterpret_cast<float *>(take(nst)) : nullptr;
        float *dso = state_out ? reinterpret_cast<float *>(take(nso)) : nullptr;

        struct Cp { void *dst; const void *src; size_t n; };
        const Cp h2d[] = {{dq, q, nqk}, {dk_, k, nqk}, {dv_, v, nv}, {db, beta, ng}, {da, decay, ng},
                          {dsi, state_in, dsi ? nst : 0}};
        for (const Cp &c : h2d)
            if (c.n && e == cudaSuccess)
                e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, stream);
        if (e != cudaSuccess) rc = fail(GDN_ERR_CUDA, "host->device copy: %s", cudaGetErrorString(e));
        if (rc == GDN_OK) {
            gdn::FwdArgs a = make_args(dq, dk_, dv_, db, da, dsi, dso, dout, B, H, T, dk, dv, mode);
            rc = ordered_dispatch(a, mode, stream);
        }
        if (rc == GDN_OK) {
            e = cudaMemcpyAsync(o, dout, nv, cudaMemcpyDeviceToHost, stream);
            if (e == cudaSuccess && dso)
                e = cudaMemcpyAsync(state_out, dso, nso, cudaMemcpyDeviceToHost, stream);
            if (e != cudaSuccess) rc = fail(GDN_ERR_CUDA, "device->host copy: %s", cudaGetErrorString(e));
        }
        e = gdn::ws_free(base, stream);
        cudaError_t es2 = sync ? cudaStreamSynchronize(stream) : cudaSuccess;
        if (rc == GDN_OK && (e != cudaSuccess || es2 != cudaSuccess))
            rc = fail(GDN_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e != cudaSuccess ? e : es2));
        return rc == GDN_OK ? ok() : rc;
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in %s", name);
    }
}


}  // namespace

extern "C" {

int gdn_version(void) { return 10000; }

const char *gdn_last_error(void) { return g_msg; }

int gdn_forward(const void *q, const void *k, const void *v, const float *beta,
                const float *decay, const float *state_in, float *state_out, void *o,
                int B, int H, int T, int dk, int dv, int mode, void *stream)
{
    try {
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        gdn::FwdArgs a = make_args(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                                   mode);
        return dispatch(a, mode, static_cast<cudaStream_t>(stream));
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_forward");
    }
}

int gdn_rollout(const void *q, const void *k, const void *v, const float *beta,
                const float *decay, const float *state_in, float *state_out,
                float *chunk_states, void *o, int B, int H, int n_chunks, int Tc, int dk,
                int dv, int mode, void *stream_)
{
    try {
        if (n_chunks <= 0) return fail(GDN_ERR_INVALID_ARG, "n_chunks must be positive");
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, Tc, dk, dv,
                              mode, "Tc");
        if (rc != GDN_OK) return rc;
        if (misaligned(chunk_states))
            return fail(GDN_ERR_MISALIGNED, "chunk_states is not 16-byte aligned");
        if (mode & GDN_BIDI)
            return fail(GDN_ERR_UNSUPPORTED, "gdn_rollout is causal only (GDN_BIDI given)");
        cudaStream_t stream = static_cast<cudaStream_t>(stream_);
        const size_t BH = (size_t)B * H;
        const size_t st = (size_t)dk * dv;
        const size_t es = dtype_size(mode);
        const size_t tok = BH * (size_t)Tc;

        float *ws = nullptr;   // ping-pong states when the caller keeps none
        if (n_chunks > 1 && !chunk_states) {
            cudaError_t e = gdn::ws_alloc(reinterpret_cast<void **>(&ws), 2 * BH * st * sizeof(float),
                                            stream);
            if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "workspace: %s", cudaGetErrorString(e));
        }
        const float *cur = state_in;
        rc = GDN_OK;
        for (int c = 0; c < n_chunks && rc == GDN_OK; ++c) {
            float *dst;
            if (chunk_states) dst = chunk_states + (size_t)c * BH * st;
            else if (c == n_chunks - 1) dst = state_out;
            else dst = ws + (size_t)(c & 1) * BH * st;
            const size_t off = (size_t)c * tok;
            gdn::FwdArgs a = make_args(
                static_cast<const char *>(q) + off * dk * es, static_cast<const char *>(k) + off * dk * es,
                static_cast<const char *>(v) + off * dv * es, beta + off, decay + off, cur, dst,
                static_cast<char *>(o) + off * dv * es, B, H, Tc, dk, dv, mode);
            rc = dispatch(a, mode, stream);
            cur = dst;
        }
        if (rc == GDN_OK && chunk_states && state_out) {
            cudaError_t e = cudaMemcpyAsync(state_out, chunk_states + (size_t)(n_chunks - 1) * BH * st,
                                            BH * st * sizeof(float), cudaMemcpyDeviceToDevice, stream);
            if (e != cudaSuccess) rc = fail(GDN_ERR_CUDA, "state copy: %s", cudaGetErrorString(e));
        }
        if (ws) {
            cudaError_t e = gdn::ws_free(ws, stream);
            if (rc == GDN_OK && e != cudaSuccess) rc = fail(GDN_ERR_CUDA, "workspace free: %s", cudaGetErrorString(e));
        }
        return rc == GDN_OK ? ok() : rc;
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_rollout");
    }
}

int gdn_forward_host(const void *q, const void *k, const void *v, const float *beta,
                     const float *decay, const float *state_in, float *state_out, void *o,
                     int B, int H, int T, int dk, int dv, int mode, void *stream)
{
    return host_call(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv, mode, stream, true,
                     "gdn_forward_host");
}

int gdn_forward_host_async(const void *q, const void *k, const void *v, const float *beta,
                           const float *decay, const float *state_in, float *state_out, void *o,
                           int B, int H, int T, int dk, int dv, int mode, void *stream)
{
    return host_call(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv, mode, stream, false,
                     "gdn_forward_host_async");
}

int gdn_forward_noalloc(const void *q, const void *k, const void *v, const float *beta,
                        const float *decay, const float *state_in, float *state_out, void *o,
                        int B, int H, int T, int dk, int dv, int mode, void *stream)
{
    try {
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        if (mode & (GDN_FP32 | GDN_RECURRENT))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_noalloc runs the bf16 chunkwise kernel only (no GDN_FP32 / "
                        "GDN_RECURRENT)");
        gdn::FwdArgs a = make_args(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                                   mode);
        if (!gdn::chunk_tc_supported(a))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_noalloc needs dk = 128 and dv in {64, 128} (got dk=%d, dv=%d)",
                        dk, dv);
        if (a.bidi) {
            const size_t need = (size_t)B * H * (size_t)((T + 63) / 64) * (size_t)(dv / 64);
            if (need > gdn::noalloc_capacity())
                return fail(GDN_ERR_UNSUPPORTED,
                            "gdn_forward_noalloc: bidirectional call needs %zu arrival counters "
                            "(B*H*ceil(T/64)*dv/64) but the static scratch holds %zu; split the "
                            "batch or use gdn_forward", need, gdn::noalloc_capacity());
        }
        cudaError_t err = gdn::launch_chunk_tc_noalloc(a, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return fail(GDN_ERR_CUDA, "launch failed: %s", cudaGetErrorString(err));
        return ok();
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_forward_noalloc");
    }
}

int gdn_forward_segmented(const void *q, const void *k, const void *v, const float *beta,
                          const float *decay, const float *state_in, float *state_out, void *o,
                          int B, int H, int T, int dk, int dv, int n_segments, int mode,
                          void *stream)
{
    try {
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        if (n_segments < 1) return fail(GDN_ERR_INVALID_ARG, "n_segments must be >= 1 (got %d)", n_segments);
        if (mode & (GDN_BIDI | GDN_FP32 | GDN_RECURRENT))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_segmented is causal and runs the bf16 chunkwise kernel only "
                        "(no GDN_BIDI / GDN_FP32 / GDN_RECURRENT)");
        gdn::FwdArgs a = make_args(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                                   mode);
        if (!gdn::chunk_tc_supported(a))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_segmented needs dk = 128 and dv in {64, 128} (got dk=%d, dv=%d)",
                        dk, dv);
        int seg_chunks = 0;
        const int S = gdn::segment_count(T, n_segments, &seg_chunks);
        if ((long long)B * H * S > 65535)
            return fail(GDN_ERR_UNSUPPORTED, "B*H*segments = %lld exceeds 65535", (long long)B * H * S);
        cudaError_t err = gdn::launch_segmented(a, n_segments, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return fail(GDN_ERR_CUDA, "launch failed: %s", cudaGetErrorString(err));
        return ok();
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_forward_segmented");
    }
}

int gdn_forward_blockcausal(const void *q, const void *k, const void *v, const float *beta,
                            const float *decay, const float *state_in, float *state_out, void *o,
                            int B, int H, int T, int dk, int dv, int block, int mode, void *stream)
{
    try {
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        if (block < 1 || T % block != 0)
            return fail(GDN_ERR_INVALID_ARG, "block must be >= 1 and divide T (got block=%d, T=%d)", block, T);
        if (mode & (GDN_BIDI | GDN_FP32 | GDN_RECURRENT))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_blockcausal is causal and runs the bf16 chunkwise kernel only "
                        "(no GDN_BIDI / GDN_FP32 / GDN_RECURRENT)");
        gdn::FwdArgs a = make_args(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                                   mode);
        if (!gdn::chunk_tc_supported(a))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_blockcausal needs dk = 128 and dv in {64, 128} (got dk=%d, dv=%d)",
                        dk, dv);
        if ((long long)B * H * (T / block) > 65535)
            return fail(GDN_ERR_UNSUPPORTED, "B*H*T/block = %lld exceeds 65535",
                        (long long)B * H * (T / block));
        cudaError_t err = gdn::launch_blockcausal(a, block, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return fail(GDN_ERR_CUDA, "launch failed: %s", cudaGetErrorString(err));
        return ok();
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_forward_blockcausal");
    }
}

int gdn_forward_normalized(const void *q, const void *k, const void *v, const float *beta,
                           const float *decay, const float *state_in, const float *state_z_in,
                           float *state_out, float *state_z_out, void *o, int B, int H, int T, int dk,
                           int dv, float eps, int mode, void *stream)
{
    try {
        int rc = check_common(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        if ((reinterpret_cast<uintptr_t>(state_z_in) | reinterpret_cast<uintptr_t>(state_z_out)) & 15)
            return fail(GDN_ERR_MISALIGNED, "state_z_in / state_z_out is not 16-byte aligned");
        if (mode & (GDN_FP32 | GDN_RECURRENT))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_normalized runs the bf16 chunkwise kernel only (no GDN_FP32 / "
                        "GDN_RECURRENT)");
        gdn::FwdArgs a = make_args(q, k, v, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                                   mode);
        if (!gdn::chunk_tc_supported(a))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_normalized needs dk = 128 and dv in {64, 128} (got dk=%d, dv=%d)",
                        dk, dv);
        cudaError_t err = gdn::launch_normalized(a, state_z_in, state_z_out, eps,
                                                 static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return fail(GDN_ERR_CUDA, "launch failed: %s", cudaGetErrorString(err));
        return ok();
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_forward_normalized");
    }
}

int gdn_forward_fp8(const void *q8, const void *k8, const void *v8, const float *q_scale,
                    const float *k_scale, const float *v_scale, const float *beta, const float *decay,
                    const float *state_in, float *state_out, void *o, int B, int H, int T, int dk, int dv,
                    int mode, void *stream)
{
    try {
        int rc = check_common(q8, k8, v8, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                              mode, "T");
        if (rc != GDN_OK) return rc;
        if (!q_scale || !k_scale || !v_scale)
            return fail(GDN_ERR_INVALID_ARG, "q_scale, k_scale and v_scale must be non-NULL");
        if (mode & (GDN_FP32 | GDN_RECURRENT))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_fp8 takes E4M3 inputs and writes bf16 o (no GDN_FP32 / GDN_RECURRENT)");
        gdn::FwdArgs a = make_args(q8, k8, v8, beta, decay, state_in, state_out, o, B, H, T, dk, dv,
                                   mode);
        if (!gdn::chunk_tc_supported(a))
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_forward_fp8 needs dk = 128 and dv in {64, 128} (got dk=%d, dv=%d)", dk, dv);
        cudaError_t err = gdn::launch_fp8(a, q_scale, k_scale, v_scale, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return fail(GDN_ERR_CUDA, "launch failed: %s", cudaGetErrorString(err));
        return ok();
    } catch (...) {
        return fail(GDN_ERR_CUDA, "internal error in gdn_forward_fp8");
    }
}

int gdn_device_status(void *stream)
{
    int err = 0;
    cudaError_t e = gdn::read_and_clear_device_error(static_cast<cudaStream_t>(stream), &err);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "device status: %s", cudaGetErrorString(e));
    if (err) return fail(GDN_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up (code %d)", err);
    return ok();
}

int gdn_debug_wait_limit(unsigned long long ns)
{
    const unsigned long long v = ns ? ns : 4000000000ull;
    cudaError_t e = gdn::set_wait_limit_pool(v);
    if (e == cudaSuccess) e = gdn::set_wait_limit_tc(v);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "wait limit: %s", cudaGetErrorString(e));
    return ok();
}

int gdn_workspace_release(int device)
{
    cudaError_t e = gdn::ws_release(device);
    if (e == cudaErrorInvalidDevice) return fail(GDN_ERR_INVALID_ARG, "no device %d", device);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "workspace release: %s", cudaGetErrorString(e));
    return ok();
}

int gdn_workspace_reserved(int device, unsigned long long *bytes)
{
    if (!bytes) return fail(GDN_ERR_INVALID_ARG, "bytes must be non-NULL");
    uint64_t v = 0;
    cudaError_t e = gdn::ws_reserved(device, &v);
    *bytes = v;
    if (e == cudaErrorInvalidDevice) return fail(GDN_ERR_INVALID_ARG, "no device %d", device);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "workspace size: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"
