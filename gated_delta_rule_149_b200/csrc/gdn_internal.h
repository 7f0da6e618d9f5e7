// Internal declarations shared by the libgdn translation units.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace gdn {

// One forward/bidi pass, already validated on the host.
struct FwdArgs {
    const void *q, *k, *v;
    const float *beta, *decay;
    const float *state_in;    // [B,H,dk,dv] or nullptr
    float *state_out;         // causal [B,H,dk,dv]; bidi [2,B,H,dk,dv]; or nullptr
    void *o;                  // [B,H,T,dv]
    int B, H, T, dk, dv;
    bool bidi;
    bool fp32;                // q/k/v/o dtype: fp32 (else bf16)
    // Segments (chunkwise kernel, causal only): the launch runs n_seg
    // consecutive segments seg0 .. seg0 + n_seg - 1 of seg_chunks 64-token
    // chunks of every head (the last one may be shorter); state_in/state_out
    // then hold one [dk][dv] state per (head, segment), head-major.
    // seg_chunks = 0: one segment, the whole sequence.
    int seg0 = 0, n_seg = 1, seg_chunks = 0;
};

// Token-by-token fp32 SIMT kernel (any dtype; dk, dv multiples of 32, <= 128).
cudaError_t launch_recurrent(const FwdArgs &a, cudaStream_t stream);

// Chunkwise tcgen05 kernel (bf16; dk = 128; dv in {64, 128}).
bool chunk_tc_supported(const FwdArgs &a);
cudaError_t launch_chunk_tc(const FwdArgs &a, cudaStream_t stream);

// Chunkwise kernel with one CTA per SM: a state chain per scan beside a pool of
// preparation workers that serve every scan (bf16, dk = dv = 128, whole
// sequences, no segments).  launch_chunk_tc hands such calls to it.
bool chunk_pool_supported(const FwdArgs &a);
// The pooled chunkwise kernel; with q_scale (and k_scale, v_scale) given, a.q,
// a.k and a.v are E4M3 codes with one fp32 scale per head, widened in-kernel.
cudaError_t launch_chunk_pool(const FwdArgs &a, cudaStream_t stream, const float *q_scale = nullptr,
                              const float *k_scale = nullptr, const float *v_scale = nullptr);

// Allocation-free variant of launch_chunk_tc: the bidirectional arrival
// counters come from a fixed static device array of noalloc_capacity() ints.
size_t noalloc_capacity();
cudaError_t launch_chunk_tc_noalloc(const FwdArgs &a, cudaStream_t stream);

// Segment-parallel causal scan (chunkwise kernel): splits each head's sequence
// into about n_segments whole-chunk segments, runs them in parallel and threads
// the state through them (three kernel passes and a combine).  segment_count
// returns the number of segments used and their length in chunks.
int segment_count(int T, int n_segments, int *seg_chunks);
cudaError_t launch_segmented(const FwdArgs &a, int n_segments, cudaStream_t stream);

// Frame-block read-out (chunkwise kernel, causal): every token of block f of
// `block` tokens is read out with the state after the whole block.  T must be
// a multiple of block.
cudaError_t launch_blockcausal(const FwdArgs &a, int block, cudaStream_t stream);

// Normalised read-out o = (S q) / (z.q + eps), z the same recurrence driven by a
// value of 1; state_z_in [B,H,dk] or nullptr, state_z_out [B,H,dk] (bidi
// [2,B,H,dk]) or nullptr.
cudaError_t launch_normalized(const FwdArgs &a, const float *state_z_in, float *state_z_out, float eps,
                              cudaStream_t stream);

// fp8 (E4M3) q, k, v with per-(batch, head) fp32 scales: dequantised to bf16
// workspace copies, then the chunkwise kernel (a.q, a.k, a.v are the fp8 codes).
cudaError_t launch_fp8(const FwdArgs &a, const float *q_scale, const float *k_scale, const float *v_scale,
                       cudaStream_t stream);

// Scratch memory: stream-ordered allocations from the library's own pool on
// the current device, which keeps its reservation across synchronisations;
// ws_release trims it to nothing, ws_reserved reads its size.
cudaError_t ws_alloc(void **ptr, size_t bytes, cudaStream_t stream);
cudaError_t ws_free(void *ptr, cudaStream_t stream);
cudaError_t ws_release(int dev);
cudaError_t ws_reserved(int dev, uint64_t *bytes);

// Device-side error word (set by bounded waits that gave up).
cudaError_t device_error_word(int **ptr);

// The limit of the bounded waits in the chunkwise kernels (each module holds
// its own copy), on the current device.
cudaError_t set_wait_limit_pool(unsigned long long ns);
cudaError_t set_wait_limit_tc(unsigned long long ns);

// Launch accounting (gdn_kernel_launches).
void count_launches(int n);
cudaError_t read_and_clear_device_error(cudaStream_t stream, int *err);

}  // namespace gdn
