/*
 * gdn_debug.h -- test and profiling hooks of libgdn.  Not part of the
 * operation's ABI (gdn.h): they change how the next calls of this process run
 * (which kernel, where intermediate values go, how long a device wait lasts),
 * never what a call computes when they are off.  All are off by default, are
 * process-wide (not per thread), and must not be changed while a call that
 * they affect is in flight.
 */
#ifndef GDN_DEBUG_H_
#define GDN_DEBUG_H_

#ifdef __cplusplus
extern "C" {
#endif

/*
 * gdn_debug_kernel_select -- which chunkwise kernel bf16 calls use: 0 (default)
 * chooses by shape (the pooled kernel for whole sequences with dk = dv = 128,
 * the single-CTA kernel otherwise); 1 forces the single-CTA kernel for every
 * bf16 call.  Other values act as 0.
 */
void gdn_debug_kernel_select(int which);

/*
 * gdn_debug_ring -- a device buffer of at least dirs*B*H*8*33792 bytes (dirs
 * = 2 for GDN_BIDI, else 1) that the pooled kernel uses as its operand ring
 * instead of workspace, so that a test can read back the operands prepared
 * for each scan's last eight chunks.  NULL (default) turns it off.  Caller-owned.
 */
void gdn_debug_ring(void *device_buffer);

/*
 * gdn_debug_dump -- a device buffer of 53248 floats where the next chunkwise
 * launches write the first chunk's intermediates of their first scan, in
 * builds with GDN_DEBUG_DUMP (ignored otherwise).  NULL (default) turns it off.
 */
void gdn_debug_dump(float *device_buffer);

/*
 * gdn_debug_profile -- a device buffer of long longs (zeroed by the caller)
 * for per-phase clock64() marks, in builds with GDN_PROFILE or GDN_TRACE
 * (ignored otherwise).  NULL (default) turns it off.
 */
void gdn_debug_profile(long long *device_buffer);

/*
 * gdn_debug_stall -- chunk c >= 0 makes scan 0's state chain in the pooled
 * kernel wait for chunk c's operands with a target that nothing reaches, so
 * that the wait runs out, the kernel records GDN_ERR_DEVICE_TIMEOUT in the
 * device error word and returns; -1 (default) turns it off.  Combine with
 * gdn_debug_wait_limit to keep the run short.
 */
void gdn_debug_stall(int chunk);

/*
 * gdn_debug_plain_launch -- 1 launches the pooled kernel without the
 * cooperative attribute (same grid: one CTA per SM), for profilers that replay
 * one launch at a time with the GPU otherwise idle; 0 (default) restores the
 * cooperative launch, which guarantees that every CTA is resident.
 */
void gdn_debug_plain_launch(int on);

/*
 * gdn_debug_wait_limit -- the limit, in nanoseconds, of every bounded wait in
 * the chunkwise kernels on the current device; 0 restores the default (4 s).
 * Synchronous.  Returns GDN_OK or GDN_ERR_CUDA.
 */
int gdn_debug_wait_limit(unsigned long long ns);

#ifdef __cplusplus
}
#endif

#endif /* GDN_DEBUG_H_ */
