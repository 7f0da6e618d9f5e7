"""Thin ctypes binding of libgdn's C ABI (argument marshalling only).

Every function takes torch tensors, checks dtype/shape/device/contiguity,
and passes raw pointers and sizes to the library; all computation happens in
the library's CUDA kernels.  There is no CPU or fallback path: if libgdn.so
cannot be loaded, calls raise.
"""
import ctypes
import os

import torch

GDN_CAUSAL = 0
GDN_BIDI = 1
GDN_BF16 = 0
GDN_FP32 = 2
GDN_RECURRENT = 4

_STATUS = {0: "GDN_OK", -1: "GDN_ERR_INVALID_ARG", -2: "GDN_ERR_UNSUPPORTED",
           -3: "GDN_ERR_MISALIGNED", -4: "GDN_ERR_CUDA", -5: "GDN_ERR_DEVICE_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class GDNError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{_STATUS.get(code, code)}: {msg}")
        self.code = code


def lib_path():
    return os.environ.get("GDN_LIB", os.path.join(_HERE, "lib", "libgdn.so"))


def load_library():
    """Loads libgdn.so and declares the ABI's argument types."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise GDNError(-4, f"libgdn.so not found at {path}; run "
                               f"`python -m gated_delta_rule_149_b200.build` first")
        lib = ctypes.CDLL(path)
        vp, i = ctypes.c_void_p, ctypes.c_int
        lib.gdn_forward.argtypes = [vp] * 8 + [i] * 6 + [vp]
        lib.gdn_forward.restype = i
        lib.gdn_forward_host.argtypes = [vp] * 8 + [i] * 6 + [vp]
        lib.gdn_forward_host.restype = i
        lib.gdn_forward_host_async.argtypes = [vp] * 8 + [i] * 6 + [vp]
        lib.gdn_forward_host_async.restype = i
        lib.gdn_forward_noalloc.argtypes = [vp] * 8 + [i] * 6 + [vp]
        lib.gdn_forward_noalloc.restype = i
        lib.gdn_forward_segmented.argtypes = [vp] * 8 + [i] * 7 + [vp]
        lib.gdn_forward_segmented.restype = i
        lib.gdn_forward_blockcausal.argtypes = [vp] * 8 + [i] * 7 + [vp]
        lib.gdn_forward_blockcausal.restype = i
        lib.gdn_forward_normalized.argtypes = [vp] * 10 + [i] * 5 + [ctypes.c_float, i, vp]
        lib.gdn_forward_normalized.restype = i
        lib.gdn_forward_fp8.argtypes = [vp] * 11 + [i] * 6 + [vp]
        lib.gdn_forward_fp8.restype = i
        lib.gdn_rollout.argtypes = [vp] * 9 + [i] * 7 + [vp]
        lib.gdn_rollout.restype = i
        lib.gdn_device_status.argtypes = [vp]
        lib.gdn_device_status.restype = i
        lib.gdn_last_error.argtypes = []
        lib.gdn_last_error.restype = ctypes.c_char_p
        lib.gdn_version.argtypes = []
        lib.gdn_version.restype = i
        lib.gdn_kernel_launches.argtypes = []
        lib.gdn_kernel_launches.restype = ctypes.c_longlong
        lib.gdn_workspace_release.argtypes = [i]
        lib.gdn_workspace_release.restype = i
        lib.gdn_workspace_reserved.argtypes = [i, ctypes.POINTER(ctypes.c_ulonglong)]
        lib.gdn_workspace_reserved.restype = i
        lib.gdn_debug_kernel_select.argtypes = [i]
        lib.gdn_debug_kernel_select.restype = None
        lib.gdn_debug_ring.argtypes = [vp]
        lib.gdn_debug_ring.restype = None
        lib.gdn_debug_stall.argtypes = [i]
        lib.gdn_debug_stall.restype = None
        lib.gdn_debug_plain_launch.argtypes = [i]
        lib.gdn_debug_plain_launch.restype = None
        lib.gdn_debug_wait_limit.argtypes = [ctypes.c_ulonglong]
        lib.gdn_debug_wait_limit.restype = i
        _lib = lib
    return _lib


def _check(rc):
    if rc != 0:
        raise GDNError(rc, load_library().gdn_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _mode(q, bidi, recurrent):
    if q.dtype == torch.float32:
        m = GDN_FP32
    elif q.dtype == torch.bfloat16:
        m = GDN_BF16
    else:
        raise TypeError(f"q/k/v must be bf16 or fp32, got {q.dtype}")
    return m | (GDN_BIDI if bidi else 0) | (GDN_RECURRENT if recurrent else 0)


def _expect(t, name, shape, dtype, device):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gdn_forward(q, k, v, beta, decay, state_in=None, *, bidi=False, recurrent=False,
                o=None, state_out=None, want_state=True, stream=None):
    """o, state_out = gdn_forward(q, k, v, beta, decay, state_in) on CUDA tensors.

    q, k [B,H,T,dk] and v [B,H,T,dv] (bf16 or fp32, same dtype); beta, decay
    [B,H,T] fp32; state_in [B,H,dk,dv] fp32 or None.  Returns o [B,H,T,dv]
    (dtype of q) and the final state ([B,H,dk,dv], or [2,B,H,dk,dv] for bidi:
    forward then reverse), or None if want_state is False.
    """
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_forward runs on CUDA tensors only")
    _expect(k, "k", (B, H, T, dk), q.dtype, dev)
    _expect(v, "v", (B, H, T, dv), q.dtype, dev)
    _expect(beta, "beta", (B, H, T), torch.float32, dev)
    _expect(decay, "decay", (B, H, T), torch.float32, dev)
    _expect(q, "q", (B, H, T, dk), q.dtype, dev)
    if state_in is not None:
        _expect(state_in, "state_in", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    _expect(o, "o", (B, H, T, dv), q.dtype, dev)
    s_shape = ((2,) if bidi else ()) + (B, H, dk, dv)
    if state_out is None and want_state:
        state_out = torch.empty(s_shape, dtype=torch.float32, device=dev)
    if state_out is not None:
        _expect(state_out, "state_out", s_shape, torch.float32, dev)
    lib = load_library()
    _check(lib.gdn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(state_in),
                           _ptr(state_out), _ptr(o), B, H, T, dk, dv,
                           _mode(q, bidi, recurrent), _stream_handle(stream, dev)))
    return o, state_out


def gdn_forward_segmented(q, k, v, beta, decay, state_in=None, *, n_segments=4, o=None,
                          state_out=None, want_state=True, stream=None):
    """Causal gdn_forward with each head's sequence split into about n_segments
    time segments that run in parallel (same arguments and results; bf16,
    dk = 128, dv in {64, 128})."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_forward_segmented runs on CUDA tensors only")
    for t, name, shape, dt in ((k, "k", (B, H, T, dk), q.dtype), (v, "v", (B, H, T, dv), q.dtype),
                               (beta, "beta", (B, H, T), torch.float32),
                               (decay, "decay", (B, H, T), torch.float32), (q, "q", (B, H, T, dk), q.dtype)):
        _expect(t, name, shape, dt, dev)
    if state_in is not None:
        _expect(state_in, "state_in", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    _expect(o, "o", (B, H, T, dv), q.dtype, dev)
    if state_out is None and want_state:
        state_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    if state_out is not None:
        _expect(state_out, "state_out", (B, H, dk, dv), torch.float32, dev)
    lib = load_library()
    _check(lib.gdn_forward_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(state_in),
                                     _ptr(state_out), _ptr(o), B, H, T, dk, dv, int(n_segments),
                                     _mode(q, False, False), _stream_handle(stream, dev)))
    return o, state_out


def gdn_forward_blockcausal(q, k, v, beta, decay, state_in=None, *, block, o=None,
                            state_out=None, want_state=True, stream=None):
    """Frame-block causal read-out: every token of block f (frames of `block`
    tokens, T a multiple of it) is read out with the state after the whole
    block.  Arguments and layouts as gdn_forward (bf16, dk = 128, dv in
    {64, 128}); returns o and the final state."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_forward_blockcausal runs on CUDA tensors only")
    for t, name, shape, dt in ((k, "k", (B, H, T, dk), q.dtype), (v, "v", (B, H, T, dv), q.dtype),
                               (beta, "beta", (B, H, T), torch.float32),
                               (decay, "decay", (B, H, T), torch.float32), (q, "q", (B, H, T, dk), q.dtype)):
        _expect(t, name, shape, dt, dev)
    if state_in is not None:
        _expect(state_in, "state_in", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    _expect(o, "o", (B, H, T, dv), q.dtype, dev)
    if state_out is None and want_state:
        state_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    if state_out is not None:
        _expect(state_out, "state_out", (B, H, dk, dv), torch.float32, dev)
    lib = load_library()
    _check(lib.gdn_forward_blockcausal(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(state_in),
                                       _ptr(state_out), _ptr(o), B, H, T, dk, dv, int(block),
                                       _mode(q, False, False), _stream_handle(stream, dev)))
    return o, state_out


def gdn_forward_normalized(q, k, v, beta, decay, state_in=None, state_z_in=None, *, eps=1e-6,
                           bidi=False, o=None, stream=None):
    """Normalised read-out o = (S q) / (z.q + eps), z the same recurrence driven
    by a value of 1.  Arguments as gdn_forward (bf16, dk = 128, dv in
    {64, 128}) plus state_z_in [B,H,dk] fp32 or None.  Returns o, the kv state
    and the z state ([B,H,dk], bidi [2,B,H,dk])."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_forward_normalized runs on CUDA tensors only")
    for t, name, shape, dt in ((k, "k", (B, H, T, dk), q.dtype), (v, "v", (B, H, T, dv), q.dtype),
                               (beta, "beta", (B, H, T), torch.float32),
                               (decay, "decay", (B, H, T), torch.float32), (q, "q", (B, H, T, dk), q.dtype)):
        _expect(t, name, shape, dt, dev)
    if state_in is not None:
        _expect(state_in, "state_in", (B, H, dk, dv), torch.float32, dev)
    if state_z_in is not None:
        _expect(state_z_in, "state_z_in", (B, H, dk), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    _expect(o, "o", (B, H, T, dv), q.dtype, dev)
    lead = (2,) if bidi else ()
    s_kv = torch.empty(lead + (B, H, dk, dv), dtype=torch.float32, device=dev)
    s_z = torch.empty(lead + (B, H, dk), dtype=torch.float32, device=dev)
    lib = load_library()
    _check(lib.gdn_forward_normalized(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(state_in),
                                      _ptr(state_z_in), _ptr(s_kv), _ptr(s_z), _ptr(o), B, H, T, dk, dv,
                                      ctypes.c_float(eps), _mode(q, bidi, False), _stream_handle(stream, dev)))
    return o, s_kv, s_z


def gdn_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, beta, decay, state_in=None, *, bidi=False,
                    o=None, state_out=None, want_state=True, stream=None):
    """gdn_forward on fp8 (E4M3) q, k, v given as uint8 codes [B,H,T,d] with
    fp32 scales [B,H] (x = scale * decode(x8)); o is bf16."""
    B, H, T, dk = q8.shape
    dv = v8.shape[-1]
    dev = q8.device
    if dev.type != "cuda":
        raise ValueError("gdn_forward_fp8 runs on CUDA tensors only")
    for t, name, shape, dt in ((q8, "q8", (B, H, T, dk), torch.uint8), (k8, "k8", (B, H, T, dk), torch.uint8),
                               (v8, "v8", (B, H, T, dv), torch.uint8),
                               (q_scale, "q_scale", (B, H), torch.float32), (k_scale, "k_scale", (B, H), torch.float32),
                               (v_scale, "v_scale", (B, H), torch.float32),
                               (beta, "beta", (B, H, T), torch.float32), (decay, "decay", (B, H, T), torch.float32)):
        _expect(t, name, shape, dt, dev)
    if state_in is not None:
        _expect(state_in, "state_in", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=torch.bfloat16, device=dev)
    _expect(o, "o", (B, H, T, dv), torch.bfloat16, dev)
    s_shape = ((2,) if bidi else ()) + (B, H, dk, dv)
    if state_out is None and want_state:
        state_out = torch.empty(s_shape, dtype=torch.float32, device=dev)
    if state_out is not None:
        _expect(state_out, "state_out", s_shape, torch.float32, dev)
    lib = load_library()
    _check(lib.gdn_forward_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                               _ptr(beta), _ptr(decay), _ptr(state_in), _ptr(state_out), _ptr(o),
                               B, H, T, dk, dv, GDN_BIDI if bidi else 0, _stream_handle(stream, dev)))
    return o, state_out


def gdn_rollout(q, k, v, beta, decay, state_in=None, *, recurrent=False, chunk_states=False,
                o=None, state_out=None, stream=None):
    """Streaming rollout over chunk-major inputs q,k [n,B,H,Tc,dk], v [n,B,H,Tc,dv],
    gates [n,B,H,Tc].  Returns (o, state_out, chunk_states or None)."""
    n, B, H, Tc, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn_rollout runs on CUDA tensors only")
    _expect(k, "k", (n, B, H, Tc, dk), q.dtype, dev)
    _expect(v, "v", (n, B, H, Tc, dv), q.dtype, dev)
    _expect(beta, "beta", (n, B, H, Tc), torch.float32, dev)
    _expect(decay, "decay", (n, B, H, Tc), torch.float32, dev)
    _expect(q, "q", (n, B, H, Tc, dk), q.dtype, dev)
    if state_in is not None:
        _expect(state_in, "state_in", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(n, B, H, Tc, dv, dtype=q.dtype, device=dev)
    if state_out is None:
        state_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    cs = torch.empty(n, B, H, dk, dv, dtype=torch.float32, device=dev) if chunk_states else None
    lib = load_library()
    _check(lib.gdn_rollout(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(state_in),
                           _ptr(state_out), _ptr(cs), _ptr(o), B, H, n, Tc, dk, dv,
                           _mode(q, False, recurrent), _stream_handle(stream, dev)))
    return o, state_out, cs


def gdn_forward_host(q, k, v, beta, decay, state_in=None, *, bidi=False, recurrent=False,
                     o=None, state_out=None, want_state=True, stream=None, device=None):
    """gdn_forward on CPU (ideally pinned) tensors through the library's host-buffer
    entry point: the library copies inputs in, runs, copies o/state back and
    synchronises.  Returns CPU tensors."""
    return _host(False, q, k, v, beta, decay, state_in, bidi, recurrent, o, state_out, want_state,
                 stream, device)


def gdn_forward_host_async(q, k, v, beta, decay, state_in=None, *, bidi=False, recurrent=False,
                           o=None, state_out=None, want_state=True, stream=None, device=None):
    """gdn_forward_host without the final synchronise: returns once the copies
    and kernels are enqueued on `stream`.  Keep every tensor alive and the
    outputs unread until the stream has passed the call."""
    return _host(True, q, k, v, beta, decay, state_in, bidi, recurrent, o, state_out, want_state,
                 stream, device)


def _host(asynchronous, q, k, v, beta, decay, state_in, bidi, recurrent, o, state_out, want_state,
          stream, device):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("beta", beta), ("decay", decay)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, pin_memory=q.is_pinned())
    s_shape = ((2,) if bidi else ()) + (B, H, dk, dv)
    if state_out is None and want_state:
        state_out = torch.empty(s_shape, dtype=torch.float32, pin_memory=q.is_pinned())
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    lib = load_library()
    fn = lib.gdn_forward_host_async if asynchronous else lib.gdn_forward_host
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(state_in), _ptr(state_out),
              _ptr(o), B, H, T, dk, dv, _mode(q, bidi, recurrent), _stream_handle(stream, dev)))
    return o, state_out


def gdn_device_status(stream=None, device=None):
    """Synchronises the stream and raises GDNError if a bounded device wait gave up."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check(load_library().gdn_device_status(_stream_handle(stream, dev)))


def _device_index(device):
    if device is None:
        return torch.cuda.current_device()
    if isinstance(device, int):
        return device
    d = torch.device(device)
    return torch.cuda.current_device() if d.index is None else d.index


def gdn_workspace_release(device=None):
    """Returns the library's reserved workspace memory on `device` (default: the
    current CUDA device) to the driver; synchronise its streams first."""
    _check(load_library().gdn_workspace_release(_device_index(device)))


def gdn_workspace_reserved(device=None):
    """Bytes of device memory the library's workspace pool on `device` holds."""
    v = ctypes.c_ulonglong(0)
    _check(load_library().gdn_workspace_reserved(_device_index(device), ctypes.byref(v)))
    return v.value


def debug_kernel_select(which):
    """Test hook: 0 picks the bf16 chunkwise kernel by shape (the pooled kernel
    for dk = dv = 128 whole-sequence calls), 1 forces the single-CTA chunkwise
    kernel for every bf16 call (for A/B comparisons of the two)."""
    load_library().gdn_debug_kernel_select(int(which))


def debug_ring(buf):
    """Test hook: a CUDA uint8 tensor of at least dirs*B*H*8*33792 bytes that the
    pooled kernel uses as its operand ring (None: workspace), so that the
    prepared operands of the last eight chunks of every scan can be read back."""
    load_library().gdn_debug_ring(None if buf is None else ctypes.c_void_p(buf.data_ptr()))


def debug_stall(chunk):
    """Test hook: chunk >= 0 makes scan 0's state chain of the pooled kernel wait
    for that chunk's operands with a target nothing reaches, so the wait runs
    out and the call ends with a device timeout status; -1 turns it off."""
    load_library().gdn_debug_stall(int(chunk))


def debug_plain_launch(on):
    """Test hook: launch the pooled kernel without the cooperative attribute (for
    profilers that replay one launch at a time); False restores the default."""
    load_library().gdn_debug_plain_launch(1 if on else 0)


def debug_wait_limit(ns):
    """Test hook: the limit in nanoseconds of every bounded device wait of the
    chunkwise kernels on the current device; 0 restores the default (4 s)."""
    _check(load_library().gdn_debug_wait_limit(int(ns)))
