"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments with the documented codes before
launching anything.  No call here reaches a CUDA API (every case fails
validation first), so these run without a GPU."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_149_b200 import build, gdn
    build.build()
    return gdn.load_library()


def declared_functions(header=None):
    names = set()
    for h in ([header] if header else sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))):
        src = open(os.path.join(ROOT, "include", h) if header else h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names.update(re.findall(r"^[A-Za-z_][\w ]*[\s*]+(gdn_\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_header_declares_the_abi():
    names = declared_functions("gdn.h")
    for n in ("gdn_forward", "gdn_rollout", "gdn_forward_host", "gdn_forward_host_async", "gdn_forward_noalloc",
              "gdn_forward_segmented", "gdn_forward_blockcausal", "gdn_forward_normalized",
              "gdn_forward_fp8",
              "gdn_device_status",
              "gdn_kernel_launches", "gdn_workspace_release", "gdn_workspace_reserved",
              "gdn_last_error", "gdn_version"):
        assert n in names


def test_debug_header_declares_the_hooks():
    names = declared_functions("gdn_debug.h")
    assert names == sorted(["gdn_debug_kernel_select", "gdn_debug_ring", "gdn_debug_dump", "gdn_debug_profile",
                            "gdn_debug_stall", "gdn_debug_plain_launch", "gdn_debug_wait_limit"])


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in a header under include/ but not exported"


def test_version(lib):
    assert lib.gdn_version() >= 10000


# Fake but 16-byte-aligned addresses: never dereferenced, because every case
# below fails host-side validation before any CUDA call.
P = ctypes.c_void_p(0x10000)
PM = ctypes.c_void_p(0x10008)   # misaligned


def fwd(lib, q=P, k=P, v=P, beta=P, decay=P, sin=None, sout=None, o=P,
        B=1, H=1, T=64, dk=128, dv=128, mode=0):
    return lib.gdn_forward(q, k, v, beta, decay, sin, sout, o, B, H, T, dk, dv, mode, None)


@pytest.mark.parametrize("which", ["q", "k", "v", "beta", "decay", "o"])
def test_null_required_pointer(lib, which):
    rc = fwd(lib, **{which: None})
    assert rc == -1 and b"non-NULL" in lib.gdn_last_error()


@pytest.mark.parametrize("B,H,T", [(0, 1, 1), (1, 0, 1), (1, 1, 0), (1, 1, -5), (-1, 2, 3)])
def test_nonpositive_sizes(lib, B, H, T):
    assert fwd(lib, B=B, H=H, T=T) == -1


def test_bad_mode_bits(lib):
    assert fwd(lib, mode=8) == -1
    assert b"mode" in lib.gdn_last_error()


@pytest.mark.parametrize("dk,dv", [(48, 128), (128, 40), (160, 128), (128, 256), (0, 64), (16, 16)])
def test_unsupported_head_dims(lib, dk, dv):
    assert fwd(lib, dk=dk, dv=dv) == -2


def test_too_many_heads(lib):
    assert fwd(lib, B=256, H=256) == -2


@pytest.mark.parametrize("which", ["q", "k", "v", "beta", "decay", "o", "sin", "sout"])
def test_misaligned_pointer(lib, which):
    rc = fwd(lib, **{which: PM})
    assert rc == -3 and b"aligned" in lib.gdn_last_error()


def test_rollout_rejects_bidi_and_bad_chunks(lib):
    r = lambda **kw: lib.gdn_rollout(P, P, P, P, P, None, None, kw.get("cs"), P, 1, 1,
                                     kw.get("n", 2), 64, 128, 128, kw.get("mode", 0), None)
    assert r(mode=1) == -2
    assert r(n=0) == -1
    assert r(cs=PM) == -3


def test_host_entry_validates_first(lib):
    for fn in (lib.gdn_forward_host, lib.gdn_forward_host_async):
        assert fn(None, P, P, P, P, None, None, P, 1, 1, 64, 128, 128, 0, None) == -1
        assert fn(P, P, P, P, P, None, None, P, 1, 1, 0, 128, 128, 0, None) == -1
        assert fn(P, P, P, P, P, None, None, PM, 1, 1, 64, 128, 128, 0, None) == -3


def test_last_error_is_per_call(lib):
    fwd(lib, B=0)
    assert lib.gdn_last_error() != b""


def test_noalloc_rejects_before_launch(lib):
    """The allocation-free entry point refuses what its static scratch cannot
    hold, and the modes it does not run, before any CUDA call."""
    f = lambda T=64, dk=128, dv=128, mode=1: lib.gdn_forward_noalloc(
        P, P, P, P, P, None, None, P, 1, 1, T, dk, dv, mode, None)
    assert f(T=64 * 262145) == -2                      # 524290 counters > 262144
    assert b"262144" in lib.gdn_last_error()
    assert f(mode=1 | 2) == -2                          # fp32
    assert f(mode=1 | 4) == -2                          # recurrent kernel
    assert f(dk=64) == -2
    assert f(T=0) == -1


def test_segmented_rejects_before_launch(lib):
    """The segment-parallel entry point is causal, bf16 chunkwise only, and
    needs at least one segment; each refusal happens before any CUDA call."""
    f = lambda T=640, dk=128, dv=128, nseg=4, mode=0: lib.gdn_forward_segmented(
        P, P, P, P, P, None, None, P, 1, 1, T, dk, dv, nseg, mode, None)
    assert f(nseg=0) == -1 and b"n_segments" in lib.gdn_last_error()
    assert f(mode=1) == -2                               # bidirectional
    assert f(mode=2) == -2                               # fp32
    assert f(mode=4) == -2                               # recurrent kernel
    assert f(dk=64) == -2
    assert f(dv=96) == -2
    assert f(T=0) == -1
    assert lib.gdn_forward_segmented(P, P, P, P, P, None, None, P, 1, 64, 64 * 4000, 128, 128, 2000, 0,
                                     None) == -2         # B*H*segments > 65535


def test_blockcausal_rejects_before_launch(lib):
    """The frame-block entry point needs a block that divides T, runs causal
    bf16 chunkwise only, and refuses each bad case before any CUDA call."""
    f = lambda T=640, dk=128, dv=128, block=64, mode=0: lib.gdn_forward_blockcausal(
        P, P, P, P, P, None, None, P, 1, 1, T, dk, dv, block, mode, None)
    assert f(block=0) == -1 and b"block" in lib.gdn_last_error()
    assert f(block=100) == -1                            # 640 is not a multiple of 100
    assert f(mode=1) == -2                               # bidirectional
    assert f(mode=2) == -2                               # fp32
    assert f(dk=64) == -2
    assert f(T=70000, block=1) == -2                     # 70000 blocks > 65535


def test_normalized_rejects_before_launch(lib):
    """The normalised read-out runs the bf16 chunkwise kernel only and checks
    its z-state pointers, before any CUDA call."""
    f = lambda dk=128, dv=128, mode=0, zin=None, zout=None: lib.gdn_forward_normalized(
        P, P, P, P, P, None, zin, None, zout, P, 1, 1, 640, dk, dv, ctypes.c_float(1e-6), mode, None)
    assert f(mode=2) == -2                               # fp32
    assert f(mode=4) == -2                               # recurrent kernel
    assert f(dk=64) == -2
    assert f(zin=PM) == -3 and b"state_z" in lib.gdn_last_error()
    assert f(zout=PM) == -3


def test_fp8_rejects_before_launch(lib):
    """The fp8 entry point needs its three scales and runs bf16-output chunkwise
    shapes only; each refusal happens before any CUDA call."""
    f = lambda sq=P, dk=128, dv=128, mode=0: lib.gdn_forward_fp8(
        P, P, P, sq, P, P, P, P, None, None, P, 1, 1, 640, dk, dv, mode, None)
    assert f(sq=None) == -1 and b"scale" in lib.gdn_last_error()
    assert f(mode=2) == -2
    assert f(mode=4) == -2
    assert f(dk=64) == -2


def test_workspace_calls_validate_and_start_empty(lib):
    """Bad device indices and a NULL out-pointer are rejected before any CUDA
    call; a pool no call has used reports 0 bytes and releases as a no-op."""
    v = ctypes.c_ulonglong(123)
    for dev in (-1, 64):
        assert lib.gdn_workspace_reserved(dev, ctypes.byref(v)) == -1
        assert lib.gdn_workspace_release(dev) == -1
    assert lib.gdn_workspace_reserved(0, None) == -1
    assert lib.gdn_workspace_reserved(0, ctypes.byref(v)) == 0 and v.value == 0
    assert lib.gdn_workspace_release(0) == 0

