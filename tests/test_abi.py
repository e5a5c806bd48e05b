"""The C-ABI library without a GPU: it loads, it exports every entry point the
header declares, and the host-side argument checks reject bad calls before
anything touches CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep_b200.h")


@pytest.fixture(scope="module")
def ep():
    import __graft_entry__

    __graft_entry__.build()
    import combine_get_dispatch_05_b200 as m

    return m


def _declared():
    text = open(HEADER).read()
    return re.findall(r"^EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_calls():
    names = set(_declared())
    for n in ("ep_get_dispatch_layout", "ep_dispatch", "ep_combine", "ep_low_latency_dispatch",
              "ep_low_latency_combine"):
        assert n in names


def test_library_exports_every_declared_symbol(ep):
    lib = ctypes.CDLL(ep.LIB_PATH)
    declared = _declared()
    assert declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(ep._lib.EXPORTED)


def test_built_for_sm100a_only():
    import __graft_entry__

    build = __graft_entry__._load_by_path("_ep_build_check", "combine_get_dispatch_05_b200/build.py")

    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "--use_fast_math" not in build.NVCC_FLAGS and "-prec-div=true" in build.NVCC_FLAGS


def test_version_and_strings(ep):
    assert ep.lib.ep_abi_version() == 2
    assert ep.status_string(ep.EP_ERR_SHAPE) == "unsupported size"
    assert ep.status_string(99) == "unknown status"


def test_workspace_bytes(ep):
    b = ep.ep_workspace_bytes(4096, 256, 8)
    # header + one int per (expert or partition, layout chunk of up to 128 tokens)
    assert b == ((256 + 4 * 32 * (256 + 8)) + 255) // 256 * 256
    assert ep.ep_workspace_bytes(0, 256, 8) > 0
    assert ep.ep_workspace_bytes(-1, 256, 8) == 0
    assert ep.ep_workspace_bytes(10, 0, 1) == 0
    assert ep.ep_workspace_bytes(32768, 288, 8) >= ep.ep_workspace_bytes(4096, 288, 8)


class _Fake:
    """Aligned non-null addresses: the checks below fail before any dereference."""
    P = 0x100000


def _layout_struct(ep, valid=True):
    p = _Fake.P if valid else None
    return ep._lib.ep_layout(p, p, p, p, p, p, p)


def _dispatch(ep, T=16, H=256, K=4, E=8, P=2, quant=1, ws_bytes=1 << 20, **over):
    f = _Fake.P
    args = dict(T=T, H=H, K=K, E=E, P=P, quant=quant, x=f, idx=f, w=f, rx=f, rs=f, ri=f, rw=f,
                lay=_layout_struct(ep), ws=f, ws_bytes=ws_bytes)
    args.update(over)
    lay = args["lay"]
    return ep.lib.ep_dispatch(args["T"], args["H"], args["K"], args["E"], args["P"], args["quant"],
                              args["x"], args["idx"], args["w"], args["rx"], args["rs"],
                              args["ri"], args["rw"], ctypes.byref(lay) if lay is not None else None,
                              args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("over,status", [
    (dict(K=0), 2), (dict(K=33), 2), (dict(E=7, P=2), 2), (dict(P=65, E=65 * 2), 2),
    (dict(E=4097, P=1), 2), (dict(T=-1), 2), (dict(H=200), 2), (dict(H=0), 2),
    (dict(H=16512), 2), (dict(quant=1, H=136), 2), (dict(quant=5), 1), (dict(x=None), 1),
    (dict(quant=2, H=136), 2), (dict(quant=2, rs=None), 1), (dict(quant=3), 1),
    (dict(quant=0x100), 1), (dict(quant=0x200 | 1), 1), (dict(quant=0x101, rs=None), 1),
    (dict(quant=0x102, H=136), 2),
    (dict(rs=None), 1), (dict(x=_Fake.P + 8), 1), (dict(rx=_Fake.P + 4), 1), (dict(rs=_Fake.P + 4), 1),
    (dict(ws=None), 1), (dict(ws=_Fake.P + 8), 1), (dict(lay=None), 1), (dict(ws_bytes=64), 3),
    (dict(T=1 << 28, K=8), 2),
])
def test_dispatch_host_checks(ep, over, status):
    assert _dispatch(ep, **over) == status


def test_dispatch_bf16_needs_no_scales_but_checks_hidden(ep):
    # quant NONE accepts H % 8 == 0 and a NULL recv_scales; it then reaches CUDA,
    # which on a machine without a GPU reports a runtime error, not a crash
    import torch

    st = _dispatch(ep, quant=0, H=136, rs=None)
    if torch.cuda.is_available():
        pytest.skip("only meaningful without a GPU")
    assert st == ep.EP_ERR_CUDA
    assert _dispatch(ep, quant=0, H=132) == ep.EP_ERR_SHAPE


def test_layout_host_checks(ep):
    f = _Fake.P
    lay = _layout_struct(ep)
    L = ep.lib
    assert L.ep_get_dispatch_layout(4, 0, 8, 2, f, ctypes.byref(lay), f, 1 << 20, None) == 2
    assert L.ep_get_dispatch_layout(4, 2, 8, 3, f, ctypes.byref(lay), f, 1 << 20, None) == 2
    assert L.ep_get_dispatch_layout(4, 2, 8, 2, None, ctypes.byref(lay), f, 1 << 20, None) == 1
    bad = ep._lib.ep_layout(f, f, f, f, None, f, f)
    assert L.ep_get_dispatch_layout(4, 2, 8, 2, f, ctypes.byref(bad), f, 1 << 20, None) == 1
    assert L.ep_get_dispatch_layout(4, 2, 8, 2, f, ctypes.byref(lay), f, 16, None) == 3


def test_combine_host_checks(ep):
    f = _Fake.P
    lay = _layout_struct(ep)
    L = ep.lib
    assert L.ep_combine(4, 100, 2, f, 8, ctypes.byref(lay), f, f, f, 4096, None) == 2  # H % 8
    assert L.ep_combine(4, 128, 0, f, 8, ctypes.byref(lay), f, f, f, 4096, None) == 2
    assert L.ep_combine(4, 128, 2, f, -1, ctypes.byref(lay), f, f, f, 4096, None) == 2
    assert L.ep_combine(4, 128, 2, f, 8, None, f, f, f, 4096, None) == 1
    assert L.ep_combine(4, 128, 2, f, 8, ctypes.byref(lay), f, f + 2, f, 4096, None) == 1
    assert L.ep_combine(4, 128, 2, f, 8, ctypes.byref(lay), None, f, f, 4096, None) == 1
    assert L.ep_combine(4, 128, 2, f, 8, ctypes.byref(lay), f, f, f, 8, None) == 1
    # an empty batch is a no-op that succeeds without touching the device
    assert L.ep_combine(0, 128, 2, None, 0, ctypes.byref(lay), None, None, f, 4096, None) == 0


def test_low_latency_host_checks(ep):
    f = _Fake.P
    h = ep._lib.ep_ll_handle(f, f)
    L = ep.lib
    ok = dict(T=8, H=256, K=4, E=16, cap=8)

    def call(**o):
        a = dict(ok)
        a.update(o)
        return L.ep_low_latency_dispatch(a["T"], a["H"], a["K"], a["E"], a["cap"], f, f, f, f, f,
                                         ctypes.byref(h), f, 4096, None)

    assert call(T=9) == 2            # more tokens than capacity
    assert call(cap=0) == 2
    assert call(H=136) == 2          # FP8 needs H % 128 == 0
    assert call(K=33) == 2
    assert call(E=1 << 20, cap=1 << 12) == 2
    assert L.ep_low_latency_combine(8, 256, 4, 0, 8, f, ctypes.byref(h), f, f, f, 4096, None) == 2
    assert L.ep_low_latency_combine(8, 256, 4, 16, 8, f, None, f, f, f, 4096, None) == 1


def test_read_status_and_probe_argument_checks(ep):
    L = ep.lib
    bits = ctypes.c_uint32(0)
    assert L.ep_read_status(None, 4096, None, ctypes.byref(bits)) == 1
    assert L.ep_read_status(_Fake.P, 16, None, ctypes.byref(bits)) == 1
    assert L.ep_debug_wait_probe(1000, None, 4096, None) == 1
    assert L.ep_workspace_init(None, 4096, None) == 1


def test_backward_host_checks(ep):
    f = _Fake.P
    lay = _layout_struct(ep)
    L = ep.lib
    # dispatch backward: both weight-gradient pointers or neither
    assert L.ep_dispatch_backward(4, 128, 2, f, 8, ctypes.byref(lay), f, f, None, f, 4096, None) == 1
    assert L.ep_dispatch_backward(4, 124, 2, f, 8, ctypes.byref(lay), None, f, None, f, 4096, None) == 2
    assert L.ep_dispatch_backward(4, 128, 33, f, 8, ctypes.byref(lay), None, f, None, f, 4096, None) == 2
    assert L.ep_dispatch_backward(4, 128, 2, f, 8, ctypes.byref(lay), None, f + 8, None, f, 4096,
                                  None) == 1
    assert L.ep_dispatch_backward(0, 128, 2, None, 0, ctypes.byref(lay), None, None, None, f, 4096,
                                  None) == 0
    # combine backward
    assert L.ep_combine_backward(4, 128, 2, f, f, 8, ctypes.byref(lay), None, f, f, f, 4096, None) == 1
    assert L.ep_combine_backward(4, 128, 2, f, f, -1, ctypes.byref(lay), f, f, f, f, 4096, None) == 2
    assert L.ep_combine_backward(4, 128, 2, f, f + 4, 8, ctypes.byref(lay), f, f, f, f, 4096,
                                 None) == 1
    assert L.ep_combine_backward(0, 128, 2, None, None, 0, ctypes.byref(lay), None, None, None, f,
                                 4096, None) == 0


def test_dedup_host_checks(ep):
    f = _Fake.P
    lay = _layout_struct(ep)
    L = ep.lib

    def call(T=16, H=256, K=4, E=64, P=8, quant=1, ws=f):
        return L.ep_dispatch_dedup(T, H, K, E, P, quant, f, f, f, f, f, f, f, ctypes.byref(lay),
                                   ws, 1 << 20, None)

    assert call(P=64, E=128) == 2   # one storer lane per partition: P <= 32
    assert call(E=60) == 2           # E % P
    assert call(quant=3) == 1
    assert call(ws=f + 8) == 1
    assert L.ep_combine_dedup(4, 128, 33, f, 8, ctypes.byref(lay), f, f, 4096, None) == 2
    assert L.ep_combine_dedup(4, 128, 8, f, 8, None, f, f, 4096, None) == 1
    assert L.ep_combine_dedup(0, 128, 8, None, 0, ctypes.byref(lay), None, f, 4096, None) == 0


def test_lb_host_checks(ep):
    f = _Fake.P
    L = ep.lib
    pre, red = L.ep_lb_prefetch_weights, L.ep_lb_reduce_grads
    assert pre(0, 16, f, f, f, 4096, None) == 2          # no slots
    assert pre(4097, 16, f, f, f, 4096, None) == 2       # too many slots
    assert pre(4, 24, f, f, f, 4096, None) == 2          # blob not a multiple of 16 bytes
    assert pre(4, 16, None, f, f, 4096, None) == 1
    assert pre(4, 16, f, f + 8, f, 4096, None) == 1      # weights not 16-byte aligned
    assert pre(4, 16, f, f, f, 64, None) == 1            # workspace too small
    assert red(4, 6, f, f, f, 4096, None) == 2           # n not a multiple of 4
    assert red(4, -4, f, f, f, 4096, None) == 2
    assert red(4, 8, f, f + 4, f, 4096, None) == 1       # grads not 16-byte aligned
    assert red(4, 0, f, None, f, 4096, None) == 0        # nothing to reduce


def test_peer_host_checks(ep):
    f = _Fake.P
    lay = _layout_struct(ep)
    L = ep.lib
    plan = L.ep_peer_plan
    assert plan(0, 0, 8, f, f, 64, f, f, f, f, 4096, None) == 2         # no ranks
    assert plan(65, 0, 130, f, f, 64, f, f, f, f, 4096, None) == 2      # too many ranks
    assert plan(3, 0, 8, f, f, 64, f, f, f, f, 4096, None) == 2         # E % W
    assert plan(2, 2, 8, f, f, 64, f, f, f, f, 4096, None) == 2         # rank >= W
    assert plan(2, 0, 8, f, f, -1, f, f, f, f, 4096, None) == 2         # capacity < 0
    assert plan(2, 0, 8, f, f, 1 << 31, f, f, f, f, 4096, None) == 2    # capacity >= 2^31
    assert plan(2, 0, 8, None, f, 64, f, f, f, f, 4096, None) == 1
    assert plan(2, 0, 8, f, f, 64, f, None, f, f, 4096, None) == 1
    assert plan(2, 0, 8, f, f, 64, f, f, f, f, 64, None) == 1          # workspace too small

    peers = ep._lib.ep_peer_buffers(f, f, f, f, 64)

    def disp(T=16, H=256, K=4, E=8, W=2, quant=1, x=f, dst=f, pb=peers, ws=f):
        return L.ep_peer_dispatch(T, H, K, E, W, quant, x, f, f, ctypes.byref(lay), dst,
                                  ctypes.byref(pb) if pb is not None else None, ws, 4096, None)

    assert disp(quant=0x101) == 1       # block-major scales are not offered
    assert disp(quant=4) == 1
    assert disp(E=7) == 2
    assert disp(H=136) == 2             # FP8 needs H % 128 == 0
    assert disp(pb=None) == 2
    assert disp(pb=ep._lib.ep_peer_buffers(f, f, f, f, 1 << 31)) == 2
    assert disp(pb=ep._lib.ep_peer_buffers(f, None, f, f, 64)) == 1     # FP8 needs scales
    assert disp(pb=ep._lib.ep_peer_buffers(None, f, f, f, 64)) == 1
    assert disp(x=f + 8) == 1
    assert disp(dst=None) == 1
    assert disp(ws=f + 8) == 1
    assert disp(T=0, x=None, dst=None) == 0   # an empty batch touches nothing

    comb = L.ep_peer_combine
    assert comb(4, 100, 2, 8, 2, f, 64, ctypes.byref(lay), f, f, f, f, f, 4096, None) == 2  # H % 8
    assert comb(4, 128, 2, 8, 3, f, 64, ctypes.byref(lay), f, f, f, f, f, 4096, None) == 2  # E % W
    assert comb(4, 128, 2, 8, 2, f, -1, ctypes.byref(lay), f, f, f, f, f, 4096, None) == 2
    assert comb(4, 128, 2, 8, 2, None, 64, ctypes.byref(lay), f, f, f, f, f, 4096, None) == 1
    assert comb(4, 128, 2, 8, 2, f, 64, ctypes.byref(lay), None, f, f, f, f, 4096, None) == 1
    assert comb(4, 128, 2, 8, 2, f, 64, ctypes.byref(lay), f, f, f, f + 4, f, 4096, None) == 1
    assert comb(4, 128, 2, 8, 2, f, 64, None, f, f, f, f, f, 4096, None) == 1
    assert comb(0, 128, 2, 8, 2, None, 64, ctypes.byref(lay), None, None, None, None, f, 4096,
                None) == 0

    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(ep.EP_IPC_HANDLE_BYTES)
    assert L.ep_ipc_alloc(0, ctypes.byref(ptr), handle) == 1
    assert L.ep_ipc_alloc(256, None, handle) == 1
    assert L.ep_ipc_alloc(256, ctypes.byref(ptr), None) == 1
    assert L.ep_ipc_free(None) == 1
    assert L.ep_ipc_open(None, ctypes.byref(ptr)) == 1
    assert L.ep_ipc_open(handle, None) == 1
    assert L.ep_ipc_close(None) == 1


def test_peer_dedup_host_checks(ep):
    f = _Fake.P
    lay = _layout_struct(ep)
    L = ep.lib
    lo = L.ep_get_dispatch_layout_dedup
    assert lo(4, 2, 64, 33, f, ctypes.byref(lay), f, 1 << 20, None) == 2   # P > 32
    assert lo(4, 2, 60, 8, f, ctypes.byref(lay), f, 1 << 20, None) == 2    # E % P
    assert lo(4, 2, 64, 8, None, ctypes.byref(lay), f, 1 << 20, None) == 1
    assert lo(4, 2, 64, 8, f, ctypes.byref(lay), f, 16, None) == 3          # workspace
    peers = ep._lib.ep_peer_buffers(f, f, f, f, 64)

    def disp(T=16, H=256, K=4, E=64, W=8, quant=1, pb=peers):
        return L.ep_peer_dispatch_dedup(T, H, K, E, W, quant, f, f, f, ctypes.byref(lay), f,
                                        ctypes.byref(pb) if pb is not None else None, f, 4096,
                                        None)

    assert disp(W=64, E=128) == 2       # one storer lane per rank: W <= 32
    assert disp(quant=0x101) == 1
    assert disp(H=136) == 2
    assert disp(pb=None) == 2
    assert disp(pb=ep._lib.ep_peer_buffers(f, None, f, f, 64)) == 1
    assert disp(T=0) == 0
    comb = L.ep_peer_combine_dedup
    assert comb(4, 128, 33, f, 64, ctypes.byref(lay), f, f, f, 4096, None) == 2
    assert comb(4, 100, 8, f, 64, ctypes.byref(lay), f, f, f, 4096, None) == 2
    assert comb(4, 128, 8, None, 64, ctypes.byref(lay), f, f, f, 4096, None) == 1
    assert comb(4, 128, 8, f, 64, ctypes.byref(lay), None, f, f, 4096, None) == 1
    assert comb(0, 128, 8, None, 64, ctypes.byref(lay), None, None, f, 4096, None) == 0


def test_peer_low_latency_host_checks(ep):
    f = _Fake.P
    h = ep._lib.ep_ll_handle(f, f)
    L = ep.lib

    def disp(T=8, H=256, K=4, E=16, W=2, rank=0, cap=8, x=f, tx=f):
        return L.ep_peer_low_latency_dispatch(T, H, K, E, W, rank, cap, x, f, tx, f, f,
                                              ctypes.byref(h), f, 4096, None)

    assert disp(T=9) == 2           # more tokens than capacity
    assert disp(rank=2) == 2        # rank >= W
    assert disp(E=15) == 2          # E % W
    assert disp(H=136) == 2         # FP8 needs H % 128 == 0
    assert disp(tx=None) == 1
    assert disp(x=f + 8) == 1
    comb = L.ep_peer_low_latency_combine

    def cmb(T=8, H=256, K=4, E=16, W=2, rank=0, cap=8, eo=f, y=f):
        return comb(T, H, K, E, W, rank, cap, eo, f, ctypes.byref(h), f, y, f, 4096, None)

    assert cmb(rank=-1) == 2
    assert cmb(cap=0) == 2
    assert cmb(H=100) == 2
    assert cmb(eo=None) == 1
    assert cmb(y=f + 2) == 1
    assert cmb(T=0, eo=None, y=None) == 0


def test_plain_c_client(ep, tmp_path):
    """The header compiles as C11 (warnings as errors), a C program links the library
    and its host-side checks answer the same as through the binding."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(ep.LIB_PATH)
    exe = tmp_path / "abi_c_check"
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_c_check.c"), "-L", lib_dir, "-lep_b200",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
