"""CPU checks of the C ABI: the library loads, exports every entry point that
include/moe.h declares, and rejects bad arguments on the host before any
device work.  No compute call is made here (these run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")
LIB = os.path.join(ROOT, "moe_layer_forward_b200", "libmoe.so")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA, DEVICE = range(6)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import __graft_entry__

        __graft_entry__.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["moe_rmsnorm", "moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_unpermute_combine",
              "moe_forward", "moe_expert_gate_up", "moe_expert_down", "moe_status_string", "moe_abi_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(lib, n)


def test_status_strings_and_version(lib):
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [ctypes.c_int]
    texts = [lib.moe_status_string(s).decode() for s in range(6)]
    assert texts[0] == "ok" and len(set(texts)) == 6
    assert lib.moe_status_string(99).decode() == "unknown status"
    assert lib.moe_abi_version() == 2


def test_launch_counter_counts_no_rejected_call(lib):
    # arguments rejected on the host enqueue nothing, so the counter stays where it was
    lib.moe_kernel_launches.restype = ctypes.c_uint64
    n0 = lib.moe_kernel_launches()
    assert lib.moe_rmsnorm(None, 1, None, -1, 64, ctypes.c_float(1e-5), None, 1, None) != 0
    assert lib.moe_kernel_launches() == n0


def test_library_does_not_link_the_oracle():
    out = subprocess.run(["nm", "-D", LIB], capture_output=True, text=True, check=True).stdout
    assert "oracle_" not in out
    deps = subprocess.run(["readelf", "-d", LIB], capture_output=True, text=True, check=True).stdout
    assert "oracle" not in deps and "libcuda.so" not in deps


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "moe_layer_forward_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\boracle\b", src), f


V = ctypes.c_void_p
NULL = None


def _p(n=0x1000):
    return ctypes.c_void_p(n)  # a fake, 16-byte aligned address; validation fails before any use


def test_rmsnorm_rejects_bad_shapes_on_host(lib):
    f = lib.moe_rmsnorm
    f.argtypes = [V, ctypes.c_int, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, V, ctypes.c_int, V]
    assert f(_p(), 1, _p(), 4, 12, 1e-5, _p(), 1, NULL) == UNSUPPORTED  # d % 8
    assert f(_p(), 1, _p(), -1, 16, 1e-5, _p(), 1, NULL) == INVALID
    assert f(_p(), 7, _p(), 4, 16, 1e-5, _p(), 1, NULL) == INVALID  # dtype
    assert f(_p(), 1, _p(), 0, 16, 1e-5, _p(), 1, NULL) == OK  # T == 0 queues nothing
    assert f(ctypes.c_void_p(0x1004), 1, _p(), 4, 16, 1e-5, _p(), 1, NULL) == INVALID  # misaligned


def test_router_rejects_bad_shapes_on_host(lib):
    f = lib.moe_router_topk
    f.argtypes = [V, ctypes.c_int, V, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, V, V, V, V,
                  V, ctypes.POINTER(ctypes.c_size_t), V]
    n = ctypes.c_size_t(0)
    args = lambda T, d, E, k: f(_p(), 1, _p(), _p(), T, d, E, k, _p(), _p(), NULL, NULL, NULL, ctypes.byref(n), NULL)
    assert args(8, 64, 32, 9) == UNSUPPORTED  # top_k > 8
    assert args(8, 64, 300, 8) == UNSUPPORTED  # E > 256
    assert args(8, 64, 4, 8) == UNSUPPORTED  # k > E
    assert args(8, 60, 32, 8) == UNSUPPORTED  # d % 8
    assert args(8, 64, 32, 0) == INVALID


def test_permute_workspace_query_needs_no_device(lib):
    f = lib.moe_permute
    f.argtypes = [V, ctypes.c_int, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, V, V, V, V, V,
                  V, ctypes.POINTER(ctypes.c_size_t), V, V]
    n = ctypes.c_size_t(0)
    assert f(_p(), 1, _p(), 1000, 64, 16, 8, _p(), _p(), _p(), _p(), _p(), NULL, ctypes.byref(n), NULL, NULL) == OK
    assert n.value == 4 * 16 * 4  # 4 chunks of 256 tokens x 16 experts x int32
    small = ctypes.c_size_t(16)
    ws = ctypes.c_void_p(0x100000)
    assert f(_p(), 1, _p(), 1000, 64, 16, 8, _p(), _p(), _p(), _p(), _p(), ws, ctypes.byref(small), NULL, NULL) == \
        WORKSPACE
    assert small.value == 256
    unaligned = ctypes.c_void_p(0x100010)
    big = ctypes.c_size_t(1 << 20)
    assert f(_p(), 1, _p(), 1000, 64, 16, 8, _p(), _p(), _p(), _p(), _p(), unaligned, ctypes.byref(big), NULL,
             NULL) == INVALID


def test_expert_and_combine_reject_bad_shapes_on_host(lib):
    g = lib.moe_expert_gate_up
    g.argtypes = [V, V, V, ctypes.c_int, V, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, V, V, V]
    assert g(_p(), _p(), _p(), 1, _p(), _p(), 64, 8, 96, 256, _p(), NULL, NULL) == UNSUPPORTED  # bf16 needs d % 128
    assert g(_p(), _p(), _p(), 1, _p(), _p(), 64, 8, 128, 200, _p(), NULL, NULL) == UNSUPPORTED  # d_ff % 128
    assert g(_p(), _p(), _p(), 1, _p(), _p(), 64, 300, 128, 256, _p(), NULL, NULL) == UNSUPPORTED
    assert g(_p(), _p(), _p(), 0, _p(), _p(), 64, 8, 12, 256, _p(), NULL, NULL) == UNSUPPORTED  # f32 needs d % 8
    assert g(_p(), _p(), _p(), 1, _p(), _p(), 0, 8, 128, 256, _p(), NULL, NULL) == OK  # no rows: nothing to do
    assert g(NULL, _p(), _p(), 1, _p(), _p(), 64, 8, 128, 256, _p(), NULL, NULL) == INVALID
    m = lib.moe_grouped_swiglu_masked
    m.argtypes = [V, V, V, V, ctypes.c_int, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, V, V,
                  V, V]
    assert m(_p(), _p(), _p(), _p(), 1, _p(), 8, 0, 128, 256, _p(), _p(), NULL, NULL) == INVALID  # cap >= 1
    assert m(_p(), _p(), _p(), _p(), 1, _p(), 8, 1 << 28, 128, 256, _p(), _p(), NULL, NULL) == INVALID  # E*cap
    assert m(_p(), _p(), _p(), _p(), 0, _p(), 8, 16, 128, 256, _p(), _p(), NULL, NULL) == UNSUPPORTED  # bf16 only
    assert m(_p(), _p(), _p(), _p(), 1, _p(), 8, 16, 96, 256, _p(), _p(), NULL, NULL) == UNSUPPORTED  # d % 128
    assert m(_p(), _p(), _p(), _p(), 1, NULL, 8, 16, 128, 256, _p(), _p(), NULL, NULL) == INVALID  # counts
    qz = lib.moe_quantize_fp8
    qz.argtypes = [V, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, V, V, V]
    assert qz(_p(), 1, 64, 256, 64, _p(), _p(), NULL) == INVALID  # block of 1 or 128 rows
    assert qz(_p(), 1, 64, 200, 128, _p(), _p(), NULL) == UNSUPPORTED  # cols % 128
    assert qz(_p(), 7, 64, 256, 1, _p(), _p(), NULL) == INVALID  # dtype
    assert qz(_p(), 1, 0, 256, 1, _p(), _p(), NULL) == OK  # nothing to do
    c = lib.moe_unpermute_combine
    c.argtypes = [V, ctypes.c_int, V, V, V, ctypes.c_int, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, V,
                  ctypes.c_int, V]
    assert c(_p(), 1, _p(), _p(), _p(), 1, 4, 64, 9, _p(), 1, NULL) == UNSUPPORTED
    assert c(_p(), 1, _p(), _p(), _p(), 1, 4, 60, 8, _p(), 1, NULL) == UNSUPPORTED
    assert c(_p(), 1, _p(), _p(), _p(), 5, 4, 64, 8, _p(), 1, NULL) == INVALID


def test_peer_memory_and_sized_entries_reject_bad_arguments_on_host(lib):
    i32 = ctypes.c_int32
    sz = lib.moe_grouped_swiglu_sized
    sz.argtypes = [V, V, V, V, ctypes.c_int, V, V, i32, i32, i32, i32, i32, V, V, V, V]
    assert sz(_p(), _p(), _p(), _p(), 1, _p(), _p(), 64, 0, 8, 128, 256, _p(), _p(), NULL, NULL) == INVALID
    assert sz(_p(), _p(), _p(), _p(), 1, _p(), _p(), 64, 65, 8, 128, 256, _p(), _p(), NULL, NULL) == INVALID
    assert sz(_p(), _p(), _p(), _p(), 1, _p(), _p(), 64, 32, 8, 96, 256, _p(), _p(), NULL, NULL) == UNSUPPORTED
    assert sz(_p(), _p(), _p(), _p(), 1, NULL, _p(), 64, 32, 8, 128, 256, _p(), _p(), NULL, NULL) == INVALID
    dsp = lib.moe_ep_dispatch
    i64 = ctypes.c_int64
    dsp.argtypes = [V, ctypes.c_int, V, V, V, V, i32, i32, i32, i32, i32, i32, V, i64, V, V]
    assert dsp(_p(), 1, _p(), _p(), _p(), _p(), 0, 3, 16, 4, 64, 8, _p(), 64, NULL, NULL) == UNSUPPORTED  # E % N
    assert dsp(_p(), 1, _p(), _p(), _p(), _p(), 2, 2, 16, 4, 64, 8, _p(), 64, NULL, NULL) == INVALID  # rank < N
    assert dsp(_p(), 1, _p(), _p(), _p(), NULL, 0, 2, 16, 4, 64, 8, _p(), 64, NULL, NULL) == INVALID  # table
    assert dsp(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, 4, 60, 8, _p(), 64, NULL, NULL) == UNSUPPORTED  # d % 8
    assert dsp(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, 4, 64, 8, NULL, 64, NULL, NULL) == INVALID  # recv_bufs
    assert dsp(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, 4, 64, 8, _p(), -1, NULL, NULL) == INVALID  # recv_rows
    assert dsp(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, 0, 64, 8, _p(), 64, NULL, NULL) == OK  # no tokens
    lay = lib.moe_ep_layout
    lay.argtypes = [V, i32, i32, i32, V, V, V]
    assert lay(NULL, 0, 2, 16, _p(), _p(), NULL) == INVALID
    assert lay(_p(), 0, 2, 16, NULL, _p(), NULL) == INVALID
    assert lay(_p(), 0, 5, 16, _p(), _p(), NULL) == UNSUPPORTED
    cmb = lib.moe_ep_combine
    cmb.argtypes = [V, ctypes.c_int, V, V, V, V, i32, i32, i32, V, V, ctypes.c_int, i32, i32, i32, V, ctypes.c_int,
                    i64, V, V]
    assert cmb(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, _p(), _p(), 1, 4, 64, 9, _p(), 1, 64, NULL,
               NULL) == UNSUPPORTED
    assert cmb(NULL, 1, _p(), _p(), _p(), _p(), 0, 2, 16, _p(), _p(), 1, 4, 64, 8, _p(), 1, 64, NULL, NULL) == INVALID
    assert cmb(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, _p(), _p(), 7, 4, 64, 8, _p(), 1, 64, NULL, NULL) == INVALID
    assert cmb(_p(), 1, _p(), _p(), _p(), _p(), 0, 2, 16, _p(), _p(), 1, 4, 64, 8, _p(), 1, -1, NULL, NULL) == INVALID


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("eps", ctypes.c_float), ("x_dtype", ctypes.c_int),
                ("w_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int)]


def test_forward_rejects_bad_shapes_on_host(lib):
    f = lib.moe_forward
    f.argtypes = [ctypes.POINTER(Shape), V, V, V, V, V, V, V, ctypes.POINTER(ctypes.c_size_t), V, V]
    n = ctypes.c_size_t(0)
    w = ctypes.create_string_buffer(48)
    assert f(None, w, NULL, NULL, NULL, NULL, NULL, NULL, ctypes.byref(n), NULL, NULL) == INVALID
    bad = [Shape(8, 4096, 128, 9, 1536, 1e-5, 1, 1, 1),   # top_k
           Shape(8, 4096, 512, 8, 1536, 1e-5, 1, 1, 1),   # E
           Shape(8, 4000, 128, 8, 1536, 1e-5, 1, 1, 1),   # bf16 experts need d % 128
           Shape(8, 4096, 128, 8, 1500, 1e-5, 1, 1, 1)]   # bf16 experts need d_ff % 128
    for s in bad:
        assert f(ctypes.byref(s), w, NULL, NULL, NULL, NULL, NULL, NULL, ctypes.byref(n), NULL, NULL) == UNSUPPORTED
    s = Shape(8, 4096, 128, 8, 1536, 1e-5, 3, 1, 1)
    assert f(ctypes.byref(s), w, NULL, NULL, NULL, NULL, NULL, NULL, ctypes.byref(n), NULL, NULL) == INVALID


def test_route_and_gate_up_raw_reject_bad_arguments_on_host(lib):
    i32, V = ctypes.c_int32, ctypes.c_void_p
    r = lib.moe_route
    r.argtypes = [V, ctypes.c_int, V, V, V, i32, i32, i32, i32, ctypes.c_float, V, V, V, V, V,
                  ctypes.POINTER(ctypes.c_size_t), V]
    n = ctypes.c_size_t(0)
    p = ctypes.c_void_p(16)
    assert r(p, 1, p, p, p, 8, 4096, 128, 9, 1e-5, p, p, None, None, None, ctypes.byref(n), None) == UNSUPPORTED
    assert r(p, 1, p, p, p, 8, 4096, 512, 8, 1e-5, p, p, None, None, None, ctypes.byref(n), None) == UNSUPPORTED
    assert r(p, 1, p, p, p, 8, 4100, 128, 8, 1e-5, p, p, None, None, None, ctypes.byref(n), None) == UNSUPPORTED
    assert r(p, 3, p, p, p, 8, 4096, 128, 8, 1e-5, p, p, None, None, None, ctypes.byref(n), None) == INVALID
    assert r(p, 1, p, p, p, -1, 4096, 128, 8, 1e-5, p, p, None, None, None, ctypes.byref(n), None) == INVALID
    g = lib.moe_expert_gate_up_raw
    g.argtypes = [V, V, V, V, V, i32, i32, i32, i32, V, V, V]
    assert g(p, p, p, p, p, 64, 8, 4000, 1536, p, None, None) == UNSUPPORTED  # bf16 needs d % 128
    assert g(p, p, p, p, p, -1, 8, 4096, 1536, p, None, None) == INVALID
    assert g(p, None, p, p, p, 64, 8, 4096, 1536, p, None, None) == INVALID
    assert g(p, p, p, p, p, 0, 8, 4096, 1536, p, None, None) == OK  # no rows: nothing to do
