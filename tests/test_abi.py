"""The C-ABI library builds for sm_100a, loads without a GPU, exports every call that
include/mla.h declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("mla_build", os.path.join(ROOT, "attention_mla_get_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    path = b.build()
    L = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.mla_decode_kvcache.argtypes = [vp, vp, i64, vp, i32, vp, i32, i32, i32, i32, i32, vp, i32, vp,
                                     ctypes.c_float, i32, i32, vp, vp, vp, sz, vp]
    L.mla_decode_kvcache.restype = i32
    L.mla_get_metadata.argtypes = [vp, i32, i32, i32, vp, i32, vp, vp]
    L.mla_workspace_size.argtypes = [i32, i32, i32, i32]
    L.mla_workspace_size.restype = sz
    L.mla_strerror.restype = ctypes.c_char_p
    L.mla_version.restype = ctypes.c_char_p
    return L


def _declared():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    return re.findall(r"^MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text, flags=re.M)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert set(names) == {"mla_num_sm_parts", "mla_get_metadata", "mla_workspace_size", "mla_decode_kvcache",
                          "mla_decode_kvcache_noalloc", "mla_noalloc_read_status", "mla_get_metadata_sparse", "mla_decode_kvcache_sparse",
                          "mla_sparse_prefill", "mla_session_create", "mla_session_decode", "mla_session_join",
                          "mla_session_status", "mla_session_destroy",
                          "mla_read_status", "mla_fault_injection_arm", "mla_strerror", "mla_version"}
    so = os.path.join(ROOT, "attention_mla_get_b200", "libmla.so")
    nm = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (mla_\w+)", nm))
    assert set(names) == exported
    for n in names:
        assert hasattr(lib, n)


def test_no_cuda_runtime_dependency():
    so = os.path.join(ROOT, "attention_mla_get_b200", "libmla.so")
    deps = subprocess.run(["ldd", so], capture_output=True, text=True).stdout
    assert "libcudart" not in deps and "libtorch" not in deps


def test_built_for_sm100a():
    so = os.path.join(ROOT, "attention_mla_get_b200", "libmla.so")
    # the embedded fatbin names its target architecture
    data = open(so, "rb").read()
    assert b"sm_100a" in data


def test_noalloc_read_status_rejects_null(lib):
    lib.mla_noalloc_read_status.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    lib.mla_noalloc_read_status.restype = ctypes.c_int
    assert lib.mla_noalloc_read_status(0, None, None) == -1


def test_fault_injection_arm_argument_errors(lib):
    lib.mla_fault_injection_arm.argtypes = [ctypes.c_longlong, ctypes.c_int]
    lib.mla_fault_injection_arm.restype = ctypes.c_int
    assert lib.mla_fault_injection_arm(-1, -1) == -7
    assert lib.mla_fault_injection_arm(100, -2) == -7
    assert lib.mla_fault_injection_arm(0, -1) == 0   # disarmed: the default bound, no withheld fill


def test_strerror_and_version(lib):
    assert lib.mla_version() == b"0.1.0"
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10, -100, 12345):
        assert lib.mla_strerror(code)


def test_workspace_size(lib):
    # header 256 B, lse [b+P, R] rounded to 256 B, O [b+P, R, 512] fp32
    assert lib.mla_workspace_size(128, 148, 16, 1) == 256 + 276 * 16 * 4 + 276 * 16 * 512 * 4
    assert lib.mla_workspace_size(0, 148, 16, 1) == 0
    assert lib.mla_workspace_size(4, 0, 16, 1) == 0
    assert lib.mla_workspace_size(4, 10, 16, 2) == 0
    assert lib.mla_workspace_size(4, 10, 5000, 1) == 0


def _call(lib, **kw):
    fake = ctypes.c_void_p(0x10000)   # 16-byte aligned, never dereferenced on these paths
    a = dict(q=fake, kv=fake, nb=10, bt=fake, maxb=4, sl=fake, b=2, s_q=1, h_q=16, h_kv=1, d_v=512, md=fake,
             parts=4, ns=fake, scale=0.04, causal=0, dt=0, out=fake, lse=fake, ws=fake, wsb=1 << 30, st=None)
    a.update(kw)
    return lib.mla_decode_kvcache(a["q"], a["kv"], a["nb"], a["bt"], a["maxb"], a["sl"], a["b"], a["s_q"],
                                  a["h_q"], a["h_kv"], a["d_v"], a["md"], a["parts"], a["ns"], a["scale"],
                                  a["causal"], a["dt"], a["out"], a["lse"], a["ws"], a["wsb"], a["st"])


def test_argument_errors_are_reported_before_any_launch(lib):
    assert _call(lib, q=None) == -1
    assert _call(lib, ws=None) == -1
    assert _call(lib, out=ctypes.c_void_p(0x10008)) == -2
    assert _call(lib, lse=ctypes.c_void_p(0x10002)) == -2
    assert _call(lib, d_v=256) == -3
    assert _call(lib, h_kv=2) == -4
    assert _call(lib, h_q=0) == -4
    assert _call(lib, dt=7) == -5
    assert _call(lib, b=0) == -7
    assert _call(lib, s_q=0) == -7
    assert _call(lib, nb=0) == -7
    assert _call(lib, nb=1 << 25) == -7          # 2^25 pages * 64 tokens reaches 2^31
    assert _call(lib, h_q=4097) == -7
    assert _call(lib, parts=0) == -8
    assert _call(lib, wsb=100) == -6
    fake = ctypes.c_void_p(0x10000)
    assert lib.mla_get_metadata(None, 2, 16, 1, fake, 4, fake, None) == -1
    assert lib.mla_get_metadata(fake, 0, 16, 1, fake, 4, fake, None) == -7
    assert lib.mla_get_metadata(fake, 2, 16, 2, fake, 4, fake, None) == -4
    assert lib.mla_get_metadata(fake, 2, 16, 1, fake, 0, fake, None) == -8


def _call_sparse(lib, **kw):
    """mla_decode_kvcache_sparse with plausible fake pointers (never dereferenced: every case
    below fails an argument check before anything is enqueued)."""
    fake = ctypes.c_void_p(0x10000)
    a = dict(q=fake, kv=fake, nb=8, bt=fake, mb=4, sl=fake, b=2, s_q=1, h_q=16, h_kv=1, d_v=512, idx=fake,
             topk=64, md=fake, parts=4, ns=fake, scale=0.04, dt=0, out=fake, lse=fake, ws=fake, wsb=1 << 30)
    a.update(kw)
    f = lib.mla_decode_kvcache_sparse
    i32, i64, vp, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    f.argtypes = [vp, vp, i64, vp, i32, vp, i32, i32, i32, i32, i32, vp, i32, vp, i32, vp, ctypes.c_float, i32,
                  vp, vp, vp, sz, vp]
    f.restype = i32
    return f(a["q"], a["kv"], a["nb"], a["bt"], a["mb"], a["sl"], a["b"], a["s_q"], a["h_q"], a["h_kv"], a["d_v"],
             a["idx"], a["topk"], a["md"], a["parts"], a["ns"], a["scale"], a["dt"], a["out"], a["lse"], a["ws"],
             a["wsb"], None)


def test_sparse_argument_errors_are_reported_before_any_launch(lib):
    assert _call_sparse(lib, idx=None) == -1
    assert _call_sparse(lib, idx=ctypes.c_void_p(0x10002)) == -2
    assert _call_sparse(lib, d_v=256) == -3
    assert _call_sparse(lib, h_kv=2) == -4
    assert _call_sparse(lib, dt=1) == -5             # token-sparse decode reads bf16 caches only
    assert _call_sparse(lib, topk=0) == -7
    assert _call_sparse(lib, s_q=0) == -7
    assert _call_sparse(lib, parts=0) == -8
    assert _call_sparse(lib, wsb=100) == -6
    fake = ctypes.c_void_p(0x10000)
    g = lib.mla_get_metadata_sparse
    g.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    assert g(2, 1, 64, 16, 1, None, 4, fake, None) == -1
    assert g(2, 1, 0, 16, 1, fake, 4, fake, None) == -7
    assert g(2, 1, 64, 16, 2, fake, 4, fake, None) == -4
    assert g(2, 1, 64, 16, 1, fake, 0, fake, None) == -8
    # the scheduler's cost sums are 32-bit: batch * s_q * (ceil(topk / 128) + 2) must stay below 2^31
    assert g(1 << 29, 1, 256, 16, 1, fake, 4, fake, None) == -7       # 2^29 * 4 = 2^31
    assert g(1 << 20, 1, 128 * 2046, 16, 1, fake, 4, fake, None) == -7  # 2^20 * 2048 = 2^31


def test_session_argument_errors(lib):
    """mla_session_create checks its arguments before any CUDA call; without a usable device a
    valid request fails with MLA_ERR_NO_DEVICE; the per-step calls reject a NULL session."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.mla_session_create.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]
    lib.mla_session_create.restype = i32
    h = vp()
    ref = ctypes.byref(h)
    # device, batch, s_q, h_q, h_kv, max_blocks, topk, kv_dtype, num_sm_parts
    assert lib.mla_session_create(0, 4, 1, 16, 1, 8, 0, 0, 74, None) == -1
    assert lib.mla_session_create(0, 4, 1, 16, 2, 8, 0, 0, 74, ref) == -4      # h_kv != 1
    assert lib.mla_session_create(0, 4, 1, 0, 1, 8, 0, 0, 74, ref) == -4       # h_q < 1
    assert lib.mla_session_create(0, 4, 1, 16, 1, 8, 0, 7, 74, ref) == -5      # kv_dtype
    assert lib.mla_session_create(0, 4, 1, 16, 1, 8, 64, 1, 74, ref) == -5     # sparse needs bf16
    assert lib.mla_session_create(0, 0, 1, 16, 1, 8, 0, 0, 74, ref) == -7      # batch
    assert lib.mla_session_create(0, 4, 1, 16, 1, 0, 0, 0, 74, ref) == -7      # max_blocks
    assert lib.mla_session_create(0, 4, 1, 16, 1, 8, -1, 0, 74, ref) == -7     # topk < 0
    assert lib.mla_session_create(0, 4, 64, 128, 1, 8, 0, 0, 74, ref) == -7    # 8192 rows
    assert lib.mla_session_create(0, 4, 1, 16, 1, 8, 0, 0, 0, ref) == -8       # parts
    import torch
    if not torch.cuda.is_available():
        assert lib.mla_session_create(0, 4, 1, 16, 1, 8, 0, 0, 74, ref) == -9
        assert not h.value
    lib.mla_session_decode.argtypes = [vp] * 3 + [ctypes.c_int64] + [vp] * 3 + [ctypes.c_float, i32, vp, vp, vp]
    lib.mla_session_decode.restype = i32
    assert lib.mla_session_decode(None, 1, 1, 1, 1, 1, None, 1.0, 0, 1, 1, None) == -1
    lib.mla_session_join.argtypes = [vp, vp]
    assert lib.mla_session_join(None, None) == -1
    lib.mla_session_status.argtypes = [vp, i32, ctypes.POINTER(i32)]
    assert lib.mla_session_status(None, 0, ctypes.byref(i32())) == -1
    lib.mla_session_destroy.argtypes = [vp]
    assert lib.mla_session_destroy(None) == -1
