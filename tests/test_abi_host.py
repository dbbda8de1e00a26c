"""Host-side checks of the C ABI that need no GPU.

The library must load and export every function include/had.h declares;
argument checks, workspace sizing and status strings run on the host and
return before anything touches the device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "had.h")
LIB = os.path.join(ROOT, "sparse_attention_sigma_b200", "libhad.so")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(had_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from sparse_attention_sigma_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("had_binarize_pack", "had_hamming_topn", "had_sparse_softmax_av",
                 "had_attention_fwd", "had_workspace_bytes", "had_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    lib.had_status_string.restype = ctypes.c_char_p
    lib.had_status_string.argtypes = [ctypes.c_int]
    assert lib.had_status_string(0) == b"HAD_OK"
    assert lib.had_status_string(5) == b"HAD_ERR_BAD_SIGMA"
    assert lib.had_status_string(99) == b"HAD_ERR_UNKNOWN"


def test_workspace_and_launch_counts(lib):
    lib.had_workspace_bytes.restype = ctypes.c_size_t
    lib.had_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.had_launch_count.argtypes = [ctypes.c_int] * 6
    bad = ctypes.c_size_t(-1).value
    assert lib.had_workspace_bytes(2, 4, 16, 4096, 64, 512) > 0
    assert lib.had_workspace_bytes(2, 4, 16, 4096, 96, 512) == bad      # d unsupported
    assert lib.had_workspace_bytes(2, 4, 16, 4096, 64, 4097) == bad     # N > n
    assert lib.had_workspace_bytes(0, 1, 1, 8, 64, 1) == 0
    assert lib.had_launch_count(0, 1, 1, 8, 64, 1) == 1
    assert lib.had_launch_count(2, 1, 1, 8, 64, 0) == -1


def test_wait_limit_setter_swaps_and_restores_the_default(lib):
    lib.had_set_wait_limit_ns.restype = ctypes.c_ulonglong
    lib.had_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    default = 2_000_000_000
    assert lib.had_set_wait_limit_ns(1000) == default
    assert lib.had_set_wait_limit_ns(0) == 1000          # 0 restores the default
    assert lib.had_set_wait_limit_ns(0) == default


def test_argument_errors_return_before_any_cuda_call(lib):
    f = lib.had_attention_fwd
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    f.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, ctypes.c_float, vp, vp, vp, vp, sz, vp, vp]
    f.restype = ctypes.c_int
    fake = vp(4096)        # never dereferenced: the checks fail first
    # d = 96 is unsupported
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 96, 2, 0.1, fake, None, None,
             fake, 1 << 20, None, None) == 2
    # N > n
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 9, 0.1, fake, None, None,
             fake, 1 << 20, None, None) == 1
    # null Q
    assert f(None, fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, 0.1, fake, None, None,
             fake, 1 << 20, None, None) == 1
    # workspace too small
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, 0.1, fake, None, None,
             fake, 16, None, None) == 3
    # misaligned pointer
    assert f(vp(4097), fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, 0.1, fake, None, None,
             fake, 1 << 20, None, None) == 1


def test_topn_mass_argument_errors_return_before_any_cuda_call(lib):
    f = lib.had_topn_mass
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, i, i, i, i, ctypes.c_float, vp, i, vp, vp, vp]
    f.restype = ctypes.c_int
    fake = vp(4096)        # never dereferenced: the checks fail first
    good = (ctypes.c_double * 3)(0.5, 0.9, 1.0)
    bad = (ctypes.c_double * 1)(1.5)
    p = lambda a: ctypes.cast(a, vp)
    assert f(fake, fake, 1, 1, 8, 96, 0.1, p(good), 3, fake, None, None) == 2    # d
    assert f(fake, fake, 1, 1, 8, 64, 0.1, p(good), 0, fake, None, None) == 1    # np = 0
    assert f(fake, fake, 1, 1, 8, 64, 0.1, p(good), 9, fake, None, None) == 1    # np > 8
    assert f(fake, fake, 1, 1, 8, 64, 0.1, p(bad), 1, fake, None, None) == 1     # p > 1
    assert f(fake, fake, 1, 1, 8, 64, -0.1, p(good), 3, fake, None, None) == 1   # tau < 0
    assert f(fake, fake, 1, 1, 8, 64, 0.1, None, 3, fake, None, None) == 1       # no p
    lib.had_workspace_bytes.restype = ctypes.c_size_t
    lib.had_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.had_launch_count.argtypes = [ctypes.c_int] * 6
    assert lib.had_workspace_bytes(6, 1, 1, 8, 64, 0) == 0
    assert lib.had_launch_count(6, 1, 1, 8, 64, 0) == 1


def test_causal_argument_errors_return_before_any_cuda_call(lib):
    f = lib.had_attention_causal_fwd
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    f.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, ctypes.c_float, vp, vp, vp, vp, sz, vp,
                  vp]
    f.restype = ctypes.c_int
    fake = vp(4096)        # never dereferenced: the checks fail first
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 96, 2, 0.1, fake, None, None, fake,
             1 << 20, None, None) == 2                                           # d
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 9, 0.1, fake, None, None, fake,
             1 << 20, None, None) == 1                                           # N > n
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, 0.1, fake, None, None, None,
             1 << 20, None, None) == 3                                           # no workspace
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, 0.1, fake, None, None, fake,
             16, None, None) == 3                                                # too small
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, float("nan"), fake, None, None,
             fake, 1 << 20, None, None) == 1                                     # tau NaN
    assert f(fake, fake, fake, 0, fake, fake, 1, 1, 8, 64, 2, 0.1, fake, vp(4100), None, fake,
             1 << 20, None, None) == 1                                           # misaligned
    g = lib.had_hamming_topn_causal
    g.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, vp]
    g.restype = ctypes.c_int
    assert g(fake, fake, 1, 1, 8, 64, 0, fake, fake, None, None) == 1            # N = 0
    assert g(fake, None, 1, 1, 8, 64, 2, fake, fake, None, None) == 1            # no kbits
    assert g(fake, fake, 1, 1, 8, 64, 2, vp(4100), fake, None, None) == 1        # misaligned
    lib.had_workspace_bytes.restype = ctypes.c_size_t
    lib.had_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.had_launch_count.argtypes = [ctypes.c_int] * 6
    # the causal call runs the fused path: same workspace and launches
    for shape in ((1, 1, 128, 64, 16), (4, 16, 4096, 64, 512), (1, 32, 16384, 128, 2048)):
        assert lib.had_workspace_bytes(7, *shape) == lib.had_workspace_bytes(2, *shape)
        assert lib.had_launch_count(7, *shape) == 4
    assert lib.had_workspace_bytes(7, 1, 1, 128, 64, 129) == ctypes.c_size_t(-1).value


def test_soft_argument_errors_return_before_any_cuda_call(lib):
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    fake = vp(4096)        # never dereferenced: the checks fail first
    b = lib.had_soft_binarize
    b.argtypes = [vp, i, vp, f, i, i, i, i, vp, vp, vp]
    b.restype = ctypes.c_int
    assert b(fake, 0, fake, 1.0, 1, 1, 8, 96, fake, None, None) == 2            # d
    assert b(fake, 0, fake, 0.0, 1, 1, 8, 64, fake, None, None) == 1            # c = 0
    assert b(fake, 0, fake, float("inf"), 1, 1, 8, 64, fake, None, None) == 1   # c = inf
    assert b(fake, 0, fake, 1.0, 1, 1, 8, 64, vp(4100), None, None) == 1        # misaligned
    t = lib.had_soft_topn
    t.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, sz, vp, vp]
    t.restype = ctypes.c_int
    assert t(fake, fake, 1, 1, 8, 64, 9, fake, fake, fake, 1 << 30, None, None) == 1   # N > n
    assert t(fake, fake, 1, 1, 40000, 64, 9, fake, fake, fake, 1 << 40, None, None) == 2
    assert t(fake, fake, 1, 1, 8, 64, 2, fake, fake, fake, 16, None, None) == 3        # ws
    a = lib.had_soft_attention_fwd
    a.argtypes = [vp, vp, vp, i, vp, vp, f, i, i, i, i, i, f, vp, vp, sz, vp, vp]
    a.restype = ctypes.c_int
    assert a(fake, fake, fake, 0, fake, fake, -1.0, 1, 1, 8, 64, 2, 0.1, fake, fake, 1 << 30,
             None, None) == 1                                                    # c < 0
    assert a(fake, fake, fake, 0, fake, fake, 1.0, 1, 1, 8, 64, 2, 0.1, fake, fake, 64,
             None, None) == 3                                                    # ws
    lib.had_workspace_bytes.restype = ctypes.c_size_t
    lib.had_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.had_launch_count.argtypes = [ctypes.c_int] * 6
    # long workload: 64 heads of 64 MiB logits, 32 heads per 2 GiB group -> 2 groups
    assert lib.had_workspace_bytes(9, 4, 16, 4096, 64, 512) == 2 << 30
    assert lib.had_launch_count(9, 4, 16, 4096, 64, 512) == 4
    assert lib.had_launch_count(11, 4, 16, 4096, 64, 512) == 7
    assert lib.had_launch_count(8, 4, 16, 4096, 64, 512) == 1
    # ragged n: rows padded to a multiple of 4 floats
    assert lib.had_workspace_bytes(9, 1, 1, 130, 64, 5) >= 130 * 132 * 4
    assert lib.had_workspace_bytes(11, 1, 1, 130, 64, 5) >= 130 * (2 * 64 * 4 + 8 * 5) + 130 * 132 * 4


def test_bwd_argument_errors_return_before_any_cuda_call(lib):
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    fake = vp(4096)        # never dereferenced: the checks fail first
    b = lib.had_attention_bwd
    b.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, f, f, vp, vp, vp, vp, sz,
                  vp, vp]
    b.restype = ctypes.c_int
    ok = (fake, fake, fake, 0, fake, fake, fake, None, None, 1, 1, 8, 64, 2, 0.1, 1.0, fake,
          fake, fake, fake, 1 << 30, None, None)

    def call(**kw):
        a = list(ok)
        for pos, val in kw.items():
            a[int(pos[1:])] = val
        return b(*a)

    assert call(a12=96) == 2                      # d
    assert call(a13=9) == 1                       # N > n
    assert call(a15=-1.0) == 1                    # clip < 0
    assert call(a15=float("nan")) == 1            # clip NaN
    assert call(a14=float("inf")) == 1            # tau
    assert call(a6=None) == 1                     # no dout
    assert call(a7=fake) == 1                     # idx without logits
    assert call(a17=vp(4100)) == 1                # misaligned dk
    assert call(a20=64) == 3                      # workspace
    assert call(a15=float("inf"), a20=64) == 3    # clip = inf is allowed; fails on ws
    assert call(a7=fake, a8=fake, a20=64) == 3    # a given kept set; fails on ws
    lib.had_workspace_bytes.restype = ctypes.c_size_t
    lib.had_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.had_launch_count.argtypes = [ctypes.c_int] * 6
    # per query row: codes 16 B, per-key count, offset and cursor 16 B; per kept
    # pair: idx 4 B, logit 2 B, p and ds 8 B, a 16-byte key-list record
    assert lib.had_workspace_bytes(12, 1, 1, 128, 64, 16) >= 128 * (16 + 16 + 30 * 16)
    assert lib.had_launch_count(12, 4, 16, 4096, 64, 512) == 8
