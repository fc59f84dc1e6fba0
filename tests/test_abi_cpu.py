"""Host-only checks of the C ABI: the library loads without a GPU, exports
every entry point that include/magicpig.h declares, and rejects bad arguments
on the host (no kernel is launched, no CUDA call is made)."""
import ctypes
import os
import re

import pytest

import lsh_sampled_sparse_simhash_b200 as mp
from lsh_sampled_sparse_simhash_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "magicpig.h")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    return mp.library()


def good_shape(**kw):
    d = dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, capacity=1024, k_bits=8, n_tables=75,
             sink=4, window=64, code_layout=0)
    d.update(kw)
    return B._CShape(*d.values())


def test_exports_every_declared_symbol(lib):
    decl = re.findall(r"^\s*(?:int|const char \*)\s*(mp_\w+)\s*\(", open(HEADER).read(), re.M)
    assert len(decl) >= 8
    for name in decl:
        assert hasattr(lib, name), name
    # and nothing undeclared under the mp_ prefix
    import subprocess
    syms = subprocess.run(["nm", "-D", "--defined-only", mp.library_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (mp_\w+)$", syms, re.M))
    assert exported == set(decl), exported ^ set(decl)


def test_library_has_no_driver_link_dependency(lib):
    import subprocess
    out = subprocess.run(["ldd", mp.library_path], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert mp.status_string(code).startswith("MP_")


def test_codes_bytes_formula(lib):
    n = ctypes.c_size_t()
    for K, L, lay in [(8, 75, 0), (10, 150, 0), (8, 75, 2), (8, 75, 1), (10, 150, 2)]:
        s = good_shape(k_bits=K, n_tables=L, code_layout=lay)
        assert lib.mp_codes_bytes(ctypes.byref(s), ctypes.byref(n)) == 0
        assert n.value == 2 * 2 * L * K * 1024 // 8


@pytest.mark.parametrize("bad", [
    dict(head_dim=64), dict(k_bits=9), dict(n_tables=1), dict(n_tables=256), dict(n_q_heads=6),
    dict(n_q_heads=32, n_kv_heads=2), dict(capacity=1000), dict(capacity=0), dict(batch=0),
    dict(sink=-1), dict(window=-1), dict(n_kv_heads=0), dict(code_layout=3), dict(code_layout=-1),
    dict(k_bits=10, n_tables=150, code_layout=1)])
def test_bad_shapes_rejected(lib, bad):
    n = ctypes.c_size_t()
    s = good_shape(**bad)
    assert lib.mp_codes_bytes(ctypes.byref(s), ctypes.byref(n)) == mp.MP_ERR_SHAPE
    assert lib.mp_hash_keys(ctypes.byref(s), 16, 16, None, 10, 16, None, None) == mp.MP_ERR_SHAPE
    assert lib.mp_decode_workspace_bytes(ctypes.byref(s), 10, ctypes.byref(n)) == mp.MP_ERR_SHAPE


def test_null_and_misaligned_pointers_rejected(lib):
    s = good_shape()
    assert lib.mp_hash_keys(ctypes.byref(s), None, 16, None, 10, 16, None, None) == mp.MP_ERR_ARG
    assert lib.mp_hash_keys(ctypes.byref(s), 16, 18, None, 10, 16, None, None) == mp.MP_ERR_ALIGN
    assert lib.mp_hash_keys(ctypes.byref(s), 16, 16, 18, 10, 16, None, None) == mp.MP_ERR_ALIGN
    assert lib.mp_hash_keys(ctypes.byref(s), 16, 16, None, 10, 16, 18, None) == mp.MP_ERR_ALIGN
    assert lib.mp_hash_queries(ctypes.byref(s), 16, 16, None, None) == mp.MP_ERR_ARG
    assert lib.mp_append_token(ctypes.byref(s), 16, 16, 16, 16, 16, 16, None, None, None) == mp.MP_ERR_ARG
    assert lib.mp_append_token(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, 18, None) == mp.MP_ERR_ALIGN
    assert lib.mp_read_status(None, None, None) == mp.MP_ERR_ARG


def test_lengths_and_workspace_checked(lib):
    s = good_shape()
    n = ctypes.c_size_t()
    assert lib.mp_hash_keys(ctypes.byref(s), 16, 16, None, 1025, 16, None, None) == mp.MP_ERR_CAPACITY
    assert lib.mp_hash_keys(ctypes.byref(s), 16, 16, None, -1, 16, None, None) == mp.MP_ERR_CAPACITY
    assert lib.mp_decode_workspace_bytes(ctypes.byref(s), 1025, ctypes.byref(n)) == mp.MP_ERR_CAPACITY
    assert lib.mp_decode_workspace_bytes(ctypes.byref(s), 1000, ctypes.byref(n)) == 0
    need = n.value
    args = [16] * 6 + [1000] + [16] * 4
    assert lib.mp_decode_attend(ctypes.byref(s), *args, need - 1, None, None) == mp.MP_ERR_WORKSPACE
    args[6] = 2000
    assert lib.mp_decode_attend(ctypes.byref(s), *args, need, None, None) == mp.MP_ERR_CAPACITY


def test_workspace_grows_with_max_len(lib):
    s = good_shape(capacity=65536)
    sizes = []
    for m in (0, 1, 2048, 2049, 65536):
        n = ctypes.c_size_t()
        assert lib.mp_decode_workspace_bytes(ctypes.byref(s), m, ctypes.byref(n)) == 0
        sizes.append(n.value)
    assert sizes == sorted(sizes) and sizes[1] < sizes[3]


def test_decode_path_selector_checked(lib):
    """mp_decode_debug.path: out-of-range values are MP_ERR_ARG; the fused path
    needs bit-plane codes and at most 4 query heads per kv head (MP_ERR_SHAPE).
    Rejected on the host, so nothing launches."""
    A = 1 << 12  # aligned fake device pointers (never dereferenced)
    for lay, G, path, want in [(1, 4, 2, mp.MP_ERR_SHAPE), (2, 8, 2, mp.MP_ERR_SHAPE), (2, 4, 7, mp.MP_ERR_ARG),
                               (2, 4, 4, mp.MP_ERR_ARG), (2, 4, -1, mp.MP_ERR_ARG)]:
        s = good_shape(code_layout=lay, n_q_heads=2 * G)
        need = ctypes.c_size_t()
        assert lib.mp_decode_workspace_bytes(ctypes.byref(s), 1024, ctypes.byref(need)) == 0
        dbg = B._CDebug(None, None, None, path)
        rc = lib.mp_decode_attend(ctypes.byref(s), A, A, A, A, A, A, 1024, A, A, A, A, need.value, ctypes.byref(dbg),
                                  None)
        assert rc == want, (lay, G, path, rc)


def test_hash_range_checked(lib):
    """mp_hash_keys_range: the range starts on a 128-token tile and ends within
    the capacity; rejected on the host, so nothing launches."""
    s = good_shape()
    A = 1 << 12
    f = lib.mp_hash_keys_range
    assert f(ctypes.byref(s), A, A, 64, 10, A, None, None) == mp.MP_ERR_ALIGN
    assert f(ctypes.byref(s), A, A, 896, 129, A, None, None) == mp.MP_ERR_CAPACITY
    assert f(ctypes.byref(s), A, A, -128, 10, A, None, None) == mp.MP_ERR_CAPACITY
    assert f(ctypes.byref(s), A, A, 0, -1, A, None, None) == mp.MP_ERR_CAPACITY


def test_binding_declares_argument_types_for_every_entry_point(lib):
    """Every C entry point has ctypes argument types, so no 64-bit pointer or
    stream handle is ever passed as a C int."""
    decl = re.findall(r"^\s*(?:int|const char \*)\s*(mp_\w+)\s*\(", open(HEADER).read(), re.M)
    for name in decl:
        assert getattr(lib, name).argtypes is not None, name


def test_int8_key_entry_points_checked(lib):
    """mp_quantize_keys / mp_append_token_q8 / mp_decode_attend_q8 reject null
    and misaligned pointers, out-of-range token ranges and the bf16-only
    kernel paths on the host, so nothing launches."""
    s = good_shape()
    A = 1 << 12
    q = lib.mp_quantize_keys
    assert q(ctypes.byref(s), None, None, 0, 10, A, None) == mp.MP_ERR_ARG
    assert q(ctypes.byref(s), A, None, 0, 10, None, None) == mp.MP_ERR_ARG
    assert q(ctypes.byref(s), A, None, 0, 10, A + 8, None) == mp.MP_ERR_ALIGN
    assert q(ctypes.byref(s), A, A + 2, 0, 10, A, None) == mp.MP_ERR_ALIGN
    assert q(ctypes.byref(s), A, None, 1000, 25, A, None) == mp.MP_ERR_CAPACITY
    assert q(ctypes.byref(s), A, None, -1, 10, A, None) == mp.MP_ERR_CAPACITY
    assert q(ctypes.byref(s), A, None, 0, -1, A, None) == mp.MP_ERR_CAPACITY
    ap = lib.mp_append_token_q8
    assert ap(ctypes.byref(s), A, A, A, A, A, A, A, None, None, None) == mp.MP_ERR_ARG
    assert ap(ctypes.byref(s), A, A, A, A, A, A, A, A + 4, None, None) == mp.MP_ERR_ALIGN
    assert ap(ctypes.byref(s), A, A, A, A, A, A, A, A, A + 2, None) == mp.MP_ERR_ALIGN
    assert ap(ctypes.byref(s), A, A, A, A + 2, A, A, A, A, None, None) == mp.MP_ERR_ALIGN  # k_cache may be NULL
    assert ap(ctypes.byref(s), A, A, A, A, None, A, A, A, None, None) == mp.MP_ERR_ARG     # v_cache may not
    need = ctypes.c_size_t()
    assert lib.mp_decode_workspace_bytes(ctypes.byref(s), 1024, ctypes.byref(need)) == 0
    d = lib.mp_decode_attend_q8
    assert d(ctypes.byref(s), A, A, A, None, A, A, 1024, A, A, A, A, need.value, None, None) == mp.MP_ERR_ARG
    assert d(ctypes.byref(s), A, A, A, A + 4, A, A, 1024, A, A, A, A, need.value, None, None) == mp.MP_ERR_ALIGN
    assert d(ctypes.byref(s), A, A, A, A, A, A, 1024, A, A, A, A, need.value - 1, None, None) == mp.MP_ERR_WORKSPACE
    assert d(ctypes.byref(s), A, A, A, A, A, A, 1025, A, A, A, A, need.value, None, None) == mp.MP_ERR_CAPACITY
    for path, want in [(mp.MP_PATH_FUSED, mp.MP_ERR_SHAPE), (mp.MP_PATH_TC, mp.MP_ERR_SHAPE), (4, mp.MP_ERR_ARG)]:
        dbg = B._CDebug(None, None, None, path)
        assert d(ctypes.byref(s), A, A, A, A, A, A, 1024, A, A, A, A, need.value, ctypes.byref(dbg),
                 None) == want, path
    m = re.search(r"#define MP_Q8_ROW_BYTES (\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == B.Q8_ROW_BYTES == 144


def test_auto_layout_threshold_matches_header():
    """The binding's copy of the MP_CODES_AUTO rule uses the header's threshold."""
    m = re.search(r"#define MP_CODES_AUTO_PLANES_MIN \(1 << (\d+)\)", open(HEADER).read())
    assert m and mp.MP_CODES_AUTO_PLANES_MIN == 1 << int(m.group(1))
    assert not mp.auto_planes(1, 8, 16512, 8)        # a 16k-token layer: byte codes
    assert mp.auto_planes(4, 8, 131200, 8)           # four 128k-token sequences: bit planes
    assert mp.auto_planes(1, 1, 128, 10)             # K = 10: always bit planes


def test_skip_scan_hook_only_on_the_split_path(lib):
    """mp_decode_debug.skip_scan (the failure-path test hook) is refused with
    the fused and tcgen05 paths, whose kernels would not wait for the scan's
    flags; rejected on the host, so nothing launches."""
    A = 1 << 12
    s = good_shape(code_layout=2, n_q_heads=8)
    need = ctypes.c_size_t()
    assert lib.mp_decode_workspace_bytes(ctypes.byref(s), 1024, ctypes.byref(need)) == 0
    for path in (mp.MP_PATH_FUSED, mp.MP_PATH_TC):
        dbg = B._CDebug(None, None, None, path, 1)
        rc = lib.mp_decode_attend(ctypes.byref(s), A, A, A, A, A, A, 1024, A, A, A, A, need.value, ctypes.byref(dbg),
                                  None)
        assert rc == mp.MP_ERR_ARG, (path, rc)
