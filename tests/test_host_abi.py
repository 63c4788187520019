"""Host-side tests of the C ABI (no GPU): the library loads, exports every symbol the
header declares with the binding's signatures, generates the same permutations as the
oracle's independent generator, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import poetx_ref as ref
from orthogonal_reparameterized_cnp_b200 import poetx as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "poetx.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(poetx_[a-z0-9_]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = P.lib()
    names = _declared_functions()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(P.SIGNATURES) == names  # the binding declares exactly the header's calls


def test_status_strings_and_version():
    lib = P.lib()
    for st in range(8):
        assert lib.poetx_status_string(st)
    assert lib.poetx_status_string(99) == b"unknown status"
    assert b"sm_100a" in lib.poetx_version()


@pytest.mark.parametrize("seed,n", [(0, 4), (1, 1), (0, 0), (12345, 2048), (2 ** 64 - 1, 5120),
                                    ((2 << 32) | (0 << 8) | 1, 14336)])
def test_perm_generator_bit_exact_against_oracle(seed, n):
    p, inv = P.make_perm(seed, n)
    q, jnv = ref.make_perm(seed, n)
    assert np.array_equal(p, q) and np.array_equal(inv, jnv)


def test_make_perm_rejects_bad_arguments():
    lib = P.lib()
    assert lib.poetx_make_perm(0, -1, None, None) == P.POETX_ERR_INVALID_ARG
    assert lib.poetx_make_perm(0, 3, None, None) == P.POETX_ERR_INVALID_ARG
    assert b"perm" in lib.poetx_last_error()


def test_cnp_validation_before_launch():
    lib = P.lib()
    fake = ctypes.c_void_p(0x10000)
    assert lib.poetx_cnp_fwd(fake, fake, None, 2, 0, 4, fake, 1 << 20, None) == P.POETX_ERR_SHAPE
    assert lib.poetx_cnp_fwd(fake, fake, None, 2, 8, 0, fake, 1 << 20, None) == P.POETX_ERR_SHAPE
    assert lib.poetx_cnp_fwd(fake, fake, None, 2, 8, 17, fake, 1 << 20, None) == P.POETX_ERR_SHAPE
    assert lib.poetx_cnp_fwd(None, fake, None, 2, 8, 4, fake, 1 << 20, None) == \
        P.POETX_ERR_INVALID_ARG
    assert lib.poetx_cnp_fwd(fake, fake, None, -1, 8, 4, fake, 1 << 20, None) == \
        P.POETX_ERR_INVALID_ARG
    odd = ctypes.c_void_p(0x10004)
    assert lib.poetx_cnp_fwd(odd, fake, None, 2, 8, 4, fake, 1 << 20, None) == P.POETX_ERR_ALIGN
    # scratch below one block's need
    assert lib.poetx_cnp_fwd(fake, fake, None, 2, 64, 4, fake, 1024, None) == \
        P.POETX_ERR_WORKSPACE
    assert lib.poetx_cnp_bwd(fake, None, fake, 2, 8, 4, fake, 1 << 20, None) == \
        P.POETX_ERR_INVALID_ARG
    # nothing to do is fine
    assert lib.poetx_cnp_fwd(None, None, None, 0, 8, 4, None, 0, None) == P.POETX_OK


def test_cnp_workspace_query():
    assert P.cnp_workspace(16, 256, 4) >= 16 * 4 * 256 * 256 * 4
    assert P.cnp_workspace(0, 256, 4) == 0
    assert P.cnp_workspace(4, 0, 4) == 0
    # large block counts are processed in chunks: the query stays bounded
    assert P.cnp_workspace(44032, 64, 6) < 8 << 30


def _desc(T=64, n=512, m=256, b=128, dtype=P.POETX_BF16, maps=True):
    fake = 0x20000 if maps else None
    return P.LinearDesc(T, n, m, b, dtype, fake, fake, fake, fake)


def test_linear_validation_before_launch():
    lib = P.lib()
    f = ctypes.c_void_p(0x30000)
    ws = ctypes.c_void_p(0x40000)
    big = 1 << 40

    def fwd(d, x=f, ws_bytes=big):
        return lib.poetx_linear_fwd(ctypes.byref(d), x, f, f, f, f, None, None, ws, ws_bytes, None)

    assert lib.poetx_linear_fwd(None, f, f, f, f, f, None, None, ws, big, None) == \
        P.POETX_ERR_INVALID_ARG
    assert fwd(_desc(n=500)) == P.POETX_ERR_SHAPE               # n % b
    assert fwd(_desc(b=64)) == P.POETX_ERR_SHAPE                # bf16 b outside {128,256,512}
    assert fwd(_desc(dtype=7)) == P.POETX_ERR_DTYPE
    assert fwd(_desc(maps=False)) == P.POETX_ERR_INVALID_ARG
    assert fwd(_desc(), x=None) == P.POETX_ERR_INVALID_ARG
    assert fwd(_desc(), x=ctypes.c_void_p(0x30002)) == P.POETX_ERR_ALIGN
    assert fwd(_desc(), ws_bytes=16) == P.POETX_ERR_WORKSPACE
    assert fwd(_desc(T=0)) == P.POETX_OK                        # empty token set: no-op
    assert fwd(_desc(T=-1)) == P.POETX_ERR_INVALID_ARG
    d = _desc()
    assert lib.poetx_linear_bwd(ctypes.byref(d), f, f, f, f, f, f, f, f, f, f, 2, ws, big, None) \
        == P.POETX_ERR_INVALID_ARG                              # accumulate not 0/1
    assert lib.poetx_linear_bwd(ctypes.byref(d), f, f, f, f, f, f, f, f, None, f, 0, ws, big,
                                None) == P.POETX_ERR_INVALID_ARG


def test_linear_workspace_queries():
    d = _desc(T=8192, n=2048, m=2048, b=256)
    fs = P.linear_fwd_workspace(d, True, True)
    assert fs >= 2 * 8192 * 2048 * 2          # V and Z scratch
    assert P.linear_fwd_workspace(d, False, False) >= fs + 2 * 8192 * 2048 * 2
    assert P.linear_bwd_workspace(d, False, False) > P.linear_bwd_workspace(d, True, True)


def test_outer_merge_validation_before_launch():
    lib = P.lib()
    f = ctypes.c_void_p(0x50000)
    big = 1 << 40

    def call(m=512, n=256, b=128, dtype=P.POETX_BF16, w=f, out=ctypes.c_void_p(0x60000),
             ws_bytes=big):
        return lib.poetx_outer_merge(w, f, f, m, n, b, f, f, f, f, out, dtype, f, ws_bytes, None)

    assert call(m=500) == P.POETX_ERR_SHAPE                 # m % b
    assert call(b=64) == P.POETX_ERR_SHAPE                  # bf16 needs b % 128 == 0
    assert call(b=0) == P.POETX_ERR_INVALID_ARG
    assert call(dtype=9) == P.POETX_ERR_DTYPE
    assert call(w=None) == P.POETX_ERR_INVALID_ARG
    assert call(out=f) == P.POETX_ERR_INVALID_ARG           # output aliases the input
    assert call(w=ctypes.c_void_p(0x50008)) == P.POETX_ERR_ALIGN
    assert call(ws_bytes=1024) == P.POETX_ERR_WORKSPACE
    assert P.outer_merge_workspace(2048, 2048, P.POETX_BF16) >= 2 * 2048 * 2048 * 2
    assert P.outer_merge_workspace(0, 2048, P.POETX_BF16) == 0


def test_int8_weight_validation_before_launch():
    lib = P.lib()
    f = ctypes.c_void_p(0x70000)
    assert lib.poetx_quantize_rows(f, f, f, 4, 8, 9, None) == P.POETX_ERR_DTYPE
    assert lib.poetx_quantize_rows(None, f, f, 4, 8, P.POETX_BF16, None) == \
        P.POETX_ERR_INVALID_ARG
    assert lib.poetx_quantize_rows(ctypes.c_void_p(0x70004), f, f, 4, 8, P.POETX_BF16, None) == \
        P.POETX_ERR_ALIGN
    assert lib.poetx_quantize_rows(f, f, f, 0, 8, P.POETX_BF16, None) == P.POETX_OK
    d32 = _desc(dtype=P.POETX_F32)
    assert P.linear_q8_scratch(d32) == 0
    d = _desc(T=64, n=512, m=256, b=128)
    assert P.linear_q8_scratch(d) >= 512 * 256 * 2
    ws = ctypes.c_void_p(0x80000)
    assert lib.poetx_linear_fwd_q8(ctypes.byref(d32), f, f, f, f, f, f, None, None, ws, 1 << 40,
                                   None) == P.POETX_ERR_DTYPE
    assert lib.poetx_linear_fwd_q8(ctypes.byref(d), f, f, f, None, f, f, None, None, ws, 1 << 40,
                                   None) == P.POETX_ERR_INVALID_ARG
    assert lib.poetx_linear_fwd_q8(ctypes.byref(d), f, f, f, f, f, f, None, None, ws, 16,
                                   None) == P.POETX_ERR_WORKSPACE


def test_merge_perm_q8_validation_before_launch():
    lib = P.lib()
    f = ctypes.c_void_p(0xA0000)
    assert lib.poetx_merge_perm_q8(f, f, f, 4, 8, f, f, 9, None) == P.POETX_ERR_DTYPE
    assert lib.poetx_merge_perm_q8(None, f, f, 4, 8, f, f, P.POETX_BF16, None) == \
        P.POETX_ERR_INVALID_ARG
    assert lib.poetx_merge_perm_q8(f, f, f, 4, 8, ctypes.c_void_p(0xA0004), f, P.POETX_BF16,
                                   None) == P.POETX_ERR_ALIGN
    assert lib.poetx_merge_perm_q8(f, f, f, 4, 200000, f, f, P.POETX_F32, None) == \
        P.POETX_ERR_SHAPE
    assert lib.poetx_merge_perm_q8(f, f, f, 0, 8, f, f, P.POETX_BF16, None) == P.POETX_OK


def test_profile_and_launch_counter_without_launches():
    n0 = P.launch_count()
    assert P.launch_count() == n0


def test_invert_perm_matches_the_generators_inverse():
    for seed, n in [(0, 1), (7, 64), (123, 5120)]:
        p, inv = P.make_perm(seed, n)
        assert np.array_equal(P.invert_perm(p), inv)
    assert P.invert_perm(np.zeros(0, dtype=np.int32)).shape == (0,)


def test_invert_perm_rejects_maps_that_are_not_bijections():
    lib = P.lib()
    with pytest.raises(P.PoetxError) as e:
        P.invert_perm([0, 2, 2, 1])              # 2 twice, 3 missing
    assert e.value.status == P.POETX_ERR_INVALID_ARG and "twice" in str(e.value)
    with pytest.raises(P.PoetxError) as e:
        P.invert_perm([0, 1, 4])                 # out of range
    assert e.value.status == P.POETX_ERR_INVALID_ARG and "outside" in str(e.value)
    with pytest.raises(P.PoetxError):
        P.invert_perm([-1, 0])
    a = (ctypes.c_int32 * 3)(0, 1, 2)
    assert lib.poetx_invert_perm(a, 3, a) == P.POETX_ERR_INVALID_ARG   # in place
    assert lib.poetx_invert_perm(None, 3, a) == P.POETX_ERR_INVALID_ARG
    assert lib.poetx_invert_perm(a, -1, a) == P.POETX_ERR_INVALID_ARG
    # nothing is written when the map is rejected
    inv = (ctypes.c_int32 * 3)(-7, -7, -7)
    bad = (ctypes.c_int32 * 3)(1, 1, 0)
    assert lib.poetx_invert_perm(bad, 3, inv) == P.POETX_ERR_INVALID_ARG
    assert list(inv) == [-7, -7, -7]


def test_layer_object_validates_index_maps_before_any_device_work():
    # PoetxLinear takes the inverse maps from the library; a map with a duplicate entry is
    # rejected there (the CUDA check comes after, so this holds without a GPU too)
    with pytest.raises(P.PoetxError) as e:
        P.PoetxLinear.__init__(object.__new__(P.PoetxLinear), _FakeW0(), None, None,
                               [0, 0, 1, 2], [0, 1, 2, 3], 2, 4, 8)
    assert e.value.status == P.POETX_ERR_INVALID_ARG and "bijection" in str(e.value)


class _FakeW0:
    shape = (4, 4)
    device = "cpu"
    dtype = None


def test_gemm_pairs_setter():
    prev = P.set_gemm_pairs(False)
    try:
        assert P.set_gemm_pairs(True) is False
        assert P.set_gemm_pairs(True) is True
        assert P.lib().poetx_set_gemm_pairs(2, None) == P.POETX_ERR_INVALID_ARG
    finally:
        P.set_gemm_pairs(prev)


def test_wait_limit_setter():
    prev = P.set_wait_limit(50_000_000)
    try:
        assert P.set_wait_limit(0) == 50_000_000   # 0 restores the 2 s default
        assert P.set_wait_limit(0) == 2_000_000_000
        with pytest.raises(P.PoetxError):
            P.set_wait_limit(61 * 10 ** 9)
    finally:
        P.set_wait_limit(prev)


def test_new_entry_points_validate_before_launch():
    lib = P.lib()
    f = ctypes.c_void_p(0x90000)
    assert lib.poetx_fma_probe(f, 0, 10, None) == P.POETX_ERR_INVALID_ARG
    assert lib.poetx_fma_probe(None, 1, 10, None) == P.POETX_ERR_INVALID_ARG
    assert lib.poetx_fma_probe(ctypes.c_void_p(0x90004), 1, 10, None) == P.POETX_ERR_ALIGN
    # the timeout self-test runs only on task-graph shapes and needs room for every block
    assert lib.poetx_selftest_wait_timeout(f, f, 2, 100, 4, f, 1 << 30, None) == \
        P.POETX_ERR_SHAPE
    assert lib.poetx_selftest_wait_timeout(f, f, 2, 64, 4, f, 1024, None) == \
        P.POETX_ERR_WORKSPACE
    assert lib.poetx_selftest_wait_timeout(f, f, 0, 64, 4, f, 1 << 30, None) == \
        P.POETX_ERR_INVALID_ARG
