"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""

import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "pisa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pisa_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    raw = lib.raw_lib()
    names = _header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(raw, n), n
    assert set(names) == set(lib.EXPORTS)


def test_keep_count_matches_the_oracle_reading(lib):
    for L, B, r in [(1024, 64, 0.25), (4608, 64, 0.25), (32760, 128, 0.15), (75600, 128, 0.10),
                    (119040, 128, 0.08), (1000, 128, 1.0), (1000, 64, 0.001), (50, 64, 0.3)]:
        assert lib.keep_count(L, B, r) == oracle.keep_count(L, B, r)
    assert lib.keep_count(0, 64, 0.5) == -1
    assert lib.keep_count(100, 64, 0.0) == -1
    assert lib.keep_count(100, 64, float("nan")) == -1


def test_workspace_sizes(lib):
    assert lib.workspace_size(1, 40, 75600, 128, 128, 60) > 0
    assert lib.workspace_size(1, 1, 1024, 64, 64, 4) > 0
    assert lib.stats_workspace_size(1, 24, 4608, 128, 64) > 0
    assert lib.workspace_size(1, 1, 1024, 96, 64, 4) == 0      # unsupported d
    assert lib.workspace_size(1, 1, 1024, 64, 32, 4) == 0      # unsupported block
    assert lib.workspace_size(1, 1, 1024, 64, 64, 17) == 0     # k > nb
    a = lib.workspace_size(1, 2, 1000, 128, 128, 2)
    b = lib.workspace_size(2, 2, 1000, 128, 128, 2)
    assert b > a


def test_status_strings(lib):
    for code in range(-6, 1):
        assert lib.status_string(code)
    assert "unknown" in lib.status_string(-99)


FAKE = ctypes.c_void_p(0x10000)        # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def test_invalid_arguments_are_rejected_on_the_host(lib):
    raw = lib.raw_lib()
    f = raw.pisa_attn_fwd
    ok_args = [FAKE, FAKE, FAKE, FAKE, 0, 1, 2, 1000, 128, 128, ctypes.c_float(0.25), FAKE,
               ctypes.c_size_t(1 << 40), None]

    def call(**over):
        a = list(ok_args)
        for i, val in over.items():
            a[int(i[1:])] = val
        return f(*a)

    assert call(a0=None) == lib.PISA_ERR_INVALID_ARG            # null q
    assert call(a3=MISALIGNED) == lib.PISA_ERR_INVALID_ARG      # misaligned out
    assert call(a8=96) == lib.PISA_ERR_UNSUPPORTED              # d = 96
    assert call(a9=32) == lib.PISA_ERR_UNSUPPORTED              # block = 32
    assert call(a7=0) == lib.PISA_ERR_INVALID_ARG               # L = 0
    assert call(a4=7) == lib.PISA_ERR_INVALID_ARG               # bad dtype
    assert call(a10=ctypes.c_float(-1.0)) == lib.PISA_ERR_INVALID_ARG
    assert call(a11=None) == lib.PISA_ERR_WORKSPACE
    assert call(a12=ctypes.c_size_t(1024)) == lib.PISA_ERR_WORKSPACE


def test_stage_entry_points_validate(lib):
    raw = lib.raw_lib()
    # pisa_select: k out of range, null pointers
    assert raw.pisa_select(FAKE, FAKE, FAKE, 1, 1, 1000, 128, 128, 9, FAKE, None) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_select(None, FAKE, FAKE, 1, 1, 1000, 128, 128, 2, FAKE, None) == lib.PISA_ERR_INVALID_ARG
    # pisa_block_stats: workspace too small
    assert raw.pisa_block_stats(FAKE, FAKE, FAKE, 0, 1, 1, 1000, 128, 128, FAKE, FAKE, FAKE, FAKE,
                                FAKE, ctypes.c_size_t(16), None) == lib.PISA_ERR_WORKSPACE
    # pisa_cov_norm / pisa_block_first_order: unsupported d
    assert raw.pisa_cov_norm(FAKE, FAKE, 0, 1, 1, 1000, 80, 128, FAKE, FAKE, FAKE, FAKE, None) == \
        lib.PISA_ERR_UNSUPPORTED
    assert raw.pisa_block_first_order(FAKE, FAKE, 0, 1, 1, 1000, 128, 128, None, FAKE, FAKE, None) == \
        lib.PISA_ERR_INVALID_ARG
    # pisa_attn_fwd_with_sel: k_sel out of range
    assert raw.pisa_attn_fwd_with_sel(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 1000, 128, 128, FAKE, FAKE, FAKE,
                                      FAKE, 0, FAKE, ctypes.c_size_t(1 << 30), None) == \
        lib.PISA_ERR_INVALID_ARG


def test_host_workspace_size(lib):
    import torch
    kk = 60
    full = lib.host_workspace_size(torch.bfloat16, 1, 40, 75600, 128, 128, kk, 8)
    assert full > 0
    assert lib.host_workspace_size(torch.float32, 1, 40, 75600, 128, 128, kk, 8) > full
    assert lib.host_workspace_size(torch.bfloat16, 1, 40, 75600, 128, 128, kk, 0) == 0   # chunk < 1
    assert lib.host_workspace_size(torch.float16, 1, 40, 75600, 128, 128, kk, 8) == 0    # bad dtype
    assert lib.host_workspace_size(torch.bfloat16, 1, 40, 75600, 96, 128, kk, 8) == 0    # d = 96
    # the forward's scratch is not monotonic in the slice count (the statistics
    # chunking depends on it), so the size must cover both chunk shapes that
    # occur: full chunks and the shorter last one
    sizes = [lib.workspace_size(1, n, 75600, 128, 128, kk) for n in range(1, 41)]
    assert any(sizes[n] < sizes[n - 1] for n in range(1, 40))      # a real non-monotonic case
    for chunk in (3, 7, 8, 16):
        need = max(sizes[chunk - 1], sizes[40 % chunk - 1] if 40 % chunk else 0)
        assert lib.host_workspace_size(torch.bfloat16, 1, 40, 75600, 128, 128, kk, chunk) > need
    # a chunk larger than the slice count is clamped to it
    assert lib.host_workspace_size(torch.bfloat16, 1, 3, 1000, 128, 128, 2, 64) == \
        lib.host_workspace_size(torch.bfloat16, 1, 3, 1000, 128, 128, 2, 3)


def test_host_entry_point_validates_before_any_cuda_call(lib):
    raw = lib.raw_lib()
    f = raw.pisa_attn_fwd_host
    ok = [FAKE, FAKE, FAKE, FAKE, 0, 1, 2, 1000, 128, 128, ctypes.c_float(0.25), 2, FAKE,
          ctypes.c_size_t(1 << 40), None]

    def call(**over):
        a = list(ok)
        for i, val in over.items():
            a[int(i[1:])] = val
        return f(*a)

    assert call(a1=None) == lib.PISA_ERR_INVALID_ARG            # null k_host
    assert call(a3=None) == lib.PISA_ERR_INVALID_ARG            # null out_host
    assert call(a11=0) == lib.PISA_ERR_INVALID_ARG              # chunk = 0
    assert call(a8=80) == lib.PISA_ERR_UNSUPPORTED              # d = 80
    assert call(a4=3) == lib.PISA_ERR_INVALID_ARG               # bad dtype
    assert call(a10=ctypes.c_float(0.0)) == lib.PISA_ERR_INVALID_ARG
    assert call(a12=None) == lib.PISA_ERR_WORKSPACE
    assert call(a13=ctypes.c_size_t(4096)) == lib.PISA_ERR_WORKSPACE
    assert call(a12=MISALIGNED) == lib.PISA_ERR_INVALID_ARG


def test_routing_variant_entry_points_validate(lib):
    raw = lib.raw_lib()
    # unknown route value
    assert raw.pisa_select_route(FAKE, FAKE, None, 1, 1, 1000, 128, 128, 2, 7, FAKE, None) == \
        lib.PISA_ERR_INVALID_ARG
    # the pooled route reads no M, covariance needs it
    assert raw.pisa_select_route(None, FAKE, None, 1, 1, 1000, 128, 128, 2, lib.PISA_ROUTE_POOLED, FAKE,
                                 None) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_select_route(FAKE, FAKE, None, 1, 1, 1000, 128, 128, 2, lib.PISA_ROUTE_COVARIANCE, FAKE,
                                 None) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_select_route(FAKE, FAKE, None, 1, 1, 1000, 128, 128, 9, lib.PISA_ROUTE_POOLED, FAKE,
                                 None) == lib.PISA_ERR_INVALID_ARG      # k > nb
    # spectral norm: null H, unsupported d, misaligned M
    assert raw.pisa_cov_norm_spectral(None, FAKE, 1, 1, 1000, 128, 128, FAKE, None) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_cov_norm_spectral(FAKE, FAKE, 1, 1, 1000, 96, 128, FAKE, None) == lib.PISA_ERR_UNSUPPORTED
    assert raw.pisa_cov_norm_spectral(FAKE, FAKE, 1, 1, 1000, 128, 128, MISALIGNED, None) == \
        lib.PISA_ERR_INVALID_ARG


def test_blockwise_entry_point_validates_before_any_cuda_call(lib):
    raw = lib.raw_lib()
    f = raw.pisa_attn_fwd_blockwise_with_sel
    args = lambda H=FAKE, d=128, k=2, sel=FAKE, dt=lib.PISA_BF16: (
        FAKE, FAKE, FAKE, FAKE, dt, 1, 1, 1000, d, 128, FAKE, FAKE, H, sel, k, None)
    assert f(*args(H=None)) == lib.PISA_ERR_INVALID_ARG          # no block matrices
    assert f(*args(H=MISALIGNED)) == lib.PISA_ERR_INVALID_ARG
    assert f(*args(sel=None)) == lib.PISA_ERR_INVALID_ARG
    assert f(*args(d=96)) == lib.PISA_ERR_UNSUPPORTED
    assert f(*args(k=0)) == lib.PISA_ERR_INVALID_ARG
    assert f(*args(k=9)) == lib.PISA_ERR_INVALID_ARG              # k > nb = 8
    assert f(*args(dt=7)) == lib.PISA_ERR_INVALID_ARG


def test_tuning_entry_points_validate_before_any_cuda_call(lib):
    raw = lib.raw_lib()
    t = lib._Tuning(0, 40, 0)  # select rows above 32
    assert raw.pisa_set_tuning(1, 2, 1000, 128, 128, ctypes.byref(t)) == lib.PISA_ERR_INVALID_ARG
    t = lib._Tuning(-1, 0, 0)
    assert raw.pisa_set_tuning(1, 2, 1000, 128, 128, ctypes.byref(t)) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_set_tuning(1, 2, 1000, 96, 128, None) == lib.PISA_ERR_UNSUPPORTED
    assert raw.pisa_get_tuning(1, 2, 1000, 128, 128, None) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_tuning_save(None) == lib.PISA_ERR_INVALID_ARG
    assert raw.pisa_tuning_load(None) == lib.PISA_ERR_INVALID_ARG
    f = raw.pisa_autotune
    ok = [FAKE, FAKE, FAKE, FAKE, 0, 1, 2, 1000, 128, 128, ctypes.c_float(0.25), FAKE, ctypes.c_size_t(1 << 40),
          None, None]
    a = list(ok); a[3] = None
    assert f(*a) == lib.PISA_ERR_INVALID_ARG                    # no output buffer
    a = list(ok); a[12] = ctypes.c_size_t(64)
    assert f(*a) == lib.PISA_ERR_WORKSPACE
