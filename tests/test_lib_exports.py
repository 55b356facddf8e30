"""The C-ABI library builds for sm_100a, loads, and exports every symbol that
include/lora.h declares; host-side argument checks answer before any launch.
No compute call is made here (no GPU needed)."""
import ctypes
import os
import re

import numpy as np

import pytest

from adapter_gemm_builder_b200 import build as lbuild
from adapter_gemm_builder_b200 import lora as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    lbuild.build()
    return L.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "lora.h")).read()
    return re.findall(r"LORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(_declared())
    for n in ["lora_build_segments", "lora_shrink", "lora_expand", "lora_apply",
              "fp8_gemm_lora_epilogue"]:
        assert n in names
    assert names == set(L.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_library_is_sm100a_only():
    # every object is compiled with -gencode arch=compute_100a,code=sm_100a
    assert lbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_version_and_constants(lib):
    assert lib.lora_version() >= 1
    assert lib.lora_tile_tokens() == 64
    # decode-like batches (T <= 64 and T <= 2 * n_adapters) get 4-token tiles
    assert lib.lora_tile_tokens_for(36, 32) == 4
    assert lib.lora_tile_tokens_for(64, 32) == 4
    assert lib.lora_tile_tokens_for(1, 1) == 4
    assert lib.lora_tile_tokens_for(64, 4) == 64
    assert lib.lora_tile_tokens_for(65, 1000) == 64
    assert lib.lora_tile_tokens_for(-1, 4) == -1 and lib.lora_tile_tokens_for(4, 0) == -1
    # floor((T + (t - 1) * min(n, T)) / t)
    assert lib.lora_max_tiles(36, 32) == (36 + 3 * 32) // 4
    assert lib.lora_max_tiles(512, 256) == (512 + 63 * 256) // 64
    assert lib.lora_max_tiles(-1, 4) == -1
    assert lib.lora_status_string(L.LORA_ERR_TIMEOUT).decode()


def _pool(**kw):
    d = dict(A=16, B=32, ranks=None, scales=None, n_slices=1, n_adapters=4, h_in=64, h_out=64,
             r_max=16)
    d.update(kw)
    return L.lora_pool_t(d["A"], d["B"], d["ranks"], d["scales"], d["n_slices"], d["n_adapters"],
                         d["h_in"], d["h_out"], d["r_max"])


def test_workspace_sizes(lib):
    assert lib.lora_workspace_size(L.LORA_OP_SHRINK, 10, 0, None) == 0
    assert lib.lora_workspace_size(L.LORA_OP_APPLY, 10, 0, None) == ctypes.c_size_t(-1).value
    pa = _pool(n_slices=4, n_adapters=256, h_in=5120, h_out=5120, r_max=64)
    assert lib.lora_workspace_size(L.LORA_OP_APPLY, 36, 0, ctypes.byref(_pool(n_adapters=32))) == 0
    # a general batch: the tile rows in cost order, 16 bytes per row of lora_max_tiles
    n = lib.lora_workspace_size(L.LORA_OP_APPLY, 512, 0, ctypes.byref(pa))
    assert n >= 16 * lib.lora_max_tiles(512, 256) and n % 256 == 0
    # long segments (T >= 32 n_adapters, h_out >= 128): the shrink's planes of v in fp32
    # (one per part of h_in, at most 8), n_slices x T x r_max x 4 bytes each, rounded up to 256
    pl = _pool(n_slices=2, n_adapters=8, h_in=4096, h_out=11008, r_max=64)
    assert lib.lora_workspace_size(L.LORA_OP_APPLY, 2704, 0, ctypes.byref(pl)) == \
        -(-8 * 2 * 2704 * 64 * 4 // 256) * 256
    pl = _pool(n_slices=1, n_adapters=2, h_in=192, h_out=128, r_max=16)
    assert lib.lora_workspace_size(L.LORA_OP_APPLY, 64, 0, ctypes.byref(pl)) == -(-3 * 64 * 16 * 4 // 256) * 256
    # ... but not with a narrow y (h_out < 128) or fewer tokens per adapter
    assert lib.lora_workspace_size(L.LORA_OP_APPLY, 2704, 0, ctypes.byref(_pool(n_adapters=8, h_out=120))) \
        == -(-16 * lib.lora_max_tiles(2704, 8) // 256) * 256
    assert lib.lora_workspace_size(L.LORA_OP_APPLY, 255, 0, ctypes.byref(_pool(n_adapters=8, h_out=256))) \
        == -(-16 * lib.lora_max_tiles(255, 8) // 256) * 256
    p = _pool(h_in=8192, h_out=28672)
    n = lib.lora_workspace_size(L.LORA_OP_FP8_GEMM, 256, 8192, ctypes.byref(p))
    assert n >= 256 + 256 * 8192 + 256 * 4 + 256 * 16 * 4
    n0 = lib.lora_workspace_size(L.LORA_OP_FP8_GEMM, 256, 8192, None)
    assert n0 < n
    # a prefill through a GEMM call (M > 1024, long segments): the split path's apply
    # holds the tensor-core shrink's eight planes of v in the same workspace
    pp = _pool(n_adapters=8, h_in=4096, h_out=11008, r_max=64)
    for op in (L.LORA_OP_FP8_GEMM, L.LORA_OP_BF16_GEMM):
        big = lib.lora_workspace_size(op, 2704, 4096, ctypes.byref(pp))
        base = lib.lora_workspace_size(op, 2704, 4096, None)
        assert big - base >= 8 * 2704 * 64 * 4
    assert lib.lora_workspace_size(99, 1, 1, None) == ctypes.c_size_t(-1).value
    assert lib.lora_workspace_size(L.LORA_OP_FP8_GEMM, 4, 0, None) == ctypes.c_size_t(-1).value


def _seg(T=8, n=4):
    return L.lora_segments_t(16, 32, 48, 64, 80, 96, T, n)


@pytest.mark.parametrize("bad,code", [
    (dict(r_max=72), L.LORA_ERR_UNSUPPORTED),
    (dict(r_max=12), L.LORA_ERR_INVALID_ARG),
    (dict(r_max=24), L.LORA_ERR_UNSUPPORTED),
    (dict(h_in=100), L.LORA_ERR_INVALID_ARG),
    (dict(A=None), L.LORA_ERR_INVALID_ARG),
    (dict(A=24), L.LORA_ERR_INVALID_ARG),            # misaligned
    (dict(n_adapters=0), L.LORA_ERR_INVALID_ARG),
    (dict(n_adapters=20000), L.LORA_ERR_UNSUPPORTED),
])
def test_pool_checks_before_launch(lib, bad, code):
    p = _pool(**bad)
    s = _seg(n=p.n_adapters)
    st = lib.lora_apply(ctypes.c_void_p(1024), 0, ctypes.byref(p), ctypes.byref(s),
                        ctypes.c_void_p(2048), None, 0, None)
    assert st == code


def test_segment_and_pointer_checks(lib):
    p = _pool()
    s = _seg(n=5)  # n_adapters mismatch
    assert lib.lora_shrink(ctypes.c_void_p(1024), 0, ctypes.byref(p), ctypes.byref(s),
                           ctypes.c_void_p(2048), None, 0, None) == L.LORA_ERR_INVALID_ARG
    s = _seg()
    assert lib.lora_shrink(None, 0, ctypes.byref(p), ctypes.byref(s), ctypes.c_void_p(2048), None,
                           0, None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_shrink(ctypes.c_void_p(1024), 12, ctypes.byref(p), ctypes.byref(s),
                           ctypes.c_void_p(2048), None, 0, None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_expand(ctypes.c_void_p(1028), ctypes.byref(p), ctypes.byref(s),
                           ctypes.c_void_p(2048), None, 0, None) == L.LORA_ERR_INVALID_ARG
    # empty batch: nothing to do, no launch
    s0 = _seg(T=0)
    assert lib.lora_apply(ctypes.c_void_p(1024), 0, ctypes.byref(p), ctypes.byref(s0),
                          ctypes.c_void_p(2048), None, 0, None) == L.LORA_OK


def test_fp8_checks_before_launch(lib):
    x, w, sw, y = (ctypes.c_void_p(v) for v in (1024, 2048, 4096, 8192))
    ws = ctypes.c_void_p(16384)
    # K not a multiple of 16
    assert lib.fp8_gemm_lora_epilogue(x, 4, 24, 64, w, sw, None, None, y, ws, 1 << 20,
                                      None) == L.LORA_ERR_INVALID_ARG
    # workspace too small
    assert lib.fp8_gemm_lora_epilogue(x, 4, 64, 64, w, sw, None, None, y, ws, 16,
                                      None) == L.LORA_ERR_WORKSPACE
    # LoRA pool that does not match the GEMM
    p = _pool(h_in=64, h_out=128)
    s = _seg(T=4)
    assert lib.fp8_gemm_lora_epilogue(x, 4, 64, 64, w, sw, ctypes.byref(p), ctypes.byref(s), y, ws,
                                      1 << 20, None) == L.LORA_ERR_INVALID_ARG
    # segments for a different token count
    p = _pool(h_in=64, h_out=64)
    s = _seg(T=5)
    assert lib.fp8_gemm_lora_epilogue(x, 4, 64, 64, w, sw, ctypes.byref(p), ctypes.byref(s), y, ws,
                                      1 << 20, None) == L.LORA_ERR_INVALID_ARG
    assert lib.fp8_quantize_rows(x, 4, 8, w, sw, None) == L.LORA_ERR_INVALID_ARG
    assert lib.fp8_quantize_rows(x, 0, 16, w, sw, None) == L.LORA_OK


def test_build_segments_checks(lib):
    s = _seg(T=8, n=4)
    assert lib.lora_build_segments(None, 8, 4, ctypes.byref(s), 0, None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_build_segments(ctypes.c_void_p(64), 9, 4, ctypes.byref(s), 0,
                                   None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_build_segments(ctypes.c_void_p(64), 8, 0, ctypes.byref(s), 0,
                                   None) == L.LORA_ERR_INVALID_ARG
    big = _seg(T=8, n=20000)
    assert lib.lora_build_segments(ctypes.c_void_p(64), 8, 20000, ctypes.byref(big), 0,
                                   None) == L.LORA_ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(tmp_path):
    missing = str(tmp_path / "liblora.so")
    saved = L._lib
    L._lib = None
    try:
        with pytest.raises(L.LoraLibraryMissing):
            L.load(missing)
    finally:
        L._lib = saved


def test_max_tiles_bounds_every_id_mix(lib):
    """The tile-row bound holds for the worst cases of the tile rule: every adapter
    one token more than a multiple of the tile size, all tokens on one adapter,
    and random mixes (rows counted by the tile rule over the oracle's grouping)."""
    import oracle
    from tile_rule import expected_tiles, tile_tokens
    rng = np.random.default_rng(7)
    cases = [(36, 32), (64, 32), (48, 24), (5, 2), (64, 4), (300, 7), (1000, 999), (130, 64)]
    for T, n in cases:
        t = lib.lora_tile_tokens_for(T, n)
        assert t == tile_tokens(T, n), (T, n)
        bound = lib.lora_max_tiles(T, n)
        mixes = [rng.integers(0, n, T), np.zeros(T, np.int64), np.arange(T) % n,
                 np.repeat(np.arange(n), t + 1)[:T]]
        for ids in mixes:
            seg = oracle.build_segments(ids.astype(np.int32), n)
            rows = expected_tiles(seg["indptr"], seg["active"], seg["counts"][1], t)
            assert len(rows) <= bound, (T, n, t)


def test_debug_wait_limit_validates_and_restores(lib):
    assert lib.lora_debug_set_wait_limit(999, 0) == L.LORA_ERR_INVALID_ARG       # below 1 us
    assert lib.lora_debug_set_wait_limit(3_000_000_000, 0) == L.LORA_ERR_INVALID_ARG  # above 2 s
    assert lib.lora_debug_set_wait_limit(1_000_000, 2) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_debug_set_wait_limit(1_000_000, 1) == L.LORA_OK
    assert lib.lora_debug_set_wait_limit(0, 0) == L.LORA_OK                      # default again


def test_bench_launch_rule_matches_the_library(lib):
    """bench.py counts this library's launches per apply (gpu_launches) with its own copy
    of the rule that sends a batch to the tensor-core shrink and expand; the library's
    rule shows in the APPLY workspace size (planes of v instead of the tile order)."""
    import sys
    from types import SimpleNamespace
    sys.path.insert(0, ROOT)
    import bench
    for T, n, h_in, h_out in [(2704, 8, 4096, 11008), (512, 256, 5120, 5120), (36, 32, 4096, 4096),
                              (64, 2, 4096, 4096), (63, 2, 4096, 4096), (256, 8, 512, 128),
                              (256, 8, 512, 120), (255, 8, 512, 128), (1100, 16, 8192, 28672),
                              (64, 64, 1024, 1024), (4096, 1, 64, 200)]:
        pool = _pool(n_adapters=n, h_in=h_in, h_out=h_out, r_max=64)
        got = lib.lora_workspace_size(L.LORA_OP_APPLY, T, 0, ctypes.byref(pool))
        planes = min(8, -(-h_in // 64))
        tc_size = -(-max(planes * T * 64 * 4, 16 * lib.lora_max_tiles(T, n)) // 256) * 256
        p = SimpleNamespace(T=T, n_adapters=n, h_in=h_in, h_out=h_out)
        assert bench.tc_path(p) == (got == tc_size and got != 0), (T, n, h_in, h_out, got)


def test_bench_launches_per_apply(lib):
    """The launches per lora_apply that bench.py multiplies into gpu_launches, on the
    bench workloads' shapes (148 SMs): the decode kernel alone; the tile-ordering kernel
    and the cluster kernel when the clusters need more than one wave; the tensor-core
    shrink and expand for long segments; the cluster kernel alone otherwise."""
    import sys
    from types import SimpleNamespace as NS
    sys.path.insert(0, ROOT)
    import bench
    cases = {
        "bgmv_decode": (NS(T=36, n_adapters=32, n_slices=1, h_in=4096, h_out=4096), 1),
        "identical": (NS(T=36, n_adapters=32, n_slices=1, h_in=4096, h_out=4096), 1),
        "sgmv_tiny": (NS(T=64, n_adapters=4, n_slices=1, h_in=1024, h_out=1024), 1),
        "sgmv_prefill": (NS(T=2704, n_adapters=8, n_slices=1, h_in=4096, h_out=11008), 2),
        "many_tenants": (NS(T=512, n_adapters=256, n_slices=4, h_in=5120, h_out=5120), 2),
    }
    for name, (p, want) in cases.items():
        assert bench.apply_launches(p, sm_count=148) == want, name
