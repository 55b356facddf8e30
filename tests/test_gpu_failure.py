"""Failure detection without a GPU fault: a bounded device-side wait is made to
run out, and the kernel must return, the status call must report
LORA_ERR_TIMEOUT, and the next normal call must be correct.

The wait that runs out is one on a barrier that nothing completes (a test hook,
lora_debug_set_wait_limit(limit, inject_stall=1)): one CTA of each launch
waits on it before its first copy, under a limit of 1 ms, then takes the same
abort path a real stall would take (drain what it issued, still take part in
every barrier of its cluster, leave). No trap, assert, bad address or endless
loop is involved, and the limit is restored before the test ends."""
import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from gpu_util import (TOL_BF16, TOL_FP8, DeviceProblem, assert_close, dev, dev_bf16, f64,
                      host_bf16_bits, oracle_apply)

pytestmark = pytest.mark.gpu

# status bits of the SGMV kernels' waits (copies, v exchange, the stall, v counters) and of
# the FP8 GEMM's stall; which SGMV wait runs out first depends on timing (the CTAs that
# exchange v with the stalled one, or wait for its part, give up as well)
SGMV_WAIT_BITS = 0x100 | 0x200 | 0x400 | 0x800 | 0x2000 | 0x4000
STALL_FP8 = 0x400


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()
    yield
    L.lora_debug_set_wait_limit(0, False)


def _stalled(fn):
    L.lora_debug_set_wait_limit(1_000_000, inject_stall=True)  # 1 ms
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        L.lora_debug_set_wait_limit(0, False)


def test_sgmv_wait_runs_out_then_next_call_is_correct():
    # 150 tokens over 6 adapters: 64-token tiles, clusters of 2 CTAs, one-phase exchange
    p = wl.make_lora_problem("t", 11, T=150, n_adapters=6, h_in=520, h_out=392, r_max=32,
                             ids_kind="zipf", none_frac=0.1, rank_choices=(1, 5, 8, 13, 24, 32))
    d = DeviceProblem(p)
    y = d.y_in()
    _stalled(lambda: L.lora_apply(d.x, d.pool, d.seg, y))
    st, detail = L.lora_segments_status(d.seg)
    assert st == L.LORA_ERR_TIMEOUT and detail & SGMV_WAIT_BITS, hex(detail)
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK  # the query cleared the word
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, "after a timeout")


def test_sgmv_shrink_wait_runs_out_then_next_call_is_correct():
    # 300 tokens on 3 adapters (multi-tile segments), shrink only
    p = wl.make_lora_problem("t", 12, T=300, n_adapters=3, h_in=1024, h_out=256, r_max=16,
                             ids_kind="sorted_zipf", none_frac=0.1)
    d = DeviceProblem(p)
    v = torch.full((1, p.T, p.r_max), float("nan"), device="cuda")
    _stalled(lambda: L.lora_shrink(d.x, d.pool, d.seg, v))
    st, detail = L.lora_segments_status(d.seg)
    assert st == L.LORA_ERR_TIMEOUT and detail & SGMV_WAIT_BITS, hex(detail)
    L.lora_shrink(d.x, d.pool, d.seg, v)
    torch.cuda.synchronize()
    want = oracle.lora_shrink(p.x[0], p.A[0], p.ranks, p.ids)
    has = p.ids >= 0
    assert_close(v.cpu().numpy()[0][has].astype(np.float64), want[has], TOL_BF16, "shrink")


def test_sgmv_tc_expand_wait_runs_out_then_next_call_is_correct():
    # 300 tokens on 3 adapters: long segments, so lora_expand runs the tensor-core expand
    # (its stalled CTA drains its copies and MMAs and releases TMEM before it leaves)
    p = wl.make_lora_problem("t", 13, T=300, n_adapters=3, h_in=256, h_out=392, r_max=32,
                             ids_kind="zipf", none_frac=0.1, rank_choices=(5, 32))
    d = DeviceProblem(p)
    rng = np.random.default_rng(13)
    v = rng.standard_normal((1, p.T, p.r_max)).astype(np.float32)
    y = d.y_in()
    _stalled(lambda: L.lora_expand(dev(v), d.pool, d.seg, y))
    st, detail = L.lora_segments_status(d.seg)
    assert st == L.LORA_ERR_TIMEOUT and detail & SGMV_WAIT_BITS, hex(detail)
    y = d.y_in()
    L.lora_expand(dev(v), d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    want = oracle.lora_expand(v[0], p.B[0], p.ranks, p.scales, p.ids, p.y_in[0])
    assert_close(f64(host_bf16_bits(y))[0], want, TOL_BF16, "tc expand after a timeout")


def test_sgmv_tc_apply_wait_runs_out_then_next_call_is_correct():
    # long segments with a workspace: the tensor-core shrink into planes of v, then the
    # tensor-core expand; one CTA of each launch stalls
    p = wl.make_lora_problem("t", 14, T=300, n_adapters=3, h_in=640, h_out=392, r_max=64,
                             ids_kind="zipf", none_frac=0.1, rank_choices=(8, 40, 64))
    d = DeviceProblem(p)
    y = d.y_in()
    _stalled(lambda: L.lora_apply(d.x, d.pool, d.seg, y))
    st, detail = L.lora_segments_status(d.seg)
    assert st == L.LORA_ERR_TIMEOUT and detail & SGMV_WAIT_BITS, hex(detail)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, "tc apply after a timeout")


def test_fp8_gemm_wait_runs_out_then_next_call_is_correct():
    M, K, N = 64, 512, 640
    rng = np.random.default_rng(5)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=5, r=16, seed=9, ids_kind="zipf", none_frac=0.1, W=W)
    Wq_o, sw_o = oracle.quantize_rows(p.W)
    x, Wq, sw = dev_bf16(p.x), dev(Wq_o), dev(sw_o)
    pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
    seg = L.Segments(M, 5)
    L.lora_build_segments(dev(p.ids), 5, seg)
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, pool)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    _stalled(lambda: L.fp8_gemm_lora_epilogue(x, Wq, sw, pool, seg, y, ws))
    st, detail = L.lora_workspace_status(ws)
    assert st == L.LORA_ERR_TIMEOUT and detail & STALL_FP8, hex(detail)
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    L.fp8_gemm_lora_epilogue(x, Wq, sw, pool, seg, y, ws)
    torch.cuda.synchronize()
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    xq, sx = oracle.quantize_rows(p.x)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = oracle.fp8_gemm_lora_sampled(xq, sx, Wq_o, sw_o, rows, cols, x=p.x, A=p.A, B=p.B,
                                        ranks=p.ranks, scales=p.scales, ids=p.ids).reshape(M, N)
    assert_close(f64(host_bf16_bits(y)), want, TOL_FP8, "fp8 after a timeout")


def test_fp8_gemm_base_only_wait_runs_out_then_recovers():
    M, K, N = 16, 256, 384
    rng = np.random.default_rng(6)
    xb = wl.normal_bf16(rng, (M, K))
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    Wq_o, sw_o = oracle.quantize_rows(W)
    x, Wq, sw = dev_bf16(xb), dev(Wq_o), dev(sw_o)
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, None)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    _stalled(lambda: L.fp8_gemm_lora_epilogue(x, Wq, sw, None, None, y, ws))
    st, detail = L.lora_workspace_status(ws)
    assert st == L.LORA_ERR_TIMEOUT and detail & STALL_FP8, hex(detail)
    L.fp8_gemm_lora_epilogue(x, Wq, sw, None, None, y, ws)
    torch.cuda.synchronize()
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    xq, sx = oracle.quantize_rows(xb)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = oracle.fp8_gemm_lora_sampled(xq, sx, Wq_o, sw_o, rows, cols).reshape(M, N)
    assert_close(f64(host_bf16_bits(y)), want, TOL_FP8, "fp8 base after a timeout")
