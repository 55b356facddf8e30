"""GPU parity of the 16-bit base GEMM with the fused LoRA term
(bf16_gemm_lora_epilogue: tcgen05 kind::f16, the same kernel as the FP8 path)
against the fp64 oracle's whole layer, y_ref = sum_k x.W + s.(x.A).B, through
the C ABI. Tolerance: the bf16 bar, max |gpu - oracle| <= 2e-2 (1 + |oracle|)."""
import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from gpu_util import TOL_BF16, assert_close, dev, dev_bf16, f64, host_bf16_bits, rne_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()


def _run(x, W, A, B, ranks, scales, ids, lora=True):
    M, K = x.shape
    N = W.shape[0]
    n_ad = A.shape[0]
    pool = seg = None
    if lora:
        pool = L.Pool(dev_bf16(A), dev_bf16(B), dev(ranks), dev(scales))
        seg = L.Segments(M, n_ad)
        L.lora_build_segments(dev(ids), n_ad, seg)
    ws = L.workspace(L.LORA_OP_BF16_GEMM, M, K, pool)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.bf16_gemm_lora_epilogue(dev_bf16(x), dev_bf16(W), pool, seg, y, ws)
    torch.cuda.synchronize()
    st, detail = L.lora_workspace_status(ws)
    assert st == L.LORA_OK, hex(detail)
    return host_bf16_bits(y)


def _oracle(x, W, A, B, ranks, scales, ids, rows, lora=True):
    """y_ref on the given token rows, every column."""
    N = W.shape[0]
    rr = np.repeat(np.asarray(rows), N).astype(np.int32)
    cols = np.tile(np.arange(N), len(rows)).astype(np.int32)
    base = oracle.linear_bf16_sampled(x, W, rr, cols).reshape(len(rows), N)
    if not lora:
        return base
    zeros = np.zeros((len(rows), N), np.uint16)
    return base + oracle.lora_apply(x[rows], A, B, ranks, scales, ids[rows], zeros)


@pytest.mark.parametrize("M,K,N,n_ad,r,kind,lora", [
    (16, 256, 256, 4, 16, "zipf", False), (16, 256, 256, 4, 16, "zipf", True),
    (37, 1040, 392, 5, 16, "zipf", True), (64, 512, 640, 64, 16, "distinct", True),
    (1, 128, 128, 2, 16, "zipf", True), (200, 384, 256, 6, 32, "uniform", True),
    (300, 256, 256, 5, 16, "zipf", True), (48, 512, 256, 6, 8, "zipf", True),
    (96, 512, 256, 40, 64, "uniform", True),
])
def test_bf16_gemm_lora_full_grid(M, K, N, n_ad, r, kind, lora):
    rng = np.random.default_rng(M + K + N + r)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=r, seed=M + N, ids_kind=kind,
                       none_frac=0.1 if kind == "zipf" else 0.0, W=W,
                       rank_choices=(8, 16, 40, 64) if r == 64 else None)
    got = _run(p.x, p.W, p.A, p.B, p.ranks, p.scales, p.ids, lora)
    want = _oracle(p.x, p.W, p.A, p.B, p.ranks, p.scales, p.ids, np.arange(M), lora)
    assert_close(f64(got), want, TOL_BF16, f"bf16 gemm M{M} K{K} N{N} lora={lora}")


def test_bf16_gemm_small_integers_exact():
    """Small-integer inputs: every product and partial sum is exact in fp32 and
    s.v exact in bf16, so y must equal the exact value rounded once to bf16."""
    rng = np.random.default_rng(8)
    M, K, N, n_ad, r = 40, 64, 256, 3, 16
    x = wl.to_bf16_bits(rng.integers(-1, 2, (M, K)).astype(np.float32))
    W = wl.to_bf16_bits(rng.integers(-2, 3, (N, K)).astype(np.float32))
    A = wl.to_bf16_bits(rng.integers(-1, 2, (n_ad, K, r)).astype(np.float32))
    B = wl.to_bf16_bits(rng.integers(-2, 3, (n_ad, r, N)).astype(np.float32))
    ranks = np.full(n_ad, r, np.int32)
    scales = np.full(n_ad, 2.0, np.float32)
    ids = rng.integers(-1, n_ad, M).astype(np.int32)
    got = _run(x, W, A, B, ranks, scales, ids)
    want = _oracle(x, W, A, B, ranks, scales, ids, np.arange(M))
    assert np.array_equal(got, rne_bf16_bits(want))


@pytest.mark.parametrize("kind", ["all_none", "out_of_range"])
def test_bf16_gemm_ids_without_adapter(kind):
    M, K, N, n_ad = 48, 256, 384, 4
    rng = np.random.default_rng(78)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=16, seed=78, W=W)
    p.ids[:] = -1 if kind == "all_none" else rng.integers(-3, n_ad + 3, size=M)
    got = _run(p.x, p.W, p.A, p.B, p.ranks, p.scales, p.ids)
    want = _oracle(p.x, p.W, p.A, p.B, p.ranks, p.scales, p.ids, np.arange(M))
    assert_close(f64(got), want, TOL_BF16, f"bf16 gemm ids {kind}")


def _layer(p, W, rows, s=0):
    return (_run(p.x[s], W[s], p.A[s], p.B[s], p.ranks, p.scales, p.ids)[rows],
            _oracle(p.x[s], W[s], p.A[s], p.B[s], p.ranks, p.scales, p.ids, rows))


def test_bf16_gemm_whole_layer_sgmv_tiny():
    p = wl.sgmv_tiny()
    got, want = _layer(p, p.W, np.arange(p.T))
    assert_close(f64(got), want, TOL_BF16, "sgmv_tiny, one fused call")


def test_bf16_gemm_whole_layer_bgmv_decode():
    p = wl.bgmv_decode()
    W = wl.weight_bf16(p.h_out, p.h_in, seed=101)[None]
    got, want = _layer(p, W, np.arange(p.T))
    assert_close(f64(got), want, TOL_BF16, "bgmv_decode, one fused call")


def test_bf16_gemm_whole_layer_sgmv_prefill_sampled():
    p = wl.sgmv_prefill()
    W = wl.weight_bf16(p.h_out, p.h_in, seed=102)[None]
    starts = np.concatenate([[0], np.cumsum(np.bincount(p.ids))])
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([rng.choice(p.T, 12, replace=False), starts[1:-1], starts[1:] - 1]))
    got, want = _layer(p, W, rows)
    assert_close(f64(got), want, TOL_BF16, "sgmv_prefill, one fused call")


def test_bf16_gemm_whole_layer_many_tenants_sampled():
    """Four projections: one fused call per slice (each its own W, A, B, x)."""
    p = wl.many_tenants()
    rng = np.random.default_rng(4)
    rows = np.sort(rng.choice(p.T, 16, replace=False))
    for s in range(p.n_slices):
        W = wl.weight_bf16(p.h_out, p.h_in, seed=103 + s)
        got, want = _layer(p, {s: W}, rows, s)
        assert_close(f64(got), want, TOL_BF16, f"many_tenants slice {s}, one fused call")
