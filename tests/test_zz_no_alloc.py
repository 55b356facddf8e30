"""The FP8 GEMM + LoRA epilogue entry point that allocates nothing.

Some callers cannot allocate device memory (a plugin inside a serving engine
that plans all memory itself, or a hot path that must not call cudaMalloc),
so they cannot pass the workspace that fp8_gemm_lora_epilogue needs.
fp8_gemm_lora_epilogue_noalloc keeps that scratch space inside the library.
These tests call it through the C ABI twice in a row and check each result
against the fp64 oracle and against the workspace entry point on the same
inputs, within the FP8 path's tolerance, at a small shape and at the decode
shapes where such a caller would use it (K 8192, N 28672, M 16 and 64, on
sampled outputs), with and without adapters. The file is named so that pytest
collects it last."""
import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from gpu_util import TOL_FP8, assert_close, dev, dev_bf16, f64, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()


_W_FULL = {}


def _weights(N, K, seed):
    """Wq, sw on the device and the oracle's codes for checked rows. Small weights are
    quantised by the oracle; the full-size one on the GPU, its sampled rows checked
    bit-exact against the oracle by the caller."""
    rng = np.random.default_rng(seed)
    if N * K <= 1 << 23:
        W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
        Wq_o, sw_o = oracle.quantize_rows(W)
        return W, dev(Wq_o), dev(sw_o)
    if (N, K) not in _W_FULL:
        W = wl.weight_bf16(N, K, seed=seed)
        Wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        sw = torch.empty(N, dtype=torch.float32, device="cuda")
        L.fp8_quantize_rows(dev_bf16(W), Wq, sw)
        _W_FULL[(N, K)] = (W, Wq, sw)
    return _W_FULL[(N, K)]


def _case(M, K, N, lora, seed):
    W, Wq, sw = _weights(N, K, seed)
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=16 if K >= 8192 else 6, r=16, seed=seed,
                       ids_kind="zipf", none_frac=0.1, W=np.zeros((1, 1), np.uint16))
    x = dev_bf16(p.x)
    pool = seg = None
    if lora:
        pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
        seg = L.Segments(M, p.A.shape[0])
        L.lora_build_segments(dev(p.ids), p.A.shape[0], seg)
    return p, W, x, Wq, sw, pool, seg


def _oracle(p, W, Wq, sw, rows, cols, lora):
    need = np.unique(cols)
    Wq_h = Wq.cpu().numpy()
    sw_h = sw.cpu().numpy()
    Wq_o, sw_o = oracle.quantize_rows(W[need])
    assert np.array_equal(Wq_h[need], Wq_o) and np.array_equal(sw_h[need], sw_o)
    xq, sx = oracle.quantize_rows(p.x)
    kw = dict(x=p.x, A=p.A, B=p.B, ranks=p.ranks, scales=p.scales, ids=p.ids) if lora else {}
    return oracle.fp8_gemm_lora_sampled(xq, sx, Wq_h, sw_h, rows, cols, **kw)


@pytest.mark.parametrize("M,K,N,lora", [(96, 1024, 640, True), (96, 1024, 640, False),
                                        (16, 8192, 28672, True), (64, 8192, 28672, True),
                                        (16, 8192, 28672, False)])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(M, K, N, lora):
    p, W, x, Wq, sw, pool, seg = _case(M, K, N, lora, seed=12)
    limit = L.load().lora_noalloc_scratch_bytes()
    assert L.lora_workspace_size(L.LORA_OP_FP8_GEMM, M, K, pool) <= limit
    if N * K <= 1 << 23:
        rows = np.repeat(np.arange(M), N).astype(np.int32)
        cols = np.tile(np.arange(N), M).astype(np.int32)
    else:
        rng = np.random.default_rng(M)
        rows = rng.integers(0, M, 1200).astype(np.int32)
        cols = rng.integers(0, N, 1200).astype(np.int32)
        cols[:56] = np.arange(0, N, N // 56)[:56]   # every W row block boundary region
        cols[56:64] = np.arange(N - 8, N)
    want = _oracle(p, W, Wq, sw, rows, cols, lora)
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, pool)
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    L.fp8_gemm_lora_epilogue(x, Wq, sw, pool, seg, y_ref, ws)
    torch.cuda.synchronize()
    ref = f64(host_bf16_bits(y_ref))[rows, cols]
    assert_close(ref, want, TOL_FP8, "workspace entry point vs oracle")
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.fp8_gemm_lora_epilogue_noalloc(x, Wq, sw, pool, seg, y)
        torch.cuda.synchronize()
        got = f64(host_bf16_bits(y))[rows, cols]
        assert_close(got, want, TOL_FP8, "no-alloc entry point vs oracle")
        assert_close(got, ref, TOL_FP8, "no-alloc vs workspace entry point")
        st, detail = L.lora_noalloc_status()
        assert st == L.LORA_OK, hex(detail)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    limit = L.load().lora_noalloc_scratch_bytes()
    assert limit == 8 << 20
    M, K, N = 2048, 8192, 256  # M*K bytes of activations alone exceed the scratch
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LoraError) as e:
        L.fp8_gemm_lora_epilogue_noalloc(x, Wq, sw, None, None, y)
    assert e.value.status == L.LORA_ERR_WORKSPACE


def test_noalloc_checks_arguments_like_the_workspace_entry_point():
    """A bad argument gets the same status from both entry points, whatever the size."""
    M, K, N = 4096, 8200, 256  # K % 16 != 0 at a size whose workspace exceeds the scratch
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LoraError) as e:
        L.fp8_gemm_lora_epilogue_noalloc(x, Wq, sw, None, None, y)
    assert e.value.status == L.LORA_ERR_INVALID_ARG
