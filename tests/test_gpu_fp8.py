"""GPU parity of the FP8 quantiser (bit-exact codes and scales) and of the
fused FP8 GEMM + LoRA epilogue (tolerance 6e-2 * (1 + |oracle|), the bar for
the FP8 path) against the fp64 oracle, through the C ABI."""
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


def _quantize_gpu(x_bits):
    M, K = x_bits.shape
    xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    L.fp8_quantize_rows(dev_bf16(x_bits), xq, sx)
    torch.cuda.synchronize()
    return xq, sx


@pytest.mark.parametrize("M,K,std", [(1, 16, 1.0), (37, 1040, 1.0), (256, 8192, 1.0),
                                     (64, 4096, 1e-3), (8, 64, 300.0)])
def test_quantize_rows_bitexact(M, K, std):
    rng = np.random.default_rng(M * 7 + K)
    x = wl.normal_bf16(rng, (M, K), std)
    x[0, : min(K, 16)] = 0  # a partly zero row
    if M > 1:
        x[1] = 0  # an all-zero row: scale 1
    xq, sx = _quantize_gpu(x)
    want_q, want_s = oracle.quantize_rows(x)
    assert np.array_equal(sx.cpu().numpy(), want_s)
    assert np.array_equal(xq.cpu().numpy(), want_q)


ORACLE_QUANT_MAX = 1 << 23  # weights up to this many codes are quantised by the oracle


def _fp8_case(M, K, N, n_adapters=5, r=16, lora=True, seed=0, kind="zipf", none_frac=0.1,
              rank_choices=None):
    rng = np.random.default_rng(seed + 1000)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_adapters, r=r, seed=seed, ids_kind=kind,
                       none_frac=none_frac, W=W, rank_choices=rank_choices)
    x = dev_bf16(p.x)
    if N * K <= ORACLE_QUANT_MAX:
        # the weight codes and scales come from the oracle (the GPU quantiser has its own
        # bit-exact test), so nothing the oracle consumes comes from the CUDA path
        Wq_o, sw_o = oracle.quantize_rows(p.W)
        Wq, sw = dev(Wq_o), dev(sw_o)
    else:
        # the full-size weight (235 M codes) is quantised on the GPU; the tests that use
        # it check the sampled rows bit-exact against the oracle before using them
        Wq, sw = _quantize_gpu(p.W)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    pool = seg = None
    if lora:
        pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
        seg = L.Segments(M, n_adapters)
        L.lora_build_segments(dev(p.ids), n_adapters, seg)
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, pool)
    L.fp8_gemm_lora_epilogue(x, Wq, sw, pool, seg, y, ws)
    torch.cuda.synchronize()
    st, detail = L.lora_workspace_status(ws)
    assert st == L.LORA_OK, hex(detail)
    return p, Wq.cpu().numpy(), sw.cpu().numpy(), host_bf16_bits(y)


def _oracle_fp8(p, Wq, sw, rows, cols, lora):
    xq, sx = oracle.quantize_rows(p.x)
    kw = dict(x=p.x, A=p.A, B=p.B, ranks=p.ranks, scales=p.scales, ids=p.ids) if lora else {}
    return oracle.fp8_gemm_lora_sampled(xq, sx, Wq, sw, rows, cols, **kw)


@pytest.mark.parametrize("M,K,N,lora", [
    (16, 256, 256, False), (16, 256, 256, True), (37, 1040, 392, True), (64, 512, 640, True),
    (1, 128, 128, True), (200, 384, 256, True), (256, 256, 384, True), (300, 256, 256, True),
    (130, 2048, 1024, False),
])
def test_fp8_gemm_lora_full_grid(M, K, N, lora):
    p, Wq, sw, y = _fp8_case(M, K, N, lora=lora, seed=M + K + N)
    # the weight codes are the oracle's, bit for bit
    Wq_o, sw_o = oracle.quantize_rows(p.W)
    assert np.array_equal(Wq, Wq_o) and np.array_equal(sw, sw_o)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = _oracle_fp8(p, Wq, sw, rows, cols, lora).reshape(M, N)
    assert_close(f64(y), want, TOL_FP8, f"fp8 M{M} K{K} N{N} lora={lora}")


def test_fp8_gemm_adapters_beyond_vq_capacity():
    """256 tokens over 48 adapters of rank up to 64: the shared-memory plan holds V'
    tiles for 8 adapters per token block (64-byte k-blocks, 4 slots, two phases), so
    the others take the CUDA-core path in the epilogue."""
    M, K, N = 256, 512, 256
    p, Wq, sw, y = _fp8_case(M, K, N, n_adapters=48, r=64, seed=21, kind="uniform",
                             rank_choices=(8, 16, 40, 64))
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = _oracle_fp8(p, Wq, sw, rows, cols, True).reshape(M, N)
    assert_close(f64(y), want, TOL_FP8, "adapters beyond V' capacity")


def test_fp8_gemm_mixed_ranks_many_adapters():
    p, Wq, sw, y = _fp8_case(96, 512, 256, n_adapters=40, r=64, seed=5, kind="uniform",
                             rank_choices=(8, 16, 64))
    M, N = 96, 256
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = _oracle_fp8(p, Wq, sw, rows, cols, True).reshape(M, N)
    assert_close(f64(y), want, TOL_FP8, "mixed ranks")


@pytest.mark.parametrize("M", [16, 64, 256])
def test_fp8_gemm_lora_full_size_sampled(M):
    """The full decode shape (K=8192, N=28672, 16 adapters, r=16, Zipf ids) in the
    launch configuration the benchmark times, checked on sampled outputs."""
    K, N = 8192, 28672
    p, Wq, sw, y = _fp8_case(M, K, N, n_adapters=16, r=16, seed=3, none_frac=0.0)
    rng = np.random.default_rng(M)
    n_s = 1500
    rows = rng.integers(0, M, n_s).astype(np.int32)
    cols = rng.integers(0, N, n_s).astype(np.int32)
    # every W row block boundary and the last columns
    cols[:64] = np.arange(0, N, N // 64)[:64]
    cols[64:72] = np.arange(N - 8, N)
    need = np.unique(cols)
    Wq_o, sw_o = oracle.quantize_rows(p.W[need])
    assert np.array_equal(Wq[need], Wq_o) and np.array_equal(sw[need], sw_o)
    want = _oracle_fp8(p, Wq, sw, rows, cols, True)
    assert_close(f64(y[rows, cols]), want, TOL_FP8, f"fp8 full M{M}")


@pytest.mark.parametrize("M,K,N,n_adapters,r,kind", [
    (48, 512, 256, 6, 8, "zipf"),         # r_max 8: B staged as 8-row boxes, rank steps of 16
    (48, 512, 256, 6, 32, "zipf"),        # r_max 32: two rank steps per adapter
    (64, 256, 256, 64, 16, "distinct"),   # one adapter per token: more adapters than slots
    (40, 256, 384, 3, 16, "identical"),   # a single adapter over the whole token block
])
def test_fp8_gemm_lora_rank_and_id_mixes(M, K, N, n_adapters, r, kind):
    p, Wq, sw, y = _fp8_case(M, K, N, n_adapters=n_adapters, r=r, seed=M + r, kind=kind,
                             none_frac=0.0 if kind != "zipf" else 0.1)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = _oracle_fp8(p, Wq, sw, rows, cols, True).reshape(M, N)
    assert_close(f64(y), want, TOL_FP8, f"fp8 r{r} {kind}")



def test_fp8_gemm_rejects_unaligned_y():
    """y must start on a 16-byte boundary (the epilogue writes 16-byte row pieces):
    a y two bytes past one is refused before anything is launched."""
    M, K, N = 16, 256, 256
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y_buf = torch.full((M * N + 1,), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, None)
    with pytest.raises(L.LoraError) as err:
        L.fp8_gemm_lora_epilogue(x, Wq, sw, None, None, y_buf[1:].view(M, N), ws)
    assert err.value.status == L.LORA_ERR_INVALID_ARG
    L.fp8_gemm_lora_epilogue(x, Wq, sw, None, None, y_buf[:-1].view(M, N), ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y_buf[:-1]).item() == 0  # all-zero x: y = 0


@pytest.mark.parametrize("kind", ["all_none", "out_of_range"])
def test_fp8_gemm_lora_ids_without_adapter(kind):
    """Every token without an adapter (pure base GEMM through the LoRA path), and ids
    outside [-1, n_adapters) (served as -1): the oracle leaves those rows base-only."""
    M, K, N, n_ad = 48, 256, 384, 4
    rng = np.random.default_rng(77)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=16, seed=77, W=W)
    if kind == "all_none":
        p.ids[:] = -1
    else:
        p.ids[:] = rng.integers(-3, n_ad + 3, size=M).astype(np.int32)
    Wq_o, sw_o = oracle.quantize_rows(p.W)
    pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
    seg = L.Segments(M, n_ad)
    L.lora_build_segments(dev(p.ids), n_ad, seg)
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, K, pool)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.fp8_gemm_lora_epilogue(dev_bf16(p.x), dev(Wq_o), dev(sw_o), pool, seg, y, ws)
    torch.cuda.synchronize()
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = _oracle_fp8(p, Wq_o, sw_o, rows, cols, True).reshape(M, N)
    assert_close(f64(host_bf16_bits(y)), want, TOL_FP8, f"fp8 ids {kind}")


def test_fp8_gemm_lora_many_tokens_split_path():
    """More than 1024 tokens: the call runs the base GEMM, then the SGMV apply on its
    output with the tile rows in cost order from the GEMM workspace; y = bf16(bf16(base)
    + term), within the FP8 bar on every element."""
    M, K, N = 1100, 256, 264
    p, Wq, sw, y = _fp8_case(M, K, N, n_adapters=6, r=16, seed=17, none_frac=0.1)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = _oracle_fp8(p, Wq, sw, rows, cols, True).reshape(M, N)
    assert_close(f64(y), want, TOL_FP8, "fp8 split path, 1100 tokens")
