"""GPU parity of the 4-bit base (OCP MX FP4 weights, bf16 activations) with the
fused LoRA term, mxfp4_gemm_lora_epilogue, and of its weight quantiser,
mxfp4_quantize_rows, against the fp64 oracle through the C ABI.

The quantiser is integer work: codes and scales bit-exact. The GEMM dequantises
exactly (an E2M1 value times a power of two is a bf16 value) and accumulates in
fp32, so it is held to the bf16 bar, max |gpu - oracle| <= 2e-2 (1 + |oracle|);
with small-integer activations and exactly representable weights every sum is
exact and y must equal the oracle rounded once to bf16. The GEMM tests take
their codes and scales from the oracle's quantiser (laid out as the library
expects), not from the GPU's."""
import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from gpu_util import TOL_BF16, TOL_FP8, assert_close, dev, dev_bf16, f64, host_bf16_bits, rne_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()


def _pack(codes, scales):
    """The library's storage of oracle codes / scales (a pure rearrangement): two codes per
    byte (element 2i in the low nibble) in tiles of 128 rows x 64 values, and the scales
    per group of 128 rows, block-major. Padding rows are zero."""
    N, K = codes.shape
    Np = (N + 127) // 128 * 128
    pk = np.zeros((Np, K // 2), np.uint8)
    pk[:N] = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    Wp = np.ascontiguousarray(pk.reshape(Np // 128, 128, K // 64, 32).transpose(0, 2, 1, 3)).reshape(-1)
    nb = K // 32
    sc = np.zeros((Np, nb), np.uint8)
    sc[:N] = scales
    Wsc = np.ascontiguousarray(sc.reshape(Np // 128, 128, nb).transpose(0, 2, 1)).reshape(-1)
    return Wp, Wsc


def _unpack_rows(Wp, N, K):
    """Row-major packed codes [N, K / 2] from the tiled storage."""
    Np = (N + 127) // 128 * 128
    return np.ascontiguousarray(Wp.reshape(Np // 128, K // 64, 128, 32).transpose(0, 2, 1, 3)).reshape(Np, K // 2)[:N]


def _gpu_quantize(W):
    N, K = W.shape
    Wp = torch.zeros(L.mxfp4_code_bytes(N, K), dtype=torch.uint8, device="cuda")
    Wsc = torch.zeros(L.mxfp4_scale_bytes(N, K), dtype=torch.uint8, device="cuda")
    L.mxfp4_quantize_rows(dev_bf16(W), Wp, Wsc)
    torch.cuda.synchronize()
    return Wp, Wsc


@pytest.mark.parametrize("N,K,std", [(128, 64, 1.0), (200, 256, 0.02), (64, 1024, 30.0), (300, 128, 1e-30)])
def test_mxfp4_quantize_bitexact(N, K, std):
    rng = np.random.default_rng(N + K)
    W = wl.normal_bf16(rng, (N, K), std)
    W[0, :32] = 0                     # an all-zero block
    W[1, 5] = wl.to_bf16_bits(np.array([-0.0], np.float32))[0]
    Wp, Wsc = _gpu_quantize(W)
    codes, scales = oracle.mxfp4_quantize(W)
    want_p, want_s = _pack(codes, scales)
    assert np.array_equal(_unpack_rows(Wp.cpu().numpy(), N, K), _unpack_rows(want_p, N, K))
    got_s = Wsc.cpu().numpy()
    # rows past N in the last 128-row group are padding: compare the real rows only
    n_groups = (N + 127) // 128
    got = got_s.reshape(n_groups, K // 32, 128).transpose(0, 2, 1).reshape(-1, K // 32)[:N]
    assert np.array_equal(got, scales)


def _run(x, Wp, Wsc, N, A=None, B=None, ranks=None, scales=None, ids=None):
    M, K = x.shape
    pool = seg = None
    if A is not None:
        n_ad = A.shape[0]
        pool = L.Pool(dev_bf16(A), dev_bf16(B), dev(ranks), dev(scales))
        seg = L.Segments(M, n_ad)
        L.lora_build_segments(dev(ids), n_ad, seg)
    ws = L.workspace(L.LORA_OP_MXFP4_GEMM, M, K, pool)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.mxfp4_gemm_lora_epilogue(dev_bf16(x), dev(Wp) if isinstance(Wp, np.ndarray) else Wp,
                               dev(Wsc) if isinstance(Wsc, np.ndarray) else Wsc, pool, seg, y, ws)
    torch.cuda.synchronize()
    st, detail = L.lora_workspace_status(ws)
    assert st == L.LORA_OK, hex(detail)
    return host_bf16_bits(y)


@pytest.mark.parametrize("M,K,N,n_ad,r,lora", [
    (16, 256, 256, 4, 16, False), (16, 256, 256, 4, 16, True), (37, 1024, 392, 5, 16, True),
    (64, 512, 640, 6, 32, True), (200, 384, 256, 6, 16, True), (300, 256, 264, 5, 16, True),
    (64, 512, 256, 40, 16, True),   # more than 16 adapters: the base GEMM then the SGMV apply
])
def test_mxfp4_gemm_lora_full_grid(M, K, N, n_ad, r, lora):
    rng = np.random.default_rng(M + K + N)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=r, seed=M + N, ids_kind="zipf", none_frac=0.1, W=W)
    codes, scales = oracle.mxfp4_quantize(W)
    Wp, Wsc = _pack(codes, scales)
    kw = dict(A=p.A, B=p.B, ranks=p.ranks, scales=p.scales, ids=p.ids) if lora else {}
    got = _run(p.x, Wp, Wsc, N, **kw)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    ka = dict(A=p.A, B=p.B, ranks=p.ranks, scales_lora=p.scales, ids=p.ids) if lora else {}
    want = oracle.mxfp4_gemm_lora_sampled(p.x, codes, scales, rows, cols, **ka).reshape(M, N)
    assert_close(f64(got), want, TOL_BF16, f"mxfp4 M{M} K{K} N{N} lora={lora}")


def test_mxfp4_gemm_small_integers_exact():
    rng = np.random.default_rng(41)
    M, K, N = 24, 128, 136
    x = wl.to_bf16_bits(rng.integers(-2, 3, (M, K)).astype(np.float32))
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    scales = rng.integers(126, 129, (N, K // 32)).astype(np.uint8)   # 0.5, 1, 2
    Wp, Wsc = _pack(codes, scales)
    got = _run(x, Wp, Wsc, N)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = oracle.mxfp4_gemm_lora_sampled(x, codes, scales, rows, cols).reshape(M, N)
    assert np.array_equal(got, rne_bf16_bits(want))


@pytest.mark.parametrize("M", [16, 256])
def test_mxfp4_gemm_lora_decode_shape_sampled(M):
    """K 8192, N 28672, 16 adapters of rank 16, Zipf ids: the GPU quantises the weight
    (its sampled rows checked bit-exact against the oracle's quantiser first)."""
    K, N = 8192, 28672
    W = wl.weight_bf16(N, K, seed=3 + 7000)
    Wp, Wsc = _gpu_quantize(W)
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=16, r=16, seed=3, none_frac=0.0, W=np.zeros((1, 1), np.uint16))
    rng = np.random.default_rng(M)
    rows = rng.integers(0, M, 1200).astype(np.int32)
    cols = rng.integers(0, N, 1200).astype(np.int32)
    cols[:56] = np.arange(0, N, N // 56)[:56]
    cols[56:64] = np.arange(N - 8, N)
    need = np.unique(cols)
    codes, scales = oracle.mxfp4_quantize(W[need])
    got_p = _unpack_rows(Wp.cpu().numpy(), N, K)[need]
    assert np.array_equal(got_p, (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8))
    sc_all = Wsc.cpu().numpy().reshape((N + 127) // 128, K // 32, 128).transpose(0, 2, 1).reshape(-1, K // 32)
    assert np.array_equal(sc_all[need], scales)
    y = _run(p.x, Wp, Wsc, N, A=p.A, B=p.B, ranks=p.ranks, scales=p.scales, ids=p.ids)
    full_codes = np.zeros((N, K), np.uint8)
    full_codes[need] = codes
    full_scales = np.zeros((N, K // 32), np.uint8)
    full_scales[need] = scales
    want = oracle.mxfp4_gemm_lora_sampled(p.x, full_codes, full_scales, rows, cols, A=p.A, B=p.B,
                                          ranks=p.ranks, scales_lora=p.scales, ids=p.ids)
    assert_close(f64(y[rows, cols]), want, TOL_BF16, f"mxfp4 full M{M}")


# ------------------------------------------------------------------ W8A16: FP8 weights, bf16 activations
#
# W8A16 is on the FP8 path (its weights are E4M3): the fused adapter term folds the
# per-channel scale into the adapter operand (B / w_scale rounded to bf16) besides s.v,
# two bf16 roundings where the bf16 path has one, so it is held to the FP8 bar,
# 6e-2 (1 + |oracle|).

@pytest.mark.parametrize("M,K,N,n_ad,lora", [
    (16, 256, 256, 4, False), (16, 256, 256, 4, True), (37, 1024, 392, 5, True),
    (200, 384, 256, 6, True), (64, 512, 256, 40, True),
])
def test_w8a16_gemm_lora_full_grid(M, K, N, n_ad, lora):
    rng = np.random.default_rng(M + K + N + 1)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_ad, r=16, seed=M + N + 1, ids_kind="zipf", none_frac=0.1, W=W)
    Wq, sw = oracle.quantize_rows(W)
    pool = seg = None
    if lora:
        pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
        seg = L.Segments(M, n_ad)
        L.lora_build_segments(dev(p.ids), n_ad, seg)
    ws = L.workspace(L.LORA_OP_W8A16_GEMM, M, K, pool)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.w8a16_gemm_lora_epilogue(dev_bf16(p.x), dev(Wq), dev(sw), pool, seg, y, ws)
    torch.cuda.synchronize()
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    ka = dict(A=p.A, B=p.B, ranks=p.ranks, scales=p.scales, ids=p.ids) if lora else {}
    want = oracle.w8a16_gemm_lora_sampled(p.x, Wq, sw, rows, cols, **ka).reshape(M, N)
    assert_close(f64(host_bf16_bits(y)), want, TOL_FP8, f"w8a16 M{M} K{K} N{N} lora={lora}")


def test_w8a16_gemm_small_integers_exact():
    """Integer weights that E4M3 holds exactly, power-of-two channel scales and activations
    in -2..2: every product and partial sum is exact in fp32, so y must equal the oracle
    rounded once to bf16."""
    rng = np.random.default_rng(43)
    M, K, N = 24, 192, 136
    x = wl.to_bf16_bits(rng.integers(-2, 3, (M, K)).astype(np.float32))
    ints = rng.integers(-4, 5, (N, K))
    Wq = np.vectorize(oracle.e4m3_encode)(ints.astype(np.float64)).astype(np.uint8)
    sw = np.float32(2.0) ** rng.integers(-2, 3, N).astype(np.float32)
    ws = L.workspace(L.LORA_OP_W8A16_GEMM, M, K, None)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.w8a16_gemm_lora_epilogue(dev_bf16(x), dev(Wq), dev(sw), None, None, y, ws)
    torch.cuda.synchronize()
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    want = oracle.w8a16_gemm_lora_sampled(x, Wq, sw, rows, cols).reshape(M, N)
    assert np.array_equal(host_bf16_bits(y), rne_bf16_bits(want))


def test_w8a16_gemm_lora_decode_shape_sampled():
    """K 8192, N 28672, M 16, 16 adapters of rank 16, Zipf ids; the weight quantised by
    the library (its sampled rows checked bit-exact against the oracle's quantiser)."""
    M, K, N = 16, 8192, 28672
    W = wl.weight_bf16(N, K, seed=3 + 7000)
    Wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N,), dtype=torch.float32, device="cuda")
    L.fp8_quantize_rows(dev_bf16(W), Wq, sw)
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=16, r=16, seed=3, none_frac=0.0, W=np.zeros((1, 1), np.uint16))
    rng = np.random.default_rng(77)
    rows = rng.integers(0, M, 1200).astype(np.int32)
    cols = rng.integers(0, N, 1200).astype(np.int32)
    cols[:8] = np.arange(N - 8, N)
    need = np.unique(cols)
    q_need, s_need = oracle.quantize_rows(W[need])
    assert np.array_equal(Wq[torch.from_numpy(need).cuda()].cpu().numpy(), q_need)
    assert np.array_equal(sw[torch.from_numpy(need).cuda()].cpu().numpy(), s_need)
    pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
    seg = L.Segments(M, 16)
    L.lora_build_segments(dev(p.ids), 16, seg)
    ws = L.workspace(L.LORA_OP_W8A16_GEMM, M, K, pool)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.w8a16_gemm_lora_epilogue(dev_bf16(p.x), Wq, sw, pool, seg, y, ws)
    torch.cuda.synchronize()
    assert L.lora_workspace_status(ws)[0] == L.LORA_OK
    full_q = np.zeros((N, K), np.uint8)
    full_q[need] = q_need
    full_s = np.ones(N, np.float32)
    full_s[need] = s_need
    want = oracle.w8a16_gemm_lora_sampled(p.x, full_q, full_s, rows, cols, A=p.A, B=p.B, ranks=p.ranks,
                                          scales=p.scales, ids=p.ids)
    assert_close(f64(host_bf16_bits(y)[rows, cols]), want, TOL_FP8, "w8a16 decode shape")
