"""GPU parity of the adapter-training backward on a frozen FP8 base
(fp8_lora_backward) against the fp64 oracle, through the C ABI.

dX mixes the 8-bit base GEMM with the adapter term: the FP8 bar,
max |gpu - oracle| <= 6e-2 (1 + |oracle|). dA and dB are bf16 inputs with fp32
accumulation and fp32 outputs: the bf16 bar 2e-2 (1 + |oracle|); with
small-integer inputs every product and sum is exact in fp32 and they must
equal the oracle exactly. The oracle's base term takes the weight codes WqT /
swT from the oracle's own quantisation of W^T and dY's codes from the oracle's
quantisation of dY (the GPU quantiser is tested bit-exact on its own)."""
import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from gpu_util import TOL_BF16, TOL_FP8, assert_close, dev, dev_bf16, f64, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()


def _case(M, K, N, n_ad, r_max, seed, kind="zipf", rank_choices=None, ints=False, none_frac=0.1):
    rng = np.random.default_rng(seed)
    ids = wl.make_ids(kind, rng, M, n_ad, none_frac)
    ranks = (rng.choice(np.asarray(rank_choices, np.int32), n_ad) if rank_choices
             else np.full(n_ad, r_max, np.int32)).astype(np.int32)

    def draw(shape, std):
        if ints:
            return wl.to_bf16_bits(rng.integers(-2, 3, size=shape).astype(np.float32))
        return wl.normal_bf16(rng, shape, std)
    x = draw((M, K), 1.0)
    dY = draw((M, N), 1.0)
    W = draw((N, K), 1.0 / np.sqrt(K))
    A = np.full((n_ad, K, r_max), wl.BF16_NAN, np.uint16)
    B = np.full((n_ad, r_max, N), wl.BF16_NAN, np.uint16)
    for a in range(n_ad):
        r = int(ranks[a])
        A[a, :, :r] = draw((K, r), 1.0 / np.sqrt(K))
        B[a, :r, :] = draw((r, N), 1.0 / np.sqrt(r))
    scales = np.full(n_ad, 2.0, np.float32)
    return x, dY, W, A, B, ranks, scales, ids


def _run(x, dY, W, A, B, ranks, scales, ids):
    M, K = x.shape
    N = dY.shape[1]
    n_ad, _, r_max = A.shape
    WqT, swT = oracle.quantize_rows(np.ascontiguousarray(W.T))
    pool = L.Pool(dev_bf16(A), dev_bf16(B), dev(ranks), dev(scales))
    seg = L.Segments(M, n_ad)
    L.lora_build_segments(dev(ids), n_ad, seg)
    ws = L.workspace(L.LORA_OP_FP8_BACKWARD, M, K, pool)
    dX = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device="cuda")
    dA = torch.full((n_ad, K, r_max), float("nan"), device="cuda")
    dB = torch.full((n_ad, r_max, N), float("nan"), device="cuda")
    L.fp8_lora_backward(dev_bf16(x), dev_bf16(dY), dev(WqT), dev(swT), pool, seg, dX, dA, dB, ws)
    torch.cuda.synchronize()
    st, detail = L.lora_workspace_status(ws)
    assert st == L.LORA_OK, hex(detail)
    dYq, sd = oracle.quantize_rows(dY)
    want = oracle.lora_backward(x, dY, A, B, ranks, scales, ids, dYq, sd, WqT, swT)
    return (f64(host_bf16_bits(dX)), dA.cpu().numpy().astype(np.float64),
            dB.cpu().numpy().astype(np.float64)), want


@pytest.mark.parametrize("M,K,N,n_ad,r_max,kind,ranks", [
    (16, 256, 384, 4, 16, "zipf", None),
    (64, 512, 256, 6, 32, "zipf", (8, 16, 24, 32)),
    (37, 264, 512, 40, 16, "uniform", (4, 16)),
    (150, 256, 256, 3, 64, "sorted_zipf", (16, 64)),
    (36, 1024, 1024, 32, 16, "distinct", None),
])
def test_backward_parity(M, K, N, n_ad, r_max, kind, ranks):
    got, want = _run(*_case(M, K, N, n_ad, r_max, seed=M + K, kind=kind, rank_choices=ranks))
    assert_close(got[0], want[0], TOL_FP8, "dX")
    assert_close(got[1], want[1], TOL_BF16, "dA")
    assert_close(got[2], want[2], TOL_BF16, "dB")


def test_backward_small_integers_adapter_gradients_exact():
    """dA and dB only: with integer operands in the hundreds, dX's base and adapter
    terms cancel to small values, where the 6e-2 (1 + |oracle|) bar does not fit the
    bf16 rounding of the adapter operand (dX is checked on the random cases)."""
    got, want = _run(*_case(48, 128, 256, 5, 16, seed=3, ints=True, rank_choices=(5, 16)))
    assert np.array_equal(got[1], want[1]) and np.array_equal(got[2], want[2])


def test_backward_decode_batch_mid_size():
    """A decode batch (16 tokens, Zipf over 16 adapters of rank 16) at K 2048, N 4096."""
    M, K, N = 16, 2048, 4096
    x, dY, W, A, B, ranks, scales, ids = _case(M, K, N, 16, 16, seed=5, none_frac=0.0)
    got, want = _run(x, dY, W, A, B, ranks, scales, ids)
    assert_close(got[0], want[0], TOL_FP8, "dX")
    assert_close(got[1], want[1], TOL_BF16, "dA")
    assert_close(got[2], want[2], TOL_BF16, "dB")
    idle = np.setdiff1d(np.arange(16), np.unique(ids))
    assert not got[1][idle].any() and not got[2][idle].any()
