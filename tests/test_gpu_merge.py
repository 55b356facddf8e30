"""GPU parity of the token-wise adapter merge (lora_switch_merge) against the
fp64 oracle, through the C ABI.

Tolerance. The kernel multiplies bf16 values exactly into fp32, sums at most
256 products in fp32 per adapter, applies gate * scale in fp32 and rounds the
merged weight once to bf16, so |gpu - oracle| <= 2^-8 (|oracle| + |delta|_abs)
elementwise, with |delta|_abs = sum_e |g_e s_a| sum_j |A[k][j] B[j][n]| (one
bf16 rounding, 2^-9 |oracle|, plus fp32 summation error far below it). With
small-integer operands and power-of-two gates every intermediate is exact and
the result must equal the oracle rounded once to bf16. The merged weight is
also checked where it is used: y = x.W_out^T against the oracle's layer, at the
bf16 bar 2e-2 (1 + |y|)."""
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


def _problem(seed, N, K, n_ad, r_max, ranks=None, ints=False):
    rng = np.random.default_rng(seed)
    if ranks is None:
        ranks = rng.choice(np.array([r for r in (4, 8, 16, 32, 64) if r <= r_max], np.int32), size=n_ad)
    ranks = np.asarray(ranks, np.int32)
    if ints:
        W = wl.to_bf16_bits(rng.integers(-4, 5, (N, K)).astype(np.float32))
    else:
        W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    A = np.full((n_ad, K, r_max), wl.BF16_NAN, np.uint16)
    B = np.full((n_ad, r_max, N), wl.BF16_NAN, np.uint16)
    for a in range(n_ad):
        r = int(ranks[a])
        if ints:
            A[a, :, :r] = wl.to_bf16_bits(rng.integers(-1, 2, (K, r)).astype(np.float32))
            B[a, :r, :] = wl.to_bf16_bits(rng.integers(-1, 2, (r, N)).astype(np.float32))
        else:
            A[a, :, :r] = wl.normal_bf16(rng, (K, r), 1.0 / np.sqrt(K))
            B[a, :r, :] = wl.normal_bf16(rng, (r, N), 1.0 / np.sqrt(r))
    scales = np.full(n_ad, 2.0, np.float32)
    return W, A, B, ranks, scales


def _gpu_merge(W, A, B, ranks, scales, sel, gates, in_place=False):
    Wd = dev_bf16(W)
    pool = L.Pool(dev_bf16(A), dev_bf16(B), dev(ranks), dev(scales))
    out = Wd if in_place else torch.full_like(Wd, float("nan"))
    L.lora_switch_merge(Wd, pool, dev(np.asarray(sel, np.int32)), dev(np.asarray(gates, np.float32)), out)
    torch.cuda.synchronize()
    return host_bf16_bits(out)


def _abs_delta(A, B, ranks, scales, sel, gates, N, K):
    d = np.zeros((N, K))
    for e, a in enumerate(sel):
        if not 0 <= a < A.shape[0]:
            continue
        r = int(ranks[a])
        Af = np.abs(oracle.bf16_to_f64(A[a][:, :r]))
        Bf = np.abs(oracle.bf16_to_f64(B[a][:r, :]))
        d += abs(float(gates[e]) * float(scales[a])) * (Bf.T @ Af.T)
    return d


def _check(got, want, absd, what):
    err = np.abs(f64(got) - want)
    bound = 2.0 ** -8 * (np.abs(want) + absd) + 1e-30
    assert np.isfinite(f64(got)).all(), what
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} outside the bound; worst {np.max(err / bound)}"


@pytest.mark.parametrize("N,K,n_ad,r_max,sel,gates", [
    (256, 512, 8, 16, [3, 5], [0.7, 0.3]),
    (200, 264, 6, 64, [0, 2, 4], [0.5, 0.25, 0.25]),      # ragged tiles, mixed ranks
    (64, 128, 4, 8, [1], [1.0]),
    (512, 384, 8, 32, [7, -1, 2, 9], [0.4, 0.9, 0.35, 0.8]),  # -1 and out-of-range entries
    (128, 1024, 16, 16, [1, 3, 5, 7, 9, 11, 13, 15], [0.125] * 8),  # eight at once
])
def test_merge_parity(N, K, n_ad, r_max, sel, gates):
    W, A, B, ranks, scales = _problem(N + K, N, K, n_ad, r_max)
    got = _gpu_merge(W, A, B, ranks, scales, sel, gates)
    want = oracle.lora_switch_merge(W, A, B, ranks, scales, np.array(sel, np.int32),
                                    np.array(gates, np.float32))
    _check(got, want, _abs_delta(A, B, ranks, scales, sel, gates, N, K), f"merge N{N} K{K}")


def test_merge_small_integers_exact_and_in_place():
    N, K, n_ad, r_max = 192, 320, 5, 32
    W, A, B, ranks, scales = _problem(4, N, K, n_ad, r_max, ranks=[3, 8, 16, 32, 5], ints=True)
    sel, gates = [4, 1, 3], [0.5, 0.25, 1.0]
    want = rne_bf16_bits(oracle.lora_switch_merge(W, A, B, ranks, scales, np.array(sel, np.int32),
                                                  np.array(gates, np.float32)))
    assert np.array_equal(_gpu_merge(W, A, B, ranks, scales, sel, gates), want)
    assert np.array_equal(_gpu_merge(W, A, B, ranks, scales, sel, gates, in_place=True), want)


def test_merge_zero_gates_or_no_adapter_leave_the_backbone():
    W, A, B, ranks, scales = _problem(5, 128, 256, 4, 16)
    assert np.array_equal(_gpu_merge(W, A, B, ranks, scales, [0, 1], [0.0, 0.0]), W)
    assert np.array_equal(_gpu_merge(W, A, B, ranks, scales, [-1, 7], [1.0, 1.0]), W)


def test_merged_backbone_decodes_the_token():
    """Llama-2-7B q_proj shape (4096 x 4096), 8 adapters of rank 16, a token routed to two
    of them: y = x.W_out^T on the GPU against the oracle's merged layer."""
    N = K = 4096
    W, A, B, ranks, scales = _problem(6, N, K, 8, 16, ranks=[16] * 8)
    sel, gates = [2, 6], [0.62, 0.38]
    Wm = _gpu_merge(W, A, B, ranks, scales, sel, gates)
    rng = np.random.default_rng(7)
    x = wl.normal_bf16(rng, (4, K))
    y = (dev_bf16(x) @ dev_bf16(Wm).t()).float().cpu().numpy()
    merged = oracle.lora_switch_merge(W, A, B, ranks, scales, np.array(sel, np.int32),
                                      np.array(gates, np.float32))
    assert_close(y, f64(x) @ merged.T, TOL_BF16, "decode with the merged backbone")


def test_merge_llama70b_shape_sampled_rows():
    """28672 x 8192 (the FP8 section's up_proj shape), top-2 of 16 adapters of rank 16:
    rows of the merged weight checked against the oracle on the same rows."""
    N, K, n_ad = 28672, 8192, 16
    rng = np.random.default_rng(70)
    W = wl.weight_bf16(N, K, seed=71)
    ranks = np.full(n_ad, 16, np.int32)
    A = wl.normal_bf16(rng, (n_ad, K, 16), 1.0 / np.sqrt(K))
    B = wl.normal_bf16(rng, (n_ad, 16, N), 0.25)
    scales = np.full(n_ad, 2.0, np.float32)
    sel, gates = [3, 12], [0.55, 0.45]
    got = _gpu_merge(W, A, B, ranks, scales, sel, gates)
    rows = np.unique(np.concatenate([rng.choice(N, 48, replace=False), [0, 63, 64, N - 1]]))
    want = oracle.lora_switch_merge(W[rows], A, np.ascontiguousarray(B[:, :, rows]), ranks, scales,
                                    np.array(sel, np.int32), np.array(gates, np.float32))
    absd = _abs_delta(A, np.ascontiguousarray(B[:, :, rows]), ranks, scales, sel, gates, len(rows), K)
    _check(got[rows], want, absd, "merge 28672 x 8192")


def test_merge_rejects_overlap_and_too_many_adapters():
    W, A, B, ranks, scales = _problem(8, 64, 128, 12, 64)
    pool = L.Pool(dev_bf16(A), dev_bf16(B), dev(ranks), dev(scales))
    sel, gates = dev(np.array([0, 1], np.int32)), dev(np.array([0.5, 0.5], np.float32))
    n = W.size
    buf = torch.zeros(n + 8, dtype=torch.bfloat16, device="cuda")
    w_in, w_out = buf[:n].view(W.shape), buf[8:8 + n].view(W.shape)  # shifted by 16 bytes
    with pytest.raises(L.LoraError) as e:
        L.lora_switch_merge(w_in, pool, sel, gates, w_out)
    assert e.value.status == L.LORA_ERR_INVALID_ARG
    with pytest.raises(L.LoraError) as e:
        L.lora_switch_merge(w_in, pool, dev(np.arange(5, dtype=np.int32)), dev(np.ones(5, np.float32)),
                            torch.empty_like(w_in))
    assert e.value.status == L.LORA_ERR_UNSUPPORTED  # 5 x 64 > 256
