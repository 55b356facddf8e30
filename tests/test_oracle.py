"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something the pages or mathematics fix:
format definitions (OCP FP8 E4M3, bfloat16) re-checked against torch's own
conversions, hand-worked examples (tests/golden/), brute force in exact
rationals on tiny shapes, closed forms and invariants of the LoRA algebra
(Punica README, "How?"), and a library sort for the segment order.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- formats

def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def _golden_e4m3():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_key_values.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            rows.append((int(c, 16), float(v)))
    return rows


def test_e4m3_decode_golden_values():
    for c, v in _golden_e4m3():
        got = oracle.e4m3_decode(c)
        if math.isnan(v):
            assert math.isnan(got), hex(c)
        else:
            assert got == v and math.copysign(1, got) == math.copysign(1, v), hex(c)


def test_e4m3_encode_roundtrip_every_finite_code():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(123)
    vals = np.concatenate([
        rng.uniform(-448, 448, 4000),
        rng.standard_normal(4000) * 3,
        rng.standard_normal(2000) * 0.01,          # subnormal region
        rng.uniform(-2 ** -9, 2 ** -9, 500),
    ]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(v)) for v in vals], np.uint8)
    assert np.array_equal(ours, ref)


def test_e4m3_encode_ties_to_even_and_saturation():
    # midpoint of 1.0 (0x38) and 1.125 (0x39): even code wins
    assert oracle.e4m3_encode(1.0625) == 0x38
    # midpoint of 1.125 (0x39) and 1.25 (0x3A)
    assert oracle.e4m3_encode(1.1875) == 0x3A
    # half the smallest subnormal ties between 0 and 2^-9: goes to 0
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00
    assert oracle.e4m3_encode(1.5 * 2.0 ** -10) == 0x01
    # every midpoint between consecutive positive codes goes to the even one
    for c in range(0, 0x7E):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mid = (lo + hi) / 2
        if float(np.float32(mid)) != mid:
            continue
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == want, hex(c)
    # saturating conversion: beyond the largest finite value -> +-448
    for v in (448.0, 449.0, 464.0, 480.0, 1e30, float("inf")):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F


# ---------------------------------------------------------------- segments

def _segments_by_sort(ids, n_adapters):
    T = len(ids)
    key = [(ids[t] if 0 <= ids[t] < n_adapters else n_adapters, t) for t in range(T)]
    order = sorted(range(T), key=lambda t: key[t])  # library sort, stable key
    counts = [sum(1 for t in range(T) if key[t][0] == a) for a in range(n_adapters + 1)]
    indptr = [sum(counts[:a]) for a in range(n_adapters + 1)]
    active = [a for a in range(n_adapters) if counts[a] > 0]
    n_bad = sum(1 for i in ids if i != -1 and not (0 <= i < n_adapters))
    return order, indptr, active, n_bad


SEG_KINDS = ["distinct", "identical", "uniform", "zipf", "sorted_zipf", "none", "bad", "single"]


@pytest.mark.parametrize("kind", SEG_KINDS)
def test_segments_match_sorted_order(kind):
    rng = np.random.default_rng(SEG_KINDS.index(kind))
    n_adapters = 12
    if kind == "none":
        ids = np.full(17, -1, np.int32)
    elif kind == "bad":
        ids = rng.integers(-3, n_adapters + 3, size=40).astype(np.int32)
    elif kind == "single":
        ids = np.array([5], np.int32)
    elif kind == "distinct":
        ids = wl.make_ids("distinct", rng, 12, n_adapters, none_frac=0.2)
    else:
        ids = wl.make_ids(kind, rng, 50, n_adapters, none_frac=0.1)
    seg = oracle.build_segments(ids, n_adapters)
    order, indptr, active, n_bad = _segments_by_sort(list(ids), n_adapters)
    assert seg["perm"].tolist() == order
    assert seg["indptr"].tolist() == indptr
    n_active = len(active)
    assert seg["counts"].tolist() == [indptr[n_adapters], n_active, n_bad]
    assert seg["active"][:n_active].tolist() == active
    assert (seg["active"][n_active:] == -1).all()
    want_tok = [i if 0 <= i < n_adapters else -1 for i in ids]
    assert seg["tok_adapter"].tolist() == want_tok


def test_segments_empty_batch():
    seg = oracle.build_segments(np.zeros(0, np.int32), 3)
    assert seg["counts"].tolist() == [0, 0, 0]
    assert seg["indptr"].tolist() == [0, 0, 0, 0]
    assert seg["active"].tolist() == [-1, -1, -1]


# ---------------------------------------------------------------- LoRA algebra

def _read_worked_example():
    d = {}
    with open(os.path.join(GOLDEN, "lora_how_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *vals = line.split()
            d.setdefault(k, []).append([float(v) for v in vals])
    return d


@pytest.mark.parametrize("s", [1.0, 2.0])
def test_worked_example_of_how_section(s):
    d = _read_worked_example()
    W_h1h2 = np.array(d["W_row0"] + d["W_row1"])           # [H1=2, H2=3]
    W = wl.to_bf16_bits(W_h1h2.T.copy())                    # stored [N=3][K=2]
    A = np.stack([wl.to_bf16_bits(np.array(d["A0"][0]).reshape(2, 1)),
                  wl.to_bf16_bits(np.array(d["A1"][0]).reshape(2, 1))])
    B = np.stack([wl.to_bf16_bits(np.array(d["B0"][0]).reshape(1, 3)),
                  wl.to_bf16_bits(np.array(d["B1"][0]).reshape(1, 3))])
    toks = np.array(d["tok"])
    ids = toks[:, 0].astype(np.int32)
    x = wl.to_bf16_bits(toks[:, 1:])
    rows = np.repeat(np.arange(3), 3).astype(np.int32)
    cols = np.tile(np.arange(3), 3).astype(np.int32)
    base = oracle.linear_bf16_sampled(x, W, rows, cols).reshape(3, 3)
    assert np.array_equal(base, np.array(d["base"]))
    y = oracle.lora_apply(x, A, B, np.array([1, 1], np.int32), np.array([s, s], np.float32),
                          ids, wl.to_bf16_bits(base))
    want = np.array(d["y_s1"] if s == 1.0 else d["y_s2"])
    assert np.array_equal(y, want)


def _frac_bf16(a):
    return [[Fraction(float(v)) for v in row] for row in oracle.bf16_to_f64(a)]


def _brute_force_apply(x, A, B, ranks, scales, ids, y_in):
    """Exact rationals, straight from y = y_in + s * (x A) B per token."""
    T = x.shape[0]
    n_adapters, h_in, r_max = A.shape
    h_out = B.shape[2]
    X = _frac_bf16(x)
    Y = _frac_bf16(y_in)
    out = []
    for t in range(T):
        a = int(ids[t])
        row = list(Y[t])
        if 0 <= a < n_adapters:
            r = int(ranks[a])
            Aa = _frac_bf16(A[a][:, :r])
            Ba = _frac_bf16(B[a][:r, :])
            s = Fraction(float(scales[a]))
            v = [sum(X[t][k] * Aa[k][j] for k in range(h_in)) for j in range(r)]
            for n in range(h_out):
                row[n] += s * sum(v[j] * Ba[j][n] for j in range(r))
        out.append(row)
    return out


def _tiny_problem(seed, T=5, n_adapters=3, h_in=7, h_out=5, r_max=3, ints=False):
    rng = np.random.default_rng(seed)
    ids = rng.integers(-1, n_adapters, size=T).astype(np.int32)
    ranks = rng.integers(1, r_max + 1, size=n_adapters).astype(np.int32)
    scales = rng.choice(np.array([0.5, 1.0, 2.0, -1.5], np.float32), size=n_adapters)

    def draw(shape, std):
        if ints:
            return wl.to_bf16_bits(rng.integers(-2, 3, size=shape).astype(np.float32))
        return wl.normal_bf16(rng, shape, std)
    x = draw((T, h_in), 1.0)
    A = np.full((n_adapters, h_in, r_max), wl.BF16_NAN, np.uint16)
    B = np.full((n_adapters, r_max, h_out), wl.BF16_NAN, np.uint16)
    for a in range(n_adapters):
        A[a, :, :ranks[a]] = draw((h_in, ranks[a]), 0.4)
        B[a, :ranks[a], :] = draw((ranks[a], h_out), 0.6)
    y_in = draw((T, h_out), 1.0)
    return x, A, B, ranks, scales, ids, y_in


@pytest.mark.parametrize("seed", range(6))
def test_apply_exact_rationals_small_ints(seed):
    args = _tiny_problem(seed, ints=True)
    got = oracle.lora_apply(*args)
    want = _brute_force_apply(*args)
    assert [[Fraction(float(v)) for v in row] for row in got] == want


@pytest.mark.parametrize("seed", range(6))
def test_apply_rationals_random_bf16(seed):
    args = _tiny_problem(100 + seed, T=6, n_adapters=2, h_in=8, h_out=4, r_max=3)
    got = oracle.lora_apply(*args)
    want = np.array([[float(v) for v in row] for row in _brute_force_apply(*args)])
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_shrink_then_expand_equals_apply():
    x, A, B, ranks, scales, ids, y_in = _tiny_problem(7, T=9, n_adapters=4, h_in=16, h_out=12,
                                                      r_max=4)
    v = oracle.lora_shrink(x, A, ranks, ids)
    y = oracle.lora_expand(v, B, ranks, scales, ids, y_in)
    assert np.array_equal(y, oracle.lora_apply(x, A, B, ranks, scales, ids, y_in))
    # padding beyond each adapter's rank is NaN in A and B and is never read
    assert np.isfinite(v).all() and np.isfinite(y).all()


def _random_problem(seed, T=24, n_adapters=5, h_in=64, h_out=40, r_max=8):
    p = wl.make_lora_problem("t", seed, T=T, n_adapters=n_adapters, h_in=h_in, h_out=h_out,
                             r_max=r_max, ids_kind="uniform", none_frac=0.2,
                             rank_choices=(1, 3, 8), with_W=True)
    return p


def test_invariant_zero_B_gives_base_output():
    p = _random_problem(1)
    B0 = np.where(p.B[0] == wl.BF16_NAN, p.B[0], np.uint16(0))
    y = oracle.lora_apply(p.x[0], p.A[0], B0, p.ranks, p.scales, p.ids, p.y_in[0])
    assert np.array_equal(y, oracle.bf16_to_f64(p.y_in[0]))


def test_invariant_no_adapter_rows_untouched():
    p = _random_problem(2)
    y = oracle.lora_apply(p.x[0], p.A[0], p.B[0], p.ranks, p.scales, p.ids, p.y_in[0])
    none = p.ids == -1
    assert none.any()
    assert np.array_equal(y[none], oracle.bf16_to_f64(p.y_in[0][none]))
    assert not np.array_equal(y[~none], oracle.bf16_to_f64(p.y_in[0][~none]))


def test_invariant_permuting_tokens_permutes_outputs():
    p = _random_problem(3)
    y = oracle.lora_apply(p.x[0], p.A[0], p.B[0], p.ranks, p.scales, p.ids, p.y_in[0])
    pi = np.random.default_rng(0).permutation(p.T)
    y2 = oracle.lora_apply(p.x[0][pi], p.A[0], p.B[0], p.ranks, p.scales, p.ids[pi],
                           p.y_in[0][pi])
    assert np.array_equal(y2, y[pi])


def test_invariant_merged_weight():
    """x.W^T + s.(x.A).B == x.(W + s.(A.B)^T)^T, the README's identity, with the
    merged product formed by numpy's matmul."""
    p = _random_problem(4)
    T, K, N = p.T, p.h_in, p.h_out
    rows = np.repeat(np.arange(T), N).astype(np.int32)
    cols = np.tile(np.arange(N), T).astype(np.int32)
    base = oracle.linear_bf16_sampled(p.x[0], p.W[0], rows, cols).reshape(T, N)
    # feed the exact fp64 base in through y_in = 0 and add it afterwards
    zeros = np.zeros((T, N), np.uint16)
    lora = oracle.lora_apply(p.x[0], p.A[0], p.B[0], p.ranks, p.scales, p.ids, zeros)
    y = base + lora
    X = oracle.bf16_to_f64(p.x[0])
    W = oracle.bf16_to_f64(p.W[0])
    for t in range(T):
        a = p.ids[t]
        if a < 0:
            want = X[t] @ W.T
        else:
            r = p.ranks[a]
            Aa = oracle.bf16_to_f64(p.A[0][a][:, :r])
            Ba = oracle.bf16_to_f64(p.B[0][a][:r, :])
            merged = W + float(p.scales[a]) * (Aa @ Ba).T
            want = X[t] @ merged.T
        assert np.allclose(y[t], want, rtol=1e-9, atol=1e-9)


def test_rank1_closed_form():
    """A = e_j (unit column), B = c * ones -> s * x[t, j] * c, exactly."""
    T, h_in, h_out, j, c, s = 7, 32, 9, 5, 0.75, 2.0
    rng = np.random.default_rng(9)
    x = wl.normal_bf16(rng, (T, h_in))
    A = np.zeros((1, h_in, 1), np.uint16)
    A[0, j, 0] = wl.to_bf16_bits(np.array([1.0]))[0]
    B = wl.to_bf16_bits(np.full((1, 1, h_out), c))
    y = oracle.lora_apply(x, A, B, np.array([1], np.int32), np.array([s], np.float32),
                          np.zeros(T, np.int32), np.zeros((T, h_out), np.uint16))
    want = s * oracle.bf16_to_f64(x)[:, j:j + 1] * c * np.ones((1, h_out))
    assert np.array_equal(y, want)


def test_expand_uses_v_exactly():
    rng = np.random.default_rng(5)
    T, r, h_out = 4, 2, 3
    v = rng.standard_normal((T, r)).astype(np.float32)
    B = wl.to_bf16_bits(np.array([[[1.0, 2.0, 0.5], [-1.0, 0.25, 4.0]]]))
    ids = np.array([0, -1, 0, 0], np.int32)
    y = oracle.lora_expand(v, B, None, np.array([3.0], np.float32), ids,
                           np.zeros((T, h_out), np.uint16))
    Bf = np.array([[1.0, 2.0, 0.5], [-1.0, 0.25, 4.0]])
    for t in range(T):
        want = np.zeros(h_out) if ids[t] < 0 else 3.0 * (v[t].astype(np.float64) @ Bf)
        assert np.allclose(y[t], want, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- FP8 path

def test_quantize_rows_exact_row():
    vals = np.array([[448, 224, 1, -2, 0.5, 0]], np.float32)
    xq, sx = oracle.quantize_rows(wl.to_bf16_bits(vals))
    assert sx[0] == 1.0
    assert xq[0].tolist() == [0x7E, 0x76, 0x38, 0xC0, 0x30, 0x00]


def test_quantize_rows_zero_row_scale_one():
    xq, sx = oracle.quantize_rows(np.zeros((2, 16), np.uint16))
    assert sx.tolist() == [1.0, 1.0] and not xq.any()


def test_quantize_rows_scale_and_error_bound():
    rng = np.random.default_rng(11)
    x = wl.normal_bf16(rng, (8, 256), 3.0)
    xq, sx = oracle.quantize_rows(x)
    X = oracle.bf16_to_f64(x)
    amax = np.abs(X).max(axis=1)
    assert np.array_equal(sx, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    deq = oracle.e4m3_to_f64(xq) * sx[:, None].astype(np.float64)
    # the largest element lands on the top code
    for m in range(8):
        k = int(np.argmax(np.abs(X[m])))
        assert xq[m, k] & 0x7F == 0x7E
    # relative error of a normal E4M3 value is at most 2^-4 (half of 2^-3)
    big = np.abs(X) >= 2.0 ** -6 * sx[:, None]
    rel = np.abs(deq - X)[big] / np.abs(X)[big]
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
    # agrees with a library E4M3 cast of the fp32 quotient
    q = (X.astype(np.float32) / sx[:, None]).astype(np.float32)
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(xq, ref)


def _brute_force_fp8(xq, sx, Wq, sw, x, A, B, ranks, scales, ids, m, n):
    K = xq.shape[1]
    acc = sum(Fraction(oracle.e4m3_decode(int(xq[m, k]))) *
              Fraction(oracle.e4m3_decode(int(Wq[n, k]))) for k in range(K))
    y = Fraction(float(sx[m])) * Fraction(float(sw[n])) * acc
    a = int(ids[m])
    if A is not None and 0 <= a < A.shape[0]:
        r = int(ranks[a])
        Xr = [Fraction(v) for v in oracle.bf16_to_f64(x[m])]
        Aa = _frac_bf16(A[a][:, :r])
        Ba = _frac_bf16(B[a][:r, :])
        v = [sum(Xr[k] * Aa[k][j] for k in range(K)) for j in range(r)]
        y += Fraction(float(scales[a])) * sum(v[j] * Ba[j][n] for j in range(r))
    return y


@pytest.mark.parametrize("with_lora", [False, True])
def test_fp8_gemm_lora_bruteforce(with_lora):
    rng = np.random.default_rng(21)
    M, K, N = 4, 16, 6
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=3, r=2, seed=5, ids_kind="uniform",
                       none_frac=0.3, W=wl.normal_bf16(rng, (N, K), 0.25))
    xq, sx = oracle.quantize_rows(p.x)
    Wq, sw = oracle.quantize_rows(p.W)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    kw = dict(x=p.x, A=p.A, B=p.B, ranks=p.ranks, scales=p.scales, ids=p.ids) if with_lora else {}
    got = oracle.fp8_gemm_lora_sampled(xq, sx, Wq, sw, rows, cols, **kw)
    for i in range(M * N):
        want = _brute_force_fp8(xq, sx, Wq, sw, p.x, p.A if with_lora else None, p.B, p.ranks,
                                p.scales, p.ids, rows[i], cols[i])
        assert abs(got[i] - float(want)) <= 1e-12 * (1 + abs(float(want)))


def test_fp8_gemm_small_int_exact():
    """Small integers are exact in E4M3 with unit scales: the GEMM is exact."""
    rng = np.random.default_rng(3)
    M, K, N = 3, 32, 5
    xi = rng.integers(-8, 9, size=(M, K)).astype(np.float32)
    xi[:, 0] = 448.0  # pin amax so that sx == 1
    wi = rng.integers(-8, 9, size=(N, K)).astype(np.float32)
    wi[:, 0] = 448.0
    xq, sx = oracle.quantize_rows(wl.to_bf16_bits(xi))
    Wq, sw = oracle.quantize_rows(wl.to_bf16_bits(wi))
    assert (sx == 1).all() and (sw == 1).all()
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    got = oracle.fp8_gemm_lora_sampled(xq, sx, Wq, sw, rows, cols)
    assert np.array_equal(got.reshape(M, N), xi.astype(np.float64) @ wi.T.astype(np.float64))


def test_linear_bf16_matches_numpy():
    rng = np.random.default_rng(8)
    x = wl.normal_bf16(rng, (5, 33))
    W = wl.normal_bf16(rng, (7, 33))
    rows = np.repeat(np.arange(5), 7).astype(np.int32)
    cols = np.tile(np.arange(7), 5).astype(np.int32)
    got = oracle.linear_bf16_sampled(x, W, rows, cols).reshape(5, 7)
    want = oracle.bf16_to_f64(x) @ oracle.bf16_to_f64(W).T
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- token-wise merge (LoRA-Switch)

def _merge_problem(seed, N=6, K=7, n_adapters=4, r_max=3, n_sel=2, ints=False):
    rng = np.random.default_rng(seed)
    ranks = rng.integers(1, r_max + 1, size=n_adapters).astype(np.int32)
    scales = rng.choice(np.array([0.5, 1.0, 2.0, -1.5], np.float32), size=n_adapters)

    def draw(shape, std):
        if ints:
            return wl.to_bf16_bits(rng.integers(-2, 3, size=shape).astype(np.float32))
        return wl.normal_bf16(rng, shape, std)
    W = draw((N, K), 0.5)
    A = np.full((n_adapters, K, r_max), wl.BF16_NAN, np.uint16)
    B = np.full((n_adapters, r_max, N), wl.BF16_NAN, np.uint16)
    for a in range(n_adapters):
        A[a, :, :ranks[a]] = draw((K, ranks[a]), 0.4)
        B[a, :ranks[a], :] = draw((ranks[a], N), 0.6)
    sel = rng.choice(n_adapters, size=n_sel, replace=False).astype(np.int32)
    gates = (rng.choice(np.array([0.25, 0.5, 0.75, 1.0], np.float32), size=n_sel) if ints
             else rng.random(n_sel).astype(np.float32))
    return W, A, B, ranks, scales, sel, gates


def _brute_force_merge(W, A, B, ranks, scales, sel, gates):
    """Exact rationals: W + sum_e g_e s_a (A_a B_a)^T, elementwise."""
    N, K = W.shape
    Wf = _frac_bf16(W)
    out = [list(row) for row in Wf]
    for e, a in enumerate(sel):
        a = int(a)
        if not 0 <= a < A.shape[0]:
            continue
        r = int(ranks[a])
        Af = _frac_bf16(A[a][:, :r])
        Bf = _frac_bf16(B[a][:r, :])
        c = Fraction(float(gates[e])) * Fraction(float(scales[a]))
        for n in range(N):
            for k in range(K):
                out[n][k] += c * sum(Af[k][j] * Bf[j][n] for j in range(r))
    return out


@pytest.mark.parametrize("seed", range(4))
def test_merge_exact_rationals_small_ints(seed):
    args = _merge_problem(seed, ints=True)
    got = oracle.lora_switch_merge(*args)
    assert [[Fraction(float(v)) for v in row] for row in got] == _brute_force_merge(*args)


@pytest.mark.parametrize("seed", range(4))
def test_merge_rationals_random_bf16(seed):
    args = _merge_problem(50 + seed, N=5, K=9, n_sel=3)
    got = oracle.lora_switch_merge(*args)
    want = np.array([[float(v) for v in row] for row in _brute_force_merge(*args)])
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_merge_zero_gates_and_no_adapter_give_the_backbone():
    W, A, B, ranks, scales, sel, gates = _merge_problem(9, N=12, K=10)
    base = oracle.bf16_to_f64(W)
    assert np.array_equal(oracle.lora_switch_merge(W, A, B, ranks, scales, sel, gates * 0), base)
    none = np.full_like(sel, -1)
    assert np.array_equal(oracle.lora_switch_merge(W, A, B, ranks, scales, none, gates), base)
    bad = np.array([A.shape[0], 99], np.int32)  # ids outside the pool add nothing
    assert np.array_equal(oracle.lora_switch_merge(W, A, B, ranks, scales, bad, gates), base)


def test_merge_is_linear_in_the_gates():
    W, A, B, ranks, scales, sel, gates = _merge_problem(10, N=16, K=12, n_sel=2)
    base = oracle.bf16_to_f64(W)
    both = oracle.lora_switch_merge(W, A, B, ranks, scales, sel, gates) - base
    one = oracle.lora_switch_merge(W, A, B, ranks, scales, sel[:1], gates[:1]) - base
    two = oracle.lora_switch_merge(W, A, B, ranks, scales, sel[1:], gates[1:]) - base
    assert np.allclose(both, one + two, rtol=1e-12, atol=1e-15)


def test_merged_weight_reproduces_the_unmerged_layer():
    """Punica README, "How?": x.(W + A.B) = x.W + x.A.B. A token routed to one adapter
    with gate 1 gets the same output from the merged backbone as from the base layer
    plus the separately pinned LoRA apply."""
    p = _random_problem(11, T=8, n_adapters=4, h_in=24, h_out=20, r_max=8)
    a = 2
    merged = oracle.lora_switch_merge(p.W[0], p.A[0], p.B[0], p.ranks, p.scales,
                                      np.array([a], np.int32), np.array([1.0], np.float32))
    xf = oracle.bf16_to_f64(p.x[0])
    y_merged = xf @ merged.T
    rows = np.repeat(np.arange(p.T), p.h_out).astype(np.int32)
    cols = np.tile(np.arange(p.h_out), p.T).astype(np.int32)
    base = oracle.linear_bf16_sampled(p.x[0], p.W[0], rows, cols).reshape(p.T, p.h_out)
    ids = np.full(p.T, a, np.int32)
    lora = oracle.lora_apply(p.x[0], p.A[0], p.B[0], p.ranks, p.scales, ids,
                             np.zeros((p.T, p.h_out), np.uint16))
    assert np.allclose(y_merged, base + lora, rtol=1e-10, atol=1e-12)


def test_merge_rank1_closed_form():
    """A_a = e_j0 (one nonzero row k0, column 0) and rank 1: the delta is g s B[0][n] at
    column k0 only."""
    N, K, r_max = 6, 8, 8
    W = wl.normal_bf16(np.random.default_rng(3), (N, K), 0.3)
    A = np.zeros((1, K, r_max), np.uint16)
    k0 = 5
    A[0, k0, 0] = wl.to_bf16_bits(np.array([1.0], np.float32))[0]
    B = np.zeros((1, r_max, N), np.uint16)
    B[0, 0] = wl.to_bf16_bits(np.linspace(-1, 1, N).astype(np.float32))
    out = oracle.lora_switch_merge(W, A, B, np.array([1], np.int32), np.array([2.0], np.float32),
                                   np.array([0], np.int32), np.array([0.5], np.float32))
    delta = out - oracle.bf16_to_f64(W)
    want = np.zeros((N, K))
    want[:, k0] = 0.5 * 2.0 * oracle.bf16_to_f64(B[0, 0])
    assert np.array_equal(delta, want)


# ---------------------------------------------------------------- gradients (adapter training)

def _loss_lora(x, A, B, ranks, scales, ids, dY):
    """L = sum dY * (s (x A) B) through the separately pinned forward oracle."""
    y = oracle.lora_apply(x, A, B, ranks, scales, ids, np.zeros(dY.shape, np.uint16))
    return float(np.sum(oracle.bf16_to_f64(dY) * y))


def _int_bits(rng, shape, lo=-2, hi=3):
    return wl.to_bf16_bits(rng.integers(lo, hi, size=shape).astype(np.float32))


def _grad_problem(seed, M=7, K=6, N=5, n_ad=3, r_max=3):
    rng = np.random.default_rng(seed)
    x = _int_bits(rng, (M, K))
    dY = _int_bits(rng, (M, N))
    ranks = rng.integers(1, r_max + 1, size=n_ad).astype(np.int32)
    A = np.full((n_ad, K, r_max), wl.BF16_NAN, np.uint16)
    B = np.full((n_ad, r_max, N), wl.BF16_NAN, np.uint16)
    for a in range(n_ad):
        A[a, :, :ranks[a]] = _int_bits(rng, (K, ranks[a]))
        B[a, :ranks[a], :] = _int_bits(rng, (ranks[a], N))
    scales = rng.choice(np.array([0.5, 1.0, 2.0, -1.5], np.float32), size=n_ad)
    ids = rng.integers(-1, n_ad, size=M).astype(np.int32)
    return rng, x, dY, A, B, ranks, scales, ids


@pytest.mark.parametrize("seed", range(4))
def test_backward_adjoint_identities(seed):
    """The layer is linear in x, in A (B fixed) and in B (A fixed), so for any
    direction d: L(. + d) - L(.) = <grad, d> exactly (small integers: every value
    and sum is exact in fp64)."""
    rng, x, dY, A, B, ranks, scales, ids = _grad_problem(seed)
    dX, dA, dB = oracle.lora_backward(x, dY, A, B, ranks, scales, ids)
    L0 = _loss_lora(x, A, B, ranks, scales, ids, dY)
    d = _int_bits(rng, x.shape, -1, 2)
    xd = wl.to_bf16_bits((oracle.bf16_to_f64(x) + oracle.bf16_to_f64(d)).astype(np.float32))
    assert _loss_lora(xd, A, B, ranks, scales, ids, dY) - L0 == float(np.sum(dX * oracle.bf16_to_f64(d)))
    dAdir = np.zeros(A.shape, np.float64)
    Ad = A.copy()
    for a in range(A.shape[0]):
        r = ranks[a]
        step = rng.integers(-1, 2, size=(A.shape[1], r)).astype(np.float64)
        dAdir[a, :, :r] = step
        Ad[a, :, :r] = wl.to_bf16_bits((oracle.bf16_to_f64(A[a, :, :r]) + step).astype(np.float32))
    assert _loss_lora(x, Ad, B, ranks, scales, ids, dY) - L0 == float(np.sum(dA * dAdir))
    dBdir = np.zeros(B.shape, np.float64)
    Bd = B.copy()
    for a in range(B.shape[0]):
        r = ranks[a]
        step = rng.integers(-1, 2, size=(r, B.shape[2])).astype(np.float64)
        dBdir[a, :r, :] = step
        Bd[a, :r, :] = wl.to_bf16_bits((oracle.bf16_to_f64(B[a, :r, :]) + step).astype(np.float32))
    assert _loss_lora(x, A, Bd, ranks, scales, ids, dY) - L0 == float(np.sum(dB * dBdir))


def test_backward_brute_force_rationals():
    """Every output from its definition in exact rationals (u, v, then the sums)."""
    rng, x, dY, A, B, ranks, scales, ids = _grad_problem(9, M=5, K=4, N=3)
    dX, dA, dB = oracle.lora_backward(x, dY, A, B, ranks, scales, ids)
    X, D = _frac_bf16(x), _frac_bf16(dY)
    M, K, N = len(X), len(X[0]), len(D[0])
    n_ad, _, r_max = A.shape
    wdX = [[Fraction(0)] * K for _ in range(M)]
    wdA = np.zeros(A.shape, dtype=object); wdA[:] = Fraction(0)
    wdB = np.zeros(B.shape, dtype=object); wdB[:] = Fraction(0)
    for m in range(M):
        a = int(ids[m])
        if a < 0:
            continue
        r = int(ranks[a])
        Af, Bf = _frac_bf16(A[a][:, :r]), _frac_bf16(B[a][:r, :])
        s = Fraction(float(scales[a]))
        u = [sum(D[m][n] * Bf[j][n] for n in range(N)) for j in range(r)]
        v = [sum(X[m][k] * Af[k][j] for k in range(K)) for j in range(r)]
        for k in range(K):
            wdX[m][k] = s * sum(u[j] * Af[k][j] for j in range(r))
            for j in range(r):
                wdA[a, k, j] += s * X[m][k] * u[j]
        for j in range(r):
            for n in range(N):
                wdB[a, j, n] += s * v[j] * D[m][n]
    assert [[Fraction(float(t)) for t in row] for row in dX] == wdX
    assert all(Fraction(float(g)) == w for g, w in zip(dA.ravel(), wdA.ravel()))
    assert all(Fraction(float(g)) == w for g, w in zip(dB.ravel(), wdB.ravel()))


def test_backward_base_term_is_the_adjoint_of_the_8bit_product():
    """The base term of dX is the adjoint of y = x . W'^T, W'[n][k] = swT[k] WqT[k][n],
    under the quantised upstream dY' = sd . dYq: <base, d> = <dY', d . W'^T>."""
    rng = np.random.default_rng(21)
    M, K, N = 6, 40, 24
    x = wl.normal_bf16(rng, (M, K))
    dY = wl.normal_bf16(rng, (M, N))
    WT = wl.normal_bf16(rng, (K, N), 0.2)
    WqT, swT = oracle.quantize_rows(WT)
    dYq, sd = oracle.quantize_rows(dY)
    A = np.zeros((1, K, 8), np.uint16)
    B = np.zeros((1, 8, N), np.uint16)
    ids = np.full(M, -1, np.int32)
    dX, dA, dB = oracle.lora_backward(x, dY, A, B, None, None, ids, dYq, sd, WqT, swT)
    Wp = (swT[:, None].astype(np.float64) * oracle.e4m3_to_f64(WqT)).T   # [N][K]
    dYp = sd[:, None].astype(np.float64) * oracle.e4m3_to_f64(dYq)       # [M][N]
    d = rng.standard_normal((M, K))
    assert np.isclose(np.sum(dX * d), np.sum(dYp * (d @ Wp.T)), rtol=1e-12)
    assert not dA.any() and not dB.any()   # no token has an adapter


def test_backward_invariants():
    rng, x, dY, A, B, ranks, scales, ids = _grad_problem(12, M=9)
    dX, dA, dB = oracle.lora_backward(x, dY, A, B, ranks, scales, ids)
    # tokens without an adapter get no adapter term; permuting tokens permutes dX only
    assert not dX[ids < 0].any()
    pi = rng.permutation(len(ids))
    dX2, dA2, dB2 = oracle.lora_backward(x[pi], dY[pi], A, B, ranks, scales, ids[pi])
    assert np.array_equal(dX2, dX[pi]) and np.allclose(dA2, dA) and np.allclose(dB2, dB)
    # B = 0: u = 0, so dX and dA vanish while dB does not
    B0 = np.where(B == wl.BF16_NAN, B, np.uint16(0))
    dX0, dA0, dB0 = oracle.lora_backward(x, dY, A, B0, ranks, scales, ids)
    assert not dX0.any() and not dA0.any() and dB0.any()
    # the padding past each rank is never written
    for a in range(A.shape[0]):
        assert not dA[a, :, ranks[a]:].any() and not dB[a, ranks[a]:, :].any()


# ---------------------------------------------------------------- MX FP4 (4-bit base)

def test_e2m1_decode_golden_values():
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_decode(int(code, 16))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_e8m0_decode():
    assert oracle.e8m0_decode(127) == 1.0 and oracle.e8m0_decode(128) == 2.0
    assert oracle.e8m0_decode(0) == 2.0 ** -127 and oracle.e8m0_decode(254) == 2.0 ** 127
    assert math.isnan(oracle.e8m0_decode(255))


def test_e2m1_encode_round_trip_ties_and_saturation():
    for c in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_decode(c)) == (c if c != 8 else 8)
    # midpoints go to the code with fraction bit 0
    for mid, want in [(0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
                      (5.0, 0x6)]:
        assert oracle.e2m1_encode(mid) == want, mid
        assert oracle.e2m1_encode(-mid) == want | 8, -mid
    for big in (6.0, 6.5, 7.9, 100.0):
        assert oracle.e2m1_encode(big) == 0x7 and oracle.e2m1_encode(-big) == 0xF
    assert oracle.e2m1_encode(0.26) == 0x1 and oracle.e2m1_encode(0.24) == 0x0


def _mx_representable_rows(rng, N, K):
    """Rows whose every 32-block is E2M1 codes times 2^k with the block's largest
    magnitude 4 or 6 times 2^k: exactly representable in MXFP4 (and in bf16)."""
    W = np.zeros((N, K), np.float32)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    for n in range(N):
        for b in range(K // 32):
            k = int(rng.integers(-6, 4))
            v = rng.choice(mags, 32) * rng.choice([-1.0, 1.0], 32)
            v[rng.integers(0, 32)] = rng.choice([4.0, 6.0]) * rng.choice([-1.0, 1.0])
            W[n, b * 32:(b + 1) * 32] = v * 2.0 ** k
    return wl.to_bf16_bits(W), W


def test_mxfp4_quantize_exact_on_representable_blocks():
    rng = np.random.default_rng(31)
    Wb, W = _mx_representable_rows(rng, 6, 96)
    codes, scales = oracle.mxfp4_quantize(Wb)
    deq = np.vectorize(oracle.e2m1_decode)(codes) * np.repeat(
        np.vectorize(oracle.e8m0_decode)(scales), 32, axis=1)
    assert np.array_equal(deq, W.astype(np.float64))


def test_mxfp4_quantize_scale_rule_and_zero_block():
    # amax 1.0 -> X = 2^(0 - 2): 1.0 / 0.25 = 4, code 6
    W = np.zeros((2, 64), np.float32)
    W[0, :32] = 1.0
    W[0, 32:] = np.linspace(-7.9, 7.9, 32)   # amax 7.9: X = 2^(2 - 2) = 1, 7.9 saturates to 6
    codes, scales = oracle.mxfp4_quantize(wl.to_bf16_bits(W))
    assert scales[0, 0] == 127 - 2 and (codes[0, :32] == 0x6).all()
    assert scales[0, 1] == 127 and codes[0, 32] == 0xF and codes[0, 63] == 0x7
    assert scales[1, 0] == 0 and (codes[1] == 0).all()      # all-zero blocks


def test_mxfp4_gemm_equals_bf16_linear_on_representable_weights():
    """With MXFP4-representable weights the 4-bit GEMM equals the (separately pinned)
    bf16 linear oracle on the same values."""
    rng = np.random.default_rng(32)
    N, K, M = 10, 128, 5
    Wb, _ = _mx_representable_rows(rng, N, K)
    x = wl.normal_bf16(rng, (M, K))
    codes, scales = oracle.mxfp4_quantize(Wb)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    got = oracle.mxfp4_gemm_lora_sampled(x, codes, scales, rows, cols)
    want = oracle.linear_bf16_sampled(x, Wb, rows, cols)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_mxfp4_gemm_lora_brute_force_rationals():
    rng = np.random.default_rng(33)
    M, K, N, n_ad, r = 3, 64, 4, 2, 2
    x = wl.to_bf16_bits(rng.integers(-2, 3, (M, K)).astype(np.float32))
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    scales = rng.integers(124, 130, (N, K // 32)).astype(np.uint8)
    A = wl.to_bf16_bits(rng.integers(-2, 3, (n_ad, K, r)).astype(np.float32))
    B = wl.to_bf16_bits(rng.integers(-2, 3, (n_ad, r, N)).astype(np.float32))
    ranks = np.array([2, 1], np.int32)
    sl = np.array([2.0, 0.5], np.float32)
    ids = np.array([0, -1, 1], np.int32)
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    got = oracle.mxfp4_gemm_lora_sampled(x, codes, scales, rows, cols, A=A, B=B, ranks=ranks,
                                         scales_lora=sl, ids=ids)
    X = _frac_bf16(x)
    E2 = [Fraction(oracle.e2m1_decode(c)) for c in range(16)]
    for i, (m, n) in enumerate(zip(rows, cols)):
        y = sum(X[m][k] * E2[codes[n, k]] * Fraction(2) ** (int(scales[n, k // 32]) - 127) for k in range(K))
        a = int(ids[m])
        if a >= 0:
            Af, Bf = _frac_bf16(A[a]), _frac_bf16(B[a])
            v = [sum(X[m][k] * Af[k][j] for k in range(K)) for j in range(ranks[a])]
            y += Fraction(float(sl[a])) * sum(v[j] * Bf[j][n] for j in range(ranks[a]))
        assert Fraction(got[i]) == y


# ---------------------------------------------------------------- W8A16 (FP8 weights, bf16 activations)

def test_w8a16_equals_bf16_linear_on_power_of_two_scales():
    """With power-of-two channel scales every dequantised weight sw * E4M3(code) is a bf16
    value, and the W8A16 product equals the (separately pinned) bf16 linear oracle."""
    rng = np.random.default_rng(51)
    M, K, N = 5, 96, 12
    x = wl.normal_bf16(rng, (M, K))
    Wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
    Wq[(Wq & 0x7F) == 0x7F] = 0x10          # no NaN codes
    sw = (2.0 ** rng.integers(-8, 3, N)).astype(np.float32)
    W = wl.to_bf16_bits((oracle.e4m3_to_f64(Wq) * sw[:, None]).astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f64(W), oracle.e4m3_to_f64(Wq) * sw[:, None])
    rows = np.repeat(np.arange(M), N).astype(np.int32)
    cols = np.tile(np.arange(N), M).astype(np.int32)
    got = oracle.w8a16_gemm_lora_sampled(x, Wq, sw, rows, cols)
    assert np.allclose(got, oracle.linear_bf16_sampled(x, W, rows, cols), rtol=1e-13, atol=1e-13)


def test_w8a16_lora_term_matches_the_apply_oracle():
    """The LoRA term of W8A16 is the pinned apply oracle's term (zero base weight)."""
    p = _random_problem(52, T=6, n_adapters=3, h_in=32, h_out=16, r_max=8)
    Wq = np.zeros((p.h_out, p.h_in), np.uint8)
    sw = np.ones(p.h_out, np.float32)
    rows = np.repeat(np.arange(p.T), p.h_out).astype(np.int32)
    cols = np.tile(np.arange(p.h_out), p.T).astype(np.int32)
    got = oracle.w8a16_gemm_lora_sampled(p.x[0], Wq, sw, rows, cols, A=p.A[0], B=p.B[0], ranks=p.ranks,
                                         scales=p.scales, ids=p.ids).reshape(p.T, p.h_out)
    want = oracle.lora_apply(p.x[0], p.A[0], p.B[0], p.ranks, p.scales, p.ids,
                             np.zeros((p.T, p.h_out), np.uint16))
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
