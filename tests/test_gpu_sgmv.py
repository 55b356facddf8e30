"""GPU parity of the segment builder and the SGMV shrink / expand / apply kernels
against the fp64 oracle, through the C ABI, on seeded inputs (workloads.py).

Tolerance (the stated bar for bf16 inputs with fp32 accumulation):
max |gpu - oracle| <= 2e-2 * (1 + |oracle|) elementwise. Integer work (the
segments) is bit-exact; small-integer inputs make the float results exact, so
there the GPU must equal the oracle rounded once to bf16."""
import numpy as np
import pytest
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from tile_rule import expected_tiles, tile_tokens
from gpu_util import (TOL_BF16, DeviceProblem, assert_close, dev, dev_bf16, f64, host_bf16_bits,
                      oracle_apply, rne_bf16_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()


# ------------------------------------------------------------------ segments

def _check_segments(ids, n_adapters):
    """The grouping (perm, indptr, active, tok_adapter, counts) bit-exact against
    the oracle; the tile table against the tile rule applied to the oracle's grouping."""
    T = len(ids)
    seg = L.Segments(T, n_adapters)
    L.lora_build_segments(dev(ids) if T else torch.empty(0, dtype=torch.int32, device="cuda"),
                          n_adapters, seg)
    torch.cuda.synchronize()
    want = oracle.build_segments(ids, n_adapters)
    counts = seg.counts.cpu().numpy()
    t = L.tile_tokens_for(T, n_adapters)
    assert t == tile_tokens(T, n_adapters)
    want_tiles = expected_tiles(want["indptr"], want["active"], want["counts"][1], t)
    assert counts[:3].tolist() == want["counts"].tolist()
    assert counts[3] == len(want_tiles)
    assert counts[4:].tolist() == [0, 0, 0, 0]
    assert seg.indptr.cpu().numpy().tolist() == want["indptr"].tolist()
    assert seg.active.cpu().numpy().tolist() == want["active"].tolist()
    got_tiles = seg.tiles.cpu().numpy()
    n_rows = L.max_tiles(T, n_adapters)
    assert len(want_tiles) <= n_rows
    assert got_tiles[:len(want_tiles)].tolist() == want_tiles
    assert all(row == [-1, 0, 0, -1] for row in got_tiles[len(want_tiles):n_rows].tolist())
    if T:
        assert seg.perm.cpu().numpy()[:T].tolist() == want["perm"].tolist()
        assert seg.tok_adapter.cpu().numpy()[:T].tolist() == want["tok_adapter"].tolist()


@pytest.mark.parametrize("kind,T,n", [
    ("distinct", 36, 32), ("identical", 36, 32), ("uniform", 1000, 7), ("zipf", 512, 256),
    ("sorted_zipf", 2300, 8), ("uniform", 5000, 3000), ("zipf", 4097, 1), ("uniform", 1, 5),
    ("zipf", 70000, 16384),
    # one-warp builder (T <= 64, n <= 64): both tile sizes, a partial second slot of lanes
    ("zipf", 64, 64), ("uniform", 50, 3), ("zipf", 17, 60), ("sorted_zipf", 40, 8),
    ("identical", 64, 1), ("uniform", 33, 64), ("distinct", 64, 64),
])
def test_segments_bitexact(kind, T, n):
    rng = np.random.default_rng(T + n)
    ids = wl.make_ids(kind if kind != "distinct" else "distinct", rng, T, n,
                      none_frac=0.05 if kind != "identical" else 0.0)
    _check_segments(ids, n)


def test_segments_edge_cases():
    _check_segments(np.zeros(0, np.int32), 4)               # empty batch
    _check_segments(np.full(300, -1, np.int32), 9)          # nobody has an adapter
    rng = np.random.default_rng(3)
    bad = rng.integers(-5, 15, size=777).astype(np.int32)    # out-of-range ids
    _check_segments(bad, 10)
    _check_segments(rng.integers(-5, 15, size=40).astype(np.int32), 10)  # the same, one warp
    _check_segments(np.full(20, -1, np.int32), 4)            # one warp, nobody has an adapter


def test_segments_sync_check_reports_bad_ids():
    ids = np.array([0, 1, 7, -1, 2], np.int32)
    seg = L.Segments(5, 3)
    with pytest.raises(L.LoraError) as e:
        L.lora_build_segments(dev(ids), 3, seg, sync_check=True)
    assert e.value.status == L.LORA_ERR_BAD_ADAPTER_ID
    L.lora_build_segments(dev(np.array([0, -1, 2], np.int32)), 3, L.Segments(3, 3),
                          sync_check=True)


# ------------------------------------------------------------------ problems

def _small(seed, T=150, n_adapters=6, h_in=520, h_out=392, r_max=32, kind="zipf", n_slices=1,
           rank_choices=(1, 5, 8, 13, 24, 32), none_frac=0.1):
    return wl.make_lora_problem("t", seed, T=T, n_adapters=n_adapters, h_in=h_in, h_out=h_out,
                                r_max=r_max, ids_kind=kind, none_frac=none_frac,
                                rank_choices=rank_choices, n_slices=n_slices)


SMALL_CASES = {
    "ragged_mixed_ranks": dict(seed=11),
    "multi_tile_segment": dict(seed=12, T=300, n_adapters=3, kind="sorted_zipf"),
    "decode_distinct": dict(seed=13, T=40, n_adapters=48, kind="distinct", h_in=2048,
                            h_out=1024, r_max=16, rank_choices=(16,)),
    "rank64_slices": dict(seed=14, T=90, n_adapters=9, r_max=64, rank_choices=(8, 16, 32, 64),
                          n_slices=3, h_in=640, h_out=512),
    "tiny_dims": dict(seed=15, T=7, n_adapters=2, h_in=8, h_out=8, r_max=8, rank_choices=(3, 8)),
    "single_token": dict(seed=16, T=1, n_adapters=1, none_frac=0.0),
    "medium_tiles": dict(seed=17, T=120, n_adapters=10, h_in=1024, h_out=768, r_max=16,
                         rank_choices=(16,), kind="uniform"),
    "rank8_pool": dict(seed=18, T=33, n_adapters=4, h_in=256, h_out=136, r_max=8,
                       rank_choices=(3, 8)),
    # decode-like (T <= 64, T <= 2 n): 4-token tiles on the decode kernel, several tiles
    # for the adapters with more tokens, mixed ranks and a ragged h_out
    "decode_zipf": dict(seed=19, T=48, n_adapters=32, kind="zipf", h_in=1024, h_out=520,
                        r_max=32, rank_choices=(1, 8, 16, 32)),
}


@pytest.mark.parametrize("case", list(SMALL_CASES))
def test_apply_parity_small(case):
    p = _small(**SMALL_CASES[case])
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    got = f64(host_bf16_bits(y))
    want = oracle_apply(p)
    assert_close(got, want, TOL_BF16, case)
    none = p.ids == -1
    assert np.array_equal(host_bf16_bits(y)[:, none], p.y_in[:, none])  # untouched, bit-exact


@pytest.mark.parametrize("case", list(SMALL_CASES))
def test_shrink_parity_small(case):
    p = _small(**SMALL_CASES[case])
    d = DeviceProblem(p)
    v = torch.full((p.n_slices, p.T, p.r_max), float("nan"), device="cuda")
    L.lora_shrink(d.x, d.pool, d.seg, v)
    torch.cuda.synchronize()
    got = v.cpu().numpy().astype(np.float64)
    for s in range(p.n_slices):
        want = oracle.lora_shrink(p.x[s], p.A[s], p.ranks, p.ids)
        has = p.ids >= 0
        assert_close(got[s][has], want[has], TOL_BF16, f"{case} slice {s}")
        assert np.isnan(got[s][~has]).all()  # rows without an adapter are not written


@pytest.mark.parametrize("case", list(SMALL_CASES))
def test_expand_parity_small(case):
    p = _small(**SMALL_CASES[case])
    d = DeviceProblem(p)
    rng = np.random.default_rng(99)
    v = rng.standard_normal((p.n_slices, p.T, p.r_max)).astype(np.float32)
    y = d.y_in()
    L.lora_expand(dev(v), d.pool, d.seg, y)
    torch.cuda.synchronize()
    got = f64(host_bf16_bits(y))
    for s in range(p.n_slices):
        want = oracle.lora_expand(v[s], p.B[s], p.ranks, p.scales, p.ids, p.y_in[s])
        assert_close(got[s], want, TOL_BF16, f"{case} slice {s}")


def test_apply_exact_small_integers():
    """Small-integer inputs: every product and sum is exact in fp32, so the GPU
    result must equal the exact value rounded once to bf16."""
    rng = np.random.default_rng(5)
    T, n_adapters, h_in, h_out, r_max = 130, 5, 1024, 264, 32
    p = _small(21, T=T, n_adapters=n_adapters, h_in=h_in, h_out=h_out, r_max=r_max,
               rank_choices=(3, 16, 32))
    p.x[:] = wl.to_bf16_bits(rng.integers(-2, 3, size=p.x.shape).astype(np.float32))
    for a in range(n_adapters):
        r = p.ranks[a]
        p.A[:, a, :, :r] = wl.to_bf16_bits(rng.integers(-2, 3, size=(1, h_in, r)).astype(np.float32))
        p.B[:, a, :r, :] = wl.to_bf16_bits(rng.integers(-2, 3, size=(1, r, h_out)).astype(np.float32))
    p.y_in[:] = wl.to_bf16_bits(rng.integers(-8, 9, size=p.y_in.shape).astype(np.float32))
    p.scales[:] = 2.0
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    v = torch.zeros((1, T, r_max), device="cuda")
    L.lora_shrink(d.x, d.pool, d.seg, v)
    torch.cuda.synchronize()
    want = oracle_apply(p)
    assert np.array_equal(host_bf16_bits(y), rne_bf16_bits(want))
    v_want = oracle.lora_shrink(p.x[0], p.A[0], p.ranks, p.ids)
    has = p.ids >= 0
    assert np.array_equal(v.cpu().numpy()[0][has].astype(np.float64), v_want[has])


def test_apply_invariants_on_gpu():
    p = _small(31, T=200, n_adapters=8, h_in=512, h_out=256, r_max=16, rank_choices=(16,))
    d = DeviceProblem(p)
    # B = 0 leaves y unchanged, bit for bit
    zB = L.Pool(d.A, torch.zeros_like(d.B), d.ranks, d.scales)
    y = d.y_in()
    L.lora_apply(d.x, zB, d.seg, y)
    torch.cuda.synchronize()
    assert np.array_equal(host_bf16_bits(y), p.y_in)
    # permuting tokens permutes outputs
    y1 = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y1)
    pi = np.random.default_rng(1).permutation(p.T)
    p2 = wl.LoraProblem("perm", p.x[:, pi], p.A, p.B, p.ids[pi], p.ranks, p.scales, p.y_in[:, pi])
    d2 = DeviceProblem(p2)
    y2 = d2.y_in()
    L.lora_apply(d2.x, d2.pool, d2.seg, y2)
    torch.cuda.synchronize()
    assert_close(f64(host_bf16_bits(y2)), f64(host_bf16_bits(y1))[:, pi], TOL_BF16, "permutation")


def test_shared_x_across_slices():
    p = _small(41, T=64, n_slices=3, h_in=256, h_out=128, r_max=16, rank_choices=(16,))
    p.x[1] = p.x[0]
    p.x[2] = p.x[0]
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x[0], d.pool, d.seg, y, x_slice_stride=0)
    torch.cuda.synchronize()
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, "shared x")


# ------------------------------------------------------------------ the named workloads, full size

def test_sgmv_tiny_full():
    p = wl.sgmv_tiny()
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, "sgmv_tiny")


@pytest.mark.parametrize("kind", ["distinct", "identical"])
def test_bgmv_decode_full(kind):
    p = wl.bgmv_decode(ids_kind=kind)
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, f"bgmv_decode {kind}")


def test_sgmv_prefill_full_sampled_tokens():
    p = wl.sgmv_prefill()
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(p.T, size=192, replace=False))
    # include the first and last token of every segment (tile boundaries)
    starts = np.concatenate([[0], np.cumsum(np.bincount(p.ids))])
    rows = np.unique(np.concatenate([rows, starts[:-1], starts[1:] - 1]))
    got = f64(host_bf16_bits(y))[:, rows]
    assert_close(got, oracle_apply(p, rows=rows), TOL_BF16, "sgmv_prefill")


def test_many_tenants_full():
    p = wl.many_tenants()
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, "many_tenants")


# ------------------------------------------------------------------ ids without an adapter

@pytest.mark.parametrize("T,n", [(36, 32), (150, 6)])
def test_apply_all_ids_none_leaves_y_untouched(T, n):
    """No token has an adapter (decode-like and general batches): y stays bit-exact."""
    p = _small(51, T=T, n_adapters=n, h_in=512, h_out=264, r_max=16, rank_choices=(16,))
    p.ids[:] = -1
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert np.array_equal(host_bf16_bits(y), p.y_in)
    assert seg_counts(d.seg)[:2] == [0, 0]


@pytest.mark.parametrize("T,n", [(40, 24), (300, 7)])
def test_apply_out_of_range_ids_served_as_none(T, n):
    """Ids outside [-1, n_adapters) are counted as bad and served as -1."""
    p = _small(52, T=T, n_adapters=n, h_in=512, h_out=264, r_max=16, rank_choices=(8, 16))
    rng = np.random.default_rng(52)
    p.ids[:] = rng.integers(-4, n + 4, size=T).astype(np.int32)
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    bad = (p.ids < -1) | (p.ids >= n)
    assert seg_counts(d.seg)[2] == int(bad.sum())
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, "out-of-range ids")
    none = (p.ids < 0) | (p.ids >= n)
    assert np.array_equal(host_bf16_bits(y)[:, none], p.y_in[:, none])


def seg_counts(seg):
    return seg.counts.cpu().numpy().tolist()


# ------------------------------------------------------------------ whole layer

def _whole_layer(p, W, rows):
    """y = x.W^T (the harness's base GEMM: torch bf16 on the GPU, stored as bf16) plus
    lora_apply, against the oracle's y_ref = sum_k x.W + s.(x.A).B in fp64, on the
    given token rows of every slice."""
    d = DeviceProblem(p)
    xs = d.x
    Wd = dev_bf16(W)
    y = torch.stack([xs[s] @ Wd[s].t() for s in range(p.n_slices)]).contiguous()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    got = f64(host_bf16_bits(y))[:, rows]
    zeros = np.zeros((len(rows), p.h_out), np.uint16)
    cols = np.tile(np.arange(p.h_out), len(rows)).astype(np.int32)
    rr = np.repeat(np.asarray(rows), p.h_out).astype(np.int32)
    for s in range(p.n_slices):
        base = oracle.linear_bf16_sampled(p.x[s], W[s], rr, cols).reshape(len(rows), p.h_out)
        lora = oracle.lora_apply(p.x[s][rows], p.A[s], p.B[s], p.ranks, p.scales, p.ids[rows], zeros)
        assert_close(got[s], base + lora, TOL_BF16, f"{p.name} whole layer, slice {s}")


def test_whole_layer_sgmv_tiny():
    p = wl.sgmv_tiny()
    _whole_layer(p, p.W, np.arange(p.T))


def test_whole_layer_bgmv_decode():
    p = wl.bgmv_decode()
    W = wl.weight_bf16(p.h_out, p.h_in, seed=101)[None]
    _whole_layer(p, W, np.arange(p.T))


def test_whole_layer_sgmv_prefill_sampled():
    p = wl.sgmv_prefill()
    W = wl.weight_bf16(p.h_out, p.h_in, seed=102)[None]
    starts = np.concatenate([[0], np.cumsum(np.bincount(p.ids))])
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([rng.choice(p.T, 12, replace=False), starts[1:-1], starts[1:] - 1]))
    _whole_layer(p, W, rows)


def test_whole_layer_many_tenants_sampled():
    p = wl.many_tenants()
    W = np.stack([wl.weight_bf16(p.h_out, p.h_in, seed=103 + s) for s in range(p.n_slices)])
    rng = np.random.default_rng(4)
    rows = np.sort(rng.choice(p.T, 24, replace=False))
    _whole_layer(p, W, rows)


# ------------------------------------------------------------------ tile rows in cost order

def _expected_order(tiles, n_used, ranks, r_max):
    """The order lora_apply's workspace holds: the used tile rows stably sorted by class
    (rows of more than four tokens first, then small rows by descending round_up(r, 8)),
    then the unused rows in place."""
    def key(row):
        if row[2] > 4:
            return 0
        r = max(1, min(int(ranks[row[0]]), r_max))
        return 1 + (64 - ((r + 7) & ~7)) // 8
    used = sorted(range(n_used), key=lambda i: key(tiles[i]))  # Python's sort is stable
    return np.concatenate([tiles[used], tiles[n_used:]]) if n_used < len(tiles) else tiles[used]


@pytest.mark.parametrize("ids_kind", ["zipf", "uniform"])
def test_apply_tile_order_same_results_and_cost_order(ids_kind):
    """With a workspace, a general batch's tile rows run in cost order: the output is
    bit-identical to the table-order launch (no workspace), and the workspace holds the
    rows in the stated order."""
    p = wl.many_tenants(seed=11, T=300, n_adapters=96, h=1024, ids_kind=ids_kind)
    d = DeviceProblem(p)
    y0 = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y0, ws=False)
    ws = L.workspace(L.LORA_OP_APPLY, p.T, 0, d.pool)
    y1 = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y1, ws=ws)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    assert np.array_equal(host_bf16_bits(y0), host_bf16_bits(y1))
    tiles = d.seg.tiles.cpu().numpy()
    n_used = int(d.seg.counts[3].item())
    got = ws[: tiles.size * 4].view(torch.int32).cpu().numpy().reshape(-1, 4)
    assert np.array_equal(got, _expected_order(tiles, n_used, p.ranks, p.r_max))
    assert_close(f64(host_bf16_bits(y1)), oracle_apply(p), TOL_BF16, f"ordered apply {ids_kind}")


# ------------------------------------------------------------------ tensor-core expand (long segments)

# Batches of long segments (on average half a tile or more per adapter, h_out >= 128):
# lora_expand runs the tcgen05 expand, and lora_apply with its workspace runs the shrink
# into the workspace and then that expand. Ragged column blocks, ranks that are not
# multiples of 16, a pool padded to 8 (rank rows past the box), several slices, gathered
# and pre-sorted tokens, tiles whose token count is not a multiple of 16.
TC_CASES = {
    "tc_ragged_mixed": dict(seed=61, T=400, n_adapters=6, h_in=264, h_out=392, r_max=32),
    "tc_rank64_slices": dict(seed=62, T=600, n_adapters=9, h_in=320, h_out=520, r_max=64,
                             rank_choices=(8, 16, 40, 48, 64), n_slices=3),
    "tc_rank8_pool": dict(seed=63, T=200, n_adapters=4, h_in=256, h_out=136, r_max=8,
                          rank_choices=(3, 8)),
    "tc_sorted_long": dict(seed=64, T=700, n_adapters=2, h_in=512, h_out=1024, r_max=16,
                           rank_choices=(16,), kind="sorted_zipf", none_frac=0.0),
    "tc_uniform_partial": dict(seed=65, T=130, n_adapters=4, h_in=128, h_out=264, r_max=16,
                               rank_choices=(1, 16), kind="uniform"),
}


def _tc_planes(h_in):
    return min(8, -(-h_in // 64))


def test_tc_cases_take_the_tensor_core_path():
    """The workspace of lora_apply on these batches holds the shrink's planes of v (fp32,
    every slice; one plane per part of h_in, at most 8)."""
    for case, kw in TC_CASES.items():
        p = _small(**kw)
        d = DeviceProblem(p, build=False)
        n = L.lora_workspace_size(L.LORA_OP_APPLY, p.T, 0, d.pool)
        v = _tc_planes(p.h_in) * p.n_slices * p.T * p.r_max * 4
        assert n == -(-max(v, 16 * L.max_tiles(p.T, p.n_adapters)) // 256) * 256, case


@pytest.mark.parametrize("case", ["tc_ragged_mixed", "tc_rank64_slices"])
def test_apply_tc_one_plane_workspace(case):
    """A workspace with room for one plane of v only: the cluster shrink, then the
    tensor-core expand."""
    p = _small(**TC_CASES[case])
    d = DeviceProblem(p)
    ws = torch.zeros(p.n_slices * p.T * p.r_max * 4, dtype=torch.uint8, device="cuda")
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y, ws=ws)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, case)


@pytest.mark.parametrize("case", list(TC_CASES))
def test_expand_tc_parity(case):
    p = _small(**TC_CASES[case])
    d = DeviceProblem(p)
    rng = np.random.default_rng(7)
    v = rng.standard_normal((p.n_slices, p.T, p.r_max)).astype(np.float32)
    y = d.y_in()
    L.lora_expand(dev(v), d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    got = f64(host_bf16_bits(y))
    for s in range(p.n_slices):
        want = oracle.lora_expand(v[s], p.B[s], p.ranks, p.scales, p.ids, p.y_in[s])
        assert_close(got[s], want, TOL_BF16, f"{case} slice {s}")
    none = p.ids == -1
    assert np.array_equal(host_bf16_bits(y)[:, none], p.y_in[:, none])


@pytest.mark.parametrize("case", list(TC_CASES))
@pytest.mark.parametrize("ws", [None, False], ids=["shrink+tc_expand", "cluster"])
def test_apply_tc_parity(case, ws):
    p = _small(**TC_CASES[case])
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y, ws=ws)
    torch.cuda.synchronize()
    assert L.lora_segments_status(d.seg)[0] == L.LORA_OK
    assert_close(f64(host_bf16_bits(y)), oracle_apply(p), TOL_BF16, case)
    none = p.ids == -1
    assert np.array_equal(host_bf16_bits(y)[:, none], p.y_in[:, none])


def test_apply_tc_exact_small_integers():
    """Small integers through the shrink and the tensor-core expand: v is an integer
    below 2^16, which its two bf16 halves hold exactly, every product and sum is exact
    in fp32, so y must be the exact value rounded once to bf16."""
    rng = np.random.default_rng(66)
    T, n_adapters, h_in, h_out, r_max = 300, 3, 1024, 392, 16
    p = _small(66, T=T, n_adapters=n_adapters, h_in=h_in, h_out=h_out, r_max=r_max,
               rank_choices=(5, 16))
    p.x[:] = wl.to_bf16_bits(rng.integers(-2, 3, size=p.x.shape).astype(np.float32))
    for a in range(n_adapters):
        r = p.ranks[a]
        p.A[:, a, :, :r] = wl.to_bf16_bits(rng.integers(-2, 3, size=(1, h_in, r)).astype(np.float32))
        p.B[:, a, :r, :] = wl.to_bf16_bits(rng.integers(-2, 3, size=(1, r, h_out)).astype(np.float32))
    p.y_in[:] = wl.to_bf16_bits(rng.integers(-8, 9, size=p.y_in.shape).astype(np.float32))
    p.scales[:] = 0.5
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y)
    torch.cuda.synchronize()
    assert np.array_equal(host_bf16_bits(y), rne_bf16_bits(oracle_apply(p)))


@pytest.mark.parametrize("ws", [None, False], ids=["shrink+tc_expand", "cluster"])
def test_sgmv_prefill_both_paths_sampled_tokens(ws):
    p = wl.sgmv_prefill()
    d = DeviceProblem(p)
    y = d.y_in()
    L.lora_apply(d.x, d.pool, d.seg, y, ws=ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(p.T, size=160, replace=False))
    starts = np.concatenate([[0], np.cumsum(np.bincount(p.ids))])
    rows = np.unique(np.concatenate([rows, starts[:-1], starts[1:] - 1]))
    got = f64(host_bf16_bits(y))[:, rows]
    assert_close(got, oracle_apply(p, rows=rows), TOL_BF16, "sgmv_prefill")
