"""The FP8 GEMM + LoRA epilogue entry point that allocates nothing.

Some callers cannot allocate device memory (a plugin inside a serving engine
that plans all memory itself, or a hot path that must not call cudaMalloc),
so they cannot pass the workspace that fp8_gemm_lora_epilogue needs.
fp8_gemm_lora_epilogue_noalloc keeps that scratch space inside the library.
This test calls it through the C ABI twice in a row and checks each result
against the workspace entry point on the same inputs, within the FP8 path's
tolerance. The file is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

from adapter_gemm_builder_b200 import lora as L
from adapter_gemm_builder_b200 import workloads as wl
from gpu_util import TOL_FP8, assert_close, dev, dev_bf16, f64, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    L.load()


def _inputs(M=96, K=1024, N=640, n_adapters=6, r=16, seed=12):
    rng = np.random.default_rng(seed)
    p = wl.fp8_problem(M, K=K, N=N, n_adapters=n_adapters, r=r, seed=seed, ids_kind="zipf",
                       none_frac=0.1, W=wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K)))
    x = dev_bf16(p.x)
    Wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    L.fp8_quantize_rows(dev_bf16(p.W), Wq, sw)
    pool = L.Pool(dev_bf16(p.A), dev_bf16(p.B), dev(p.ranks), dev(p.scales))
    seg = L.Segments(M, n_adapters)
    L.lora_build_segments(dev(p.ids), n_adapters, seg)
    return x, Wq, sw, pool, seg


def test_noalloc_matches_workspace_entry_point_twice():
    x, Wq, sw, pool, seg = _inputs()
    M, N = x.shape[0], Wq.shape[0]
    ws = L.workspace(L.LORA_OP_FP8_GEMM, M, x.shape[1], pool)
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    L.fp8_gemm_lora_epilogue(x, Wq, sw, pool, seg, y_ref, ws)
    torch.cuda.synchronize()
    want = f64(host_bf16_bits(y_ref))
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.fp8_gemm_lora_epilogue_noalloc(x, Wq, sw, pool, seg, y)
        torch.cuda.synchronize()
        assert_close(f64(host_bf16_bits(y)), want, TOL_FP8, "no-alloc entry point")


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
