"""Helpers shared by the GPU parity tests: moving generator output to the
device, running the oracle on the same inputs, and the tolerance check."""
import numpy as np
import torch

import oracle
from adapter_gemm_builder_b200 import lora as L

TOL_BF16 = 2e-2   # max |gpu - oracle| <= TOL * (1 + |oracle|), bf16 inputs, fp32 accumulate
TOL_FP8 = 6e-2    # same form, FP8 base GEMM path


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def f64(t_bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f64(t_bits)


def rne_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, one rounding to nearest even (fp64 -> fp32 is exact for
    the values this is used on: small integers)."""
    return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def assert_close(got: np.ndarray, want: np.ndarray, tol: float, what: str = ""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values in GPU output"
    err = np.abs(got - want)
    bound = tol * (1.0 + np.abs(want))
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu={got[i]!r} oracle={want[i]!r}")


class DeviceProblem:
    """A workloads.LoraProblem on the device plus built segments."""

    def __init__(self, p, build=True):
        self.p = p
        self.x = dev_bf16(p.x)
        self.A = dev_bf16(p.A)
        self.B = dev_bf16(p.B)
        self.ids = dev(p.ids)
        self.ranks = dev(p.ranks)
        self.scales = dev(p.scales)
        self.pool = L.Pool(self.A, self.B, self.ranks, self.scales)
        self.seg = L.Segments(p.T, p.n_adapters)
        if build:
            L.lora_build_segments(self.ids, p.n_adapters, self.seg)

    def y_in(self):
        return dev_bf16(self.p.y_in)


def oracle_apply(p, slices=None, rows=None):
    """fp64 oracle of y_in + s.(x.A).B for every slice (optionally a token subset)."""
    out = []
    for s in (range(p.n_slices) if slices is None else slices):
        x, ids, y_in = p.x[s], p.ids, p.y_in[s]
        if rows is not None:
            x, ids, y_in = x[rows], ids[rows], y_in[rows]
        out.append(oracle.lora_apply(x, p.A[s], p.B[s], p.ranks, p.scales, ids, y_in))
    return np.stack(out)
