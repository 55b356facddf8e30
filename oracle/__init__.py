"""fp64 CPU oracle for the multi-tenant LoRA hot path (ctypes wrapper).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA product
path never imports it, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation); this module
only builds it with gcc, loads it and marshals numpy arrays. Each function
cites the passage of the pages it follows in ``oracle.c``:

* LoRA algebra and the batched output ``Y = X.W + (x_i.A_i.B_i)``:
  Punica README, section "How?".
* Per-token adapter ids in one multi-tenant batch, -1 for none:
  EpiLoRA abstract, sentence 1.
* Token-wise merge of router-selected adapters into the backbone weight:
  LoRA-Switch abstract (shd-paper.top page).
* 4-bit (OCP MX FP4) weights with the LoRA term, bf16 activations:
  EpiLoRA abstract, sentences 2 and 6.
* Gradients of the layer for training adapters on a frozen FP8 base:
  EpiLoRA abstract, sentence 6 (with the Punica README's algebra).
* FP8 base GEMM whose epilogue adds each tenant's up-projection:
  EpiLoRA abstract, sentences 2-4 (8-bit format read as E4M3 with per-row
  scales; that reading is stated in ``oracle.c``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.orc_bf16_decode.restype = ctypes.c_double
            lib.orc_bf16_decode.argtypes = [ctypes.c_uint16]
            lib.orc_e4m3_decode.restype = ctypes.c_double
            lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_encode.restype = ctypes.c_uint8
            lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
            lib.orc_build_segments.restype = None
            lib.orc_build_segments.argtypes = [P, I, I, P, P, P, P, P]
            lib.orc_lora_shrink.restype = None
            lib.orc_lora_shrink.argtypes = [P, I, I, P, I, I, P, P, P]
            lib.orc_lora_expand.restype = None
            lib.orc_lora_expand.argtypes = [P, I, I, P, I, I, P, P, P, P, P]
            lib.orc_lora_apply.restype = None
            lib.orc_lora_apply.argtypes = [P, I, I, I, P, P, I, I, P, P, P, P, P]
            lib.orc_linear_bf16_sampled.restype = None
            lib.orc_linear_bf16_sampled.argtypes = [P, P, I, P, P, I, P]
            lib.orc_quantize_rows.restype = None
            lib.orc_quantize_rows.argtypes = [P, I, I, P, P]
            lib.orc_fp8_gemm_lora_sampled.restype = None
            lib.orc_fp8_gemm_lora_sampled.argtypes = [P, P, P, P, I, P, P, P, I, I, I,
                                                      P, P, P, P, P, I, P]
            lib.orc_lora_switch_merge.restype = None
            lib.orc_lora_switch_merge.argtypes = [P, I, I, P, P, I, I, P, P, P, P, I, P]
            lib.orc_lora_backward.restype = None
            lib.orc_lora_backward.argtypes = [P, P, I, I, I, P, P, P, P, P, P, I, I, P, P, P, P, P, P]
            lib.orc_e2m1_decode.restype = ctypes.c_double
            lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e8m0_decode.restype = ctypes.c_double
            lib.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e2m1_encode.restype = ctypes.c_uint8
            lib.orc_e2m1_encode.argtypes = [ctypes.c_double]
            lib.orc_mxfp4_quantize.restype = None
            lib.orc_mxfp4_quantize.argtypes = [P, I, I, P, P]
            lib.orc_mxfp4_gemm_lora_sampled.restype = None
            lib.orc_mxfp4_gemm_lora_sampled.argtypes = [P, P, P, I, P, P, I, I, I, P, P, P, P, P, I, P]
            lib.orc_w8a16_gemm_lora_sampled.restype = None
            lib.orc_w8a16_gemm_lora_sampled.argtypes = [P, P, P, I, P, P, I, I, I, P, P, P, P, P, I, P]
            lib.orc_num_threads.restype = I
            lib.orc_set_num_threads.argtypes = [I]
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return _load().orc_num_threads()


def set_num_threads(n: int) -> None:
    _load().orc_set_num_threads(int(n))


def bf16_decode(h: int) -> float:
    return _load().orc_bf16_decode(int(h))


def e4m3_decode(c: int) -> float:
    return _load().orc_e4m3_decode(int(c))


def e4m3_encode(f: float) -> int:
    return int(_load().orc_e4m3_encode(float(f)))


_tables = {}


def _table(name, n):
    if name not in _tables:
        f = getattr(_load(), name)
        _tables[name] = np.array([f(i) for i in range(n)], dtype=np.float64)
    return _tables[name]


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Decode an array of bf16 bit patterns (uint16) to fp64 with orc_bf16_decode."""
    flat = np.asarray(a, dtype=np.uint16).ravel()
    return _table("orc_bf16_decode", 65536)[flat].reshape(np.shape(a))


def e4m3_to_f64(a: np.ndarray) -> np.ndarray:
    return _table("orc_e4m3_decode", 256)[np.asarray(a, dtype=np.uint8)]


def build_segments(ids: np.ndarray, n_adapters: int) -> dict:
    """Stable group-by of the tokens by adapter id: perm, indptr, active,
    tok_adapter and counts = [n_valid, n_active, n_bad]."""
    lib = _load()
    ids = _c(ids, np.int32)
    T = ids.shape[0]
    out = dict(
        perm=np.zeros(T, np.int32),
        indptr=np.zeros(n_adapters + 1, np.int32),
        active=np.zeros(n_adapters, np.int32),
        tok_adapter=np.zeros(T, np.int32),
        counts=np.zeros(3, np.int32),
    )
    lib.orc_build_segments(_p(ids), T, n_adapters, _p(out["perm"]), _p(out["indptr"]),
                           _p(out["active"]), _p(out["tok_adapter"]), _p(out["counts"]))
    return out


def lora_shrink(x, A, ranks, ids) -> np.ndarray:
    """x bf16 [T, h_in]; A bf16 [n_adapters, h_in, r_max]; returns v fp64 [T, r_max]."""
    lib = _load()
    x = _c(x, np.uint16); A = _c(A, np.uint16)
    ranks = _c(ranks, np.int32); ids = _c(ids, np.int32)
    T, h_in = x.shape
    n_adapters, _, r_max = A.shape
    v = np.zeros((T, r_max), np.float64)
    lib.orc_lora_shrink(_p(x), T, h_in, _p(A), n_adapters, r_max, _p(ranks), _p(ids), _p(v))
    return v


def lora_expand(v, B, ranks, scales, ids, y_in) -> np.ndarray:
    """v [T, r_max] (any float type, used exactly); B bf16 [n_adapters, r_max, h_out];
    y_in bf16 [T, h_out]; returns y fp64 [T, h_out]."""
    lib = _load()
    v = _c(v, np.float64); B = _c(B, np.uint16)
    ranks = _c(ranks, np.int32); scales = _c(scales, np.float32)
    ids = _c(ids, np.int32); y_in = _c(y_in, np.uint16)
    T, r_max = v.shape
    n_adapters, _, h_out = B.shape
    y = np.zeros((T, h_out), np.float64)
    lib.orc_lora_expand(_p(v), T, r_max, _p(B), n_adapters, h_out, _p(ranks), _p(scales),
                        _p(ids), _p(y_in), _p(y))
    return y


def lora_apply(x, A, B, ranks, scales, ids, y_in) -> np.ndarray:
    lib = _load()
    x = _c(x, np.uint16); A = _c(A, np.uint16); B = _c(B, np.uint16)
    ranks = _c(ranks, np.int32); scales = _c(scales, np.float32)
    ids = _c(ids, np.int32); y_in = _c(y_in, np.uint16)
    T, h_in = x.shape
    n_adapters, _, r_max = A.shape
    h_out = B.shape[2]
    y = np.zeros((T, h_out), np.float64)
    lib.orc_lora_apply(_p(x), T, h_in, h_out, _p(A), _p(B), n_adapters, r_max, _p(ranks),
                       _p(scales), _p(ids), _p(y_in), _p(y))
    return y


def linear_bf16_sampled(x, W, rows, cols) -> np.ndarray:
    lib = _load()
    x = _c(x, np.uint16); W = _c(W, np.uint16)
    rows = _c(rows, np.int32); cols = _c(cols, np.int32)
    out = np.zeros(rows.shape[0], np.float64)
    lib.orc_linear_bf16_sampled(_p(x), _p(W), x.shape[1], _p(rows), _p(cols), rows.shape[0],
                                _p(out))
    return out


def quantize_rows(x):
    """x bf16 [M, K] -> (codes uint8 [M, K], scales fp32 [M])."""
    lib = _load()
    x = _c(x, np.uint16)
    M, K = x.shape
    xq = np.zeros((M, K), np.uint8)
    sx = np.zeros(M, np.float32)
    lib.orc_quantize_rows(_p(x), M, K, _p(xq), _p(sx))
    return xq, sx


def fp8_gemm_lora_sampled(xq, sx, Wq, sw, rows, cols, x=None, A=None, B=None, ranks=None,
                          scales=None, ids=None) -> np.ndarray:
    lib = _load()
    xq = _c(xq, np.uint8); sx = _c(sx, np.float32)
    Wq = _c(Wq, np.uint8); sw = _c(sw, np.float32)
    rows = _c(rows, np.int32); cols = _c(cols, np.int32)
    K = xq.shape[1]
    N = Wq.shape[0]
    if A is not None:
        x = _c(x, np.uint16); A = _c(A, np.uint16); B = _c(B, np.uint16)
        ranks = _c(ranks, np.int32); scales = _c(scales, np.float32); ids = _c(ids, np.int32)
        n_adapters, _, r_max = A.shape
    else:
        n_adapters, r_max = 0, 0
    out = np.zeros(rows.shape[0], np.float64)
    lib.orc_fp8_gemm_lora_sampled(_p(xq), _p(sx), _p(Wq), _p(sw), K, _p(x), _p(A), _p(B),
                                  n_adapters, r_max, N, _p(ranks), _p(scales), _p(ids),
                                  _p(rows), _p(cols), rows.shape[0], _p(out))
    return out


def lora_switch_merge(W, A, B, ranks, scales, sel, gates) -> np.ndarray:
    """W bf16 [N, K]; A bf16 [n_adapters, K, r_max]; B bf16 [n_adapters, r_max, N];
    sel int32 [n_sel] (-1: none); gates fp32 [n_sel]; returns the merged weight fp64 [N, K]."""
    lib = _load()
    W = _c(W, np.uint16); A = _c(A, np.uint16); B = _c(B, np.uint16)
    ranks = _c(ranks, np.int32); scales = _c(scales, np.float32)
    sel = _c(sel, np.int32); gates = _c(gates, np.float32)
    N, K = W.shape
    n_adapters, _, r_max = A.shape
    out = np.zeros((N, K), np.float64)
    lib.orc_lora_switch_merge(_p(W), N, K, _p(A), _p(B), n_adapters, r_max, _p(ranks),
                              _p(scales), _p(sel), _p(gates), sel.shape[0], _p(out))
    return out


def lora_backward(x, dY, A, B, ranks, scales, ids, dYq=None, sd=None, WqT=None, swT=None):
    """x bf16 [M, K]; dY bf16 [M, N]; A bf16 [n_adapters, K, r_max]; B bf16 [n_adapters,
    r_max, N]; optional base term from dYq/sd (dY quantised per token) and WqT/swT (W^T
    quantised per input channel). Returns (dX [M, K], dA [n_ad, K, r_max], dB [n_ad, r_max, N])
    in fp64."""
    lib = _load()
    x = _c(x, np.uint16); dY = _c(dY, np.uint16); A = _c(A, np.uint16); B = _c(B, np.uint16)
    ranks = _c(ranks, np.int32); scales = _c(scales, np.float32); ids = _c(ids, np.int32)
    dYq = _c(dYq, np.uint8); sd = _c(sd, np.float32); WqT = _c(WqT, np.uint8); swT = _c(swT, np.float32)
    M, K = x.shape
    N = dY.shape[1]
    n_adapters, _, r_max = A.shape
    dX = np.zeros((M, K), np.float64)
    dA = np.zeros((n_adapters, K, r_max), np.float64)
    dB = np.zeros((n_adapters, r_max, N), np.float64)
    lib.orc_lora_backward(_p(x), _p(dY), M, K, N, _p(dYq), _p(sd), _p(WqT), _p(swT), _p(A), _p(B),
                          n_adapters, r_max, _p(ranks), _p(scales), _p(ids), _p(dX), _p(dA), _p(dB))
    return dX, dA, dB


def e2m1_decode(c: int) -> float:
    return _load().orc_e2m1_decode(int(c))


def e8m0_decode(e: int) -> float:
    return _load().orc_e8m0_decode(int(e))


def e2m1_encode(f: float) -> int:
    return int(_load().orc_e2m1_encode(float(f)))


def mxfp4_quantize(W):
    """W bf16 [N, K] (K % 32 == 0) -> (codes uint8 [N, K], one E2M1 code per byte;
    scales uint8 [N, K / 32], E8M0)."""
    lib = _load()
    W = _c(W, np.uint16)
    N, K = W.shape
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((N, K // 32), np.uint8)
    lib.orc_mxfp4_quantize(_p(W), N, K, _p(codes), _p(scales))
    return codes, scales


def mxfp4_gemm_lora_sampled(x, codes, scales, rows, cols, A=None, B=None, ranks=None,
                            scales_lora=None, ids=None) -> np.ndarray:
    lib = _load()
    x = _c(x, np.uint16); codes = _c(codes, np.uint8); scales = _c(scales, np.uint8)
    rows = _c(rows, np.int32); cols = _c(cols, np.int32)
    K = x.shape[1]
    N = codes.shape[0]
    if A is not None:
        A = _c(A, np.uint16); B = _c(B, np.uint16); ranks = _c(ranks, np.int32)
        scales_lora = _c(scales_lora, np.float32); ids = _c(ids, np.int32)
        n_adapters, _, r_max = A.shape
    else:
        n_adapters, r_max = 0, 0
    out = np.zeros(rows.shape[0], np.float64)
    lib.orc_mxfp4_gemm_lora_sampled(_p(x), _p(codes), _p(scales), K, _p(A), _p(B), n_adapters, r_max,
                                    N, _p(ranks), _p(scales_lora), _p(ids), _p(rows), _p(cols),
                                    rows.shape[0], _p(out))
    return out


def w8a16_gemm_lora_sampled(x, Wq, sw, rows, cols, A=None, B=None, ranks=None, scales=None,
                            ids=None) -> np.ndarray:
    """y = sw . (x . E4M3(Wq)^T) + LoRA with bf16 x (W8A16), at the (rows, cols) samples."""
    lib = _load()
    x = _c(x, np.uint16); Wq = _c(Wq, np.uint8); sw = _c(sw, np.float32)
    rows = _c(rows, np.int32); cols = _c(cols, np.int32)
    K = x.shape[1]
    N = Wq.shape[0]
    if A is not None:
        A = _c(A, np.uint16); B = _c(B, np.uint16); ranks = _c(ranks, np.int32)
        scales = _c(scales, np.float32); ids = _c(ids, np.int32)
        n_adapters, _, r_max = A.shape
    else:
        n_adapters, r_max = 0, 0
    out = np.zeros(rows.shape[0], np.float64)
    lib.orc_w8a16_gemm_lora_sampled(_p(x), _p(Wq), _p(sw), K, _p(A), _p(B), n_adapters, r_max, N,
                                    _p(ranks), _p(scales), _p(ids), _p(rows), _p(cols), rows.shape[0],
                                    _p(out))
    return out
