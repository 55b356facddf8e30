"""ctypes binding of ``liblora.so`` (declared in ``include/lora.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. torch supplies device memory and the current stream. If the library
has not been built, every call raises :class:`LoraLibraryMissing` -- there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblora.so")

LORA_OK = 0
LORA_ERR_INVALID_ARG = 1
LORA_ERR_UNSUPPORTED = 2
LORA_ERR_BAD_ADAPTER_ID = 3
LORA_ERR_CUDA = 4
LORA_ERR_WORKSPACE = 5
LORA_ERR_TIMEOUT = 6

LORA_OP_SHRINK = 0
LORA_OP_EXPAND = 1
LORA_OP_APPLY = 2
LORA_OP_FP8_GEMM = 3
LORA_OP_BF16_GEMM = 4
LORA_OP_FP8_BACKWARD = 5
LORA_OP_MXFP4_GEMM = 6
LORA_OP_W8A16_GEMM = 7

EXPORTED = [
    "lora_workspace_size", "lora_workspace_init", "lora_workspace_status", "lora_build_segments",
    "lora_shrink", "lora_expand", "lora_apply", "fp8_quantize_rows", "fp8_gemm_lora_epilogue",
    "lora_status_string", "lora_version", "lora_tile_tokens", "lora_tile_tokens_for", "lora_max_tiles",
    "lora_segments_status", "fp8_gemm_lora_epilogue_noalloc", "lora_noalloc_scratch_bytes",
    "lora_noalloc_status", "lora_debug_set_wait_limit", "bf16_gemm_lora_epilogue",
    "lora_switch_merge", "fp8_lora_backward", "mxfp4_quantize_rows", "mxfp4_gemm_lora_epilogue",
    "w8a16_gemm_lora_epilogue",
]


class LoraLibraryMissing(RuntimeError):
    pass


class LoraError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


class lora_pool_t(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("ranks", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("n_slices", ctypes.c_int32),
                ("n_adapters", ctypes.c_int32), ("h_in", ctypes.c_int32),
                ("h_out", ctypes.c_int32), ("r_max", ctypes.c_int32)]


class lora_segments_t(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("indptr", ctypes.c_void_p),
                ("active", ctypes.c_void_p), ("tiles", ctypes.c_void_p),
                ("tok_adapter", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("T", ctypes.c_int32), ("n_adapters", ctypes.c_int32)]


_lib = None
_lock = threading.Lock()


def load(path: str = LIB_PATH):
    """Load liblora.so; raises LoraLibraryMissing if it was not built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise LoraLibraryMissing(
                f"{path} not found: build it with `python -m adapter_gemm_builder_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        I64 = ctypes.c_int64
        sig = {
            "lora_workspace_size": (Z, [I, I, I, P]),
            "lora_workspace_init": (I, [P, Z, P]),
            "lora_workspace_status": (I, [P, Z, P, P]),
            "lora_build_segments": (I, [P, I, I, P, I, P]),
            "lora_shrink": (I, [P, I64, P, P, P, P, Z, P]),
            "lora_expand": (I, [P, P, P, P, P, Z, P]),
            "lora_apply": (I, [P, I64, P, P, P, P, Z, P]),
            "fp8_quantize_rows": (I, [P, I, I, P, P, P]),
            "fp8_gemm_lora_epilogue": (I, [P, I, I, I, P, P, P, P, P, P, Z, P]),
            "lora_status_string": (ctypes.c_char_p, [I]),
            "lora_version": (I, []),
            "lora_tile_tokens": (I, []),
            "lora_tile_tokens_for": (I, [I, I]),
            "lora_max_tiles": (I, [I, I]),
            "lora_segments_status": (I, [P, P, P]),
            "fp8_gemm_lora_epilogue_noalloc": (I, [P, I, I, I, P, P, P, P, P, P]),
            "lora_noalloc_scratch_bytes": (Z, []),
            "lora_noalloc_status": (I, [P, P]),
            "lora_debug_set_wait_limit": (I, [ctypes.c_uint64, I]),
            "bf16_gemm_lora_epilogue": (I, [P, I, I, I, P, P, P, P, P, Z, P]),
            "lora_switch_merge": (I, [P, I, I, P, P, P, I, P, P]),
            "fp8_lora_backward": (I, [P, P, I, I, I, P, P, P, P, P, P, P, P, Z, P]),
            "mxfp4_quantize_rows": (I, [P, I, I, P, P, P]),
            "mxfp4_gemm_lora_epilogue": (I, [P, I, I, I, P, P, P, P, P, P, Z, P]),
            "w8a16_gemm_lora_epilogue": (I, [P, I, I, I, P, P, P, P, P, P, Z, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
        return lib


def _check(status: int):
    if status != LORA_OK:
        msg = load().lora_status_string(status).decode()
        raise LoraError(status, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def tile_tokens() -> int:
    return load().lora_tile_tokens()


def tile_tokens_for(T: int, n_adapters: int) -> int:
    """Tokens per row of Segments.tiles for this batch (lora_tile_tokens_for)."""
    return load().lora_tile_tokens_for(T, n_adapters)


def max_tiles(T: int, n_adapters: int) -> int:
    """Rows of Segments.tiles (lora_max_tiles)."""
    return load().lora_max_tiles(T, n_adapters)


class Pool:
    """A stacked adapter pool on the device (see lora_pool_t).

    A: bf16 [n_slices, n_adapters, h_in, r_max]; B: bf16 [n_slices, n_adapters, r_max, h_out];
    ranks: int32 [n_adapters] or None; scales: fp32 [n_adapters] or None."""

    def __init__(self, A: torch.Tensor, B: torch.Tensor, ranks=None, scales=None):
        if A.dim() == 3:
            A = A.unsqueeze(0)
        if B.dim() == 3:
            B = B.unsqueeze(0)
        self.A, self.B, self.ranks, self.scales = A, B, ranks, scales
        n_slices, n_adapters, h_in, r_max = A.shape
        self.c = lora_pool_t(A.data_ptr(), B.data_ptr(),
                             ranks.data_ptr() if ranks is not None else None,
                             scales.data_ptr() if scales is not None else None,
                             n_slices, n_adapters, h_in, B.shape[3], r_max)

    @property
    def n_adapters(self): return self.c.n_adapters


class Segments:
    """Device buffers for lora_build_segments' output (see lora_segments_t)."""

    def __init__(self, T: int, n_adapters: int, device="cuda"):
        i32 = dict(dtype=torch.int32, device=device)
        self.perm = torch.empty(max(T, 1), **i32)
        self.indptr = torch.empty(n_adapters + 1, **i32)
        self.active = torch.empty(n_adapters, **i32)
        self.tiles = torch.empty((max(max_tiles(T, n_adapters), 1), 4), **i32)
        self.tok_adapter = torch.empty(max(T, 1), **i32)
        self.counts = torch.zeros(8, **i32)
        self.c = lora_segments_t(self.perm.data_ptr(), self.indptr.data_ptr(),
                                 self.active.data_ptr(), self.tiles.data_ptr(),
                                 self.tok_adapter.data_ptr(), self.counts.data_ptr(), T,
                                 n_adapters)

    @property
    def T(self): return self.c.T


def lora_workspace_size(op: int, T: int, K: int = 0, pool: Pool | None = None) -> int:
    n = load().lora_workspace_size(op, T, K, ctypes.byref(pool.c) if pool else None)
    if n == ctypes.c_size_t(-1).value:
        raise LoraError(LORA_ERR_INVALID_ARG, "invalid workspace query")
    return n


def workspace(op: int, T: int, K: int = 0, pool: Pool | None = None, device="cuda",
              stream=None) -> torch.Tensor:
    """Allocate and zero a workspace for `op` (torch memory, caller-owned)."""
    n = lora_workspace_size(op, T, K, pool)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    _check(load().lora_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))
    return ws


def lora_workspace_status(ws: torch.Tensor, stream=None) -> tuple[int, int]:
    detail = ctypes.c_uint32(0)
    st = load().lora_workspace_status(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(detail))
    return st, detail.value


def lora_segments_status(seg: "Segments", stream=None) -> tuple[int, int]:
    detail = ctypes.c_uint32(0)
    st = load().lora_segments_status(ctypes.byref(seg.c), _stream(stream), ctypes.byref(detail))
    return st, detail.value


def lora_build_segments(ids: torch.Tensor, n_adapters: int, seg: Segments, sync_check=False,
                        stream=None) -> None:
    T = ids.numel()
    _check(load().lora_build_segments(_ptr(ids) if T else None, T, n_adapters,
                                      ctypes.byref(seg.c), 1 if sync_check else 0,
                                      _stream(stream)))


def _slice_stride(x, pool):
    if x.dim() == 2:
        return 0
    return x.stride(0) if x.shape[0] > 1 else 0


def lora_shrink(x: torch.Tensor, pool: Pool, seg: Segments, v: torch.Tensor, stream=None,
                x_slice_stride: int | None = None) -> None:
    xs = _slice_stride(x, pool) if x_slice_stride is None else x_slice_stride
    _check(load().lora_shrink(_ptr(x), xs, ctypes.byref(pool.c), ctypes.byref(seg.c), _ptr(v),
                              None, 0, _stream(stream)))


def lora_expand(v: torch.Tensor, pool: Pool, seg: Segments, y: torch.Tensor, stream=None) -> None:
    _check(load().lora_expand(_ptr(v), ctypes.byref(pool.c), ctypes.byref(seg.c), _ptr(y), None, 0,
                              _stream(stream)))


def lora_apply(x: torch.Tensor, pool: Pool, seg: Segments, y: torch.Tensor, stream=None,
               x_slice_stride: int | None = None, ws: torch.Tensor | None | bool = None) -> None:
    """y += s_a (x.A_a).B_a; ws: a workspace of lora_workspace_size(LORA_OP_APPLY, T, 0, pool)
    bytes (allocated here when None and the size is not 0; False: none). A batch of long
    segments uses it for the tensor-core shrink's planes of v, then the tensor-core expand;
    another general batch, for its tile rows in cost order. Without one, one launch of the
    cluster kernel, rows in table order."""
    xs = _slice_stride(x, pool) if x_slice_stride is None else x_slice_stride
    if ws is False:  # explicitly none: the tile rows run in table order
        ws = None
    elif ws is None:
        n = lora_workspace_size(LORA_OP_APPLY, seg.T, 0, pool)
        ws = workspace(LORA_OP_APPLY, seg.T, 0, pool, device=y.device, stream=stream) if n else None
    _check(load().lora_apply(_ptr(x), xs, ctypes.byref(pool.c), ctypes.byref(seg.c), _ptr(y),
                             _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def fp8_quantize_rows(x: torch.Tensor, xq: torch.Tensor, sx: torch.Tensor, stream=None) -> None:
    M, K = x.shape
    _check(load().fp8_quantize_rows(_ptr(x), M, K, _ptr(xq), _ptr(sx), _stream(stream)))


def fp8_gemm_lora_epilogue(x: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                           pool: Pool | None, seg: Segments | None, y: torch.Tensor,
                           ws: torch.Tensor, stream=None) -> None:
    M, K = x.shape
    N = Wq.shape[0]
    _check(load().fp8_gemm_lora_epilogue(
        _ptr(x), M, K, N, _ptr(Wq), _ptr(w_scale), ctypes.byref(pool.c) if pool else None,
        ctypes.byref(seg.c) if seg else None, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))


def bf16_gemm_lora_epilogue(x: torch.Tensor, W: torch.Tensor, pool: Pool | None,
                            seg: Segments | None, y: torch.Tensor, ws: torch.Tensor,
                            stream=None) -> None:
    """y = x.W^T + s_a (x.A_a).B_a with bf16 operands (x [M, K], W [N, K])."""
    M, K = x.shape
    N = W.shape[0]
    _check(load().bf16_gemm_lora_epilogue(
        _ptr(x), M, K, N, _ptr(W), ctypes.byref(pool.c) if pool else None,
        ctypes.byref(seg.c) if seg else None, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))


def w8a16_gemm_lora_epilogue(x: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                             pool: Pool | None, seg: Segments | None, y: torch.Tensor, ws: torch.Tensor,
                             stream=None) -> None:
    """y = w_scale . (x . E4M3(Wq)^T) + s_a (x.A_a).B_a with bf16 x (W8A16)."""
    M, K = x.shape
    N = Wq.shape[0]
    _check(load().w8a16_gemm_lora_epilogue(
        _ptr(x), M, K, N, _ptr(Wq), _ptr(w_scale), ctypes.byref(pool.c) if pool else None,
        ctypes.byref(seg.c) if seg else None, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))


def mxfp4_code_bytes(N: int, K: int) -> int:
    """Bytes of the packed E2M1 codes of an [N, K] MX FP4 weight (128 x 64 tiles)."""
    return (N + 127) // 128 * 128 * (K // 2)


def mxfp4_scale_bytes(N: int, K: int) -> int:
    """Bytes of the E8M0 scale array of an [N, K] MX FP4 weight (rows padded to 128)."""
    return (N + 127) // 128 * 128 * (K // 32)


def mxfp4_quantize_rows(W: torch.Tensor, Wp: torch.Tensor, Wsc: torch.Tensor, stream=None) -> None:
    N, K = W.shape
    _check(load().mxfp4_quantize_rows(_ptr(W), N, K, _ptr(Wp), _ptr(Wsc), _stream(stream)))


def mxfp4_gemm_lora_epilogue(x: torch.Tensor, Wp: torch.Tensor, Wsc: torch.Tensor, pool: Pool | None,
                             seg: Segments | None, y: torch.Tensor, ws: torch.Tensor,
                             stream=None) -> None:
    """y = x.W^T + s_a (x.A_a).B_a with W in MX FP4 (Wp, Wsc as mxfp4_quantize_rows makes
    them; N = the weight's rows, read from y) and bf16 x."""
    M, K = x.shape
    N = y.shape[1]
    _check(load().mxfp4_gemm_lora_epilogue(
        _ptr(x), M, K, N, _ptr(Wp), _ptr(Wsc), ctypes.byref(pool.c) if pool else None,
        ctypes.byref(seg.c) if seg else None, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))


def fp8_lora_backward(x: torch.Tensor, dY: torch.Tensor, WqT: torch.Tensor, swT: torch.Tensor,
                      pool: Pool, seg: Segments, dX: torch.Tensor, dA: torch.Tensor, dB: torch.Tensor,
                      ws: torch.Tensor, stream=None) -> None:
    """Gradients of y = x.W^T + s_a (x.A_a).B_a on a frozen FP8 base (see fp8_lora_backward)."""
    M, K = x.shape
    N = dY.shape[1]
    _check(load().fp8_lora_backward(_ptr(x), _ptr(dY), M, K, N, _ptr(WqT), _ptr(swT),
                                    ctypes.byref(pool.c), ctypes.byref(seg.c), _ptr(dX), _ptr(dA),
                                    _ptr(dB), _ptr(ws), ws.numel(), _stream(stream)))


def lora_switch_merge(W: torch.Tensor, pool: Pool, sel: torch.Tensor, gates: torch.Tensor,
                      W_out: torch.Tensor, stream=None) -> None:
    """W_out = W + sum_e gates[e] s_a (A_a B_a)^T over the selected adapters (device sel/gates)."""
    N, K = W.shape
    _check(load().lora_switch_merge(_ptr(W), N, K, ctypes.byref(pool.c), _ptr(sel), _ptr(gates),
                                    sel.numel(), _ptr(W_out), _stream(stream)))


def fp8_gemm_lora_epilogue_noalloc(x: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                                   pool: Pool | None, seg: Segments | None, y: torch.Tensor,
                                   stream=None) -> None:
    """fp8_gemm_lora_epilogue without a caller workspace (scratch inside the library)."""
    M, K = x.shape
    N = Wq.shape[0]
    _check(load().fp8_gemm_lora_epilogue_noalloc(
        _ptr(x), M, K, N, _ptr(Wq), _ptr(w_scale), ctypes.byref(pool.c) if pool else None,
        ctypes.byref(seg.c) if seg else None, _ptr(y), _stream(stream)))


def lora_noalloc_status(stream=None) -> tuple[int, int]:
    """Read and clear the status word of the no-alloc entry point's scratch array."""
    detail = ctypes.c_uint32(0)
    st = load().lora_noalloc_status(_stream(stream), ctypes.byref(detail))
    return st, detail.value


def lora_debug_set_wait_limit(limit_ns: int, inject_stall: bool = False) -> None:
    """Test hook: limit of the kernels' bounded waits (0 = default 2 s) and the stall
    that makes one CTA of each later launch run out its wait."""
    _check(load().lora_debug_set_wait_limit(int(limit_ns), 1 if inject_stall else 0))
