"""Thin Python binding of the C ABI in ``include/psa.h`` (``libpsa.so``).

Argument marshalling only: every step runs in the library's CUDA kernels.
Each function has the name of the C entry point it calls.  Tensors are
PyTorch CUDA tensors (PyTorch is used for device memory and streams); the
call is issued with the device of its main tensor current, on that device's
``torch.cuda.current_stream()`` unless a stream is given.
A non-zero status raises :class:`PSAError`.  There is no fallback: if the
library is missing, :func:`lib` raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsa.so")

PSA_OK = 0
PSA_ERR_ARG = 1
PSA_ERR_SHAPE = 2
PSA_ERR_UNSUPPORTED = 3
PSA_ERR_CAPACITY = 4
PSA_ERR_CUDA = 5
PSA_ERR_TIMEOUT = 6
PSA_ERR_CSR = 7
PSA_ERR_DEVICE = 8

EXPORTS = ("psa_status_string", "psa_version", "psa_workspace_size", "psa_route_capacity", "psa_pool",
           "psa_route_topk", "psa_route_thresh", "psa_attn", "psa_dense", "psa_read_status",
           "psa_attn_noalloc", "psa_route_thresh_prob", "psa_test_stall_next_attn",
           "psa_read_fixup_count", "psa_hyd_stat", "psa_attn_hyd", "psa_attn_bwd")

_lib = None


class PSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: status {status}: {status_text(status)}")


def _declare(L: ctypes.CDLL) -> None:
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "psa_status_string": (ctypes.c_char_p, [I]),
        "psa_version": (I, []),
        "psa_workspace_size": (Z, [I, I, I, I]),
        "psa_route_capacity": (Z, [I, I, I, I]),
        "psa_pool": (I, [P, P, P, I, I, I, I, I, P, P, P, P]),
        "psa_route_topk": (I, [P, P, I, I, I, I, F, I, P, P, Z, P, P, P, Z, P]),
        "psa_route_thresh": (I, [P, P, I, I, I, I, F, I, I, P, P, Z, P, P, P, Z, P]),
        "psa_route_thresh_prob": (I, [P, P, I, I, I, I, F, I, I, P, P, Z, P, P, P, Z, P]),
        "psa_attn": (I, [P, P, P, P, P, P, P, Z, P, I, I, I, I, I, I, P, P, P, Z, P]),
        "psa_dense": (I, [P, P, P, I, I, I, I, I, P, P, P, Z, P]),
        "psa_read_status": (I, [P, ctypes.POINTER(I), P]),
        "psa_read_fixup_count": (I, [P, ctypes.POINTER(I), ctypes.POINTER(I), P]),
        "psa_hyd_stat": (I, [P, P, P, P, I, I, I, I, P, P, Z, P]),
        "psa_attn_bwd": (I, [P, P, P, P, P, P, P, Z, I, I, I, I, I, I, P, P, P, P, P, P, P, Z, P]),
        "psa_attn_hyd": (I, [P, P, P, P, P, P, P, P, Z, P, I, I, I, I, I, I, P, P, P, Z, P]),
        "psa_test_stall_next_attn": (I, [I]),
        "psa_attn_noalloc": (I, [P, P, P, P, P, P, P, Z, P, I, I, I, I, I, I, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m block_sparse_attention_psa_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _lib = L
    return _lib


def status_text(status: int) -> str:
    return lib().psa_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != PSA_OK:
        raise PSAError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, like):
    """The caller's stream, else the current stream of the problem's device."""
    s = stream if stream is not None else torch.cuda.current_stream(like.device)
    return ctypes.c_void_p(s.cuda_stream)


def _call(fn: str, like, *args) -> None:
    """Call the C entry point with the device of ``like`` (the problem's main
    tensor) current: the library launches on the current device and sizes its
    TMA descriptors and scratch for it, so the tensors' device must be the
    current one (the library itself refuses a mismatch with PSA_ERR_DEVICE)."""
    with torch.cuda.device(like.device):
        status = getattr(lib(), fn)(*args)
    _check(fn, status)


def _shape(q):
    if q.dim() != 4 or q.dtype != torch.bfloat16:
        raise ValueError("q, k, v must be bf16 [B, H, N, d]")
    return tuple(int(x) for x in q.shape)


def _expect(name, t, like=None, shape=None, dtype=None, min_numel=None):
    """The C ABI takes plain pointers sized from the problem's dimensions, so
    every tensor is checked against them here, before any pointer is passed:
    a smaller or differently typed buffer would be read or written past its
    end on the device."""
    if t is None:
        return
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} needs at least {min_numel} elements, has {t.numel()}")
    if like is not None and t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, the problem on {like.device}")


def _expect_qkv(q, k, v):
    B, H, N, d = _shape(q)
    _expect("k", k, q, (B, H, N, d), torch.bfloat16)
    _expect("v", v, q, (B, H, N, d), torch.bfloat16)
    return B, H, N, d


def _expect_ws(ws, q, B, H, N, d):
    _expect("ws", ws, q, dtype=torch.uint8, min_numel=psa_workspace_size(B, H, N, d))


def _expect_route_out(out, q, BH, M):
    row_ptr, col_idx, nnz, row_max = out
    _expect("row_ptr", row_ptr, q, dtype=torch.int32, min_numel=BH * M + 1)
    _expect("col_idx", col_idx, q, dtype=torch.int32, min_numel=1)
    _expect("nnz", nnz, q, dtype=torch.int32, min_numel=1)
    _expect("row_max", row_max, q, dtype=torch.float32, min_numel=BH * M)


def psa_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib().psa_workspace_size(B, H, N, d))


def psa_route_capacity(B: int, H: int, M: int, causal: bool) -> int:
    return int(lib().psa_route_capacity(B, H, M, int(causal)))


def workspace(B: int, H: int, N: int, d: int, device=None) -> torch.Tensor:
    """A device workspace of psa_workspace_size bytes (256-byte aligned)."""
    n = psa_workspace_size(B, H, N, d)
    if n == 0:
        raise PSAError("psa_workspace_size", PSA_ERR_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def psa_pool(q, k, v, block_size: int = 64, out=None, stream=None):
    """Returns (qbar, kbar, vsum) float32 [B, H, M, d]."""
    B, H, N, d = _expect_qkv(q, k, v)
    M = N // block_size if block_size > 0 else 0
    if out is None:
        out = tuple(torch.empty(B, H, M, d, dtype=torch.float32, device=q.device) for _ in range(3))
    qbar, kbar, vsum = out
    for name, t in (("qbar", qbar), ("kbar", kbar), ("vsum", vsum)):
        _expect(name, t, q, (B, H, M, d), torch.float32)
    _call("psa_pool", q, _ptr(q), _ptr(k), _ptr(v), B, H, N, d, block_size,
          _ptr(qbar), _ptr(kbar), _ptr(vsum), _stream(stream, q))
    return qbar, kbar, vsum


def _expect_stats(qbar, kbar):
    if qbar.dim() != 4 or qbar.dtype != torch.float32:
        raise ValueError("qbar, kbar must be float32 [B, H, M, d]")
    _expect("kbar", kbar, qbar, tuple(qbar.shape), torch.float32)
    return tuple(int(x) for x in qbar.shape)


def _route_out(B, H, M, causal, capacity, device):
    cap = capacity if capacity is not None else psa_route_capacity(B, H, M, causal)
    return (torch.empty(B * H * M + 1, dtype=torch.int32, device=device),
            torch.empty(max(cap, 1), dtype=torch.int32, device=device),
            torch.empty(1, dtype=torch.int32, device=device),
            torch.empty(B * H * M, dtype=torch.float32, device=device))


def psa_route_topk(qbar, kbar, density: float, causal: bool = False, capacity: int | None = None,
                   out=None, ws=None, stream=None):
    """Returns (row_ptr, col_idx, nnz, row_max): device int32 tensors (nnz has
    one element) and the float32 row maxima of the block scores (``out`` may
    give row_max as None to skip it)."""
    B, H, M, d = _expect_stats(qbar, kbar)
    if ws is None:
        ws = workspace(B, H, M * 64, d, qbar.device)
    if out is None:
        out = _route_out(B, H, M, causal, capacity, qbar.device)
    _expect_ws(ws, qbar, B, H, M * 64, d)
    _expect_route_out(out, qbar, B * H, M)
    row_ptr, col_idx, nnz, row_max = out
    _call("psa_route_topk", qbar, _ptr(qbar), _ptr(kbar), B, H, M, d, float(density), int(causal),
          _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(nnz), _ptr(row_max), _ptr(ws), ws.numel(),
          _stream(stream, qbar))
    return row_ptr, col_idx, nnz, row_max


def psa_route_thresh(qbar, kbar, alpha: float, causal: bool = False, keep_first: bool = False,
                     ws=None, capacity: int | None = None, out=None, stream=None):
    """Returns (row_ptr, col_idx, nnz, row_max); nnz > col_idx.numel() means truncated."""
    B, H, M, d = _expect_stats(qbar, kbar)
    if ws is None:
        ws = workspace(B, H, M * 64, d, qbar.device)
    if out is None:
        out = _route_out(B, H, M, causal, capacity, qbar.device)
    _expect_ws(ws, qbar, B, H, M * 64, d)
    _expect_route_out(out, qbar, B * H, M)
    row_ptr, col_idx, nnz, row_max = out
    _call("psa_route_thresh", qbar, _ptr(qbar), _ptr(kbar), B, H, M, d, float(alpha), int(causal),
          int(keep_first), _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(nnz), _ptr(row_max), _ptr(ws),
          ws.numel(), _stream(stream, qbar))
    return row_ptr, col_idx, nnz, row_max


def psa_route_thresh_prob(qbar, kbar, alpha: float, causal: bool = False, keep_first: bool = False,
                          ws=None, capacity: int | None = None, out=None, stream=None):
    """Threshold routing in the probability domain: keep J iff
    s_IJ >= max_J s_IJ + ln(alpha).  Returns (row_ptr, col_idx, nnz, row_max)."""
    B, H, M, d = _expect_stats(qbar, kbar)
    if ws is None:
        ws = workspace(B, H, M * 64, d, qbar.device)
    if out is None:
        out = _route_out(B, H, M, causal, capacity, qbar.device)
    _expect_ws(ws, qbar, B, H, M * 64, d)
    _expect_route_out(out, qbar, B * H, M)
    row_ptr, col_idx, nnz, row_max = out
    _call("psa_route_thresh_prob", qbar, _ptr(qbar), _ptr(kbar), B, H, M, d, float(alpha), int(causal),
          int(keep_first), _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(nnz), _ptr(row_max), _ptr(ws),
          ws.numel(), _stream(stream, qbar))
    return row_ptr, col_idx, nnz, row_max


def _expect_attn_inputs(q, kbar, vsum, row_ptr, col_idx, row_max, B, H, M, d):
    _expect("kbar", kbar, q, (B, H, M, d), torch.float32)
    _expect("vsum", vsum, q, (B, H, M, d), torch.float32)
    _expect("row_ptr", row_ptr, q, dtype=torch.int32, min_numel=B * H * M + 1)
    _expect("col_idx", col_idx, q, dtype=torch.int32, min_numel=1)
    _expect("row_max", row_max, q, dtype=torch.float32, min_numel=B * H * M)


def psa_attn(q, k, v, kbar, vsum, row_ptr, col_idx, causal: bool = False, block_size: int = 64,
             ws=None, out=None, lse=None, want_lse: bool = False, row_max=None, stream=None):
    """Returns out (bf16 [B,H,N,d]) and, if requested, lse (float32 [B,H,N]).
    ``row_max`` (optional) is a router's row maxima, used as the softmax
    stabiliser instead of computing it in the kernel."""
    B, H, N, d = _expect_qkv(q, k, v)
    M = N // block_size if block_size > 0 else 0
    _expect_attn_inputs(q, kbar, vsum, row_ptr, col_idx, row_max, B, H, M, d)
    if ws is None:
        ws = workspace(B, H, N, d, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _expect_ws(ws, q, B, H, N, d)
    _expect("out", out, q, (B, H, N, d), torch.bfloat16)
    _expect("lse", lse, q, (B, H, N), torch.float32)
    _call("psa_attn", q, _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), _ptr(row_ptr), _ptr(col_idx),
          col_idx.numel(), _ptr(row_max), B, H, N, d, block_size, int(causal), _ptr(out), _ptr(lse), _ptr(ws),
          ws.numel(), _stream(stream, q))
    return (out, lse) if lse is not None else out


def psa_hyd_stat(k, v, kbar, vsum, ws=None, out=None, stream=None):
    """The first-order correction's global statistic: float32 [B, H, d, d],
    the mean over a head's blocks of sum_j (k_j - kbar_J) v_j^T."""
    B, H, N, d = _expect_qkv(k, v, v)
    M = N // 64
    _expect("kbar", kbar, k, (B, H, M, d), torch.float32)
    _expect("vsum", vsum, k, (B, H, M, d), torch.float32)
    if ws is None:
        ws = workspace(B, H, N, d, k.device)
    if out is None:
        out = torch.empty(B, H, d, d, dtype=torch.float32, device=k.device)
    _expect_ws(ws, k, B, H, N, d)
    _expect("hstat", out, k, (B, H, d, d), torch.float32)
    _call("psa_hyd_stat", k, _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), B, H, N, d, _ptr(out), _ptr(ws),
          ws.numel(), _stream(stream, k))
    return out


def psa_attn_hyd(q, k, v, kbar, vsum, hstat, row_ptr, col_idx, causal: bool = False, block_size: int = 64,
                 ws=None, out=None, lse=None, want_lse: bool = False, row_max=None, stream=None):
    """psa_attn plus the first-order term of the unselected blocks with the
    global statistic ``hstat`` (float32 [B, H, d, d], from psa_hyd_stat)."""
    B, H, N, d = _expect_qkv(q, k, v)
    M = N // block_size if block_size > 0 else 0
    _expect_attn_inputs(q, kbar, vsum, row_ptr, col_idx, row_max, B, H, M, d)
    _expect("hstat", hstat, q, (B, H, d, d), torch.float32)
    if ws is None:
        ws = workspace(B, H, N, d, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _expect_ws(ws, q, B, H, N, d)
    _expect("out", out, q, (B, H, N, d), torch.bfloat16)
    _expect("lse", lse, q, (B, H, N), torch.float32)
    _call("psa_attn_hyd", q, _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), _ptr(hstat), _ptr(row_ptr),
          _ptr(col_idx), col_idx.numel(), _ptr(row_max), B, H, N, d, block_size, int(causal), _ptr(out),
          _ptr(lse), _ptr(ws), ws.numel(), _stream(stream, q))
    return (out, lse) if lse is not None else out


def psa_attn_bwd(q, k, v, kbar, vsum, row_ptr, col_idx, out, lse, dout, causal: bool = False,
                 block_size: int = 64, ws=None, grads=None, stream=None):
    """Gradients (dq, dk, dv), bf16 [B, H, N, d], of the 0th-order attention
    of psa_attn for fixed block lists, given its output ``out``, its ``lse``
    and dL/dout ``dout``."""
    B, H, N, d = _expect_qkv(q, k, v)
    M = N // block_size if block_size > 0 else 0
    _expect_attn_inputs(q, kbar, vsum, row_ptr, col_idx, None, B, H, M, d)
    _expect("out", out, q, (B, H, N, d), torch.bfloat16)
    _expect("dout", dout, q, (B, H, N, d), torch.bfloat16)
    if lse is None:
        raise ValueError("lse (float32 [B, H, N]) of the forward call is required")
    _expect("lse", lse, q, (B, H, N), torch.float32)
    if ws is None:
        ws = workspace(B, H, N, d, q.device)
    if grads is None:
        grads = tuple(torch.empty_like(q) for _ in range(3))
    dq, dk, dv = grads
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _expect(name, t, q, (B, H, N, d), torch.bfloat16)
    _expect_ws(ws, q, B, H, N, d)
    _call("psa_attn_bwd", q, _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), _ptr(row_ptr), _ptr(col_idx),
          col_idx.numel(), B, H, N, d, block_size, int(causal), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
          _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(stream, q))
    return dq, dk, dv


def psa_dense(q, k, v, causal: bool = False, ws=None, out=None, lse=None, want_lse: bool = False,
              stream=None):
    """Dense softmax attention through the same tensor-core kernel."""
    B, H, N, d = _expect_qkv(q, k, v)
    if ws is None:
        ws = workspace(B, H, N, d, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _expect_ws(ws, q, B, H, N, d)
    _expect("out", out, q, (B, H, N, d), torch.bfloat16)
    _expect("lse", lse, q, (B, H, N), torch.float32)
    _call("psa_dense", q, _ptr(q), _ptr(k), _ptr(v), B, H, N, d, int(causal), _ptr(out), _ptr(lse), _ptr(ws),
          ws.numel(), _stream(stream, q))
    return (out, lse) if lse is not None else out


def psa_attn_noalloc(q, k, v, kbar, vsum, row_ptr, col_idx, causal: bool = False, block_size: int = 64,
                     out=None, lse=None, status=None, row_max=None, stream=None):
    """psa_attn without a workspace, for callers that cannot allocate device
    memory (framework plugins restricted to the framework's own pool, loops
    that forbid allocation after start-up): the library's own 16 MiB scratch
    array is used instead, and calls that overlap on the GPU race on it.  ``status`` is an optional device
    int32 tensor that receives this call's device status word."""
    B, H, N, d = _expect_qkv(q, k, v)
    M = N // block_size if block_size > 0 else 0
    _expect_attn_inputs(q, kbar, vsum, row_ptr, col_idx, row_max, B, H, M, d)
    if out is None:
        out = torch.empty_like(q)
    _expect("out", out, q, (B, H, N, d), torch.bfloat16)
    _expect("lse", lse, q, (B, H, N), torch.float32)
    _expect("status", status, q, dtype=torch.int32, min_numel=1)
    _call("psa_attn_noalloc", q, _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), _ptr(row_ptr),
          _ptr(col_idx), col_idx.numel(), _ptr(row_max), B, H, N, d, block_size, int(causal), _ptr(out),
          _ptr(lse), _ptr(status), _stream(stream, q))
    return out


def psa_test_stall_next_attn(on: bool = True) -> None:
    """Failure-path test hook: the next psa_attn call's kernel lets a bounded
    wait run out and records PSA_ERR_TIMEOUT in its workspace status word."""
    _check("psa_test_stall_next_attn", lib().psa_test_stall_next_attn(int(bool(on))))


def psa_read_status(ws, stream=None) -> int:
    """Synchronise the stream and return the device status word of ``ws``."""
    _expect("ws", ws, dtype=torch.uint8, min_numel=256)
    st = ctypes.c_int(-1)
    _call("psa_read_status", ws, _ptr(ws), ctypes.byref(st), _stream(stream, ws))
    return int(st.value)


def psa_read_fixup_count(ws, stream=None):
    """Synchronise the stream and return (rerun, exact): the query blocks the
    last attention call on ``ws`` recomputed with per-query stabilisers on the
    tensor cores, and those of them that needed the exact CUDA-core path."""
    _expect("ws", ws, dtype=torch.uint8, min_numel=256)
    rerun, exact = ctypes.c_int(-1), ctypes.c_int(-1)
    _call("psa_read_fixup_count", ws, _ptr(ws), ctypes.byref(rerun), ctypes.byref(exact), _stream(stream, ws))
    return int(rerun.value), int(exact.value)


def psa_forward(q, k, v, mode: str = "topk", density: float = 0.15, alpha: float = 0.5,
                causal: bool = False, keep_first: bool = False, hyd: bool = False, ws=None, stream=None):
    """The whole path in one call (pool -> route -> attention), as the usage
    line of the PISA summary calls it: f(q, k, v, density=0.15, block_size=64).
    ``hyd`` adds the first-order correction with the global statistic.
    Returns (out, (row_ptr, col_idx, nnz, row_max))."""
    B, H, N, d = _shape(q)
    if ws is None:
        ws = workspace(B, H, N, d, q.device)
    qbar, kbar, vsum = psa_pool(q, k, v, stream=stream)
    if mode == "topk":
        csr = psa_route_topk(qbar, kbar, density, causal, ws=ws, stream=stream)
    elif mode == "thresh":
        csr = psa_route_thresh(qbar, kbar, alpha, causal, keep_first, ws=ws, stream=stream)
    elif mode == "thresh_prob":
        csr = psa_route_thresh_prob(qbar, kbar, alpha, causal, keep_first, ws=ws, stream=stream)
    else:
        raise ValueError("mode must be 'topk', 'thresh' or 'thresh_prob'")
    if hyd:
        hstat = psa_hyd_stat(k, v, kbar, vsum, ws=ws, stream=stream)
        out = psa_attn_hyd(q, k, v, kbar, vsum, hstat, csr[0], csr[1], causal, ws=ws, row_max=csr[3],
                           stream=stream)
    else:
        out = psa_attn(q, k, v, kbar, vsum, csr[0], csr[1], causal, ws=ws, row_max=csr[3], stream=stream)
    return out, csr
