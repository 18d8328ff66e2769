"""Python binding of libawq (ctypes): argument marshalling only.

Every step of the computation runs in the CUDA kernels of ``lib/libawq.so``; this module turns torch
tensors into device pointers, allocates the caller-owned outputs and workspaces with torch, and passes
the current torch stream. It raises ``RuntimeError`` when the library is missing or a call fails; there
is no fallback path.

Tensors: X is a CUDA bfloat16 [N, K] matrix (tokens x in-features), W a CUDA bfloat16 [O, K] matrix
(torch ``nn.Linear.weight`` layout) or a list of such matrices that read the same X (stacked once).
"""
from __future__ import annotations

import ctypes
import functools
import os
from dataclasses import dataclass
from typing import Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libawq.so")

AWQ_OK = 0
STATUS_NAMES = {0: "AWQ_OK", 1: "AWQ_ERR_INVALID_ARG", 2: "AWQ_ERR_UNSUPPORTED", 3: "AWQ_ERR_WORKSPACE",
                4: "AWQ_ERR_CUDA", 5: "AWQ_ERR_TIMEOUT"}
FLAG_EXACT_DIVISION = 0x1
FLAG_EXACT_POW = 0x2
FLAG_INJECT_STALL = 0x100
FLAG_SCALES_WEIGHT_AWARE = 0x10
FLAG_SCALES_RMS = 0x20
FLAG_QUANT_INT8 = 0x40
MAX_N_GRID = 64

# name -> (restype, argtypes)
_P, _I64, _I, _U, _SZ, _D = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t,
                            ctypes.c_double)
SIGNATURES = {
    "awq_last_error": (ctypes.c_char_p, []),
    "awq_version": (_I, []),
    "awq_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "awq_set_profile_events": (None, [_P, _P]),
    "awq_act_stats_workspace_size": (_SZ, [_I64, _I64]),
    "awq_act_stats": (_I, [_P, _I64, _I64, _I64, _P, _SZ, _P, _P]),
    "awq_act_stats_noalloc": (_I, [_P, _I64, _I64, _I64, _P, _P]),
    "awq_scale_table_workspace_size": (_SZ, [_I64, _I]),
    "awq_scale_table": (_I, [_P, _I64, _I, _U, _P, _SZ, _P, _P]),
    "awq_scale_table_ex": (_I, [_P, _P, _I64, _I, _U, _P, _SZ, _P, _P]),
    "awq_search_workspace_size": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "awq_search": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _I, _I, _P, _SZ, _P, _P, _P, _P]),
    "awq_search_ex": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _I, _I, _U, _P, _SZ, _P, _P, _P, _P]),
    "awq_search_status": (_I, [_P, _SZ, _P]),
    "awq_search_get_layout": (_I, [_I64, _I64, _I64, _I, _I, _P]),
    "awq_quantize_pack": (_I, [_P, _I64, _I64, _I64, _P, _I, _P, _P, _P, _P]),
    "awq_quantize_pack_ex": (_I, [_P, _I64, _I64, _I64, _P, _I, _U, _P, _P, _P, _P]),
    "awq_quantize_pack_int8": (_I, [_P, _I64, _I64, _I64, _P, _U, _P, _P, _P]),
    "awq_scale_columns": (_I, [_P, _I64, _I64, _I64, _P, _I, _P, _I64, _P]),
    "awq_scale_rows": (_I, [_P, _I64, _I64, _I64, _P, _I, _P, _I64, _P]),
    "awq_w4a16_workspace_size": (_SZ, [_I64, _I64]),
    "awq_w4a16_gemm": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _I64, _P, _I64, _P, _SZ, _P]),
}


class SearchLayout(ctypes.Structure):
    _fields_ = [("tile_n", ctypes.c_int64), ("tile_o", ctypes.c_int64), ("tiles_n", ctypes.c_int64),
                ("tiles_o", ctypes.c_int64), ("partials_per_tile", ctypes.c_int64), ("partials_offset", ctypes.c_size_t),
                ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libawq.so (once) and declare its C signatures. Fails loudly if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libawq.so not found at {path}; build it with "
                           "`python -m weight_only_quantization_act_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class AwqError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != AWQ_OK:
        msg = load_library().awq_last_error().decode(errors="replace")
        raise AwqError(fn, status, msg)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _bf16_matrix(name: str, t: torch.Tensor) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 2:
        raise TypeError(f"{name} must be a CUDA bfloat16 matrix")
    if t.stride(1) != 1:
        t = t.contiguous()
    return t


def _float_vector_out(name: str, out: torch.Tensor, n: int, device) -> torch.Tensor:
    """A caller-given float32 output of at least n elements, contiguous, on `device`: the kernels write n
    floats from its first element."""
    if (not isinstance(out, torch.Tensor) or out.dtype != torch.float32 or not out.is_cuda
            or out.device != device or out.numel() < n or not out.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA float32 tensor of at least {n} elements on {device}")
    return out


def _on_device(fn):
    """Run an entry point with its first tensor argument's device current, so that the library launches
    there and the stream passed is that device's current stream."""

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        first = args[0] if args else next(iter(kwargs.values()))
        if isinstance(first, (list, tuple)):
            first = first[0]
        if isinstance(first, torch.Tensor) and first.is_cuda:
            with torch.cuda.device(first.device):
                return fn(*args, **kwargs)
        return fn(*args, **kwargs)

    return wrapper


def _workspace(nbytes: int, device, workspace: torch.Tensor | None) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace
    # torch's caching allocator returns 512-byte aligned blocks; over-allocate to align to 1024
    raw = torch.empty(nbytes + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + nbytes]


def set_wait_limit_ns(ns: int) -> None:
    load_library().awq_set_wait_limit_ns(int(ns))


def set_profile_events(before, after) -> None:
    """Record two torch.cuda.Event objects around the loss GEMM of later searches (None, None stops)."""
    lib = load_library()
    if before is None or after is None:
        lib.awq_set_profile_events(None, None)
        return
    for ev in (before, after):
        if not ev.cuda_event:
            ev.record()  # torch creates the underlying event lazily
    lib.awq_set_profile_events(ctypes.c_void_p(before.cuda_event), ctypes.c_void_p(after.cuda_event))


def version() -> int:
    return load_library().awq_version()


# --------------------------------------------------------------------------------------------- (1)
def act_stats_workspace_size(N: int, K: int) -> int:
    return load_library().awq_act_stats_workspace_size(N, K)


@_on_device
def act_stats(X: torch.Tensor, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """act_mean[k] = mean_i |X[i,k]| (fixed-order fp64 sum, rounded to fp32)."""
    lib = load_library()
    X = _bf16_matrix("X", X)
    N, K = X.shape
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=X.device)
    _float_vector_out("out", out, K, X.device)
    ws = _workspace(lib.awq_act_stats_workspace_size(N, K), X.device, workspace)
    _check("awq_act_stats", lib.awq_act_stats(_ptr(X), N, K, X.stride(0), _ptr(ws), ws.numel(), _ptr(out),
                                              _stream(stream)))
    return out


@_on_device
def act_stats_noalloc(X: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    """Same statistic with no workspace, for callers that cannot allocate device memory at call time
    (the scratch is a fixed 16 MiB array inside the library; ceil(N/256)*K <= 2**21). ``out`` must be
    preallocated; calls that overlap on the GPU race on the shared scratch. Nothing is allocated here
    either: X must already have unit column stride (no contiguous copy is made)."""
    lib = load_library()
    if not isinstance(X, torch.Tensor) or X.dtype != torch.bfloat16 or not X.is_cuda or X.dim() != 2:
        raise TypeError("X must be a CUDA bfloat16 matrix")
    if X.stride(1) != 1:
        raise ValueError("X must have unit column stride (this entry point makes no copy)")
    N, K = X.shape
    _float_vector_out("out", out, K, X.device)
    _check("awq_act_stats_noalloc", lib.awq_act_stats_noalloc(_ptr(X), N, K, X.stride(0), _ptr(out),
                                                              _stream(stream)))
    return out


# --------------------------------------------------------------------------------------------- (2)
@_on_device
def scale_table(act_mean: torch.Tensor, n_grid: int = 20, exact_pow: bool = False, rule: str = "p4",
                weight_mean: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """float32 [n_grid, K] table of candidate scales; rule "p4" (default), "weight_aware" (needs
    weight_mean) or "rms"."""
    lib = load_library()
    K = act_mean.shape[0]
    table = torch.empty((n_grid, K), dtype=torch.float32, device=act_mean.device)
    ws = _workspace(lib.awq_scale_table_workspace_size(K, n_grid), act_mean.device, None)
    flags = (FLAG_EXACT_POW if exact_pow else 0) | RULE_FLAGS[rule]
    wm = _ptr(weight_mean) if weight_mean is not None else None
    _check("awq_scale_table_ex", lib.awq_scale_table_ex(_ptr(act_mean), wm, K, n_grid, flags, _ptr(ws), ws.numel(),
                                                        _ptr(table), _stream(stream)))
    return table


RULE_FLAGS = {"p4": 0, "weight_aware": FLAG_SCALES_WEIGHT_AWARE, "rms": FLAG_SCALES_RMS}


# --------------------------------------------------------------------------------------------- (3)-(4)
@dataclass
class SearchResult:
    losses: torch.Tensor      # float64 [n_grid] (device)
    best_j: torch.Tensor      # int32 [1] (device)
    scales: torch.Tensor      # float32 [K] (device)
    workspace: torch.Tensor   # uint8 (device), holds the scale table and the per-tile partial sums

    def ratio(self, n_grid: int) -> float:
        return int(self.best_j.item()) / n_grid


def stack_weights(W: torch.Tensor | Sequence[torch.Tensor]) -> torch.Tensor:
    """Linears that read the same X share one scale vector: stack their rows once."""
    if isinstance(W, torch.Tensor):
        return _bf16_matrix("W", W)
    mats = [_bf16_matrix("W", w) for w in W]
    return mats[0] if len(mats) == 1 else torch.cat(mats, dim=0)


def search_workspace_size(N: int, K: int, O: int, n_grid: int = 20, group: int = 128) -> int:
    return load_library().awq_search_workspace_size(N, K, O, group, n_grid)


def search_layout(N: int, K: int, O: int, n_grid: int = 20, group: int = 128) -> SearchLayout:
    lib = load_library()
    lay = SearchLayout()
    _check("awq_search_get_layout", lib.awq_search_get_layout(N, K, O, group, n_grid, ctypes.byref(lay)))
    return lay


@_on_device
def search(X: torch.Tensor, W, act_mean: torch.Tensor, n_grid: int = 20, group: int = 128, flags: int = 0,
           workspace: torch.Tensor | None = None, out: SearchResult | None = None, rule: str = "p4",
           quant: str = "int4", stream=None) -> SearchResult:
    """Grid search of the AWQ scale ratio for one linear (or stacked linears sharing X); rule selects the
    candidate scales ("p4" default, "weight_aware", "rms"); quant the weight quantizer ("int4" in groups
    of `group`, or "int8" symmetric per output channel, for which group is ignored)."""
    lib = load_library()
    flags |= RULE_FLAGS[rule]
    if quant == "int8":
        flags |= FLAG_QUANT_INT8
        group = 0
    elif quant != "int4":
        raise ValueError(f"quant must be 'int4' or 'int8', not {quant!r}")
    X = _bf16_matrix("X", X)
    W = stack_weights(W)
    N, K = X.shape
    O = W.shape[0]
    ws = _workspace(lib.awq_search_workspace_size(N, K, O, group, n_grid), X.device, workspace)
    if out is None:
        out = SearchResult(torch.empty(n_grid, dtype=torch.float64, device=X.device),
                           torch.empty(1, dtype=torch.int32, device=X.device),
                           torch.empty(K, dtype=torch.float32, device=X.device), ws)
    else:
        out.workspace = ws
    _check("awq_search_ex", lib.awq_search_ex(
        _ptr(X), N, K, X.stride(0), _ptr(W), O, W.stride(0), _ptr(act_mean), group, n_grid, flags, _ptr(ws),
        ws.numel(), _ptr(out.losses), _ptr(out.best_j), _ptr(out.scales), _stream(stream)))
    return out


def search_status(result: SearchResult, stream=None) -> int:
    """Synchronise and return the device status of the last search on this workspace (0 = ok)."""
    lib = load_library()
    return lib.awq_search_status(_ptr(result.workspace), result.workspace.numel(), _stream(stream))


def tile_partials(result: SearchResult, N: int, K: int, O: int, n_grid: int = 20) -> torch.Tensor:
    """View of the per-tile partial sums: float64 [n_grid, tiles_o, tiles_n, partials_per_tile]; entry e of
    a tile covers tile_n / partials_per_tile consecutive token rows."""
    lay = search_layout(N, K, O, n_grid)
    count = n_grid * lay.tiles_o * lay.tiles_n * lay.partials_per_tile
    raw = result.workspace[lay.partials_offset: lay.partials_offset + 8 * count]
    return raw.view(torch.float64).view(n_grid, lay.tiles_o, lay.tiles_n, lay.partials_per_tile)


# --------------------------------------------------------------------------------------------- (5)
@_on_device
def quantize_pack(W: torch.Tensor, scales: torch.Tensor, group: int = 128, flags: int = 0, stream=None):
    """(codes uint32 [O, K/8] as int32 storage, steps float32 [O, K/g], zeros float32 [O, K/g])."""
    lib = load_library()
    W = stack_weights(W)
    O, K = W.shape
    codes = torch.empty((O, K // 8), dtype=torch.int32, device=W.device)
    steps = torch.empty((O, K // group), dtype=torch.float32, device=W.device)
    zeros = torch.empty((O, K // group), dtype=torch.float32, device=W.device)
    _check("awq_quantize_pack_ex", lib.awq_quantize_pack_ex(
        _ptr(W), O, K, W.stride(0), _ptr(scales), group, flags, _ptr(codes), _ptr(steps), _ptr(zeros),
        _stream(stream)))
    return codes, steps, zeros


@_on_device
def quantize_pack_int8(W: torch.Tensor, scales: torch.Tensor, flags: int = 0, stream=None):
    """(codes int8 [O, K], steps float32 [O]): symmetric INT8, one step per output channel."""
    lib = load_library()
    W = stack_weights(W)
    O, K = W.shape
    codes = torch.empty((O, K), dtype=torch.int8, device=W.device)
    steps = torch.empty(O, dtype=torch.float32, device=W.device)
    _check("awq_quantize_pack_int8", lib.awq_quantize_pack_int8(
        _ptr(W), O, K, W.stride(0), _ptr(scales), flags, _ptr(codes), _ptr(steps), _stream(stream)))
    return codes, steps


@_on_device
def quantize_layer(X: torch.Tensor, W, n_grid: int = 20, group: int = 128, stream=None):
    """The whole path for one layer: statistic, search, and the packed artefact at the best scales."""
    act = act_stats(X, stream=stream)
    res = search(X, W, act, n_grid=n_grid, group=group, stream=stream)
    codes, steps, zeros = quantize_pack(W, res.scales, group=group, stream=stream)
    return dict(act_mean=act, losses=res.losses, best_j=res.best_j, scales=res.scales, codes=codes,
                steps=steps, zeros=zeros)


# --------------------------------------------------------------------------------------------- (6)
SCALE_MULTIPLY = 0
SCALE_DIVIDE = 1


def _as_matrix(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError("expected a CUDA bfloat16 tensor")
    return t.view(1, -1) if t.dim() == 1 else t


@_on_device
def scale_columns(A: torch.Tensor, s: torch.Tensor, divide: bool = False, out: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """out[r, c] = bf16(A[r, c] * s[c]) (or / s[c]); a 1-D tensor is one row. ``out=A`` works in place."""
    lib = load_library()
    A2 = _as_matrix(A)
    if out is None:
        out = torch.empty_like(A)
    O2 = _as_matrix(out)
    R, C = A2.shape
    _check("awq_scale_columns", lib.awq_scale_columns(_ptr(A2), R, C, A2.stride(0), _ptr(s),
                                                      SCALE_DIVIDE if divide else SCALE_MULTIPLY, _ptr(O2),
                                                      O2.stride(0), _stream(stream)))
    return out


@_on_device
def scale_rows(A: torch.Tensor, s: torch.Tensor, divide: bool = False, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """out[r, c] = bf16(A[r, c] * s[r]) (or / s[r]); a 1-D tensor is scaled element-wise."""
    lib = load_library()
    one_d = A.dim() == 1
    A2 = A.view(-1, 1) if one_d else A
    if one_d:
        # a vector scaled element-wise by s is a 1 x C column scaling
        return scale_columns(A, s, divide=divide, out=out, stream=stream)
    if out is None:
        out = torch.empty_like(A)
    R, C = A2.shape
    _check("awq_scale_rows", lib.awq_scale_rows(_ptr(A2), R, C, A2.stride(0), _ptr(s),
                                                SCALE_DIVIDE if divide else SCALE_MULTIPLY, _ptr(out),
                                                out.stride(0), _stream(stream)))
    return out


def fold_norm_linear(norm_weight: torch.Tensor, linears: Sequence[torch.Tensor], s: torch.Tensor, stream=None):
    """NormLinearSubgraph: gamma / s for the norm, W diag(s) for every linear reading its output (in place)."""
    scale_columns(norm_weight, s, divide=True, out=norm_weight, stream=stream)
    for w in linears:
        scale_columns(w, s, out=w, stream=stream)


def fold_linear_linear(w1: torch.Tensor, b1: torch.Tensor | None, w2: torch.Tensor, s: torch.Tensor, stream=None):
    """LinearLinearSubgraph / OVSubgraph (multi-head) / UpDownSubgraph: rows (and bias) of the source linear
    divided by s, columns of the target linear multiplied by s (in place)."""
    scale_rows(w1, s, divide=True, out=w1, stream=stream)
    if b1 is not None:
        scale_columns(b1, s, divide=True, out=b1, stream=stream)
    scale_columns(w2, s, out=w2, stream=stream)


# --------------------------------------------------------------------------------------------- (7)
@_on_device
def w4a16_gemm(X: torch.Tensor, codes: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor,
               out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X' deq(W)^T (bf16 [M, O]) from packed codes [O, K/8], steps and zeros [O, K/128]."""
    lib = load_library()
    X = _bf16_matrix("X", X)
    M, K = X.shape
    O = codes.shape[0]
    if out is None:
        out = torch.empty((M, O), dtype=torch.bfloat16, device=X.device)
    if workspace is None:  # zero-filled once; the library keeps its counters zero from call to call
        workspace = torch.zeros(lib.awq_w4a16_workspace_size(K, O), dtype=torch.uint8, device=X.device)
    _check("awq_w4a16_gemm", lib.awq_w4a16_gemm(_ptr(X), M, K, X.stride(0), _ptr(codes), _ptr(steps), _ptr(zeros),
                                                O, _ptr(out), out.stride(0), _ptr(workspace), workspace.numel(),
                                                _stream(stream)))
    return out
