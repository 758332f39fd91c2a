"""Python binding of the B200 Sliding Tile Attention library (``libsta.so``).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  The functions carry the names of the C entry points declared in
``include/sta.h`` and take torch tensors (device memory owned by the caller) and
the current torch CUDA stream.  There is no fallback: if the library is missing
or the device is not a B200, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsta.so")

STATUS_NAMES = {
    0: "STA_OK", 1: "STA_ERR_NULL", 2: "STA_ERR_ALIGN", 3: "STA_ERR_ALIAS", 4: "STA_ERR_SHAPE",
    5: "STA_ERR_WINDOW", 6: "STA_ERR_HEADDIM", 7: "STA_ERR_ARCH", 8: "STA_ERR_CUDA",
    9: "STA_ERR_TIMEOUT", 10: "STA_ERR_ARG", 11: "STA_ERR_SCRATCH", 12: "STA_ERR_BOUNDS",
}
STA_OK, STA_ERR_TIMEOUT = 0, 9


class sta_dim3(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int32), ("h", ctypes.c_int32), ("w", ctypes.c_int32)]


class StaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libsta.so (built by ``sparse_attention_video_tile_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run `python -m sparse_attention_video_tile_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, U64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
    D3 = sta_dim3
    sigs = {
        "sta_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "sta_last_cuda_error": (ctypes.c_char_p, []),
        "sta_tile_index_map": (ctypes.c_int, [D3, D3, ctypes.POINTER(ctypes.c_int32)]),
        "sta_attended_pairs": (I64, [I32, I32, D3, D3, ctypes.POINTER(D3)]),
        "sta_schedule_block_pairs": (I64, [I32, I32, D3, D3, ctypes.POINTER(D3), I32, ctypes.POINTER(ctypes.c_int32), I64]),
        "sta_tile_reorder": (ctypes.c_int, [P, P, I64, I32, D3, D3, P]),
        "sta_tile_unorder": (ctypes.c_int, [P, P, I64, I32, D3, D3, P]),
        "sta_tile_reorder_tokens": (ctypes.c_int, [P, P, I32, I32, I32, D3, D3, P]),
        "sta_tile_unorder_tokens": (ctypes.c_int, [P, P, I32, I32, I32, D3, D3, P]),
        "sta_attention_fwd": (ctypes.c_int, [P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]),
        "sta_attention_fwd_raster": (ctypes.c_int, [P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]),
        "sta_attention_fwd_mixed": (ctypes.c_int, [P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]),
        "sta_tile_reorder_padded": (ctypes.c_int, [P, P, I64, I32, D3, D3, P]),
        "sta_forward_host": (ctypes.c_int, [P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, I32, P]),
        "sta_attention_fwd_lse": (ctypes.c_int, [P, P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]),
        "sta_attention_bwd": (ctypes.c_int, [P, P, P, P, P, P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]),
        "sta_check_device_status": (ctypes.c_int, [P]),
        "sta_selftest_bounded_wait": (ctypes.c_int, [U64, P]),
        "sta_shutdown": (None, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _d3(x: Sequence[int]) -> sta_dim3:
    t = tuple(int(v) for v in x)
    if len(t) != 3:
        raise ValueError(f"expected (t, h, w), got {x!r}")
    return sta_dim3(*t)


def _windows(ws: Sequence[Sequence[int]]):
    arr = (sta_dim3 * len(ws))()
    for i, w in enumerate(ws):
        arr[i] = _d3(w)
    return arr


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _stream_context(stream):
    """Makes ``stream`` (None for the current stream, a torch stream or a raw
    cudaStream_t handle) torch's current stream, so that tensors allocated inside
    belong to the stream their kernels run on: the caching allocator then reuses
    their memory only after that stream's work."""
    import contextlib
    import torch
    if stream is None:
        return contextlib.nullcontext()
    if isinstance(stream, int):
        stream = torch.cuda.ExternalStream(stream)
    return torch.cuda.stream(stream)


def _check(status: int, where: str) -> None:
    if status != STA_OK:
        detail = ""
        if status == 8:
            detail = load_library().sta_last_cuda_error().decode()
        raise StaError(status, where, detail)


def _tensor_ptr(x, name: str) -> int:
    import torch
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if x.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {x.dtype}")
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return x.data_ptr()


def sta_status_str(status: int) -> str:
    return load_library().sta_status_str(int(status)).decode()


def sta_tile_index_map(grid, tile) -> np.ndarray:
    """Raster -> tiled index map (int32 array of L entries)."""
    L = int(np.prod([int(v) for v in grid]))
    out = np.empty(L, dtype=np.int32)
    st = load_library().sta_tile_index_map(_d3(grid), _d3(tile),
                                           out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    _check(st, "sta_tile_index_map")
    return out


def sta_attended_pairs(batch: int, heads: int, grid, tile, windows) -> int:
    r = load_library().sta_attended_pairs(int(batch), int(heads), _d3(grid), _d3(tile), _windows(windows))
    if r < 0:
        raise StaError(10, "sta_attended_pairs")
    return int(r)


def sta_schedule_block_pairs(batch: int, heads: int, grid, tile, windows, transposed: bool = False) -> np.ndarray:
    """(bh, query block row, key block row) of every block pair of the forward's
    schedule or, with ``transposed``, of the backward's key-side schedule (host only)."""
    lib = load_library()
    args = (int(batch), int(heads), _d3(grid), _d3(tile), _windows(windows), int(bool(transposed)))
    n = lib.sta_schedule_block_pairs(*args, None, 0)
    if n < 0:
        raise StaError(10, "sta_schedule_block_pairs")
    out = np.empty((max(n, 1), 3), dtype=np.int32)
    lib.sta_schedule_block_pairs(*args, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n)
    return out[:n]


def sta_tile_reorder(src, dst, grid, tile, stream=None) -> None:
    """dst[..., tiled(n), :] = src[..., n, :] for [.., L, d] bf16 CUDA tensors."""
    d = int(src.shape[-1])
    bh = int(src.numel() // (src.shape[-2] * d)) if src.numel() else 0
    if tuple(dst.shape) != tuple(src.shape):
        raise ValueError("src and dst shapes differ")
    st = load_library().sta_tile_reorder(_tensor_ptr(src, "src"), _tensor_ptr(dst, "dst"), bh, d,
                                         _d3(grid), _d3(tile), _stream(stream))
    _check(st, "sta_tile_reorder")


def sta_tile_unorder(src, dst, grid, tile, stream=None) -> None:
    """dst[..., n, :] = src[..., tiled(n), :]."""
    d = int(src.shape[-1])
    bh = int(src.numel() // (src.shape[-2] * d)) if src.numel() else 0
    if tuple(dst.shape) != tuple(src.shape):
        raise ValueError("src and dst shapes differ")
    st = load_library().sta_tile_unorder(_tensor_ptr(src, "src"), _tensor_ptr(dst, "dst"), bh, d,
                                         _d3(grid), _d3(tile), _stream(stream))
    _check(st, "sta_tile_unorder")


def _token_shapes(tokens, tiled, where: str):
    """(batch, heads, d) of a token-major [B, L, heads, d] tensor and its tiled
    [B, heads, L, d] counterpart."""
    if tokens.dim() != 4 or tiled.dim() != 4:
        raise ValueError(f"{where}: expected 4-D tensors")
    b, n, h, d = (int(x) for x in tokens.shape)
    if tuple(tiled.shape) != (b, h, n, d):
        raise ValueError(f"{where}: token-major {tuple(tokens.shape)} does not match tiled {tuple(tiled.shape)}")
    return b, h, d


def sta_tile_reorder_tokens(src, dst, grid, tile, stream=None) -> None:
    """dst[b, h, tiled(n), :] = src[b, n, h, :]: token-major raster [B, L, heads, d]
    (a [B, L, heads * d] projection viewed per head) to tiled [B, heads, L, d]."""
    b, h, d = _token_shapes(src, dst, "sta_tile_reorder_tokens")
    st = load_library().sta_tile_reorder_tokens(_tensor_ptr(src, "src"), _tensor_ptr(dst, "dst"), b, h, d,
                                                _d3(grid), _d3(tile), _stream(stream))
    _check(st, "sta_tile_reorder_tokens")


def sta_tile_unorder_tokens(src, dst, grid, tile, stream=None) -> None:
    """dst[b, n, h, :] = src[b, h, tiled(n), :]: tiled [B, heads, L, d] to
    token-major raster [B, L, heads, d]."""
    b, h, d = _token_shapes(dst, src, "sta_tile_unorder_tokens")
    st = load_library().sta_tile_unorder_tokens(_tensor_ptr(src, "src"), _tensor_ptr(dst, "dst"), b, h, d,
                                                _d3(grid), _d3(tile), _stream(stream))
    _check(st, "sta_tile_unorder_tokens")


def sta_attention_fwd(q, k, v, out, grid, tile, window_per_head, scale: float, stream=None) -> None:
    """STA forward on tiled-order [B, heads, L, d] bf16 CUDA tensors."""
    if q.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    B, Hn, L, d = (int(x) for x in q.shape)
    for name, t in (("k", k), ("v", v), ("out", out)):
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} differs from q {tuple(q.shape)}")
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    st = load_library().sta_attention_fwd(_tensor_ptr(q, "q"), _tensor_ptr(k, "k"), _tensor_ptr(v, "v"),
                                          _tensor_ptr(out, "out"), B, Hn, d, _d3(grid), _d3(tile),
                                          _windows(window_per_head), float(scale), _stream(stream))
    _check(st, "sta_attention_fwd")


def sta_attention_fwd_lse(q, k, v, out, lse, grid, tile, window_per_head, scale: float, stream=None) -> None:
    """sta_attention_fwd that also writes each row's log-sum-exp into ``lse``, an fp32
    CUDA tensor [B, heads, L] (tiled order)."""
    import torch
    if q.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    B, Hn, L, d = (int(x) for x in q.shape)
    for name, t in (("k", k), ("v", v), ("out", out)):
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} differs from q {tuple(q.shape)}")
    if not isinstance(lse, torch.Tensor) or lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise TypeError("lse must be a contiguous float32 CUDA tensor")
    if tuple(lse.shape) != (B, Hn, L):
        raise ValueError(f"lse must be [batch, heads, L] = {(B, Hn, L)}")
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    st = load_library().sta_attention_fwd_lse(_tensor_ptr(q, "q"), _tensor_ptr(k, "k"), _tensor_ptr(v, "v"),
                                              _tensor_ptr(out, "out"), lse.data_ptr(), B, Hn, d, _d3(grid),
                                              _d3(tile), _windows(window_per_head), float(scale), _stream(stream))
    _check(st, "sta_attention_fwd_lse")


def sta_attention_bwd(q, k, v, out, dout, lse, dq, dk, dv, grid, tile, window_per_head, scale: float,
                      stream=None) -> None:
    """STA backward on tiled-order [B, heads, L, d] bf16 CUDA tensors: writes dq, dk,
    dv from the forward's inputs, output and log-sum-exp (fp32 [B, heads, L]) and
    the output gradient dout."""
    import torch
    if q.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    B, Hn, L, d = (int(x) for x in q.shape)
    for name, t in (("k", k), ("v", v), ("out", out), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} differs from q {tuple(q.shape)}")
    if not isinstance(lse, torch.Tensor) or lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise TypeError("lse must be a contiguous float32 CUDA tensor")
    if tuple(lse.shape) != (B, Hn, L):
        raise ValueError(f"lse must be [batch, heads, L] = {(B, Hn, L)}")
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    ptrs = [_tensor_ptr(t, n) for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout"))]
    outs = [_tensor_ptr(t, n) for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"))]
    st = load_library().sta_attention_bwd(*ptrs, lse.data_ptr(), *outs, B, Hn, d, _d3(grid), _d3(tile),
                                          _windows(window_per_head), float(scale), _stream(stream))
    _check(st, "sta_attention_bwd")


def sta_attention_fwd_raster(q, k, v, out, grid, tile, window_per_head, scale: float, stream=None) -> None:
    """STA forward on raster-order [B, heads, T*H*W, d] bf16 CUDA tensors (tile
    reorder fused into the kernel; grids that are not tile multiples are padded)."""
    if q.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    B, Hn, L, d = (int(x) for x in q.shape)
    for name, t in (("k", k), ("v", v), ("out", out)):
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} differs from q {tuple(q.shape)}")
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    if L != int(np.prod([int(x) for x in grid])):
        raise ValueError("L must equal T*H*W")
    st = load_library().sta_attention_fwd_raster(_tensor_ptr(q, "q"), _tensor_ptr(k, "k"), _tensor_ptr(v, "v"),
                                                 _tensor_ptr(out, "out"), B, Hn, d, _d3(grid), _d3(tile),
                                                 _windows(window_per_head), float(scale), _stream(stream))
    _check(st, "sta_attention_fwd_raster")


def padded_rows(grid, tile) -> int:
    """Rows per (batch, head) of the latent padded up to tile multiples."""
    return int(np.prod([-(-int(a) // int(b)) * int(b) for a, b in zip(grid, tile)]))


def sta_tile_reorder_padded(src, dst, grid, tile, stream=None) -> None:
    """Raster [.., T*H*W, d] -> tiled order of the padded latent [.., Lpad, d], pad rows zero."""
    d = int(src.shape[-1])
    lead = tuple(int(x) for x in src.shape[:-2])
    if tuple(dst.shape) != lead + (padded_rows(grid, tile), d):
        raise ValueError(f"dst must be {lead + (padded_rows(grid, tile), d)}")
    bh = int(np.prod(lead)) if lead else 1
    st = load_library().sta_tile_reorder_padded(_tensor_ptr(src, "src"), _tensor_ptr(dst, "dst"), bh, d,
                                                _d3(grid), _d3(tile), _stream(stream))
    _check(st, "sta_tile_reorder_padded")


def sta_attention_fwd_mixed(q, k_tiled, v_tiled, out, grid, tile, window_per_head, scale: float, stream=None) -> None:
    """STA forward with raster-order q and out [B, heads, T*H*W, d] and k, v in the tiled
    order of the padded latent [B, heads, Lpad, d] (``sta_tile_reorder_padded``)."""
    if q.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    B, Hn, L, d = (int(x) for x in q.shape)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be shaped like q")
    for name, t in (("k_tiled", k_tiled), ("v_tiled", v_tiled)):
        if tuple(t.shape) != (B, Hn, padded_rows(grid, tile), d):
            raise ValueError(f"{name} must be [B, heads, Lpad, d]")
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    if L != int(np.prod([int(x) for x in grid])):
        raise ValueError("L must equal T*H*W")
    st = load_library().sta_attention_fwd_mixed(_tensor_ptr(q, "q"), _tensor_ptr(k_tiled, "k_tiled"),
                                                _tensor_ptr(v_tiled, "v_tiled"), _tensor_ptr(out, "out"), B, Hn, d,
                                                _d3(grid), _d3(tile), _windows(window_per_head), float(scale),
                                                _stream(stream))
    _check(st, "sta_attention_fwd_mixed")


def raster_tile_ok(tile) -> bool:
    """Whether sta_attention_fwd_raster accepts this tile (128-row slabs of whole frames)."""
    tt, th, tw = (int(x) for x in tile)
    plane = th * tw
    return 0 < plane <= 128 and 128 % plane == 0 and tt % (128 // plane) == 0


def sta_check_device_status(stream=None) -> int:
    """Synchronises the stream; returns STA_OK or STA_ERR_TIMEOUT (raises on CUDA errors)."""
    st = load_library().sta_check_device_status(_stream(stream))
    if st not in (STA_OK, STA_ERR_TIMEOUT):
        _check(st, "sta_check_device_status")
    return st


def sta_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    st = load_library().sta_selftest_bounded_wait(int(limit_ns), _stream(stream))
    if st not in (STA_OK, STA_ERR_TIMEOUT):
        _check(st, "sta_selftest_bounded_wait")
    return st


def sta_shutdown() -> None:
    load_library().sta_shutdown()


def sta_forward(q, k, v, grid, tile, window_per_head, scale: Optional[float] = None,
                stream=None, workspace: Optional[Tuple] = None, fused: Optional[bool] = None,
                path: Optional[str] = None):
    """Full STA forward on raster-order [B, heads, L, d] bf16 CUDA tensors.

    Three ways (``path``), same result:

    * "mixed": k and v are reordered into the padded latent's tiled order (two
      launches of ``sta_tile_reorder_padded``), then ``sta_attention_fwd_mixed``
      reads q and writes out in raster order.  Needs ``raster_tile_ok`` and two
      scratch tensors [B, heads, Lpad, d] (``workspace`` may hold them); handles
      grids that are not tile multiples.

    * fused: one call does everything (``sta_attention_fwd_raster``: tile reorder in
      the kernel's loads and stores).  Needs a tile that splits into 128-row slabs
      of whole frames (``raster_tile_ok``); the only way for grids that are not tile
      multiples (padding with masking), and the one that needs no scratch memory.
    * three calls: q, k and v are reordered to tiled order, attended and the output
      reordered back, on ``stream``; ``workspace`` may hold four preallocated
      tensors shaped like q (tiled q, k, v and output).  Faster on B200 where both
      apply (the tiled kernel's K/V loads are plain 3-D boxes of 128 contiguous
      rows, the fused kernel's are 5-D boxes of whole frames).

    ``path`` is "mixed", "fused" (the one-launch raster call) or "three_call";
    ``fused=True`` / ``fused=False`` select "fused" / "three_call".  By default
    "mixed" is taken wherever the tile allows it (the fastest whole forward on
    B200), else "three_call".
    Returns the raster-order output, allocated on ``stream``: use it on another
    stream only after synchronising with that one.
    """
    import torch
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    if path is None:
        if fused is None:
            path = "mixed" if raster_tile_ok(tile) else "three_call"
        else:
            path = "fused" if fused else "three_call"
    if path not in ("mixed", "fused", "three_call"):
        raise ValueError(f"unknown path {path!r}")
    with _stream_context(stream):
        out = torch.empty_like(q)
        if path == "fused":
            sta_attention_fwd_raster(q, k, v, out, grid, tile, window_per_head, scale, stream)
            return out
        if path == "mixed":
            B, Hn, _, d = (int(x) for x in q.shape)
            if workspace is None:
                workspace = tuple(torch.empty((B, Hn, padded_rows(grid, tile), d), dtype=q.dtype, device=q.device)
                                  for _ in range(2))
            kt, vt = workspace[:2]
            sta_tile_reorder_padded(k, kt, grid, tile, stream)
            sta_tile_reorder_padded(v, vt, grid, tile, stream)
            sta_attention_fwd_mixed(q, kt, vt, out, grid, tile, window_per_head, scale, stream)
            return out
        if workspace is None:
            workspace = tuple(torch.empty_like(q) for _ in range(4))
        qt, kt, vt, ot = workspace
        sta_tile_reorder(q, qt, grid, tile, stream)
        sta_tile_reorder(k, kt, grid, tile, stream)
        sta_tile_reorder(v, vt, grid, tile, stream)
        sta_attention_fwd(qt, kt, vt, ot, grid, tile, window_per_head, scale, stream)
        sta_tile_unorder(ot, out, grid, tile, stream)
        return out


def sta_forward_tokens(q, k, v, grid, tile, window_per_head, scale: Optional[float] = None,
                       stream=None, workspace: Optional[Tuple] = None):
    """Full STA forward on token-major raster [B, L, heads, d] bf16 CUDA tensors
    (the layout of per-head views of [B, L, heads * d] projections), output in the
    same layout.  The transposes to and from [B, heads, L, d] are part of the tile
    reorders (``sta_tile_reorder_tokens`` / ``sta_tile_unorder_tokens``), so there
    is no extra pass over memory.  The grid must be a tile multiple.
    ``workspace`` may hold four preallocated tiled [B, heads, L, d] tensors."""
    import torch
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    b, n, h, d = (int(x) for x in q.shape)
    with _stream_context(stream):
        if workspace is None:
            workspace = tuple(torch.empty((b, h, n, d), dtype=q.dtype, device=q.device) for _ in range(4))
        qt, kt, vt, ot = workspace
        sta_tile_reorder_tokens(q, qt, grid, tile, stream)
        sta_tile_reorder_tokens(k, kt, grid, tile, stream)
        sta_tile_reorder_tokens(v, vt, grid, tile, stream)
        sta_attention_fwd(qt, kt, vt, ot, grid, tile, window_per_head, scale, stream)
        out = torch.empty_like(q)
        sta_tile_unorder_tokens(ot, out, grid, tile, stream)
        return out


def sta_forward_host(q_h, k_h, v_h, out_h, grid, tile, window_per_head, scale: Optional[float] = None,
                     heads_per_chunk: int = 4, stream=None) -> None:
    """The C-ABI call sta_forward_host on host tensors [B, heads, L, d] (bf16, raster
    order, contiguous; pinned for overlapped copies): the library streams the heads
    through the current device in chunks and returns once ``out_h`` holds the result."""
    import torch
    if q_h.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    for name, t in (("k", k_h), ("v", v_h), ("out", out_h)):
        if tuple(t.shape) != tuple(q_h.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} differs from q {tuple(q_h.shape)}")
    for name, t in (("q", q_h), ("k", k_h), ("v", v_h), ("out", out_h)):
        if t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a contiguous host bf16 tensor")
    B, Hn, L, d = (int(x) for x in q_h.shape)
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    if L != int(np.prod([int(x) for x in grid])):
        raise ValueError("L must equal T*H*W")
    sc = 1.0 / float(d) ** 0.5 if scale is None else float(scale)
    st = load_library().sta_forward_host(q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), out_h.data_ptr(), B, Hn, d,
                                         _d3(grid), _d3(tile), _windows(window_per_head), sc, int(heads_per_chunk),
                                         _stream(stream))
    _check(st, "sta_forward_host")


def sta_forward_from_host(q_h, k_h, v_h, out_h, grid, tile, window_per_head, scale: Optional[float] = None,
                          heads_per_chunk: int = 4, device=None) -> None:
    """STA forward from pinned host tensors [B, heads, L, d] (bf16, raster order)
    into the pinned host tensor ``out_h``, with the copies overlapped with the
    computation: heads go through in chunks, and while one chunk is computed the
    next is copied in and the previous one copied out, on three CUDA streams.  Where
    the tile splits into 128-row slabs of whole frames (``raster_tile_ok``) this is
    the C-ABI call ``sta_forward_host``; other tiles take the same pipeline built
    here from ``sta_forward``.  Per head the result equals ``sta_forward`` on device
    tensors: heads are independent.  The work starts after what is already queued
    on the device's current stream (for example a copy that fills the inputs).
    Returns once ``out_h`` holds the output."""
    import torch
    if q_h.dim() != 4:
        raise ValueError("q must be [batch, heads, L, d]")
    for name, t in (("k", k_h), ("v", v_h), ("out", out_h)):
        if tuple(t.shape) != tuple(q_h.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} differs from q {tuple(q_h.shape)}")
    for name, t in (("q", q_h), ("k", k_h), ("v", v_h), ("out", out_h)):
        if t.is_cuda or not t.is_pinned() or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a contiguous pinned host bf16 tensor")
    B, Hn = int(q_h.shape[0]), int(q_h.shape[1])
    if len(window_per_head) != Hn:
        raise ValueError("one window per head is required")
    if heads_per_chunk < 1:
        raise ValueError("heads_per_chunk must be positive")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        if raster_tile_ok(tile):
            sta_forward_host(q_h, k_h, v_h, out_h, grid, tile, window_per_head, scale, heads_per_chunk,
                             torch.cuda.current_stream(dev))
        else:
            _forward_from_host_chunks(q_h, k_h, v_h, out_h, grid, tile, window_per_head, scale, heads_per_chunk,
                                      dev)


def _forward_from_host_chunks(q_h, k_h, v_h, out_h, grid, tile, window_per_head, scale, heads_per_chunk, dev):
    import torch
    B, Hn = int(q_h.shape[0]), int(q_h.shape[1])
    chunks = [(b, h0, min(Hn, h0 + heads_per_chunk)) for b in range(B) for h0 in range(0, Hn, heads_per_chunk)]
    s_in, s_run, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    caller = torch.cuda.current_stream(dev)
    for s in (s_in, s_run, s_out):
        s.wait_stream(caller)
    shape = (1, heads_per_chunk) + tuple(q_h.shape[2:])
    bufs = [[torch.empty(shape, dtype=q_h.dtype, device=dev) for _ in range(3)] for _ in range(2)]
    outs = [None, None]
    copied, computed, drained = ([None, None] for _ in range(3))
    for i, (b, h0, h1) in enumerate(chunks):
        slot, n = i % 2, h1 - h0
        with torch.cuda.stream(s_in):
            if drained[slot] is not None:
                s_in.wait_event(computed[slot])       # the slot's inputs are no longer read
            for buf, src in zip(bufs[slot], (q_h, k_h, v_h)):
                buf[:, :n].copy_(src[b:b + 1, h0:h1], non_blocking=True)
            copied[slot] = torch.cuda.Event()
            copied[slot].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(copied[slot])
            if drained[slot] is not None:
                s_run.wait_event(drained[slot])       # the slot's previous output has been copied out
            q, k, v = (buf[:, :n] if n == heads_per_chunk else buf[:, :n].contiguous() for buf in bufs[slot])
            outs[slot] = sta_forward(q, k, v, grid, tile, list(window_per_head[h0:h1]), scale, s_run)
            computed[slot] = torch.cuda.Event()
            computed[slot].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[slot])
            outs[slot].record_stream(s_out)       # its memory is reused only after this copy
            out_h[b:b + 1, h0:h1].copy_(outs[slot], non_blocking=True)
            drained[slot] = torch.cuda.Event()
            drained[slot].record(s_out)
    s_out.synchronize()
    s_run.synchronize()

