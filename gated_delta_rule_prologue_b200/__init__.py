"""Python binding of libkda (KDA recurrence hot path for B200 / sm_100a).

Argument marshalling only: every function hands raw device pointers, sizes
and the current CUDA stream of ``torch`` to the C ABI declared in
``include/kda.h`` and raises :class:`KdaError` on a non-OK status.  All work
runs in the library's CUDA kernels; there is no other implementation behind
these names, and importing fails loudly when ``libkda.so`` has not been built
(``python -m gated_delta_rule_prologue_b200.build``).  With the environment variable
``KDA_LIB=debug`` the bounds-checked build ``libkda_debug.so`` is loaded instead.

Tensor conventions (all contiguous, on the current CUDA device):
  q, k, v              [T, H, D]       float32, bfloat16 or float16
  o                    [T, H, D]       float32 (read-outs are always float32)
  g                    [T, H, Dk]      float32 (log-decay, alpha = exp(g))
  beta                 [T, H]          float32
  state                [N, H, Dv, Dk]  float32 (key index contiguous)
  x (projections)      [T, 3*H*D]      activation dtype, channel p*H*D + h*D + d
  conv_w               [3*H*D, 4]      float32
  conv cache           [N, 3, 3*H*D]   activation dtype, oldest row first
  cu_seqlens           [N+1]           int32
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "KdaError",
    "LIB_PATH",
    "lib",
    "kda_prologue",
    "kda_chunk_fwd",
    "kda_chunk_fwd_windowed_workspace_bytes",
    "kda_decode_step",
    "kda_prologue_chunk_fwd",
    "kda_get_device_status",
    "kda_selftest_wait_timeout",
    "kda_selftest_bounds",
    "kda_debug_build",
    "kda_version",
    "KDA_OK",
    "KDA_ERR_INVALID_ARG",
    "KDA_ERR_UNSUPPORTED",
    "KDA_ERR_CUDA",
    "KDA_ERR_DEVICE_TIMEOUT",
    "KDA_ERR_DEVICE_BOUNDS",
    "KDA_ERR_DEVICE_RANGE",
]

# KDA_LIB=debug selects the bounds-checked build (libkda_debug.so, built by
# ``python -m gated_delta_rule_prologue_b200.build --debug``); anything else, the release build.
_LIB_NAME = "libkda_debug.so" if os.environ.get("KDA_LIB") == "debug" else "libkda.so"
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIB_NAME)

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_CUDA = 3
KDA_ERR_DEVICE_TIMEOUT = 4
KDA_ERR_DEVICE_BOUNDS = 5
KDA_ERR_DEVICE_RANGE = 6
_F32, _BF16, _F16 = 0, 1, 2


class KdaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libkda status {status}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m gated_delta_rule_prologue_b200.build`")

lib = ctypes.CDLL(LIB_PATH)
_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
lib.kda_prologue.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                             _vp]
lib.kda_chunk_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i, _i, _i,
                              _i, _vp, _vp, _vp]
lib.kda_chunk_fwd_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                 _i, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.kda_chunk_fwd_static.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i, _i,
                                     _i, _i, _vp, _vp, _vp]
lib.kda_prologue_chunk_fwd_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i,
                                          _i, _i, _i, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.kda_chunk_fwd_gated_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _f, _vp, _vp, _i,
                                       _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, ctypes.c_size_t,
                                       _vp]
lib.kda_prologue_chunk_fwd_gated_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _f,
                                                _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                                ctypes.c_size_t, _vp]
lib.kda_decode_step_gated.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _f, _vp, _i, _i, _i,
                                      _i, _vp, _vp]
lib.kda_output_epilogue.argtypes = [_vp, _vp, _vp, _f, _i, _i, _i, _i, _vp, _vp]
lib.kda_chunk_fwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i]
lib.kda_chunk_fwd_workspace_bytes.restype = ctypes.c_size_t
lib.kda_chunk_fwd_segmented_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
lib.kda_chunk_fwd_segmented_workspace_bytes.restype = ctypes.c_size_t
lib.kda_chunk_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i]
lib.kda_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
lib.kda_chunk_bwd_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                 _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                 _vp]
lib.kda_chunk_map_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i]
lib.kda_chunk_map_workspace_bytes.restype = ctypes.c_size_t
lib.kda_chunk_map_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp,
                                 _vp, ctypes.c_size_t, _vp]
lib.kda_state_compose.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _vp]
lib.kda_chunk_fwd_segment_chunks.argtypes = [_i, _i, _i]
lib.kda_chunk_fwd_segment_chunks.restype = ctypes.c_int
lib.kda_chunk_fwd_segmented_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i,
                                           _i, _i, _i, _vp, _vp, _i, _vp, ctypes.c_size_t, _vp]
lib.kda_chunk_fwd_windowed_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i,
                                          _i, _i, _i, _vp, _vp, _i, _vp, ctypes.c_size_t, _vp]
lib.kda_chunk_fwd_windowed_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
lib.kda_prologue_chunk_fwd_windowed_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                                                   _i, _i, _i, _i, _i, _vp, _vp, _i, _vp,
                                                   ctypes.c_size_t, _vp]
lib.kda_chunk_fwd_windowed_workspace_bytes.restype = ctypes.c_size_t
lib.kda_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _f, _vp, _i, _i, _i, _i, _vp, _vp]
lib.kda_prologue_chunk_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i,
                                       _i, _i, _vp, _vp, _vp]
lib.kda_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
lib.kda_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp]
lib.kda_selftest_bounds.argtypes = [_i, _vp]
lib.kda_debug_build.argtypes = []
lib.kda_debug_build.restype = ctypes.c_int
for _fn in (lib.kda_prologue, lib.kda_chunk_fwd, lib.kda_chunk_fwd_ws, lib.kda_chunk_fwd_static,
            lib.kda_chunk_fwd_segmented_ws, lib.kda_chunk_fwd_windowed_ws,
            lib.kda_prologue_chunk_fwd_windowed_ws,
            lib.kda_chunk_bwd_ws, lib.kda_chunk_map_ws,
            lib.kda_state_compose,
            lib.kda_prologue_chunk_fwd_ws, lib.kda_decode_step, lib.kda_chunk_fwd_gated_ws,
            lib.kda_prologue_chunk_fwd_gated_ws, lib.kda_decode_step_gated,
            lib.kda_output_epilogue,
            lib.kda_prologue_chunk_fwd, lib.kda_get_device_status,
            lib.kda_selftest_wait_timeout, lib.kda_selftest_bounds):
    _fn.restype = ctypes.c_int
lib.kda_last_error.restype = ctypes.c_char_p
lib.kda_last_error.argtypes = []
lib.kda_version.restype = ctypes.c_char_p
lib.kda_version.argtypes = []


def _check(status: int):
    if status != KDA_OK:
        raise KdaError(status, lib.kda_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


def _dtype(t) -> int:
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    if t.dtype == torch.float16:
        return _F16
    raise TypeError(f"unsupported activation dtype {t.dtype}")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None):
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def kda_version() -> str:
    return lib.kda_version().decode()


def kda_get_device_status() -> int:
    """Read and clear the current device's status word (0 = no fault)."""
    code = ctypes.c_int(0)
    _check(lib.kda_get_device_status(ctypes.byref(code)))
    return code.value


def kda_selftest_wait_timeout(limit_us: int = 1000, stream=None):
    """Launch one CTA whose bounded mbarrier wait runs out after ``limit_us``
    microseconds; it records KDA_ERR_DEVICE_TIMEOUT in the status word and
    returns without faulting (the failure path of every tensor-core kernel)."""
    _check(lib.kda_selftest_wait_timeout(int(limit_us), _stream(stream)))


def kda_debug_build() -> bool:
    """True when the loaded library is the bounds-checked build (KDA_LIB=debug)."""
    return bool(lib.kda_debug_build())


def kda_selftest_bounds(index: int, stream=None):
    """Debug build only: one checked write of a four-slot device probe at ``index``;
    outside [0, 4) it records KDA_ERR_DEVICE_BOUNDS and skips the write."""
    _check(lib.kda_selftest_bounds(int(index), _stream(stream)))


def kda_prologue(x, conv_w, q, k, v, *, H: int, D: int, cache_in=None, cache_out=None,
                 cu_seqlens=None, stream=None):
    """Short conv + SiLU + L2 on q/k: writes ``q, k, v`` [T, H, D] (and ``cache_out``).
    ``x`` and the caches share one dtype; ``q, k, v`` share another."""
    for t, n in ((x, "x"), (cache_in, "cache_in"), (cache_out, "cache_out")):
        _need(t, n, x.dtype)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(conv_w, "conv_w", torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    T = x.shape[0]
    _check(lib.kda_prologue(_ptr(x), _ptr(conv_w), _ptr(cache_in), _ptr(cache_out),
                            _ptr(cu_seqlens), N, T, H, D, _dtype(x), _dtype(q), _ptr(q),
                            _ptr(k), _ptr(v), _stream(stream)))


def kda_chunk_fwd_workspace_bytes(N: int, T: int, H: int, Dk: int, Dv: int, chunk: int,
                                  dtype: torch.dtype) -> int:
    """Scratch bytes of the two-pass tensor-core prefill (0 if it does not apply)."""
    return int(lib.kda_chunk_fwd_workspace_bytes(N, T, H, Dk, Dv, chunk, _DTYPES[dtype]))


def kda_chunk_fwd_segment_chunks(N: int, T: int, H: int) -> int:
    """Segment length (in 64-token chunks) of the sequence-parallel state pass
    that the workspace entry points pick for these sizes (0: whole sequences)."""
    return int(lib.kda_chunk_fwd_segment_chunks(N, T, H))


def kda_chunk_fwd_segmented_workspace_bytes(N: int, T: int, H: int, Dk: int, Dv: int, chunk: int,
                                            dtype: torch.dtype, segment_chunks: int) -> int:
    """Scratch bytes of the two-pass prefill at an explicit segment length."""
    return int(lib.kda_chunk_fwd_segmented_workspace_bytes(N, T, H, Dk, Dv, chunk,
                                                           _DTYPES[dtype], segment_chunks))


def kda_chunk_fwd(q, k, v, g, beta, o, *, scale: float = 1.0, initial_state=None,
                  final_state=None, cu_seqlens=None, chunk: int = 64, workspace="auto",
                  segment_chunks=None, window_chunks=None, stream=None):
    """Chunkwise prefill: writes ``o`` [T, H, Dv] and optionally ``final_state``.

    ``workspace``: ``"auto"`` allocates the two-pass path's scratch from
    torch's caching allocator; a uint8 CUDA tensor is used as given (at least
    :func:`kda_chunk_fwd_workspace_bytes`); ``None`` runs the one-pass kernels.
    ``segment_chunks``: ``None`` lets the library pick the state pass's segment
    length; an int (0: whole sequences) calls ``kda_chunk_fwd_segmented_ws``
    with it (workspace sized by :func:`kda_chunk_fwd_segmented_workspace_bytes`).
    ``window_chunks``: an int >= 1 calls ``kda_chunk_fwd_windowed_ws``: the passes run
    one window of that many chunk numbers at a time, so the workspace (sized by
    :func:`kda_chunk_fwd_windowed_workspace_bytes`) does not grow with T.
    """
    if window_chunks is not None:
        return _chunk_fwd_windowed(q, k, v, g, beta, o, scale, initial_state, final_state,
                                   cu_seqlens, chunk, workspace, int(window_chunks), stream)
    if segment_chunks is not None:
        return _chunk_fwd_segmented(q, k, v, g, beta, o, scale, initial_state, final_state,
                                    cu_seqlens, chunk, workspace, int(segment_chunks), stream)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    for t, n in ((o, "o"), (g, "g"), (beta, "beta"), (initial_state, "initial_state"),
                 (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto', None or a tensor, not {workspace!r}")
        nbytes = kda_chunk_fwd_workspace_bytes(N, T, H, Dk, Dv, chunk, q.dtype)
        workspace = (torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None)
    if workspace is None:
        _check(lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                 _ptr(initial_state), _ptr(cu_seqlens), N, T, H, Dk, Dv, chunk,
                                 _dtype(q), _ptr(o), _ptr(final_state), _stream(stream)))
        return
    _need(workspace, "workspace", torch.uint8)
    _check(lib.kda_chunk_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                _ptr(initial_state), _ptr(cu_seqlens), N, T, H, Dk, Dv, chunk,
                                _dtype(q), _ptr(o), _ptr(final_state), _ptr(workspace),
                                workspace.numel(), _stream(stream)))


def kda_chunk_fwd_windowed_workspace_bytes(N, T, H, Dk, Dv, chunk, dtype, window_chunks) -> int:
    return int(lib.kda_chunk_fwd_windowed_workspace_bytes(N, T, H, Dk, Dv, chunk,
                                                          _DTYPES[dtype], window_chunks))


def _chunk_fwd_windowed(q, k, v, g, beta, o, scale, initial_state, final_state, cu_seqlens,
                        chunk, workspace, window_chunks, stream):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    for t, n in ((o, "o"), (g, "g"), (beta, "beta"), (initial_state, "initial_state"),
                 (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto' or a tensor, not {workspace!r}")
        nbytes = kda_chunk_fwd_windowed_workspace_bytes(N, T, H, Dk, Dv, chunk, q.dtype,
                                                        window_chunks)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    _check(lib.kda_chunk_fwd_windowed_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         float(scale), _ptr(initial_state), _ptr(cu_seqlens), N,
                                         T, H, Dk, Dv, chunk, _dtype(q), _ptr(o),
                                         _ptr(final_state), int(window_chunks), _ptr(workspace),
                                         workspace.numel(), _stream(stream)))


def _chunk_fwd_segmented(q, k, v, g, beta, o, scale, initial_state, final_state, cu_seqlens,
                         chunk, workspace, segment_chunks, stream):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    for t, n in ((o, "o"), (g, "g"), (beta, "beta"), (initial_state, "initial_state"),
                 (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto' or a tensor, not {workspace!r}")
        nbytes = kda_chunk_fwd_segmented_workspace_bytes(N, T, H, Dk, Dv, chunk, q.dtype,
                                                         segment_chunks)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    _check(lib.kda_chunk_fwd_segmented_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                          float(scale), _ptr(initial_state), _ptr(cu_seqlens), N,
                                          T, H, Dk, Dv, chunk, _dtype(q), _ptr(o),
                                          _ptr(final_state), segment_chunks, _ptr(workspace),
                                          workspace.numel(), _stream(stream)))


def kda_chunk_bwd_workspace_bytes(N: int, T: int, H: int, Dk: int, Dv: int, chunk: int,
                                  dtype: torch.dtype) -> int:
    """Scratch bytes of :func:`kda_chunk_bwd` (0 off the tensor-core shapes)."""
    return int(lib.kda_chunk_bwd_workspace_bytes(N, T, H, Dk, Dv, chunk, _DTYPES[dtype]))


def kda_chunk_bwd(q, k, v, g, beta, d_o, *, scale: float = 1.0, initial_state=None,
                  d_final_state=None, cu_seqlens=None, chunk: int = 64, dq=None, dk=None,
                  dv=None, dg=None, dbeta=None, d_initial_state=None, want_d_initial_state=True,
                  workspace="auto", stream=None):
    """Gradients of :func:`kda_chunk_fwd` for L = sum(d_o * o) + sum(d_final_state *
    final_state).  Returns ``(dq, dk, dv, dg, dbeta, d_initial_state)`` (fp32; the
    last is None unless wanted); output tensors not given are allocated."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    for t, n in ((g, "g"), (beta, "beta"), (d_o, "d_o"), (initial_state, "initial_state"),
                 (d_final_state, "d_final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    dev = q.device
    dq = torch.empty((T, H, Dk), device=dev) if dq is None else dq
    dk = torch.empty((T, H, Dk), device=dev) if dk is None else dk
    dv = torch.empty((T, H, Dv), device=dev) if dv is None else dv
    dg = torch.empty((T, H, Dk), device=dev) if dg is None else dg
    dbeta = torch.empty((T, H), device=dev) if dbeta is None else dbeta
    if d_initial_state is None and want_d_initial_state:
        d_initial_state = torch.empty((N, H, Dv, Dk), device=dev)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dg, "dg"), (dbeta, "dbeta"),
                 (d_initial_state, "d_initial_state")):
        _need(t, n, torch.float32)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto' or a tensor, not {workspace!r}")
        nbytes = kda_chunk_bwd_workspace_bytes(N, T, H, Dk, Dv, chunk, q.dtype)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8)
    _check(lib.kda_chunk_bwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                _ptr(initial_state), _ptr(cu_seqlens), N, T, H, Dk, Dv, chunk,
                                _dtype(q), _ptr(d_o), _ptr(d_final_state), _ptr(dq), _ptr(dk),
                                _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(d_initial_state),
                                _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv, dg, dbeta, d_initial_state


def kda_chunk_map(q, k, v, g, beta, *, cu_seqlens=None, chunk: int = 64, M=None, B=None,
                  workspace="auto", stream=None):
    """Affine map of each sequence's prefill, final = M S0 + B: returns ``(M, B)``,
    both [N, H, D, D] fp32 stored like a state (column-major)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    for t, n in ((g, "g"), (beta, "beta")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    M = torch.empty((N, H, Dk, Dk), device=q.device) if M is None else M
    B = torch.empty((N, H, Dv, Dk), device=q.device) if B is None else B
    _need(M, "M", torch.float32)
    _need(B, "B", torch.float32)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto' or a tensor, not {workspace!r}")
        nbytes = int(lib.kda_chunk_map_workspace_bytes(N, T, H, Dk, Dv, chunk, _DTYPES[q.dtype]))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    _check(lib.kda_chunk_map_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N,
                                T, H, Dk, Dv, chunk, _dtype(q), _ptr(M), _ptr(B), _ptr(workspace),
                                workspace.numel(), _stream(stream)))
    return M, B


def kda_state_compose(M, B, E_in, E_out=None, stream=None):
    """E_out = M E_in + B per (sequence, head) (E_in None: zero); returns E_out."""
    for t, n in ((M, "M"), (B, "B"), (E_in, "E_in")):
        _need(t, n, torch.float32)
    N, H, D = B.shape[0], B.shape[1], B.shape[2]
    E_out = torch.empty_like(B) if E_out is None else E_out
    _need(E_out, "E_out", torch.float32)
    _check(lib.kda_state_compose(_ptr(M), _ptr(B), _ptr(E_in), _ptr(E_out), N, H, D,
                                 _stream(stream)))
    return E_out


# Size of the library's fixed scratch buffer (one per device) used by
# kda_chunk_fwd_static; equals KDA_CHUNK_STATIC_SCRATCH_BYTES in kda.h.
KDA_CHUNK_STATIC_SCRATCH_BYTES = 64 << 20


def kda_chunk_fwd_static(q, k, v, g, beta, o, *, scale: float = 1.0, initial_state=None,
                         final_state=None, cu_seqlens=None, chunk: int = 64, stream=None):
    """The two-pass prefill with the library's fixed scratch buffer instead of
    a workspace: allocates nothing.  Sizes needing more scratch than
    KDA_CHUNK_STATIC_SCRATCH_BYTES raise KdaError (KDA_ERR_UNSUPPORTED).  All
    calls on a device share the buffer, so calls that may overlap in time
    (different streams) race; calls in order on one stream are safe."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    for t, n in ((o, "o"), (g, "g"), (beta, "beta"), (initial_state, "initial_state"),
                 (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib.kda_chunk_fwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                    _ptr(initial_state), _ptr(cu_seqlens), N, T, H, Dk, Dv,
                                    chunk, _dtype(q), _ptr(o), _ptr(final_state),
                                    _stream(stream)))


def kda_prologue_chunk_fwd(x, conv_w, g, beta, o, *, H: int, D: int, scale: float = 1.0,
                           cache_in=None, cache_out=None, initial_state=None, final_state=None,
                           cu_seqlens=None, workspace="auto", window_chunks=None, stream=None):
    """Prologue fused into the chunkwise prefill (chunk 64): ``x`` [T, 3*H*D]
    bf16/fp16 projections in, ``o`` [T, H, D] float32 out; q, k, v stay on chip.

    ``workspace`` as in :func:`kda_chunk_fwd`: ``"auto"`` (two passes, scratch
    from torch's caching allocator), a uint8 CUDA tensor, or ``None`` (the
    one-pass kernel).  ``window_chunks``: an int >= 1 calls
    ``kda_prologue_chunk_fwd_windowed_ws`` (a workspace that does not grow with T)."""
    for t, n in ((x, "x"), (cache_in, "cache_in"), (cache_out, "cache_out")):
        _need(t, n, x.dtype)
    for t, n in ((conv_w, "conv_w"), (o, "o"), (g, "g"), (beta, "beta"),
                 (initial_state, "initial_state"), (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    T = x.shape[0]
    if window_chunks is not None:
        if isinstance(workspace, str):
            if workspace != "auto":
                raise ValueError(f"workspace must be 'auto' or a tensor, not {workspace!r}")
            nbytes = kda_chunk_fwd_windowed_workspace_bytes(N, T, H, D, D, 64, x.dtype,
                                                            int(window_chunks))
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        _need(workspace, "workspace", torch.uint8)
        _check(lib.kda_prologue_chunk_fwd_windowed_ws(
            _ptr(x), _ptr(conv_w), _ptr(cache_in), _ptr(cache_out), _ptr(g), _ptr(beta),
            float(scale), _ptr(initial_state), _ptr(cu_seqlens), N, T, H, D, _dtype(x), _ptr(o),
            _ptr(final_state), int(window_chunks), _ptr(workspace), workspace.numel(),
            _stream(stream)))
        return
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto', None or a tensor, not {workspace!r}")
        nbytes = kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, x.dtype)
        workspace = (torch.empty(nbytes, dtype=torch.uint8, device=x.device) if nbytes else None)
    if workspace is None:
        _check(lib.kda_prologue_chunk_fwd(_ptr(x), _ptr(conv_w), _ptr(cache_in), _ptr(cache_out),
                                          _ptr(g), _ptr(beta), float(scale), _ptr(initial_state),
                                          _ptr(cu_seqlens), N, T, H, D, _dtype(x), _ptr(o),
                                          _ptr(final_state), _stream(stream)))
        return
    _need(workspace, "workspace", torch.uint8)
    _check(lib.kda_prologue_chunk_fwd_ws(_ptr(x), _ptr(conv_w), _ptr(cache_in), _ptr(cache_out),
                                         _ptr(g), _ptr(beta), float(scale), _ptr(initial_state),
                                         _ptr(cu_seqlens), N, T, H, D, _dtype(x), _ptr(o),
                                         _ptr(final_state), _ptr(workspace), workspace.numel(),
                                         _stream(stream)))


def kda_decode_step(x, conv_w, conv_cache, g, beta, state, o, *, H: int, D: int,
                    scale: float = 1.0, stream=None):
    """One decode token per sequence; updates ``state`` and ``conv_cache`` in place."""
    for t, n in ((x, "x"), (conv_cache, "conv_cache")):
        _need(t, n, x.dtype)
    for t, n in ((o, "o"), (conv_w, "conv_w"), (g, "g"), (beta, "beta"), (state, "state")):
        _need(t, n, torch.float32)
    N = x.shape[0]
    _check(lib.kda_decode_step(_ptr(x), _ptr(conv_w), _ptr(conv_cache), _ptr(g), _ptr(beta),
                               float(scale), _ptr(state), N, H, D, _dtype(x), _ptr(o),
                               _stream(stream)))


def _auto_workspace(workspace, N, T, H, D, dtype, device):
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError(f"workspace must be 'auto' or a tensor, not {workspace!r}")
        nbytes = kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, dtype)
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8)
    return workspace


def kda_chunk_fwd_gated(q, k, v, g_raw, beta, o, *, A_log=None, dt_bias=None,
                        lower_bound: float = -5.0, scale: float = 1.0, initial_state=None,
                        final_state=None, cu_seqlens=None, chunk: int = 64, workspace="auto",
                        stream=None):
    """Two-pass prefill with the log-decay computed in the kernel from the gate
    pre-activations ``g_raw`` [T, H, Dk] (q's dtype):
    g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :]))."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g_raw, "g_raw")):
        _need(t, n, q.dtype)
    for t, n in ((o, "o"), (beta, "beta"), (A_log, "A_log"), (dt_bias, "dt_bias"),
                 (initial_state, "initial_state"), (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    workspace = _auto_workspace(workspace, N, T, H, Dk, q.dtype, q.device)
    _check(lib.kda_chunk_fwd_gated_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g_raw), _ptr(A_log),
                                      _ptr(dt_bias), float(lower_bound), _ptr(beta), float(scale),
                                      _ptr(initial_state), _ptr(cu_seqlens), N, T, H, Dk, Dv,
                                      chunk, _dtype(q), _ptr(o), _ptr(final_state),
                                      _ptr(workspace), workspace.numel(), _stream(stream)))


def kda_prologue_chunk_fwd_gated(x, conv_w, g_raw, beta, o, *, H: int, D: int, A_log=None,
                                 dt_bias=None, lower_bound: float = -5.0, scale: float = 1.0,
                                 cache_in=None, cache_out=None, initial_state=None,
                                 final_state=None, cu_seqlens=None, workspace="auto",
                                 stream=None):
    """Fused two-pass prefill (prologue in the prep pass) with the in-kernel gate."""
    for t, n in ((x, "x"), (g_raw, "g_raw"), (cache_in, "cache_in"), (cache_out, "cache_out")):
        _need(t, n, x.dtype)
    for t, n in ((conv_w, "conv_w"), (o, "o"), (beta, "beta"), (A_log, "A_log"),
                 (dt_bias, "dt_bias"), (initial_state, "initial_state"),
                 (final_state, "final_state")):
        _need(t, n, torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    T = x.shape[0]
    workspace = _auto_workspace(workspace, N, T, H, D, x.dtype, x.device)
    _check(lib.kda_prologue_chunk_fwd_gated_ws(_ptr(x), _ptr(conv_w), _ptr(cache_in),
                                               _ptr(cache_out), _ptr(g_raw), _ptr(A_log),
                                               _ptr(dt_bias), float(lower_bound), _ptr(beta),
                                               float(scale), _ptr(initial_state),
                                               _ptr(cu_seqlens), N, T, H, D, _dtype(x), _ptr(o),
                                               _ptr(final_state), _ptr(workspace),
                                               workspace.numel(), _stream(stream)))


def kda_decode_step_gated(x, conv_w, conv_cache, g_raw, beta, state, o, *, H: int, D: int,
                          A_log=None, dt_bias=None, lower_bound: float = -5.0,
                          scale: float = 1.0, stream=None):
    """Decode step with the in-kernel gate; ``g_raw`` [N, H, D] of x's dtype."""
    for t, n in ((x, "x"), (conv_cache, "conv_cache"), (g_raw, "g_raw")):
        _need(t, n, x.dtype)
    for t, n in ((o, "o"), (conv_w, "conv_w"), (beta, "beta"), (state, "state"),
                 (A_log, "A_log"), (dt_bias, "dt_bias")):
        _need(t, n, torch.float32)
    N = x.shape[0]
    _check(lib.kda_decode_step_gated(_ptr(x), _ptr(conv_w), _ptr(conv_cache), _ptr(g_raw),
                                     _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(beta),
                                     float(scale), _ptr(state), N, H, D, _dtype(x), _ptr(o),
                                     _stream(stream)))


def kda_output_epilogue(o, gate, weight, out, *, eps: float = 1e-5, stream=None):
    """Per-head RMSNorm of the read-out ``o`` [T, H, D] (f32) times the output
    gate: out = o / sqrt(mean(o^2) + eps) * weight * sigmoid(gate); ``gate`` and
    ``out`` share a dtype."""
    _need(o, "o", torch.float32)
    _need(weight, "weight", torch.float32)
    _need(gate, "gate", out.dtype)
    _need(out, "out", out.dtype)
    T, H, D = o.shape
    _check(lib.kda_output_epilogue(_ptr(o), _ptr(gate), _ptr(weight), float(eps), T, H, D,
                                   _dtype(out), _ptr(out), _stream(stream)))
