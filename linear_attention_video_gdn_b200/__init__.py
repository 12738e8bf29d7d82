"""B200 (sm_100a) frame-wise linear-attention recurrences: Python binding.

A thin ctypes layer over ``libgdn_b200.so`` (the C ABI declared in
``include/gdn_b200.h``).  It only marshals arguments: every step of the
recurrences runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.  There is no CPU fallback: importing this package fails
loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python linear_attention_video_gdn_b200/build.py` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NO_DEVICE, ERR_RANGE = range(7)
DTYPE_F32, DTYPE_BF16 = 0, 1
IMPL_AUTO, IMPL_SEQ, IMPL_FRAME_SIMT, IMPL_TC, IMPL_TC_PFORM = 0, 1, 2, 3, 4
OP_GDN, OP_RELU_LA, OP_GDN_BWD = 0, 1, 2
IMPLS = {"auto": IMPL_AUTO, "seq": IMPL_SEQ, "frame_simt": IMPL_FRAME_SIMT, "tc": IMPL_TC,
         "tc_pform": IMPL_TC_PFORM}

EXPORTED = ("gdn_frame_fwd", "relu_la_block_fwd", "gdn_frame_fwd_host", "gdn_frame_fwd_noalloc",
            "gdn_workspace_bytes", "gdn_workspace_bytes_host", "gdn_status_string", "gdn_status_str",
            "gdn_abi_version", "temporal_conv_fwd", "softmax_window_fwd", "gdn_frame_bwd")
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


class GdnOpts(ctypes.Structure):
    _fields_ = [("in_dtype", ctypes.c_int), ("gates_are_logits", ctypes.c_int), ("impl", ctypes.c_int),
                ("stream", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("status", ctypes.c_void_p), ("max_ctas", ctypes.c_int), ("spin_limit_us", ctypes.c_int),
                ("test_withhold_unit", ctypes.c_int), ("segments", ctypes.c_int), ("rope_grid_w", ctypes.c_int),
                ("rope_frame_offset", ctypes.c_int), ("rope_base", ctypes.c_float)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_lib.gdn_frame_fwd.argtypes = [_P] * 8 + [_I] * 6 + [ctypes.POINTER(GdnOpts)]
_lib.gdn_frame_fwd.restype = _I
_lib.gdn_frame_bwd.argtypes = [_P] * 14 + [_I] * 6 + [ctypes.POINTER(GdnOpts)]
_lib.gdn_frame_bwd.restype = _I
_lib.gdn_frame_fwd_host.argtypes = [_P] * 8 + [_I] * 6 + [ctypes.POINTER(GdnOpts)]
_lib.gdn_frame_fwd_host.restype = _I
_lib.gdn_frame_fwd_noalloc.argtypes = [_P] * 8 + [_I] * 6 + [ctypes.POINTER(GdnOpts)]
_lib.gdn_frame_fwd_noalloc.restype = _I
_lib.relu_la_block_fwd.argtypes = [_P] * 8 + [_I] * 6 + [ctypes.c_float, ctypes.POINTER(GdnOpts)]
_lib.relu_la_block_fwd.restype = _I
_lib.temporal_conv_fwd.argtypes = [_P] * 6 + [_I] * 4 + [ctypes.POINTER(GdnOpts)]
_lib.temporal_conv_fwd.restype = _I
_lib.softmax_window_fwd.argtypes = [_P] * 4 + [_I] * 7 + [ctypes.c_float, ctypes.POINTER(GdnOpts)]
_lib.softmax_window_fwd.restype = _I
_lib.gdn_workspace_bytes.argtypes = [_I] * 7 + [ctypes.POINTER(GdnOpts)]
_lib.gdn_workspace_bytes.restype = ctypes.c_size_t
_lib.gdn_workspace_bytes_host.argtypes = [_I] * 6 + [ctypes.POINTER(GdnOpts)]
_lib.gdn_workspace_bytes_host.restype = ctypes.c_size_t
_lib.gdn_status_string.argtypes = [_I]
_lib.gdn_status_string.restype = ctypes.c_char_p
_lib.gdn_abi_version.argtypes = []
_lib.gdn_abi_version.restype = _I


class GdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (code {code})")


def status_string(code: int) -> str:
    return _lib.gdn_status_string(int(code)).decode()


def abi_version() -> int:
    return int(_lib.gdn_abi_version())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def make_opts(in_dtype: int, *, gates_are_logits: bool = True, impl="auto", stream=None, workspace=None,
              status=None, max_ctas: int = 0, spin_limit_us: int = 0, test_withhold_unit: int = -1,
              segments: int = 0, rope=None) -> GdnOpts:
    o = GdnOpts()
    o.in_dtype = in_dtype
    o.gates_are_logits = int(bool(gates_are_logits))
    o.impl = IMPLS[impl] if isinstance(impl, str) else int(impl)
    o.stream = _stream_handle(stream)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    o.status = None if status is None else status.data_ptr()
    o.max_ctas = int(max_ctas)
    o.spin_limit_us = int(spin_limit_us)
    o.test_withhold_unit = int(test_withhold_unit) + 1 if test_withhold_unit >= 0 else 0
    o.segments = int(segments)
    if rope is not None:  # dict(grid_w, frame_offset=0, base=1e4): the 3D RoPE on q and k
        o.rope_grid_w = int(rope["grid_w"])
        o.rope_frame_offset = int(rope.get("frame_offset", 0))
        o.rope_base = float(rope.get("base", 1e4))
    return o


def workspace_bytes(op: int, B, H, F, L, dk, dv, opts: GdnOpts) -> int:
    return int(_lib.gdn_workspace_bytes(op, B, H, F, L, dk, dv, ctypes.byref(opts)))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned device scratch (256-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _check(t, name, shape, dtype, device, allow_none=False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gdn_frame_fwd(q, k, v, alpha, beta, *, F: int, state_in=None, state_out=None, o=None,
                  gates_are_logits: bool = True, impl="auto", workspace=None, stream=None, status=None,
                  max_ctas: int = 0, spin_limit_us: int = 0, test_withhold_unit: int = -1, segments: int = 0,
                  rope=None):
    """Frame-wise Gated DeltaNet forward on the GPU (see include/gdn_b200.h).

    q, k: [B, H, F*L, dk]; v: [B, H, F*L, dv] (float32 or bfloat16, same dtype);
    alpha: [B, H, F] float32; beta: [B, H, F*L] float32; state_in/state_out:
    [B, H, dk, dv] float32 or None.  Returns o [B, H, F*L, dv] float32.
    ``segments``: chunk segments per frame for the tensor-core kernel (0 =
    automatic; see ``gdn_opts.segments``).  ``rope``: None, or
    dict(grid_w, frame_offset=0, base=1e4) for the 3D rotary position
    embedding on q and k (see ``gdn_opts.rope_grid_w``).
    """
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if N % F:
        raise ValueError(f"token count {N} is not a multiple of F={F}")
    L = N // F
    dev = q.device
    _check(k, "k", (B, H, N, dk), q.dtype, dev)
    _check(v, "v", (B, H, N, dv), q.dtype, dev)
    _check(q, "q", (B, H, N, dk), q.dtype, dev)
    _check(alpha, "alpha", (B, H, F), torch.float32, dev)
    _check(beta, "beta", (B, H, N), torch.float32, dev)
    _check(state_in, "state_in", (B, H, dk, dv), torch.float32, dev, allow_none=True)
    _check(state_out, "state_out", (B, H, dk, dv), torch.float32, dev, allow_none=True)
    if o is None:
        o = torch.empty((B, H, N, dv), dtype=torch.float32, device=dev)
    _check(o, "o", (B, H, N, dv), torch.float32, dev)
    opts = make_opts(_dtype_code(q), gates_are_logits=gates_are_logits, impl=impl, stream=stream,
                     status=status, max_ctas=max_ctas, spin_limit_us=spin_limit_us,
                     test_withhold_unit=test_withhold_unit, segments=segments, rope=rope)
    need = workspace_bytes(OP_GDN, B, H, F, L, dk, dv, opts)
    if workspace is None and need > 0:
        workspace = alloc_workspace(need, dev)
    if workspace is not None:
        opts.workspace = workspace.data_ptr()
        opts.workspace_bytes = workspace.numel() * workspace.element_size()
    rc = _lib.gdn_frame_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in), _ptr(state_out),
                            _ptr(o), B, H, F, L, dk, dv, ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "gdn_frame_fwd")
    return o


def gdn_frame_bwd(q, k, v, alpha, beta, d_o, *, F: int, state_in=None, d_state_out=None, out=None,
                  gates_are_logits: bool = True, impl="auto", workspace=None, stream=None, status=None,
                  max_ctas: int = 0, spin_limit_us: int = 0, test_withhold_unit: int = -1, rope=None):
    """Backward of ``gdn_frame_fwd`` on the GPU (see include/gdn_b200.h).

    q, k, v, alpha, beta, state_in: the forward call's inputs; d_o: [B, H, F*L, dv]
    float32 (dL/do); d_state_out: [B, H, dk, dv] float32 or None (zero).  Returns
    a dict of float32 tensors dq, dk [B, H, F*L, dk], dv [B, H, F*L, dv],
    dalpha [B, H, F], dbeta [B, H, F*L] (with respect to the logits when
    ``gates_are_logits``) and dstate_in [B, H, dk, dv].  ``out``: an optional
    dict of preallocated tensors with those names.  ``rope``: the forward's 3D
    RoPE options (dict(grid_w, frame_offset=0, base=1e4)), or None; dq and dk are
    then with respect to the unrotated q and k.
    """
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if N % F:
        raise ValueError(f"token count {N} is not a multiple of F={F}")
    L = N // F
    dev = q.device
    _check(k, "k", (B, H, N, dk), q.dtype, dev)
    _check(v, "v", (B, H, N, dv), q.dtype, dev)
    _check(q, "q", (B, H, N, dk), q.dtype, dev)
    _check(alpha, "alpha", (B, H, F), torch.float32, dev)
    _check(beta, "beta", (B, H, N), torch.float32, dev)
    _check(state_in, "state_in", (B, H, dk, dv), torch.float32, dev, allow_none=True)
    _check(d_o, "d_o", (B, H, N, dv), torch.float32, dev)
    _check(d_state_out, "d_state_out", (B, H, dk, dv), torch.float32, dev, allow_none=True)
    shapes = dict(dq=(B, H, N, dk), dk=(B, H, N, dk), dv=(B, H, N, dv), dalpha=(B, H, F), dbeta=(B, H, N),
                  dstate_in=(B, H, dk, dv))
    out = dict(out or {})
    for name, shp in shapes.items():
        if out.get(name) is None:
            out[name] = torch.empty(shp, dtype=torch.float32, device=dev)
        _check(out[name], name, shp, torch.float32, dev)
    opts = make_opts(_dtype_code(q), gates_are_logits=gates_are_logits, impl=impl, stream=stream,
                     status=status, max_ctas=max_ctas, spin_limit_us=spin_limit_us,
                     test_withhold_unit=test_withhold_unit, rope=rope)
    need = workspace_bytes(OP_GDN_BWD, B, H, F, L, dk, dv, opts)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    opts.workspace = workspace.data_ptr()
    opts.workspace_bytes = workspace.numel() * workspace.element_size()
    rc = _lib.gdn_frame_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in), _ptr(d_o),
                            _ptr(d_state_out), *(_ptr(out[n]) for n in shapes), B, H, F, L, dk, dv,
                            ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "gdn_frame_bwd")
    return out


def relu_la_block_fwd(q, k, v, *, F: int, kv_in=None, z_in=None, kv_out=None, z_out=None, o=None,
                      eps: float = 1e-6, impl="auto", workspace=None, stream=None, status=None,
                      max_ctas: int = 0, spin_limit_us: int = 0, test_withhold_unit: int = -1):
    """Block-causal ReLU linear attention forward on the GPU (see include/gdn_b200.h)."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if N % F:
        raise ValueError(f"token count {N} is not a multiple of F={F}")
    L = N // F
    dev = q.device
    _check(k, "k", (B, H, N, dk), q.dtype, dev)
    _check(v, "v", (B, H, N, dv), q.dtype, dev)
    _check(q, "q", (B, H, N, dk), q.dtype, dev)
    for t, nm, shp in ((kv_in, "kv_in", (B, H, dk, dv)), (kv_out, "kv_out", (B, H, dk, dv)),
                       (z_in, "z_in", (B, H, dk)), (z_out, "z_out", (B, H, dk))):
        _check(t, nm, shp, torch.float32, dev, allow_none=True)
    if o is None:
        o = torch.empty((B, H, N, dv), dtype=torch.float32, device=dev)
    _check(o, "o", (B, H, N, dv), torch.float32, dev)
    opts = make_opts(_dtype_code(q), impl=impl, stream=stream, status=status, max_ctas=max_ctas,
                     spin_limit_us=spin_limit_us, test_withhold_unit=test_withhold_unit)
    need = workspace_bytes(OP_RELU_LA, B, H, F, L, dk, dv, opts)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    opts.workspace = workspace.data_ptr()
    opts.workspace_bytes = workspace.numel() * workspace.element_size()
    rc = _lib.relu_la_block_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_in), _ptr(z_in), _ptr(kv_out), _ptr(z_out),
                                _ptr(o), B, H, F, L, dk, dv, float(eps), ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "relu_la_block_fwd")
    return o


def temporal_conv_fwd(x, w, *, bias=None, cache_in=None, cache_out=None, y=None, stream=None, max_ctas: int = 0):
    """Causal temporal convolution of one block of frames with the block-boundary
    cache on the GPU (see include/gdn_b200.h).  x: [B, F, HW, C] float32 or
    bfloat16; w: [C, 3] float32; bias: [C] float32 or None; cache_in /
    cache_out: [B, HW, C] of x's dtype or None.  Returns y (x's shape and dtype)."""
    B, F, HW, C = x.shape
    dev = x.device
    _check(x, "x", (B, F, HW, C), x.dtype, dev)
    _check(w, "w", (C, 3), torch.float32, dev)
    _check(bias, "bias", (C,), torch.float32, dev, allow_none=True)
    _check(cache_in, "cache_in", (B, HW, C), x.dtype, dev, allow_none=True)
    _check(cache_out, "cache_out", (B, HW, C), x.dtype, dev, allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", (B, F, HW, C), x.dtype, dev)
    opts = make_opts(_dtype_code(x), stream=stream, max_ctas=max_ctas)
    rc = _lib.temporal_conv_fwd(_ptr(x), _ptr(w), _ptr(bias), _ptr(cache_in), _ptr(cache_out), _ptr(y),
                                B, F, HW, C, ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "temporal_conv_fwd")
    return y


def softmax_window_fwd(q, k, v, *, F: int, W: int, scale: float = 0.0, o=None, impl="auto", stream=None,
                       status=None, spin_limit_us: int = 0):
    """Windowed block-causal softmax attention on the GPU (see include/gdn_b200.h):
    q, k [B, H, F*L, dk] and v [B, H, F*L, dv] bfloat16 or float32; token t of
    frame f attends to frames max(0, f-W+1) .. f.  Returns o [B, H, F*L, dv] float32."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if N % F:
        raise ValueError(f"token count {N} is not a multiple of F={F}")
    L = N // F
    dev = q.device
    _check(q, "q", (B, H, N, dk), q.dtype, dev)
    _check(k, "k", (B, H, N, dk), q.dtype, dev)
    _check(v, "v", (B, H, N, dv), q.dtype, dev)
    if o is None:
        o = torch.empty((B, H, N, dv), dtype=torch.float32, device=dev)
    _check(o, "o", (B, H, N, dv), torch.float32, dev)
    opts = make_opts(_dtype_code(q), impl=impl, stream=stream, status=status, spin_limit_us=spin_limit_us)
    rc = _lib.softmax_window_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, F, L, dk, dv, int(W), float(scale),
                                 ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "softmax_window_fwd")
    return o


def gdn_frame_fwd_host(q, k, v, alpha, beta, *, F: int, o, state_in=None, state_out=None,
                       gates_are_logits: bool = True, impl="auto", workspace=None, stream=None, status=None,
                       rope=None):
    """gdn_frame_fwd with HOST (CPU, ideally pinned) tensors; synchronous.

    Copies inputs into ``workspace`` (a device uint8 tensor of at least
    ``host_workspace_bytes(...)`` bytes), runs, and copies o/state_out back.
    """
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    L = N // F
    for t in (q, k, v, alpha, beta, o, state_in, state_out):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError("gdn_frame_fwd_host takes contiguous CPU tensors")
    opts = make_opts(_dtype_code(q), gates_are_logits=gates_are_logits, impl=impl, stream=stream, status=status,
                     rope=rope)
    need = host_workspace_bytes(B, H, F, L, dk, dv, opts)
    if workspace is None:
        workspace = alloc_workspace(need, torch.device("cuda", torch.cuda.current_device()))
    opts.workspace = workspace.data_ptr()
    opts.workspace_bytes = workspace.numel() * workspace.element_size()
    rc = _lib.gdn_frame_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in),
                                 _ptr(state_out), _ptr(o), B, H, F, L, dk, dv, ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "gdn_frame_fwd_host")
    return o


def host_workspace_bytes(B, H, F, L, dk, dv, opts: GdnOpts) -> int:
    return int(_lib.gdn_workspace_bytes_host(B, H, F, L, dk, dv, ctypes.byref(opts)))


def gdn_frame_fwd_noalloc(q, k, v, alpha, beta, *, F: int, state_in=None, state_out=None, o=None,
                          gates_are_logits: bool = True, impl="auto", stream=None, status=None):
    """gdn_frame_fwd for callers that cannot allocate device memory.

    Same arguments and result as gdn_frame_fwd, but the frame-chain scratch is
    a fixed array inside the library (NOALLOC_SCRATCH_BYTES per GPU) instead of
    a caller workspace; sizes that need more scratch raise GdnError
    (ERR_UNSUPPORTED).  Calls share that array, so calls that could overlap on
    the GPU must be serialised.  ``o`` should be passed by callers that cannot
    allocate; when it is None this wrapper (not the library) creates it.
    """
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if N % F:
        raise ValueError(f"token count {N} is not a multiple of F={F}")
    L = N // F
    dev = q.device
    _check(k, "k", (B, H, N, dk), q.dtype, dev)
    _check(v, "v", (B, H, N, dv), q.dtype, dev)
    _check(alpha, "alpha", (B, H, F), torch.float32, dev)
    _check(beta, "beta", (B, H, N), torch.float32, dev)
    _check(state_in, "state_in", (B, H, dk, dv), torch.float32, dev, allow_none=True)
    _check(state_out, "state_out", (B, H, dk, dv), torch.float32, dev, allow_none=True)
    if o is None:
        o = torch.empty((B, H, N, dv), dtype=torch.float32, device=dev)
    _check(o, "o", (B, H, N, dv), torch.float32, dev)
    opts = make_opts(_dtype_code(q), gates_are_logits=gates_are_logits, impl=impl, stream=stream, status=status)
    rc = _lib.gdn_frame_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in),
                                    _ptr(state_out), _ptr(o), B, H, F, L, dk, dv, ctypes.byref(opts))
    if rc != OK:
        raise GdnError(rc, "gdn_frame_fwd_noalloc")
    return o
