"""CPU oracle for the frame recurrences (fp64), as a ctypes binding of oracle.c.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the library path
(``linear_attention_video_gdn_b200``) never does.  It shares no code with the
CUDA path.

What is computed, and the passages it follows, is stated at the top of
``oracle.c``.  Parity is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (brute-force dense products, closed forms,
invariants, O(N^2) masked attention) and, for the backward ``gdn_bwd``, by
``tests/test_oracle_bwd_pins.py`` (finite differences of the forward, torch
autograd through an independent loop, closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

KEY_NORM_EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile liboracle.so in place (gcc -O2, strict IEEE double: no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", _LIB, _SRC, "-lm", "-lpthread"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_gdn.argtypes = [P, P, P, P, P, ctypes.c_int, P, P, P, I64, I64, I64, I64, I64, I64,
                                   I64, I64, P, I64, I64, ctypes.c_int, I64, I64, ctypes.c_double]
        lib.oracle_rope3d.argtypes = [P, P, I64, I64, I64, I64, I64, I64, ctypes.c_double]
        lib.oracle_rope3d.restype = ctypes.c_int
        lib.oracle_softmax_window.argtypes = [P, P, P, P, I64, I64, I64, I64, I64, I64, I64, ctypes.c_double, P,
                                              ctypes.c_int]
        lib.oracle_softmax_window.restype = ctypes.c_int
        lib.oracle_temporal_conv.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64]
        lib.oracle_temporal_conv.restype = ctypes.c_int
        lib.oracle_gdn.restype = ctypes.c_int
        lib.oracle_gdn_bwd.argtypes = [P, P, P, P, P, ctypes.c_int, P, P, P, P, P, P, P, P, P,
                                       I64, I64, I64, I64, I64, I64, P, I64, ctypes.c_int, I64, I64, ctypes.c_double]
        lib.oracle_gdn_bwd.restype = ctypes.c_int
        lib.oracle_relu_la.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I64, I64, I64, ctypes.c_double,
                                       ctypes.c_int]
        lib.oracle_relu_la.restype = ctypes.c_int
        lib.oracle_gate_alpha.argtypes = [ctypes.c_double]
        lib.oracle_gate_alpha.restype = ctypes.c_double
        lib.oracle_gate_beta.argtypes = [ctypes.c_double]
        lib.oracle_gate_beta.restype = ctypes.c_double
        _lib = lib
    return _lib


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data


def gate_alpha(a: float) -> float:
    """alpha = exp(-softplus(a)) in double."""
    return float(_load().oracle_gate_alpha(float(a)))


def gate_beta(b: float) -> float:
    """beta = sigmoid(b) in double."""
    return float(_load().oracle_gate_beta(float(b)))


def gdn(q, k, v, alpha, beta, *, F: int, L: int, gates_are_logits: bool = True, state_in=None,
        cols=None, heads=None, want_o: bool = True, nthreads: int | None = None, rope=None):
    """Gated DeltaNet frame recurrence in fp64.

    q, k: [..., F*L, dk]; v: [..., F*L, dv]; alpha: [..., F]; beta: [..., F*L];
    leading dims are flattened into heads.  state_in: [..., dk, dv] or None.
    cols: (lo, hi) range of d_v columns to compute (others left as NaN).
    heads: optional subset of flat head indices (outputs still full-sized,
    other heads NaN).  rope: None, or dict(grid_w, frame_offset=0, base=1e4)
    to apply the 3D RoPE (see ``rope3d``) to q and to k before its
    normalisation.  Returns (o, state_out) as float64 arrays.
    """
    q, k, v, alpha, beta = map(_f32, (q, k, v, alpha, beta))
    lead = q.shape[:-2]
    N, dk = q.shape[-2:]
    dv = v.shape[-1]
    assert N == F * L and k.shape == q.shape and v.shape[:-1] == q.shape[:-1]
    nh = int(np.prod(lead)) if lead else 1
    assert alpha.size == nh * F and beta.size == nh * N
    s_in = _f64(state_in)
    if s_in is not None:
        assert s_in.size == nh * dk * dv
    lo, hi = (0, dv) if cols is None else cols
    o = np.full(lead + (N, dv), np.nan) if want_o else None
    s_out = np.full(lead + (dk, dv), np.nan)
    hl = None if heads is None else np.ascontiguousarray(np.asarray(heads, dtype=np.int64))
    nthreads = nthreads or (os.cpu_count() or 1)
    col_block = max(1, min(hi - lo, 16)) if hi > lo else 1
    rp = _rope_args(rope)
    rc = _load().oracle_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), int(gates_are_logits),
                            _ptr(s_in), _ptr(s_out), _ptr(o), 1, nh, F, L, dk, dv, lo, hi,
                            _ptr(hl), 0 if hl is None else hl.size, col_block, nthreads, *rp)
    if rc != 0:
        raise ValueError("oracle_gdn: invalid arguments")
    return o, s_out


def gdn_bwd(q, k, v, alpha, beta, d_o, *, F: int, L: int, gates_are_logits: bool = True, state_in=None,
            dstate_out=None, heads=None, nthreads: int | None = None, rope=None):
    """Backward of the Gated DeltaNet frame recurrence in fp64 (see oracle.c).

    Shapes as in ``gdn``; d_o: [..., F*L, dv] (dL/do), dstate_out: [..., dk, dv]
    or None (zero).  Returns a dict of float64 arrays: dq, dk [..., F*L, dk],
    dv [..., F*L, dv], dalpha [..., F] and dbeta [..., F*L] (with respect to the
    logits when ``gates_are_logits``, else the gate values) and dstate_in
    [..., dk, dv].  heads: optional subset of flat head indices (the others'
    entries are NaN).  rope: as in ``gdn`` (the gradients are with respect to
    the unrotated q and k)."""
    q, k, v, alpha, beta, d_o = map(_f32, (q, k, v, alpha, beta, d_o))
    lead = q.shape[:-2]
    N, dk = q.shape[-2:]
    dv = v.shape[-1]
    assert N == F * L and k.shape == q.shape and v.shape[:-1] == q.shape[:-1] and d_o.shape == v.shape
    nh = int(np.prod(lead)) if lead else 1
    assert alpha.size == nh * F and beta.size == nh * N
    s_in, ds_out = _f64(state_in), _f64(dstate_out)
    for x in (s_in, ds_out):
        assert x is None or x.size == nh * dk * dv
    out = dict(dq=np.full(lead + (N, dk), np.nan), dk=np.full(lead + (N, dk), np.nan),
               dv=np.full(lead + (N, dv), np.nan), dalpha=np.full(lead + (F,), np.nan),
               dbeta=np.full(lead + (N,), np.nan), dstate_in=np.full(lead + (dk, dv), np.nan))
    hl = None if heads is None else np.ascontiguousarray(np.asarray(heads, dtype=np.int64))
    nthreads = nthreads or (os.cpu_count() or 1)
    rc = _load().oracle_gdn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), int(gates_are_logits),
                                _ptr(s_in), _ptr(d_o), _ptr(ds_out), _ptr(out["dq"]), _ptr(out["dk"]),
                                _ptr(out["dv"]), _ptr(out["dalpha"]), _ptr(out["dbeta"]), _ptr(out["dstate_in"]),
                                1, nh, F, L, dk, dv, _ptr(hl), 0 if hl is None else hl.size, nthreads,
                                *_rope_args(rope))
    if rc != 0:
        raise ValueError("oracle_gdn_bwd: invalid arguments")
    return out


def _rope_args(rope):
    if rope is None:
        return (0, 0, 1e4)
    return (int(rope["grid_w"]), int(rope.get("frame_offset", 0)), float(rope.get("base", 1e4)))


def rope3d(x, *, F: int, L: int, grid_w: int, frame_offset: int = 0, base: float = 1e4):
    """The 3D rotary position embedding alone, in fp64: x [..., F*L, d] -> rotated x.

    The d dimensions are a time part (d - 4*floor(d/6)), then a height and a
    width part (2*floor(d/6) each); in each part the pair (2i, 2i+1) turns by
    pos * base**(-2i / part_length), pos being the token's frame (plus
    frame_offset), row (t // grid_w) or column (t % grid_w)."""
    x = _f32(x)
    lead = x.shape[:-2]
    N, d = x.shape[-2:]
    assert N == F * L
    nh = int(np.prod(lead)) if lead else 1
    out = np.empty(x.shape, np.float64)
    rc = _load().oracle_rope3d(_ptr(x), _ptr(out), nh, F, L, d, grid_w, frame_offset, float(base))
    if rc != 0:
        raise ValueError("oracle_rope3d: invalid arguments")
    return out


def relu_la(q, k, v, *, F: int, L: int, kv_in=None, z_in=None, eps: float = 1e-6, nthreads: int | None = None):
    """Block-causal ReLU linear attention in fp64.  Returns (o, kv_out, z_out).

    Heads are independent; ``nthreads`` threads (default: all host cores) take
    whole heads, which changes no arithmetic."""
    q, k, v = map(_f32, (q, k, v))
    lead = q.shape[:-2]
    N, dk = q.shape[-2:]
    dv = v.shape[-1]
    assert N == F * L
    nh = int(np.prod(lead)) if lead else 1
    kv_in, z_in = _f64(kv_in), _f64(z_in)
    o = np.empty(lead + (N, dv))
    kv_out = np.empty(lead + (dk, dv))
    z_out = np.empty(lead + (dk,))
    nthreads = nthreads or (os.cpu_count() or 1)
    rc = _load().oracle_relu_la(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_in), _ptr(z_in), _ptr(kv_out),
                                _ptr(z_out), _ptr(o), 1, nh, F, L, dk, dv, float(eps), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_relu_la: invalid arguments")
    return o, kv_out, z_out


def gdn_stream(step_inputs, *, steps: int, L: int, state_in=None, cols=None):
    """Streaming block-cache decode: frames of ``steps`` calls each.

    Follows the SANA-Video talk's block KV cache passage (the cache made after
    block i is what every pass over block i+1 reads): ``step_inputs(call)``
    returns dict(q, k, v, a, b) for one frame (F=1) of fresh inputs, or None
    once the stream ends (only at a frame boundary).  Every step of frame f
    starts from the committed state S_{f-1} (``state_in``, or zero, before the
    first frame); the state after the LAST step of the frame is committed and
    the other steps' states are discarded.

    Returns (outs, S, committed): the per-call outputs o in call order, the
    final committed state, and the list of committed states, one per frame.
    """
    if steps < 1:
        raise ValueError("steps must be >= 1")
    S = None if state_in is None else np.asarray(state_in, np.float64)
    outs, committed = [], []
    call = 0
    while True:
        x = step_inputs(call)
        if x is None:
            break
        last_state = None
        for s in range(steps):
            if s > 0:
                x = step_inputs(call)
                if x is None:
                    raise ValueError(f"step_inputs({call}) returned None inside a frame "
                                     f"(step {s + 1} of {steps}): a frame needs all of its steps")
            o, s_out = gdn(x["q"], x["k"], x["v"], x["a"], x["b"], F=1, L=L, state_in=S, cols=cols)
            outs.append(o)
            last_state = s_out
            call += 1
        S = last_state
        committed.append(S)
    return outs, S, committed


def temporal_conv(x, w, *, bias=None, cache_in=None):
    """Causal temporal convolution of one block of frames with the block-boundary
    cache, in fp64 (see oracle.c): x [B, F, HW, C]; w [C, 3]; bias [C] or None;
    cache_in [B, HW, C] or None (zero).  Returns (y [B, F, HW, C], cache_out
    [B, HW, C] = the block's last frame)."""
    x = _f32(x)
    B, F, HW, C = x.shape
    w = _f32(w)
    assert w.shape == (C, 3)
    b = None if bias is None else _f32(bias)
    ci = None if cache_in is None else _f32(cache_in)
    y = np.empty(x.shape, np.float64)
    co = np.empty((B, HW, C), np.float64)
    rc = _load().oracle_temporal_conv(_ptr(x), _ptr(w), _ptr(b), _ptr(ci), _ptr(y), _ptr(co), B, F, HW, C)
    if rc != 0:
        raise ValueError("oracle_temporal_conv: invalid arguments")
    return y, co


def softmax_window(q, k, v, *, F: int, L: int, W: int, scale=None, frames=None, nthreads=None):
    """Windowed block-causal softmax attention in fp64 (see oracle.c): q, k
    [B, H, F*L, dk], v [B, H, F*L, dv]; token t of frame f attends to all tokens
    of frames max(0, f-W+1) .. f with weights softmax(scale q_t . k_s), scale
    defaulting to 1/sqrt(dk).  ``frames``: compute only these query frames (the
    other rows of o are NaN)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    assert N == F * L and k.shape == q.shape and v.shape[:3] == (B, H, N)
    sc = float(dk) ** -0.5 if scale is None else float(scale)
    mask = None
    o = np.empty((B, H, N, dv), np.float64)
    if frames is not None:
        mask = np.zeros(F, np.uint8)
        mask[list(frames)] = 1
        o.fill(np.nan)
    nt = nthreads or max(1, min(64, os.cpu_count() or 1))
    rc = _load().oracle_softmax_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, F, L, dk, dv, W, sc, _ptr(mask), nt)
    if rc != 0:
        raise ValueError("oracle_softmax_window: invalid arguments")
    return o
