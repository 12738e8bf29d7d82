"""Seeded synthetic workloads for the frame recurrence (inputs only).

This package draws the random inputs that both the CUDA path and the CPU
oracle consume.  It contains no step of the method itself: it produces raw
q, k, v and the gate logits a (per head and frame) and b (per head and
token).  Keys for the Gated DeltaNet workloads are drawn as uniformly random
unit vectors, which is how the workloads are specified ("k L2-normalised per
token"); the method's own key normalisation is applied again by both sides.

Every value is a pure function of (seed, tensor id, flat index), so any head
of a multi-gigabyte workload can be regenerated alone (see ``synth.c``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

# tensor ids: the draw order q, k, v, a, b
TID_Q, TID_K, TID_V, TID_A, TID_B = 0, 1, 2, 3, 4
TID_STRIDE_PER_CALL = 8  # streaming call c uses ids base + 8 * c
TID_DO, TID_STATE_IN, TID_DSTATE_OUT = 5, 6, 7  # the backward's upstream gradients and start state


def build(force: bool = False) -> str:
    """Compile libsynth.so in place with gcc (plain C, pthreads, libm)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm", "-lpthread"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.synth_fill_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        lib.synth_fill_unit_rows.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
        lib.synth_mix.argtypes = [ctypes.c_uint64]
        lib.synth_mix.restype = ctypes.c_uint64
        lib.synth_word.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_word.restype = ctypes.c_uint64
        lib.synth_normal_one.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal_one.restype = ctypes.c_double
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def normal(seed: int, tid: int, first: int, count: int, mean: float = 0.0, std: float = 1.0,
           out: np.ndarray | None = None) -> np.ndarray:
    """Elements [first, first+count) of the N(mean, std^2) stream (seed, tid), as float32."""
    lib = _load()
    if out is None:
        out = np.empty(count, dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == count
    lib.synth_fill_normal(seed, tid, first, count, mean, std, out.ctypes.data, _threads())
    return out


def unit_rows(seed: int, tid: int, first_row: int, nrows: int, d: int,
              out: np.ndarray | None = None) -> np.ndarray:
    """Rows [first_row, first_row+nrows) of uniformly random unit vectors in R^d (float32)."""
    lib = _load()
    if out is None:
        out = np.empty((nrows, d), dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == nrows * d
    lib.synth_fill_unit_rows(seed, tid, first_row, nrows, d, out.ctypes.data, _threads())
    return out


def mix(x: int) -> int:
    """The SplitMix64 output function applied to state x (one generator step)."""
    return int(_load().synth_mix(x))


def word(seed: int, tid: int, counter: int) -> int:
    return int(_load().synth_word(seed, tid, counter))


def normal_one(seed: int, tid: int, index: int) -> float:
    return float(_load().synth_normal_one(seed, tid, index))


@dataclass(frozen=True)
class Workload:
    """Shape and input distribution of one synthetic workload."""
    name: str
    mode: str            # "gdn", "gdn_stream" or "relu"
    B: int
    H: int
    F: int
    L: int
    dk: int
    dv: int
    dtype: str           # "f32" or "bf16" (q, k, v); gates and state are fp32
    seed: int
    a_mean: float = 0.0  # gate logit a ~ N(a_mean, 1) per (b, h, f)
    steps: int = 1       # denoising steps per frame (streaming)
    unit_keys: bool = True

    @property
    def N(self) -> int:
        return self.F * self.L

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: a tiny fp32 case, the 480p 5 s and 720p 60 s latent
# shapes (15x26 and 23x40 latent grids, 21 and 240 latent frames, 20 heads of
# width 112), streaming block-cache decode at the 720p shape, and block-causal
# ReLU linear attention at the 720p grid with 81 frames.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", "gdn", 1, 2, 4, 16, 32, 32, "f32", seed=0),
    "gdn_480p_5s": Workload("gdn_480p_5s", "gdn", 1, 20, 21, 390, 112, 112, "bf16", seed=1),
    "gdn_720p_60s": Workload("gdn_720p_60s", "gdn", 1, 20, 240, 920, 112, 112, "bf16", seed=2, a_mean=-2.0),
    "gdn_stream_720p": Workload("gdn_stream_720p", "gdn_stream", 1, 20, 240, 920, 112, 112, "bf16", seed=3, steps=4),
    "relu_720p_81f": Workload("relu_720p_81f", "relu", 2, 20, 81, 920, 112, 112, "bf16", seed=4, unit_keys=False),
}


def inputs(w: Workload, heads=None, call: int = 0, frames: int | None = None) -> dict:
    """Draw q, k, v, a, b for workload ``w`` (float32 numpy arrays).

    ``heads``: None for all B*H heads (arrays shaped [B, H, ...]); else a list
    of flat head indices bh = b*H + h (arrays shaped [len(heads), ...]).
    ``call``: streaming call index (frame * steps + step); each call has its
    own fresh inputs.  For streaming workloads one call covers one frame, so
    the token count per head is L (not F*L) and a has one entry per head.
    ``frames``: draw only the first ``frames`` frames of every head (same
    values as the full draw; arrays hold frames * L tokens).
    """
    Nfull = w.L if w.mode == "gdn_stream" else w.N
    Ffull = 1 if w.mode == "gdn_stream" else w.F
    F = Ffull if frames is None else min(frames, Ffull)
    N = F * w.L
    off = TID_STRIDE_PER_CALL * call
    hl = list(range(w.B * w.H)) if heads is None else list(heads)
    n = len(hl)
    q = np.empty((n, N, w.dk), np.float32)
    k = np.empty((n, N, w.dk), np.float32)
    v = np.empty((n, N, w.dv), np.float32)
    a = np.empty((n, F), np.float32)
    b = np.empty((n, N), np.float32)
    for i, bh in enumerate(hl):
        normal(w.seed, TID_Q + off, bh * Nfull * w.dk, N * w.dk, out=q[i].reshape(-1))
        if w.unit_keys:
            unit_rows(w.seed, TID_K + off, bh * Nfull, N, w.dk, out=k[i])
        else:
            normal(w.seed, TID_K + off, bh * Nfull * w.dk, N * w.dk, out=k[i].reshape(-1))
        normal(w.seed, TID_V + off, bh * Nfull * w.dv, N * w.dv, out=v[i].reshape(-1))
        normal(w.seed, TID_A + off, bh * Ffull, F, mean=w.a_mean, out=a[i])
        normal(w.seed, TID_B + off, bh * Nfull, N, out=b[i])
    if heads is None:
        q = q.reshape(w.B, w.H, N, w.dk)
        k = k.reshape(w.B, w.H, N, w.dk)
        v = v.reshape(w.B, w.H, N, w.dv)
        a = a.reshape(w.B, w.H, F)
        b = b.reshape(w.B, w.H, N)
    return dict(q=q, k=k, v=v, a=a, b=b)



def grad_inputs(w: Workload, state_in: bool = False, dstate_out: bool = False) -> dict:
    """Inputs of the backward beyond ``inputs(w)``: dL/do [B, H, N, dv] ~ N(0, 1),
    and optionally a start state and dL/dstate_out [B, H, dk, dv] ~ N(0, 1)."""
    nh = w.B * w.H
    out = dict(d_o=normal(w.seed, TID_DO, 0, nh * w.N * w.dv).reshape(w.B, w.H, w.N, w.dv))
    out["state_in"] = (normal(w.seed, TID_STATE_IN, 0, nh * w.dk * w.dv).reshape(w.B, w.H, w.dk, w.dv)
                       if state_in else None)
    out["dstate_out"] = (normal(w.seed, TID_DSTATE_OUT, 0, nh * w.dk * w.dv).reshape(w.B, w.H, w.dk, w.dv)
                         if dstate_out else None)
    return out


# ---------------------------------------------------------------- temporal convolution inputs

@dataclass(frozen=True)
class ConvWorkload:
    """Shape and input distribution of a causal temporal convolution workload:
    x [B, F, HW, C] per block of F latent frames, depthwise kernel-3 weights
    w [C, 3] and bias [C]; ``blocks`` consecutive blocks (streaming)."""
    name: str
    B: int
    F: int
    HW: int
    C: int
    dtype: str
    seed: int
    blocks: int = 1


# tensor ids of the temporal convolution draws (block c uses ids base + 8 * c)
TID_X, TID_W, TID_BIAS = 0, 1, 2

# The 720p latent grid (23x40 = 920 positions) at the model width of 20 heads
# of 112 channels: the whole 60 s clip (240 latent frames) as one block, and
# the same clip generated in 24 blocks of 10 frames with the cache carried.
CONV_WORKLOADS = {
    "tconv_720p_60s": ConvWorkload("tconv_720p_60s", 1, 240, 920, 2240, "bf16", seed=5),
    "tconv_stream_720p": ConvWorkload("tconv_stream_720p", 1, 10, 920, 2240, "bf16", seed=6, blocks=24),
}


def conv_inputs(cw: ConvWorkload, block: int = 0, frames: int | None = None) -> dict:
    """Draw x (block ``block``; its first ``frames`` frames when given), w and
    bias for ``cw`` as float32 numpy arrays.  x ~ N(0, 1); w ~ N(0, 1/3) so that
    the output keeps about unit variance; bias ~ N(0, 0.1^2).  w and bias are
    shared by all blocks."""
    F = cw.F if frames is None else min(frames, cw.F)
    off = TID_STRIDE_PER_CALL * block
    x = normal(cw.seed, TID_X + off, 0, cw.B * cw.F * cw.HW * cw.C).reshape(cw.B, cw.F, cw.HW, cw.C) \
        if F == cw.F else None
    if x is None:  # a prefix of every batch's frames
        x = np.empty((cw.B, F, cw.HW, cw.C), np.float32)
        per_b = cw.F * cw.HW * cw.C
        for b in range(cw.B):
            normal(cw.seed, TID_X + off, b * per_b, F * cw.HW * cw.C, out=x[b].reshape(-1))
    w = normal(cw.seed, TID_W, 0, cw.C * 3, std=3.0 ** -0.5).reshape(cw.C, 3)
    bias = normal(cw.seed, TID_BIAS, 0, cw.C, std=0.1)
    return dict(x=x, w=w, bias=bias)
