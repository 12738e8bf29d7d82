"""Shared helpers for the GPU parity tests: inputs on the device, oracle runs, error metric."""
import numpy as np

import oracle
import synth

TOL_BF16 = 2e-3  # max|gpu - ref| <= TOL * max|ref| for bf16 inputs (fp32 state and outputs)
TOL_F32 = 1e-5   # same, fp32 inputs


def rel_err(x, ref):
    """max|x - ref| / max|ref| over the finite entries of ref (NaN marks uncomputed entries).

    Streams over the flattened arrays in blocks, so full-size outputs (about
    5e8 elements) need no multi-gigabyte temporaries."""
    x = np.asarray(x).reshape(-1)
    ref = np.asarray(ref).reshape(-1)
    assert x.size == ref.size
    scale, err, any_ref = 0.0, 0.0, False
    step = 1 << 24
    for i in range(0, ref.size, step):
        r = ref[i:i + step].astype(np.float64, copy=False)
        m = np.isfinite(r)
        if not m.any():
            continue
        any_ref = True
        xs = x[i:i + step].astype(np.float64, copy=False)
        if not np.isfinite(xs[m]).all():
            return float("inf")
        scale = max(scale, float(np.abs(r[m]).max()))
        err = max(err, float(np.abs(xs[m] - r[m]).max()))
    assert any_ref
    return err / max(scale, 1e-30)


def device_inputs(w, x, dev, torch):
    """Torch device tensors (q, k, v in the workload dtype; gates fp32) and the exact float32
    values the device sees (bf16-rounded q, k, v) for the oracle."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {}
    host = {}
    for n in "qkv":
        tt = torch.from_numpy(x[n]).to(dt)
        host[n] = tt.float().numpy()
        t[n] = tt.to(dev).contiguous()
    for n in "ab":
        t[n] = torch.from_numpy(x[n]).to(dev).contiguous()
        host[n] = x[n]
    return t, host


def tol_for(w):
    return TOL_BF16 if w.dtype == "bf16" else TOL_F32


def oracle_gdn(host, w, state_in=None, cols=None, heads=None):
    return oracle.gdn(host["q"], host["k"], host["v"], host["a"], host["b"], F=w.F, L=w.L,
                      state_in=state_in, cols=cols, heads=heads)


__all__ = ["rel_err", "device_inputs", "tol_for", "oracle_gdn", "synth", "oracle", "TOL_BF16", "TOL_F32"]
