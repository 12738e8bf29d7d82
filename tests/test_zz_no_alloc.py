"""gdn_frame_fwd_noalloc: the entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or carve a workspace out of an allocator
of their own (a plugin inside a host program that owns all device memory, a
runtime with a fixed memory plan).  For them the library keeps its own
fixed-size scratch array; this file checks, through the C ABI, that the
no-allocation call gives the same result as the regular call with a
caller workspace and as the fp64 oracle, on two calls in a row (the shared
scratch keeps the previous call's contents, which must not leak into the next),
and that sizes beyond the scratch limit are refused.  It is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

from helpers import device_inputs, oracle_gdn, rel_err, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import linear_attention_video_gdn_b200 as lib
    return lib


def _regular(lib, w, t, dev, S0):
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], t["a"], t["b"], F=w.F, state_in=S0, state_out=s_out)
    return o, s_out


def _noalloc_via_cabi(lib, w, t, dev, S0):
    """Direct C-ABI call of gdn_frame_fwd_noalloc with caller-provided outputs only."""
    o = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32, device=dev)
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    opts = lib.make_opts(lib.DTYPE_BF16)
    P = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())
    rc = lib._lib.gdn_frame_fwd_noalloc(P(t["q"]), P(t["k"]), P(t["v"]), P(t["a"]), P(t["b"]), P(S0), P(s_out),
                                        P(o), w.B, w.H, w.F, w.L, w.dk, w.dv, ctypes.byref(opts))
    assert rc == lib.OK, lib.status_string(rc)
    return o, s_out


def test_noalloc_matches_regular_on_two_calls(lib):
    dev = torch.device("cuda", 0)
    cases = [synth.WORKLOADS["gdn_480p_5s"].with_(F=6, L=390),            # 120 frame units
             synth.WORKLOADS["gdn_480p_5s"].with_(F=3, L=200, seed=77)]   # different sizes and inputs
    for i, w in enumerate(cases):
        x = synth.inputs(w)
        t, h = device_inputs(w, x, dev, torch)
        S0h = np.random.default_rng(i).standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)
        S0 = torch.from_numpy(S0h).to(dev)
        o_reg, s_reg = _regular(lib, w, t, dev, S0)
        o, s = _noalloc_via_cabi(lib, w, t, dev, S0)
        torch.cuda.synchronize()
        o, s = o.cpu().numpy(), s.cpu().numpy()
        assert rel_err(o, o_reg.cpu().numpy()) <= 2e-3
        assert rel_err(s, s_reg.cpu().numpy()) <= 2e-3
        o_ref, s_ref = oracle_gdn(h, w, state_in=S0h)
        assert rel_err(o, o_ref) <= 2e-3
        assert rel_err(s, s_ref) <= 2e-3


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS["gdn_720p_60s"].with_(F=1000, L=1)  # 20,000 frame units, far above the limit
    opts = lib.make_opts(lib.DTYPE_BF16)
    need = lib.workspace_bytes(lib.OP_GDN, w.B, w.H, w.F, w.L, w.dk, w.dv, opts)
    assert need > lib.NOALLOC_SCRATCH_BYTES
    buf = torch.zeros(16, dtype=torch.uint8, device=dev)
    p = ctypes.c_void_p(buf.data_ptr())
    rc = lib._lib.gdn_frame_fwd_noalloc(p, p, p, p, p, None, None, p, w.B, w.H, w.F, w.L, w.dk, w.dv,
                                        ctypes.byref(opts))
    assert rc == lib.ERR_UNSUPPORTED
