"""GPU parity of the Gated DeltaNet backward (gdn_frame_bwd, through the C ABI)
against the fp64 oracle backward, itself pinned by finite differences.

Bar, per output (dq, dk, dv, dalpha, dbeta, dstate_in):
max|gpu - oracle| <= tol * max|oracle| with tol = 2e-3 for bf16 inputs and
1e-5 for fp32 inputs, the forward's tolerances.
"""
import numpy as np
import pytest

from helpers import TOL_BF16, TOL_F32, device_inputs, oracle, rel_err, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dstate_in")


@pytest.fixture(scope="module")
def lib():
    import linear_attention_video_gdn_b200 as lib
    return lib


@pytest.fixture(scope="module")
def dev():
    return torch.device("cuda", 0)


def case(B, H, F, L, dk, dv, dtype, seed, logits=True, s_in=True, ds_out=True):
    w = synth.Workload("bwd", "gdn", B, H, F, L, dk, dv, dtype, seed=seed)
    x = synth.inputs(w)
    if not logits:  # gate values in (0, 1)
        x["a"] = (1.0 / (1.0 + np.exp(x["a"]))).astype(np.float32)
        x["b"] = (1.0 / (1.0 + np.exp(-x["b"]))).astype(np.float32)
    g = synth.grad_inputs(w, state_in=s_in, dstate_out=ds_out)
    return w, x, g["d_o"], g["state_in"], g["dstate_out"]


def run(lib, dev, w, x, d_o, si, dso, logits=True, heads=None, rope=None, **kw):
    """The GPU gradients and the oracle's; with ``heads`` (flat head indices, B = 1)
    only those heads, the oracle run on them alone (heads are independent).
    ``rope``: the 3D RoPE options, given to both sides."""
    t, h = device_inputs(w, x, dev, torch)
    tsi = None if si is None else torch.from_numpy(si).to(dev)
    tds = None if dso is None else torch.from_numpy(dso).to(dev)
    g = lib.gdn_frame_bwd(t["q"], t["k"], t["v"], t["a"], t["b"], torch.from_numpy(d_o).to(dev), F=w.F,
                          state_in=tsi, d_state_out=tds, gates_are_logits=logits, rope=rope, **kw)
    torch.cuda.synchronize()
    sel = (lambda a: a) if heads is None else (lambda a: a[:, heads])
    out = {n: sel(g[n]).cpu().numpy() for n in NAMES}
    del g, t
    ref = oracle.gdn_bwd(*(sel(h[n]) for n in ("q", "k", "v", "a", "b")), sel(d_o), F=w.F, L=w.L,
                         gates_are_logits=logits, state_in=None if si is None else sel(si),
                         dstate_out=None if dso is None else sel(dso), rope=rope)
    return out, ref


def check(out, ref, tol):
    errs = {n: rel_err(out[n], ref[n]) for n in NAMES}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, errs


# B, H, F, L, dk, dv: several 48-token chunks with ragged ends, one-token frames,
# d_k != d_v, and the 112-wide heads of the video workloads
SHAPES = [(1, 2, 3, 16, 32, 32), (1, 1, 4, 100, 64, 64), (2, 2, 3, 50, 16, 48), (1, 2, 5, 1, 32, 32),
          (1, 1, 3, 97, 112, 112), (1, 2, 2, 145, 48, 112)]


@pytest.mark.parametrize("shape", SHAPES)
def test_fp32_matches_oracle(lib, dev, shape):
    w, x, d_o, si, dso = case(*shape, "f32", seed=shape[3] + 3)
    out, ref = run(lib, dev, w, x, d_o, si, dso)
    check(out, ref, TOL_F32)


@pytest.mark.parametrize("shape", SHAPES)
def test_bf16_matches_oracle(lib, dev, shape):
    w, x, d_o, si, dso = case(*shape, "bf16", seed=shape[3] + 5)
    out, ref = run(lib, dev, w, x, d_o, si, dso)
    check(out, ref, TOL_BF16)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_values_no_state_and_edge_tokens(lib, dev, dtype):
    """Gate values instead of logits, no start state and no dL/dstate_out, a
    key of zero norm (the clamp branch), tokens with beta = 0 and a frame with
    alpha = 0 (nothing flows to the frames before it)."""
    w, x, d_o, si, dso = case(1, 2, 4, 60, 32, 32, dtype, seed=77, logits=False, s_in=False, ds_out=False)
    x["k"][0, 1, 70] = 0.0
    x["b"][0, 0, 5] = 0.0
    x["b"][0, 1, 130] = 0.0
    x["a"][0, 0, 2] = 0.0
    out, ref = run(lib, dev, w, x, d_o, si, dso, logits=False)
    check(out, ref, TOL_F32 if dtype == "f32" else TOL_BF16)


def test_recompute_kernels_agree(lib, dev):
    """bf16 inputs with the fp32 CUDA-core recompute forced: the same gradients."""
    w, x, d_o, si, dso = case(1, 2, 3, 70, 64, 64, "bf16", seed=78)
    out, ref = run(lib, dev, w, x, d_o, si, dso, impl="frame_simt")
    check(out, ref, TOL_BF16)


def test_720p_60s_two_heads(lib, dev):
    """The benchmark's workload (B=1, H=20, F=240, L=920, d=112, bf16) in the
    launch the benchmark times; the oracle recomputes heads 0 and 13 in full
    (every frame, token and column)."""
    w = synth.WORKLOADS["gdn_720p_60s"]
    x = synth.inputs(w)
    d_o = synth.grad_inputs(w)["d_o"]
    heads = [0, 13]
    out, ref = run(lib, dev, w, x, d_o, None, None, heads=heads)
    check(out, ref, TOL_BF16)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_recompute_timeout_status_is_reported(lib, dev, dtype):
    """A frame of the forward recompute that never publishes its state (the
    test option withholds frame 0 of head 0): the next frame's bounded wait runs
    out after 2 ms, GDN_ERR_TIMEOUT is latched, the call returns, and the next
    call on the same context is correct."""
    w, x, d_o, si, dso = case(1, 1, 3, 40, 32, 32, dtype, seed=91)
    t, _ = device_inputs(w, x, dev, torch)
    st = torch.zeros(4, dtype=torch.int32, device=dev)
    lib.gdn_frame_bwd(t["q"], t["k"], t["v"], t["a"], t["b"], torch.from_numpy(d_o).to(dev), F=w.F,
                      state_in=torch.from_numpy(si).to(dev), status=st, spin_limit_us=2000, test_withhold_unit=0)
    torch.cuda.synchronize()
    assert int(st[0].item()) == lib.ERR_TIMEOUT
    st.zero_()
    out, ref = run(lib, dev, w, x, d_o, si, dso, status=st)
    assert int(st[0].item()) == 0
    check(out, ref, TOL_F32 if dtype == "f32" else TOL_BF16)


def test_480p_5s_all_heads(lib, dev):
    """The 480p 5 s workload (B=1, H=20, F=21, L=390, d=112, bf16) with a start
    state and dL/dstate_out: every head, frame, token and column against the
    oracle."""
    w = synth.WORKLOADS["gdn_480p_5s"]
    x = synth.inputs(w)
    g = synth.grad_inputs(w, state_in=True, dstate_out=True)
    out, ref = run(lib, dev, w, x, g["d_o"], g["state_in"], g["dstate_out"])
    check(out, ref, TOL_BF16)


# B, H, F, L, dk, dv, grid_w, frame_offset: the 3D RoPE (time, height and width
# bands of d_k) on q and k, with ragged 48-token chunks and a resumed clip's offset
ROPE = [(1, 2, 3, 40, 32, 32, 8, 0), (1, 1, 4, 100, 112, 112, 10, 5), (2, 1, 2, 60, 48, 64, 12, 2)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", ROPE)
def test_rope_matches_oracle(lib, dev, shape, dtype):
    """The forward with the embedding on q and k (recomputed by the tensor-core
    kernel for bf16 inputs, the CUDA-core one for fp32), its gradients taken
    back through the rotation, against the oracle's."""
    *sz, gw, off = shape
    w, x, d_o, si, dso = case(*sz, dtype, seed=sz[3] + 11)
    out, ref = run(lib, dev, w, x, d_o, si, dso, rope=dict(grid_w=gw, frame_offset=off))
    check(out, ref, TOL_F32 if dtype == "f32" else TOL_BF16)


def test_rope_720p_60s_one_head(lib, dev):
    """The benchmark's workload with the embedding (40 x 23 token grid per frame):
    head 7 in full (every frame, token and column) against the oracle."""
    w = synth.WORKLOADS["gdn_720p_60s"]
    x = synth.inputs(w)
    d_o = synth.grad_inputs(w)["d_o"]
    out, ref = run(lib, dev, w, x, d_o, None, None, heads=[7], rope=dict(grid_w=40))
    check(out, ref, TOL_BF16)


def test_rope_recompute_kernels_agree(lib, dev):
    """bf16 inputs with the embedding and the fp32 CUDA-core recompute forced
    (the default is the tensor-core one): the same gradients."""
    w, x, d_o, si, dso = case(1, 2, 3, 70, 64, 64, "bf16", seed=79)
    out, ref = run(lib, dev, w, x, d_o, si, dso, impl="frame_simt", rope=dict(grid_w=10, frame_offset=1))
    check(out, ref, TOL_BF16)
