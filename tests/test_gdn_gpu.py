"""GPU parity of the Gated DeltaNet frame recurrence against the fp64 CPU oracle.

Every case compares the CUDA path (called through the C ABI) with the oracle
element by element on the same seeded inputs; the bar is
max|gpu - oracle| <= tol * max|oracle| for o and for the output state, with
tol = 2e-3 for bf16 inputs and 1e-5 for fp32 inputs.
"""
import numpy as np
import pytest

from helpers import device_inputs, oracle, oracle_gdn, rel_err, synth, tol_for

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module")
def lib():
    import linear_attention_video_gdn_b200 as lib
    return lib


@pytest.fixture(scope="module")
def dev():
    return torch.device("cuda", 0)


def run_gdn(lib, w, t, dev, impl, state_in=None, want_state=True, **kw):
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev) if want_state else None
    s_in = None if state_in is None else torch.from_numpy(np.asarray(state_in, np.float32)).to(dev)
    o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], t["a"], t["b"], F=w.F, state_in=s_in, state_out=s_out,
                          impl=impl, **kw)
    torch.cuda.synchronize()
    return o.cpu().numpy(), (None if s_out is None else s_out.cpu().numpy())


def pform_ok(dk, dv):
    """Sizes the product-form tensor-core kernel takes (its shared-memory and TMEM maps fit)."""
    ny = dk + dv
    if dk % 16 or dv % 16 or dv > dk or dk > 128 or ny + 2 * (32 + dk) > 512 or (ny // 2) // 32 == 0:
        return False
    nyb, nab, nvb = (ny + 63) // 64, (dk + 63) // 64, (dv + 63) // 64
    return nyb >= nab + nvb


def impls_for(w):
    out = ["seq", "frame_simt"]
    if w.dtype == "bf16" and w.dk % 16 == 0 and w.dv % 16 == 0:
        out.append("tc")
        if pform_ok(w.dk, w.dv):
            out.append("tc_pform")
    return out


# ------------------------------------------------------------------ the workloads

@pytest.mark.parametrize("impl", ["seq", "frame_simt"])
def test_tiny_fp32(lib, dev, impl):
    w = W["tiny_fp32"]
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    o, s = run_gdn(lib, w, t, dev, impl)
    o_ref, s_ref = oracle_gdn(h, w)
    assert rel_err(o, o_ref) <= 1e-5
    assert rel_err(s, s_ref) <= 1e-5


@pytest.mark.parametrize("impl", ["frame_simt", "tc", "tc_pform"])
def test_480p_5s(lib, dev, impl):
    w = W["gdn_480p_5s"]
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    o, s = run_gdn(lib, w, t, dev, impl)
    o_ref, s_ref = oracle_gdn(h, w)
    eo, es = rel_err(o, o_ref), rel_err(s, s_ref)
    print(f"480p {impl}: err_o={eo:.3e} err_s={es:.3e}")
    assert eo <= 2e-3 and es <= 2e-3


@pytest.mark.parametrize("impl", ["frame_simt", "tc", "tc_pform"])
def test_720p_60s_full(lib, dev, impl):
    """Full 720p-60s workload in the benchmark's launch configuration, every
    head and every d_v column (including columns 64-111, which come from the
    second, zero-padded 64-wide tile) and the final state, against the oracle
    run over all heads on every host core."""
    w = W["gdn_720p_60s"]
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    o, s = run_gdn(lib, w, t, dev, impl)
    o_ref, s_ref = oracle_gdn(h, w)
    eo, es = rel_err(o, o_ref), rel_err(s, s_ref)
    eo_hi = rel_err(o[..., 64:], o_ref[..., 64:])
    print(f"720p {impl}: err_o={eo:.3e} (cols 64-111: {eo_hi:.3e}) err_s={es:.3e}")
    assert eo <= 2e-3 and es <= 2e-3 and eo_hi <= 2e-3


def test_alpha_one_long_sequence_drift(lib, dev):
    """No forgetting (alpha = 1 given as values) over 240 frames of 128 tokens:
    the state is carried from frame to frame by the tensor-core chain for the
    whole sequence, so rounding in the carried state would accumulate here."""
    w = W["gdn_480p_5s"].with_(F=240, L=128, H=4, seed=21)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    ones = torch.ones_like(t["a"])
    beta = torch.sigmoid(t["b"])
    h1 = dict(h)
    h1["a"] = np.ones_like(h["a"])
    h1["b"] = beta.cpu().numpy()
    o_ref, s_ref = oracle.gdn(h1["q"], h1["k"], h1["v"], h1["a"], h1["b"], F=w.F, L=w.L, gates_are_logits=False)
    for impl in ("tc", "tc_pform", "frame_simt"):
        s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], ones, beta, F=w.F, gates_are_logits=False,
                              state_out=s_out, impl=impl)
        torch.cuda.synchronize()
        eo, es = rel_err(o.cpu().numpy(), o_ref), rel_err(s_out.cpu().numpy(), s_ref)
        print(f"alpha=1 drift {impl}: err_o={eo:.3e} err_s={es:.3e}")
        assert eo <= 2e-3 and es <= 2e-3, impl


# ------------------------------------------------------------------ shapes and tails

SHAPES = [  # (F, L, dk, dv, H)
    (1, 1, 32, 32, 1), (2, 16, 64, 64, 2), (3, 63, 112, 112, 1), (2, 64, 112, 112, 2), (2, 65, 112, 112, 1),
    (7, 20, 128, 128, 1), (1, 390, 112, 112, 2), (2, 129, 48, 80, 1), (3, 37, 16, 16, 3),
]


@pytest.mark.parametrize("F,L,dk,dv,H", SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shapes_all_impls(lib, dev, F, L, dk, dv, H, dtype):
    w = W["gdn_480p_5s"].with_(F=F, L=L, dk=dk, dv=dv, H=H, B=1 + (H == 1), dtype=dtype, seed=100 + F + L)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    S0 = np.random.default_rng(L).standard_normal((w.B, w.H, dk, dv)).astype(np.float32)
    o_ref, s_ref = oracle_gdn(h, w, state_in=S0)
    tol = tol_for(w)
    for impl in impls_for(w):
        o, s = run_gdn(lib, w, t, dev, impl, state_in=S0)
        assert rel_err(o, o_ref) <= tol, impl
        assert rel_err(s, s_ref) <= tol, impl


def test_streaming_equals_whole_sequence(lib, dev):
    """F=1 calls that carry the state reproduce one call over all frames (exactly up to
    the fp32 kernels' rounding; within the state hand-off's rounding on tensor cores)."""
    w = W["gdn_480p_5s"].with_(F=4, L=90, H=3)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    for impl in impls_for(w):
        o_all, s_all = run_gdn(lib, w, t, dev, impl)
        S = None
        outs = []
        for f in range(w.F):
            sl = slice(f * w.L, (f + 1) * w.L)
            s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
            o = lib.gdn_frame_fwd(t["q"][:, :, sl].contiguous(), t["k"][:, :, sl].contiguous(),
                                  t["v"][:, :, sl].contiguous(), t["a"][:, :, f:f + 1].contiguous(),
                                  t["b"][:, :, sl].contiguous(), F=1, state_in=S, state_out=s_out, impl=impl)
            outs.append(o)
            S = s_out
        torch.cuda.synchronize()
        o_str = torch.cat(outs, dim=2).cpu().numpy()
        # the fp32 kernels hand the state on in fp32 either way; the tensor-core kernel takes
        # state_in as fp16 high + low parts but hands it from frame to frame as one fp16 image
        tol = 1e-5 if impl in ("seq", "frame_simt") else 1e-3
        assert rel_err(o_str, o_all) <= tol, impl
        assert rel_err(S.cpu().numpy(), s_all) <= tol, impl
    o_ref, s_ref = oracle_gdn(h, w)
    assert rel_err(o_str, o_ref) <= 2e-3 and rel_err(S.cpu().numpy(), s_ref) <= 2e-3


def test_in_place_state_carry(lib, dev):
    w = W["gdn_480p_5s"].with_(F=2, L=50, H=2)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    S0 = np.random.default_rng(5).standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)
    o_ref, s_ref = oracle_gdn(h, w, state_in=S0)
    for impl in impls_for(w):
        S = torch.from_numpy(S0).to(dev)
        o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], t["a"], t["b"], F=w.F, state_in=S, state_out=S, impl=impl)
        torch.cuda.synchronize()
        assert rel_err(o.cpu().numpy(), o_ref) <= 2e-3, impl
        assert rel_err(S.cpu().numpy(), s_ref) <= 2e-3, impl


def test_gate_values_and_edge_gates(lib, dev):
    """Gates passed as values; alpha = 1 with beta = 0 leaves the state unchanged."""
    w = W["gdn_480p_5s"].with_(F=3, L=40, H=2)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    S0 = np.random.default_rng(2).standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)
    ones = torch.ones_like(t["a"])
    zeros = torch.zeros_like(t["b"])
    for impl in impls_for(w):
        s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], ones, zeros, F=w.F, gates_are_logits=False,
                              state_in=torch.from_numpy(S0).to(dev), state_out=s_out, impl=impl)
        torch.cuda.synchronize()
        assert rel_err(s_out.cpu().numpy(), S0) <= 2e-3, impl
        expect = np.einsum("bhnd,bhde->bhne", h["q"].astype(np.float64), S0.astype(np.float64))
        assert rel_err(o.cpu().numpy(), expect) <= 2e-3, impl
    # value gates agree with the logit gates
    al = torch.sigmoid(-t["a"])
    be = torch.sigmoid(t["b"])
    o_ref, s_ref = oracle_gdn(h, w)
    for impl in impls_for(w):
        s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], al, be, F=w.F, gates_are_logits=False, state_out=s_out,
                              impl=impl)
        torch.cuda.synchronize()
        assert rel_err(o.cpu().numpy(), o_ref) <= 2e-3, impl


def test_zero_keys_and_large_values(lib, dev):
    w = W["gdn_480p_5s"].with_(F=2, L=70, H=2, unit_keys=False)
    x = synth.inputs(w)
    x["k"][:, :, 5] = 0.0
    x["k"][:, :, 69:75] = 0.0
    x["k"] *= 7.0   # unnormalised keys
    x["v"] *= 50.0  # larger values
    t, h = device_inputs(w, x, dev, torch)
    o_ref, s_ref = oracle_gdn(h, w)
    for impl in impls_for(w):
        o, s = run_gdn(lib, w, t, dev, impl)
        assert rel_err(o, o_ref) <= 2e-3, impl
        assert rel_err(s, s_ref) <= 2e-3, impl


def test_alpha_one_720p_60s(lib, dev):
    """The 720p-60s workload with no forgetting (alpha = 1 as values) and beta =
    sigmoid of the workload's logits: 240 frames of 920 tokens chained through
    the tensor-core kernels' fp16 frame hand-off, every head and column against
    the oracle."""
    w = W["gdn_720p_60s"]
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    ones = torch.ones_like(t["a"])
    beta = torch.sigmoid(t["b"])
    o_ref, s_ref = oracle.gdn(h["q"], h["k"], h["v"], np.ones_like(h["a"]), beta.cpu().numpy(), F=w.F, L=w.L,
                              gates_are_logits=False)
    for impl in ("tc", "tc_pform"):
        s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], ones, beta, F=w.F, gates_are_logits=False,
                              state_out=s_out, impl=impl)
        torch.cuda.synchronize()
        eo, es = rel_err(o.cpu().numpy(), o_ref), rel_err(s_out.cpu().numpy(), s_ref)
        print(f"720p alpha=1 {impl}: err_o={eo:.3e} err_s={es:.3e}")
        assert eo <= 2e-3 and es <= 2e-3, impl


def test_fp16_range_is_reported(lib, dev):
    """Values the fp16 tensor-core operands cannot hold (|v| or |state_in| >= 65504) end
    with GDN_ERR_RANGE in *status instead of passing silently; in-range inputs do not."""
    w = W["gdn_480p_5s"].with_(F=2, L=80, H=2)
    x = synth.inputs(w)
    x["v"][0, 1, 17] *= 1e5
    t, h = device_inputs(w, x, dev, torch)
    for impl in ("tc", "tc_pform"):
        status = torch.zeros(4, dtype=torch.int32, device=dev)
        run_gdn(lib, w, t, dev, impl, status=status)
        assert int(status[0].item()) == lib.ERR_RANGE, impl
    w2 = w.with_(seed=5)
    x2 = synth.inputs(w2)
    t2, _ = device_inputs(w2, x2, dev, torch)
    big = np.zeros((w.B, w.H, w.dk, w.dv), np.float32)
    big[0, 0, 3, 4] = 1e5
    for impl in ("tc", "tc_pform"):
        status = torch.zeros(4, dtype=torch.int32, device=dev)
        run_gdn(lib, w2, t2, dev, impl, state_in=big, status=status)
        assert int(status[0].item()) == lib.ERR_RANGE, impl
        status.zero_()
        run_gdn(lib, w2, t2, dev, impl, status=status)
        assert int(status[0].item()) == 0, impl


def test_few_ctas_many_frames(lib, dev):
    """A persistent grid far smaller than the frame count still completes the chain."""
    w = W["gdn_480p_5s"].with_(F=30, L=33, H=3)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    o_ref, s_ref = oracle_gdn(h, w)
    for impl in impls_for(w):
        if impl == "seq":
            continue
        for ctas in (1, 2, 7):
            o, s = run_gdn(lib, w, t, dev, impl, max_ctas=ctas)
            assert rel_err(o, o_ref) <= 2e-3, (impl, ctas)
            assert rel_err(s, s_ref) <= 2e-3, (impl, ctas)


def test_deterministic(lib, dev):
    w = W["gdn_480p_5s"].with_(F=5, L=100, H=4)
    x = synth.inputs(w)
    t, _ = device_inputs(w, x, dev, torch)
    for impl in impls_for(w):
        o1, s1 = run_gdn(lib, w, t, dev, impl)
        o2, s2 = run_gdn(lib, w, t, dev, impl)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(s1, s2)


def test_host_entry_point(lib, dev):
    w = W["gdn_480p_5s"].with_(F=3, L=64, H=2)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    o_dev, s_dev = run_gdn(lib, w, t, dev, "auto")
    qh, kh, vh = (t[n].cpu().pin_memory() for n in "qkv")
    ah, bh = t["a"].cpu().pin_memory(), t["b"].cpu().pin_memory()
    o_h = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32).pin_memory()
    s_h = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32).pin_memory()
    lib.gdn_frame_fwd_host(qh, kh, vh, ah, bh, F=w.F, o=o_h, state_out=s_h)
    # frame groups pass the state through fp32 state_in (high + low fp16 parts), inside
    # one call it passes as one fp16 image: equal within that rounding, and both parity
    o_ref, s_ref = oracle_gdn(h, w)
    assert rel_err(o_h.numpy(), o_ref) <= 2e-3 and rel_err(s_h.numpy(), s_ref) <= 2e-3
    assert rel_err(o_h.numpy(), o_dev) <= 1e-3 and rel_err(s_h.numpy(), s_dev) <= 1e-3


def test_device_timeout_status_is_reported(lib, dev):
    """A chain wait that is never satisfied ends with GDN_ERR_TIMEOUT in *status.

    The test asks the kernel to withhold the publish of frame 0 of head 0, so
    the wait of frame 1 of that head runs out after 2 ms; the kernel returns
    cleanly and the context stays usable for the next call.
    """
    w = W["gdn_480p_5s"].with_(F=3, L=16, H=1)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    for impl in [i for i in impls_for(w) if i != "seq"]:
        status = torch.zeros(4, dtype=torch.int32, device=dev)
        run_gdn(lib, w, t, dev, impl, spin_limit_us=2000, status=status, test_withhold_unit=0)
        assert int(status[0].item()) == lib.ERR_TIMEOUT, impl
        status.zero_()
        o, s = run_gdn(lib, w, t, dev, impl, status=status)
        assert int(status[0].item()) == 0
        o_ref, s_ref = oracle_gdn(h, w)
        assert rel_err(o, o_ref) <= 2e-3


# ------------------------------------------------------------------ frames split into chunk segments

SEG_SHAPES = [  # (B, H, F, L, dk, dv): several chunks per frame, ragged last chunk, dk != dv
    (1, 2, 1, 390, 112, 112), (2, 3, 3, 300, 112, 112), (1, 1, 2, 200, 48, 80), (1, 4, 1, 129, 128, 128),
]


@pytest.mark.parametrize("B,H,F,L,dk,dv", SEG_SHAPES)
def test_segments_match_oracle(lib, dev, B, H, F, L, dk, dv):
    """A frame split into P segments (each its own CTA, chained in order, all
    reading out against the frame's last state) matches the oracle for every P."""
    w = W["gdn_480p_5s"].with_(B=B, H=H, F=F, L=L, dk=dk, dv=dv, seed=7 + L)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    S0 = np.random.default_rng(L + 1).standard_normal((B, H, dk, dv)).astype(np.float32)
    o_ref, s_ref = oracle_gdn(h, w, state_in=S0)
    nch = (L + 63) // 64
    outs = {}
    for P in sorted({0, 1, 2, 3, nch}):
        o, s = run_gdn(lib, w, t, dev, "tc", state_in=S0, segments=P)
        assert rel_err(o, o_ref) <= 2e-3, P
        assert rel_err(s, s_ref) <= 2e-3, P
        outs[P] = o
    # the automatic choice splits these frames (few frames, several chunks)
    assert not np.array_equal(outs[0], outs[1]) or nch == 1


def test_streaming_frame_720p_segments(lib, dev):
    """One 720p frame of 20 heads (the streaming call) against the oracle, with
    the automatic segment count, one segment, and state_out left unwritten."""
    w = W["gdn_720p_60s"].with_(F=1, seed=11)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    S0 = 0.1 * np.random.default_rng(3).standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)
    o_ref, s_ref = oracle_gdn(h, w, state_in=S0)
    for P in (0, 1):
        o, s = run_gdn(lib, w, t, dev, "tc", state_in=S0, segments=P)
        assert rel_err(o, o_ref) <= 2e-3, P
        assert rel_err(s, s_ref) <= 2e-3, P
        o2, _ = run_gdn(lib, w, t, dev, "tc", state_in=S0, want_state=False, segments=P)
        np.testing.assert_array_equal(o2, o)


def test_segment_timeout_status_is_reported(lib, dev):
    """In segment mode a withheld segment state makes the next segment's chain
    wait and the earlier segment's read-out wait run out; both end cleanly."""
    w = W["gdn_480p_5s"].with_(B=2, H=1, F=1, L=200)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    # tickets (f, segment, b*H + h): ticket 0 = segment 0 of head 0
    run_gdn(lib, w, t, dev, "tc", spin_limit_us=2000, status=status, test_withhold_unit=0, segments=2)
    assert int(status[0].item()) == lib.ERR_TIMEOUT
    status.zero_()
    o, s = run_gdn(lib, w, t, dev, "tc", status=status, segments=2)
    assert int(status[0].item()) == 0
    o_ref, s_ref = oracle_gdn(h, w)
    assert rel_err(o, o_ref) <= 2e-3
    assert rel_err(s, s_ref) <= 2e-3


# ------------------------------------------------------------------ streaming block-cache protocol

def _stream_call_inputs(w, c, dev):
    x = synth.inputs(w, call=c)
    t = {n: torch.from_numpy(x[n]).to(torch.bfloat16) for n in "qkv"}
    host = {n: t[n].float().numpy() for n in "qkv"}
    host.update(a=x["a"], b=x["b"])
    dv_ = {n: t[n].to(dev).contiguous() for n in "qkv"}
    dv_.update(a=torch.from_numpy(x["a"]).to(dev), b=torch.from_numpy(x["b"]).to(dev))
    return dv_, host


@pytest.mark.parametrize("segments", [0, 1])
def test_streaming_protocol_720p(lib, dev, segments):
    """The streaming block-cache decode at the 720p frame shape (20 heads, one
    920-token frame per call): 8 frames x 4 denoising steps, fresh q, k, v and
    gates on every call, state_out = NULL on steps 1-3 and the committed state
    on step 4, which becomes the next frame's state_in.  Every call's o and
    every committed state are compared with the streaming oracle, and a
    non-committing call must leave state_in byte for byte as it was."""
    steps, frames = 4, 8
    w = W["gdn_stream_720p"]
    calls = [_stream_call_inputs(w, c, dev) for c in range(frames * steps)]
    outs_ref, _, committed_ref = oracle.gdn_stream(lambda c: calls[c][1] if c < len(calls) else None,
                                                   steps=steps, L=w.L)
    shape_s = (w.B, w.H, w.dk, w.dv)
    s_cur = None
    worst_o = worst_s = 0.0
    for f in range(frames):
        s_next = torch.empty(shape_s, dtype=torch.float32, device=dev)
        before = None if s_cur is None else s_cur.clone()
        for st in range(steps):
            c = f * steps + st
            t = calls[c][0]
            commit = st == steps - 1
            o = lib.gdn_frame_fwd(t["q"], t["k"], t["v"], t["a"], t["b"], F=1, state_in=s_cur,
                                  state_out=s_next if commit else None, segments=segments)
            torch.cuda.synchronize()
            e = rel_err(o.cpu().numpy(), outs_ref[c])
            worst_o = max(worst_o, e)
            assert e <= 2e-3, (f, st, e)
            if not commit and before is not None:
                assert torch.equal(s_cur, before), (f, st)  # state_in untouched
        e = rel_err(s_next.cpu().numpy(), committed_ref[f])
        worst_s = max(worst_s, e)
        assert e <= 2e-3, (f, e)
        s_cur = s_next
    print(f"streaming protocol segments={segments}: worst err_o={worst_o:.3e} err_s={worst_s:.3e}")


# ------------------------------------------------------------------ 3D rotary position embedding

ROPE_SHAPES = [  # (F, L, grid_w, dk, dv, H, frame_offset)
    (3, 40, 8, 112, 112, 2, 0), (2, 129, 43, 64, 64, 1, 5), (4, 30, 6, 48, 80, 2, 11), (1, 920, 40, 112, 112, 3, 17),
]


@pytest.mark.parametrize("F,L,gw,dk,dv,H,off", ROPE_SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rope_matches_oracle(lib, dev, F, L, gw, dk, dv, H, off, dtype):
    """q and k rotated by the 3D position embedding (latent grid L / gw x gw,
    frames numbered from off) against the oracle, on every kernel that takes it."""
    w = W["gdn_480p_5s"].with_(F=F, L=L, dk=dk, dv=dv, H=H, dtype=dtype, seed=300 + L + dk)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    rope = dict(grid_w=gw, frame_offset=off)
    S0 = np.random.default_rng(L).standard_normal((w.B, w.H, dk, dv)).astype(np.float32)
    o_ref, s_ref = oracle.gdn(h["q"], h["k"], h["v"], h["a"], h["b"], F=w.F, L=w.L, state_in=S0, rope=rope)
    tol = tol_for(w)
    for impl in [i for i in impls_for(w) if i != "tc_pform"]:
        o, s = run_gdn(lib, w, t, dev, impl, state_in=S0, rope=rope)
        eo, es = rel_err(o, o_ref), rel_err(s, s_ref)
        print(f"rope {F}x{L} gw={gw} d={dk}/{dv} {dtype} {impl}: err_o={eo:.3e} err_s={es:.3e}")
        assert eo <= tol and es <= tol, impl
    if dtype == "bf16":  # the tensor-core kernel with chunk segments (several CTAs per frame)
        o, s = run_gdn(lib, w, t, dev, "tc", state_in=S0, rope=rope, segments=3)
        assert rel_err(o, o_ref) <= tol and rel_err(s, s_ref) <= tol


def test_rope_resumed_call_and_host_entry(lib, dev):
    """A sequence cut in two calls, the second with frame_offset = the frames of
    the first, gives the one-call result; the host-buffer call (which streams
    frame groups with their offsets) equals the device call."""
    w = W["gdn_480p_5s"].with_(F=6, L=60, H=2, seed=41)
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    rope = dict(grid_w=10, frame_offset=3)
    o_all, s_all = run_gdn(lib, w, t, dev, "tc", rope=rope)
    cut = 4 * w.L
    w1, w2 = w.with_(F=4), w.with_(F=2)
    t1 = {n: (t[n][:, :, :cut] if n != "a" else t[n][:, :, :4]).contiguous() for n in "qkvab"}
    t2 = {n: (t[n][:, :, cut:] if n != "a" else t[n][:, :, 4:]).contiguous() for n in "qkvab"}
    _, s1 = run_gdn(lib, w1, t1, dev, "tc", rope=rope)
    o2, s2 = run_gdn(lib, w2, t2, dev, "tc", state_in=s1, rope=dict(grid_w=10, frame_offset=7))
    assert rel_err(o2, o_all[:, :, cut:]) <= 2e-3 and rel_err(s2, s_all) <= 2e-3
    o_ref, s_ref = oracle.gdn(h["q"], h["k"], h["v"], h["a"], h["b"], F=w.F, L=w.L, rope=rope)
    assert rel_err(o_all, o_ref) <= 2e-3
    qh, kh, vh = (t[n].cpu().pin_memory() for n in "qkv")
    ah, bh = t["a"].cpu().pin_memory(), t["b"].cpu().pin_memory()
    o_h = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32).pin_memory()
    lib.gdn_frame_fwd_host(qh, kh, vh, ah, bh, F=w.F, o=o_h, rope=rope)
    assert rel_err(o_h.numpy(), o_ref) <= 2e-3
    assert rel_err(o_h.numpy(), o_all) <= 1e-3


def test_rope_720p_60s_full(lib, dev):
    """The 720p-60s workload with the 3D position embedding on its 23 x 40 latent
    grid: every head and column against the oracle."""
    w = W["gdn_720p_60s"]
    x = synth.inputs(w)
    t, h = device_inputs(w, x, dev, torch)
    rope = dict(grid_w=40)
    o, s = run_gdn(lib, w, t, dev, "tc", rope=rope)
    o_ref, s_ref = oracle.gdn(h["q"], h["k"], h["v"], h["a"], h["b"], F=w.F, L=w.L, rope=rope)
    eo, es = rel_err(o, o_ref), rel_err(s, s_ref)
    print(f"rope 720p tc: err_o={eo:.3e} err_s={es:.3e}")
    assert eo <= 2e-3 and es <= 2e-3


def test_rope_refusals(lib, dev):
    w = W["gdn_480p_5s"].with_(F=2, L=64, H=1)
    x = synth.inputs(w)
    t, _ = device_inputs(w, x, dev, torch)
    with pytest.raises(lib.GdnError) as e:
        run_gdn(lib, w, t, dev, "tc_pform", rope=dict(grid_w=8))
    assert e.value.code == lib.ERR_UNSUPPORTED
    with pytest.raises(lib.GdnError) as e:
        run_gdn(lib, w, t, dev, "tc", rope=dict(grid_w=7))  # L is not a multiple of the grid width
    assert e.value.code == lib.ERR_INVALID_ARG
