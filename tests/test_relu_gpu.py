"""GPU parity of block-causal ReLU linear attention against the fp64 CPU oracle.

Bar: max|gpu - oracle| <= tol * max|oracle| for o, kv_out and z_out; tol = 2e-3
for bf16 inputs, 1e-5 for fp32 inputs.
"""
import numpy as np
import pytest

from helpers import oracle, rel_err, synth

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


def prep(w, x, dev):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {n: torch.from_numpy(x[n]).to(dt).to(dev).contiguous() for n in "qkv"}
    h = {n: t[n].float().cpu().numpy() for n in "qkv"}
    return t, h


def impls_for(w):
    out = ["frame_simt"]
    if w.dtype == "bf16" and w.dk % 16 == 0 and w.dv % 16 == 0 and w.dv <= 112:
        out.append("tc")
    return out


def run(lib, w, t, dev, impl, kv_in=None, z_in=None, **kw):
    kv_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    z_out = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device=dev)
    to = lambda a: None if a is None else torch.from_numpy(np.asarray(a, np.float32)).to(dev)
    o = lib.relu_la_block_fwd(t["q"], t["k"], t["v"], F=w.F, kv_in=to(kv_in), z_in=to(z_in), kv_out=kv_out,
                              z_out=z_out, impl=impl, **kw)
    torch.cuda.synchronize()
    return o.cpu().numpy(), kv_out.cpu().numpy(), z_out.cpu().numpy()


@pytest.mark.parametrize("impl", ["frame_simt", "tc"])
def test_relu_720p_81f_full(lib, dev, impl):
    """Full-size workload (B=2, H=20, F=81, L=920): every head, o, kv_out and
    z_out against the oracle (heads spread over the host cores)."""
    w = W["relu_720p_81f"]
    x = synth.inputs(w)
    t, h = prep(w, x, dev)
    o, kv, z = run(lib, w, t, dev, impl)
    o_ref, kv_ref, z_ref = oracle.relu_la(h["q"], h["k"], h["v"], F=w.F, L=w.L)
    eo, ek, ez = rel_err(o, o_ref), rel_err(kv, kv_ref), rel_err(z, z_ref)
    print(f"relu 720p {impl}: err_o={eo:.3e} err_kv={ek:.3e} err_z={ez:.3e}")
    assert eo <= 2e-3 and ek <= 2e-3 and ez <= 2e-3


SHAPES = [(1, 1, 32, 32, 1), (3, 63, 112, 112, 2), (2, 64, 64, 64, 1), (2, 65, 112, 112, 1), (5, 20, 128, 128, 1),
          (2, 100, 48, 80, 1), (4, 17, 16, 16, 3)]


@pytest.mark.parametrize("F,L,dk,dv,H", SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_relu_shapes(lib, dev, F, L, dk, dv, H, dtype):
    w = W["relu_720p_81f"].with_(F=F, L=L, dk=dk, dv=dv, H=H, B=1, dtype=dtype, seed=200 + F + L)
    x = synth.inputs(w)
    t, h = prep(w, x, dev)
    rng = np.random.default_rng(L)
    kv0 = rng.standard_normal((w.B, w.H, dk, dv)).astype(np.float32)
    z0 = np.abs(rng.standard_normal((w.B, w.H, dk))).astype(np.float32) * 5
    o_ref, kv_ref, z_ref = oracle.relu_la(h["q"], h["k"], h["v"], F=F, L=L, kv_in=kv0, z_in=z0)
    tol = 2e-3 if dtype == "bf16" else 1e-5
    for impl in impls_for(w):
        o, kv, z = run(lib, w, t, dev, impl, kv_in=kv0, z_in=z0)
        assert rel_err(o, o_ref) <= tol, impl
        assert rel_err(kv, kv_ref) <= tol, impl
        assert rel_err(z, z_ref) <= tol, impl


def test_relu_zero_query_gives_zero(lib, dev):
    w = W["relu_720p_81f"].with_(F=2, L=40, H=1, B=1)
    x = synth.inputs(w)
    x["q"][0, 0, 3] = -np.abs(x["q"][0, 0, 3])
    t, h = prep(w, x, dev)
    for impl in impls_for(w):
        o, _, _ = run(lib, w, t, dev, impl)
        assert np.all(o[0, 0, 3] == 0.0), impl


def test_relu_state_carry_split(lib, dev):
    w = W["relu_720p_81f"].with_(F=6, L=50, H=2, B=1)
    x = synth.inputs(w)
    t, h = prep(w, x, dev)
    for impl in impls_for(w):
        o, kv, z = run(lib, w, t, dev, impl)
        w1 = w.with_(F=3)
        t1 = {n: t[n][:, :, :150].contiguous() for n in "qkv"}
        t2 = {n: t[n][:, :, 150:].contiguous() for n in "qkv"}
        o1, kv1, z1 = run(lib, w1, t1, dev, impl)
        o2, kv2, z2 = run(lib, w1, t2, dev, impl, kv_in=kv1, z_in=z1)
        assert rel_err(np.concatenate([o1, o2], axis=2), o) <= 1e-5, impl
        assert rel_err(kv2, kv) <= 1e-5 and rel_err(z2, z) <= 1e-5, impl


def test_relu_timeout_status(lib, dev):
    w = W["relu_720p_81f"].with_(F=3, L=16, H=1, B=1)
    x = synth.inputs(w)
    t, h = prep(w, x, dev)
    for impl in impls_for(w):
        status = torch.zeros(4, dtype=torch.int32, device=dev)
        run(lib, w, t, dev, impl, spin_limit_us=2000, status=status, test_withhold_unit=0)
        assert int(status[0].item()) == lib.ERR_TIMEOUT, impl
        status.zero_()
        o, _, _ = run(lib, w, t, dev, impl, status=status)
        assert int(status[0].item()) == 0
        o_ref, _, _ = oracle.relu_la(h["q"], h["k"], h["v"], F=w.F, L=w.L)
        assert rel_err(o, o_ref) <= 2e-3


@pytest.mark.parametrize("ctas", [1, 2, 3])
def test_relu_few_ctas_odd_tiles(lib, dev, ctas):
    """One persistent CTA runs many frames whose read-out has an odd number of
    128-token tiles (L=300: 3 tiles), so its two accumulator buffers change
    roles from one frame to the next."""
    w = W["relu_720p_81f"].with_(F=5, L=300, H=2, B=1, seed=77)
    x = synth.inputs(w)
    t, h = prep(w, x, dev)
    o_ref, kv_ref, z_ref = oracle.relu_la(h["q"], h["k"], h["v"], F=w.F, L=w.L)
    o, kv, z = run(lib, w, t, dev, "tc", max_ctas=ctas)
    assert rel_err(o, o_ref) <= 2e-3
    assert rel_err(kv, kv_ref) <= 2e-3
    assert rel_err(z, z_ref) <= 2e-3
