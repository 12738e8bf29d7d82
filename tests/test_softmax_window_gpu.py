"""GPU parity of the windowed block-causal softmax attention against the fp64
CPU oracle, called through the C ABI.

Bar: max|o - o_ref| <= 2e-3 * max|o_ref| (bf16 inputs), the bound every mode of
the library meets.  The kernel forms the scores exactly (bf16 products, fp32
sums) and rounds the probabilities and v to fp16 (11-bit significands) for the
second product, so its error sits far below the bar.
"""
import numpy as np
import pytest

from helpers import oracle, rel_err, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def lib():
    import linear_attention_video_gdn_b200 as lib
    return lib


@pytest.fixture(scope="module")
def dev():
    return torch.device("cuda", 0)


def inputs(B, H, F, L, dk, dv, seed, q_scale=1.0, dev=None):
    """bf16 device tensors and the exact float32 values they hold."""
    N = F * L
    q = synth.normal(seed, 0, 0, B * H * N * dk, std=q_scale).reshape(B, H, N, dk)
    k = synth.normal(seed, 1, 0, B * H * N * dk).reshape(B, H, N, dk)
    v = synth.normal(seed, 2, 0, B * H * N * dv).reshape(B, H, N, dv)
    t = [torch.from_numpy(x).to(torch.bfloat16).to(dev) for x in (q, k, v)]
    return t, [x.float().cpu().numpy() for x in t]


# B, H, F, L, dk, dv, W: several query and key tiles with ragged ends, one-token
# frames, windows of one frame and wider than the sequence, dk != dv
SHAPES = [(1, 2, 3, 64, 64, 64, 2), (1, 1, 4, 100, 112, 112, 3), (2, 2, 5, 37, 32, 32, 1),
          (1, 2, 2, 300, 128, 128, 2), (1, 1, 6, 20, 16, 16, 10), (1, 2, 3, 70, 64, 112, 2),
          (1, 1, 8, 1, 32, 48, 3), (1, 3, 2, 129, 112, 112, 4)]


@pytest.mark.parametrize("shape", SHAPES)
def test_matches_oracle(lib, dev, shape):
    B, H, F, L, dk, dv, W = shape
    (q, k, v), (qh, kh, vh) = inputs(B, H, F, L, dk, dv, seed=50 + L, dev=dev)
    o = lib.softmax_window_fwd(q, k, v, F=F, W=W)
    torch.cuda.synchronize()
    ref = oracle.softmax_window(qh, kh, vh, F=F, L=L, W=W)
    assert rel_err(o.cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("q_scale", [4.0, 12.0])
def test_peaked_scores_and_rescaling(lib, dev, q_scale):
    """Large scores: the running maximum moves across key tiles (O and the row
    sum are rescaled in place) and the softmax is nearly one-hot."""
    B, H, F, L, d, W = 1, 2, 4, 150, 64, 4
    (q, k, v), (qh, kh, vh) = inputs(B, H, F, L, d, d, seed=61, q_scale=q_scale, dev=dev)
    o = lib.softmax_window_fwd(q, k, v, F=F, W=W)
    torch.cuda.synchronize()
    ref = oracle.softmax_window(qh, kh, vh, F=F, L=L, W=W)
    assert rel_err(o.cpu().numpy(), ref) <= TOL


def test_growing_scores_force_every_rescale(lib, dev):
    """Keys whose scores grow from frame to frame: each new key tile exceeds the
    running maximum, so every tile takes the rescaling path."""
    B, H, F, L, d, W = 1, 1, 6, 64, 32, 6
    (q, k, v), (qh, kh, vh) = inputs(B, H, F, L, d, d, seed=62, dev=dev)
    q = torch.ones_like(q)
    ramp = torch.arange(F * L, device=dev, dtype=torch.float32).reshape(1, 1, F * L, 1) * (12.0 / (F * L))
    k = (torch.ones_like(k).float() * ramp).to(torch.bfloat16)
    o = lib.softmax_window_fwd(q, k, v, F=F, W=W)
    torch.cuda.synchronize()
    ref = oracle.softmax_window(q.float().cpu().numpy(), k.float().cpu().numpy(), vh, F=F, L=L, W=W)
    assert rel_err(o.cpu().numpy(), ref) <= TOL


def test_explicit_scale(lib, dev):
    B, H, F, L, d, W = 1, 2, 3, 90, 48, 2
    (q, k, v), (qh, kh, vh) = inputs(B, H, F, L, d, d, seed=63, dev=dev)
    o = lib.softmax_window_fwd(q, k, v, F=F, W=W, scale=0.37)
    torch.cuda.synchronize()
    assert rel_err(o.cpu().numpy(), oracle.softmax_window(qh, kh, vh, F=F, L=L, W=W, scale=0.37)) <= TOL


def test_720p_60s_window4_sampled_frames(lib, dev):
    """The benchmark's workload (B=1, H=20, F=240, L=920, d=112, W=4) in the
    launch the benchmark times; the oracle recomputes frames 0, 1, 2, 3, 117 and
    239 of every head (every query row of those frames, all columns)."""
    B, H, F, L, d, W = 1, 20, 240, 920, 112, 4
    (q, k, v), (qh, kh, vh) = inputs(B, H, F, L, d, d, seed=7, dev=dev)
    o = lib.softmax_window_fwd(q, k, v, F=F, W=W)
    torch.cuda.synchronize()
    frames = [0, 1, 2, 3, 117, 239]
    ref = oracle.softmax_window(qh, kh, vh, F=F, L=L, W=W, frames=frames)
    oh = o.cpu().numpy()
    del o, q, k, v
    assert rel_err(oh, ref) <= TOL


def test_large_values_and_refusals(lib, dev):
    (q, k, v), (qh, kh, vh) = inputs(1, 2, 3, 40, 32, 32, seed=64, dev=dev)
    big = (v.float() * 3000.0).to(torch.bfloat16)  # large values inside the fp16 range of the second product
    o = lib.softmax_window_fwd(q, k, big, F=3, W=2)
    torch.cuda.synchronize()
    assert rel_err(o.cpu().numpy(), oracle.softmax_window(qh, kh, big.float().cpu().numpy(), F=3, L=40, W=2)) <= TOL
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    huge = v.clone()
    huge[0, 1, 17, 5] = 70000.0  # past the fp16 range: reported, not silently wrong
    lib.softmax_window_fwd(q, k, huge, F=3, W=2, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == lib.ERR_RANGE
    lib.softmax_window_fwd(q, k, huge, F=3, W=2, impl="frame_simt")  # the fp32 path takes it
    torch.cuda.synchronize()
    with pytest.raises(lib.GdnError) as e:  # the tensor-core kernel takes bf16 only
        lib.softmax_window_fwd(q.float(), k.float(), v.float(), F=3, W=1, impl="tc")
    assert e.value.code == lib.ERR_UNSUPPORTED
    with pytest.raises(lib.GdnError) as e:  # ... and d a multiple of 16
        lib.softmax_window_fwd(q[..., :24].contiguous(), k[..., :24].contiguous(), v, F=3, W=1, impl="tc")
    assert e.value.code == lib.ERR_UNSUPPORTED
    with pytest.raises(lib.GdnError) as e:
        lib.softmax_window_fwd(q, k, v, F=3, W=0)
    assert e.value.code == lib.ERR_INVALID_ARG


# fp32 inputs (CUDA cores, bar 1e-5) and bf16 shapes the tensor cores do not take
@pytest.mark.parametrize("B,H,F,L,dk,dv,W,dtype", [(1, 2, 3, 37, 32, 32, 2, "f32"), (2, 1, 5, 20, 24, 40, 3, "f32"),
                                                   (1, 1, 4, 9, 128, 100, 10, "f32"), (1, 2, 3, 50, 24, 24, 2, "bf16"),
                                                   (1, 2, 3, 64, 64, 64, 2, "bf16")])
def test_cuda_core_path(lib, dev, B, H, F, L, dk, dv, W, dtype):
    N = F * L
    x = [synth.normal(70 + L, t, 0, B * H * N * d).reshape(B, H, N, d) for t, d in enumerate((dk, dk, dv))]
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    q, k, v = (torch.from_numpy(a).to(dt).to(dev) for a in x)
    o = lib.softmax_window_fwd(q, k, v, F=F, W=W, impl="frame_simt")
    torch.cuda.synchronize()
    ref = oracle.softmax_window(*(t.float().cpu().numpy() for t in (q, k, v)), F=F, L=L, W=W)
    assert rel_err(o.cpu().numpy(), ref) <= (1e-5 if dtype == "f32" else TOL)
