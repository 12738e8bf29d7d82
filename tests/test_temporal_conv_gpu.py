"""GPU parity of the causal temporal convolution with the block-boundary cache
against the fp64 CPU oracle, called through the C ABI.

Bar, per element: the kernel forms y in fp32 (three fused multiply-adds, each
rounded once) and rounds it once to the element type, so
    |y - y_ref| <= u_out * |y_ref| + 4e-7 * s,
with s = |w0 x[f-1]| + |w1 x[f]| + |w2 x[f+1]| + |bias| (fp32 rounding of the
sum, 3 * 2^-24 * s < 4e-7 * s) and u_out = 2^-8 for bf16 outputs (round to
nearest), 0 for fp32.  The cache is a copy of the block's last frame: exact.
"""
import numpy as np
import pytest

from helpers import oracle, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CW = synth.CONV_WORKLOADS


@pytest.fixture(scope="module")
def lib():
    import linear_attention_video_gdn_b200 as lib
    return lib


@pytest.fixture(scope="module")
def dev():
    return torch.device("cuda", 0)


def _dt(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_dev(x, dtype, dev):
    """Device tensor of x in the workload dtype and the exact float32 values it holds."""
    t = torch.from_numpy(np.ascontiguousarray(x)).to(_dt(dtype)).to(dev).contiguous()
    return t, t.float().cpu().numpy()


def abs_scale(x, w, bias, cache_in):
    """|w0 x[f-1]| + |w1 x[f]| + |w2 x[f+1]| + |bias| per element (fp64), the same
    neighbours as the method (cache_in before the block, zero after it)."""
    xd = x.astype(np.float64)
    prev = np.concatenate([np.zeros_like(xd[:, :1]) if cache_in is None else cache_in[:, None].astype(np.float64),
                           xd[:, :-1]], axis=1)
    nxt = np.concatenate([xd[:, 1:], np.zeros_like(xd[:, :1])], axis=1)
    wd = np.abs(w.astype(np.float64))
    s = wd[:, 0] * np.abs(prev) + wd[:, 1] * np.abs(xd) + wd[:, 2] * np.abs(nxt)
    if bias is not None:
        s = s + np.abs(bias.astype(np.float64))
    return s


def check_y(y, ref, scale, dtype):
    u = 2.0 ** -8 if dtype == "bf16" else 0.0
    y = y.astype(np.float64)
    bound = u * np.abs(ref) + 4e-7 * scale + 1e-30
    bad = np.abs(y - ref) > bound
    assert not bad.any(), (f"{int(bad.sum())} elements out of bound; worst excess "
                           f"{float(np.max(np.abs(y - ref) - bound)):.3e}")


def run_case(lib, dev, B, F, HW, C, dtype, *, seed=11, bias=True, cache=True, max_ctas=0, inplace=False):
    cw = synth.ConvWorkload("case", B, F, HW, C, dtype, seed)
    inp = synth.conv_inputs(cw)
    x, xh = to_dev(inp["x"], dtype, dev)
    w = torch.from_numpy(inp["w"]).to(dev)
    b = torch.from_numpy(inp["bias"]).to(dev) if bias else None
    if cache:
        ci_np = synth.normal(seed, 7, 0, B * HW * C).reshape(B, HW, C)
        ci, ci_h = to_dev(ci_np, dtype, dev)
    else:
        ci, ci_h = None, None
    co = ci if inplace else torch.empty((B, HW, C), dtype=_dt(dtype), device=dev)
    y = lib.temporal_conv_fwd(x, w, bias=b, cache_in=ci, cache_out=co, max_ctas=max_ctas)
    torch.cuda.synchronize()
    ref, ref_cache = oracle.temporal_conv(xh, inp["w"], bias=inp["bias"] if bias else None, cache_in=ci_h)
    check_y(y.float().cpu().numpy(), ref, abs_scale(xh, inp["w"], inp["bias"] if bias else None, ci_h), dtype)
    np.testing.assert_array_equal(co.float().cpu().numpy(), ref_cache)
    return y


# B, F, HW, C: vector columns (C % 8 == 0), several tiles of 128 columns with a
# ragged last tile, single-element columns (C not a multiple of the vector),
# one frame, frame counts around the prefetch depths, and frame counts above
# the 32-frame run of one CTA (runs that start and end inside a column, with
# a halo frame on each side), exactly two runs, and one frame past a run.
SHAPES = [(1, 5, 7, 16), (2, 13, 300, 64), (1, 1, 9, 24), (2, 6, 5, 12), (1, 9, 33, 6), (3, 4, 2, 8),
          (1, 8, 130, 40), (1, 70, 33, 16), (2, 64, 9, 24), (1, 33, 20, 8), (1, 100, 5, 6), (2, 45, 7, 12)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", SHAPES)
def test_matches_oracle(lib, dev, shape, dtype):
    run_case(lib, dev, *shape, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bias,cache", [(False, False), (True, False), (False, True)])
def test_optional_arguments(lib, dev, dtype, bias, cache):
    run_case(lib, dev, 2, 7, 20, 32, dtype, bias=bias, cache=cache)


@pytest.mark.parametrize("max_ctas", [1, 3, 7, 50])
def test_few_ctas_loop_over_runs(lib, dev, max_ctas):
    """A capped grid: every CTA loops over several runs of several column tiles,
    including runs that start and end inside a column (halo frames)."""
    run_case(lib, dev, 2, 75, 40, 32, "bf16", max_ctas=max_ctas)
    run_case(lib, dev, 1, 41, 45, 12, "f32", max_ctas=max_ctas)


def test_in_place_cache(lib, dev):
    run_case(lib, dev, 2, 9, 40, 48, "bf16", inplace=True, max_ctas=5)
    run_case(lib, dev, 1, 70, 30, 16, "bf16", inplace=True)
    run_case(lib, dev, 1, 40, 30, 20, "f32", inplace=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_streaming_blocks_equal_training_construction(lib, dev, dtype):
    """Blocks called one after another with the cache carried (in place) equal
    the oracle's block-by-block run and, through the oracle's pin, the
    zero-token training construction over the whole sequence."""
    B, HW, C, Fb = 1, 37, 24, [3, 1, 5, 4]
    w = synth.normal(21, 1, 0, C * 3, std=3.0 ** -0.5).reshape(C, 3)
    bias = synth.normal(21, 2, 0, C, std=0.1)
    wd, bd = torch.from_numpy(w).to(dev), torch.from_numpy(bias).to(dev)
    cache = torch.zeros((B, HW, C), dtype=_dt(dtype), device=dev)
    ref_cache = None
    for i, F in enumerate(Fb):
        xi, xh = to_dev(synth.normal(21, 8 * (i + 1), 0, B * F * HW * C).reshape(B, F, HW, C), dtype, dev)
        y = lib.temporal_conv_fwd(xi, wd, bias=bd, cache_in=cache if i else None, cache_out=cache)
        torch.cuda.synchronize()
        ref, ref_cache_next = oracle.temporal_conv(xh, w, bias=bias, cache_in=ref_cache)
        check_y(y.float().cpu().numpy(), ref, abs_scale(xh, w, bias, ref_cache), dtype)
        np.testing.assert_array_equal(cache.float().cpu().numpy(), ref_cache_next)
        ref_cache = ref_cache_next.astype(np.float32)


def test_720p_60s_full(lib, dev):
    """The full 720p 60 s block (B=1, F=240, HW=920, C=2240, bf16) in the launch
    the benchmark times; every element checked against the oracle."""
    cw = CW["tconv_720p_60s"]
    inp = synth.conv_inputs(cw)
    x, xh = to_dev(inp["x"], cw.dtype, dev)
    del inp["x"]
    w, b = torch.from_numpy(inp["w"]).to(dev), torch.from_numpy(inp["bias"]).to(dev)
    ci_np = synth.normal(cw.seed, 7, 0, cw.HW * cw.C).reshape(1, cw.HW, cw.C)
    ci, ci_h = to_dev(ci_np, cw.dtype, dev)
    co = torch.empty_like(ci)
    y = lib.temporal_conv_fwd(x, w, bias=b, cache_in=ci, cache_out=co)
    torch.cuda.synchronize()
    del x
    yh = y.float().cpu().numpy()
    del y
    # the oracle over slices of latent positions (columns are independent)
    for n0 in range(0, cw.HW, 92):
        sl = slice(n0, n0 + 92)
        ref, rc = oracle.temporal_conv(np.ascontiguousarray(xh[:, :, sl]), inp["w"], bias=inp["bias"],
                                       cache_in=np.ascontiguousarray(ci_h[:, sl]))
        check_y(yh[:, :, sl], ref, abs_scale(xh[:, :, sl], inp["w"], inp["bias"], ci_h[:, sl]), cw.dtype)
        np.testing.assert_array_equal(co[:, sl].float().cpu().numpy(), rc)


def test_refusals(lib, dev):
    x = torch.zeros((1, 4, 8, 16), dtype=torch.bfloat16, device=dev)
    w = torch.zeros((16, 3), dtype=torch.float32, device=dev)
    with pytest.raises(lib.GdnError) as e:           # y overlaps x
        lib.temporal_conv_fwd(x, w, y=x)
    assert e.value.code == lib.ERR_INVALID_ARG
    c = torch.zeros((1, 8, 16), dtype=torch.bfloat16, device=dev)
    with pytest.raises(lib.GdnError) as e:           # cache_out inside x
        lib.temporal_conv_fwd(x, w, cache_out=x[:, 0])
    assert e.value.code == lib.ERR_INVALID_ARG
    lib.temporal_conv_fwd(x, w, cache_in=c, cache_out=c)  # in place is allowed
    big = torch.zeros(1 + 16 * 3, dtype=torch.float32, device=dev)
    with pytest.raises(lib.GdnError) as e:           # misaligned weights
        lib.temporal_conv_fwd(x, big[1:].view(16, 3))
    assert e.value.code == lib.ERR_INVALID_ARG
    torch.cuda.synchronize()
