"""The C-ABI library: loads, exports every declared symbol, validates arguments on the host.

No compute call runs here (this file needs no GPU): calls that pass host
validation stop at the device query, which reports GDN_ERR_NO_DEVICE on a
machine without an sm_100 GPU.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn_b200.h")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    import linear_attention_video_gdn_b200 as lib
    return lib


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert "gdn_frame_fwd" in names and "relu_la_block_fwd" in names
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert set(names) == set(lib.EXPORTED)


def test_boundary_names(lib):
    """The boundary's calls: the two recurrences, the workspace query and the
    status description (under both of its names)."""
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in ("gdn_frame_fwd", "relu_la_block_fwd", "gdn_workspace_bytes", "gdn_status_str", "gdn_status_string"):
        assert hasattr(raw, n), n
    raw.gdn_status_str.restype = ctypes.c_char_p
    raw.gdn_status_string.restype = ctypes.c_char_p
    for code in range(7):
        assert raw.gdn_status_str(code) == raw.gdn_status_string(code)


def test_header_constants_match_binding(lib):
    text = open(HEADER).read()
    consts = dict((k, int(v)) for k, v in re.findall(r"#define (GDN_\w+) (\d+)", text))
    assert consts["GDN_ABI_VERSION"] == lib.abi_version()
    assert consts["GDN_ERR_TIMEOUT"] == lib.ERR_TIMEOUT and consts["GDN_IMPL_TC"] == lib.IMPL_TC
    assert consts["GDN_DTYPE_BF16"] == lib.DTYPE_BF16 and consts["GDN_OP_RELU_LA"] == lib.OP_RELU_LA
    # the ctypes mirror of gdn_opts_t has the C layout (ints, pointers, size_t in declaration order)
    fields = re.search(r"typedef struct gdn_opts \{(.*?)\} gdn_opts_t;", text, re.S).group(1)
    names = re.findall(r"^\s*(?:int|void|size_t|float)\s*\*?\s*(\w+);", fields, re.M)
    assert names == [f[0] for f in lib.GdnOpts._fields_]


def test_status_strings(lib):
    for code in range(7):
        assert isinstance(lib.status_string(code), str) and lib.status_string(code) != "unknown status"
    assert lib.status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    o = lib.make_opts(lib.DTYPE_BF16, impl="frame_simt", stream=0)
    B, H, F, L, d = 1, 20, 240, 920, 112
    n = lib.workspace_bytes(lib.OP_GDN, B, H, F, L, d, d, o)
    units = B * H * F
    assert n >= units * d * d * 4 + units * 4
    assert n % 256 == 0
    assert lib.workspace_bytes(lib.OP_GDN, 0, H, F, L, d, d, o) == 0  # invalid sizes
    assert lib.workspace_bytes(lib.OP_GDN, B, H, F, L, 129, d, o) == 0
    r = lib.workspace_bytes(lib.OP_RELU_LA, 2, 20, 81, 920, d, d, o)
    assert r >= 2 * 20 * 81 * (d + 1) * d * 4
    seq = lib.make_opts(lib.DTYPE_F32, impl="seq", stream=0)
    assert lib.workspace_bytes(lib.OP_GDN, B, H, F, L, d, d, seq) == 0


def test_workspace_sizes_with_segments(lib):
    """The tcgen05 path sizes its scratch for any launch the sizes may lead to:
    with P chunk segments (residual-form kernel, the default) fp16 states and
    flags per segment unit plus one bf16 high/low end state per frame; the
    product-form kernel (one segment per frame) fp16 high and low state images
    per frame."""
    d = 112

    def need(B, H, F, L, impl="tc", **kw):
        return lib.workspace_bytes(lib.OP_GDN, B, H, F, L, d, d, lib.make_opts(lib.DTYPE_BF16, impl=impl, stream=0,
                                                                               **kw))

    up = lambda x: (x + 255) // 256 * 256

    def residual(units, P):  # counter block, flags, fp16 states, then the end states (P > 1)
        return 256 + up(4 * units * P) + up(units * P * d * d * 2) + (up(units * d * d * 4) if P > 1 else 0)

    def pform(units):  # counter block, flags, high + low images: 2 blocks of 64 columns x d rows x 2 bytes each
        return 256 + up(4 * units) + up(units * 2 * (2 * d * 128))

    nch = (920 + 63) // 64
    assert need(1, 20, 1, 920) == residual(20, min(nch, 8))                   # a streaming call: auto bound
    assert need(1, 20, 1, 920, segments=1) == residual(20, 1)
    assert need(1, 20, 1, 920, segments=3) == residual(20, 3)
    assert need(1, 20, 1, 920, segments=99) == residual(20, nch)              # at most one chunk each
    assert need(1, 20, 240, 920) == residual(4800, 1)                         # many frames: one segment
    assert need(1, 20, 1, 64) == residual(20, 1)                              # one chunk per frame
    assert need(1, 20, 240, 920, impl="tc_pform") == pform(4800)              # product form: one segment
    assert need(1, 20, 1, 920, impl="tc_pform") == pform(20)
    simt = lib.make_opts(lib.DTYPE_BF16, impl="frame_simt", stream=0, segments=4)
    assert lib.workspace_bytes(lib.OP_GDN, 1, 20, 1, 920, d, d, simt) == 256 + 256 + 20 * d * d * 4


def test_host_argument_validation(lib):
    raw = lib._lib
    o = lib.make_opts(lib.DTYPE_BF16, stream=0)
    P = ctypes.c_void_p
    p16 = P(0x10000)  # aligned, never dereferenced: validation fails first
    p_odd = P(0x10001)
    call = lambda *a: raw.gdn_frame_fwd(*a, ctypes.byref(o))
    # null required pointer
    assert call(None, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 16, 16) == lib.ERR_INVALID_ARG
    # misaligned pointer
    assert call(p_odd, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 16, 16) == lib.ERR_INVALID_ARG
    # bad sizes
    assert call(p16, p16, p16, p16, p16, None, None, p16, 1, 1, 0, 1, 16, 16) == lib.ERR_INVALID_ARG
    assert call(p16, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 256, 16) == lib.ERR_UNSUPPORTED
    # bad dtype / impl
    o.in_dtype = 7
    assert call(p16, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 16, 16) == lib.ERR_INVALID_ARG
    o.in_dtype = lib.DTYPE_BF16
    o.impl = 9
    assert call(p16, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 16, 16) == lib.ERR_INVALID_ARG
    # null opts
    assert raw.gdn_frame_fwd(p16, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 16, 16, None) == \
        lib.ERR_INVALID_ARG
    # negative eps for the ReLU mode
    o.impl = 0
    assert raw.relu_la_block_fwd(p16, p16, p16, None, None, None, None, p16, 1, 1, 1, 1, 16, 16,
                                 ctypes.c_float(-1.0), ctypes.byref(o)) == lib.ERR_INVALID_ARG


def test_temporal_conv_argument_validation(lib):
    raw = lib._lib
    o = lib.make_opts(lib.DTYPE_BF16, stream=0)
    P = ctypes.c_void_p
    x, w, y, c = P(0x100000), P(0x200000), P(0x300000), P(0x400000)  # never dereferenced
    call = lambda *a: raw.temporal_conv_fwd(*a, ctypes.byref(o))
    assert call(None, w, None, None, None, y, 1, 4, 8, 16) == lib.ERR_INVALID_ARG       # null x
    assert call(x, w, None, None, None, None, 1, 4, 8, 16) == lib.ERR_INVALID_ARG       # null y
    assert call(x, P(0x200004), None, None, None, y, 1, 4, 8, 16) == lib.ERR_INVALID_ARG  # misaligned w
    assert call(x, w, None, None, None, y, 1, 0, 8, 16) == lib.ERR_INVALID_ARG          # F = 0
    assert call(x, w, None, None, None, P(0x100010), 1, 4, 8, 16) == lib.ERR_INVALID_ARG  # y overlaps x
    assert call(x, w, None, None, P(0x100000 + 512), y, 1, 4, 8, 16) == lib.ERR_INVALID_ARG   # cache in x
    assert call(x, w, None, c, P(0x400010), y, 1, 4, 8, 16) == lib.ERR_INVALID_ARG      # caches overlap
    o.in_dtype = 5
    assert call(x, w, None, None, None, y, 1, 4, 8, 16) == lib.ERR_INVALID_ARG          # bad dtype
    o.in_dtype = lib.DTYPE_BF16
    assert raw.temporal_conv_fwd(x, w, None, None, None, y, 1, 4, 8, 16, None) == lib.ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():  # valid arguments, in-place cache: the device check comes last
        assert call(x, w, None, c, c, y, 1, 4, 8, 16) == lib.ERR_NO_DEVICE


def test_softmax_window_argument_validation(lib):
    raw = lib._lib
    o = lib.make_opts(lib.DTYPE_BF16, stream=0)
    P = ctypes.c_void_p
    q, k, v, out = P(0x100000), P(0x200000), P(0x300000), P(0x400000)  # never dereferenced
    f32 = ctypes.c_float
    call = lambda *a: raw.softmax_window_fwd(*a, ctypes.byref(o))
    assert call(None, k, v, out, 1, 2, 3, 16, 32, 32, 2, f32(0)) == lib.ERR_INVALID_ARG     # null q
    assert call(q, k, v, None, 1, 2, 3, 16, 32, 32, 2, f32(0)) == lib.ERR_INVALID_ARG       # null o
    assert call(q, k, v, out, 1, 2, 3, 16, 32, 32, 0, f32(0)) == lib.ERR_INVALID_ARG        # W = 0
    assert call(q, k, v, out, 1, 2, 3, 16, 32, 32, 2, f32(-1)) == lib.ERR_INVALID_ARG       # negative scale
    assert call(q, k, v, out, 1, 2, 3, 16, 256, 32, 2, f32(0)) == lib.ERR_UNSUPPORTED       # dk > 128
    assert call(P(0x100004), k, v, out, 1, 2, 3, 16, 32, 32, 2, f32(0)) == lib.ERR_INVALID_ARG  # misaligned
    assert call(q, k, v, P(0x100000 + 512), 1, 2, 3, 16, 32, 32, 2, f32(0)) == lib.ERR_INVALID_ARG  # o inside q
    o.impl = lib.IMPL_TC
    assert call(q, k, v, out, 1, 2, 3, 16, 24, 32, 2, f32(0)) == lib.ERR_UNSUPPORTED        # tc: d % 16
    o.in_dtype = lib.DTYPE_F32
    assert call(q, k, v, out, 1, 2, 3, 16, 32, 32, 2, f32(0)) == lib.ERR_UNSUPPORTED        # tc: bf16 only
    o.impl = 9
    assert call(q, k, v, out, 1, 2, 3, 16, 32, 32, 2, f32(0)) == lib.ERR_INVALID_ARG        # unknown kernel
    o.impl = 0
    import torch
    if not torch.cuda.is_available():  # valid arguments: the device check comes last
        assert call(q, k, v, out, 1, 2, 3, 16, 24, 40, 2, f32(0)) == lib.ERR_NO_DEVICE


def test_no_device_is_reported_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    o = lib.make_opts(lib.DTYPE_BF16, stream=0)
    p16 = ctypes.c_void_p(0x10000)
    rc = lib._lib.gdn_frame_fwd(p16, p16, p16, p16, p16, None, None, p16, 1, 1, 1, 1, 16, 16, ctypes.byref(o))
    assert rc == lib.ERR_NO_DEVICE


def test_backward_workspace_and_argument_validation(lib):
    """gdn_frame_bwd: the workspace holds the recompute's chain scratch, then
    A_f^T, S_f and G_f of every frame, the dalpha partial sums and (with the 3D
    RoPE) its table; host checks come before any device work."""
    up = lambda x: (x + 255) // 256 * 256
    B, H, F, L, d = 1, 20, 240, 920, 112
    fr = B * H * F
    tc = lib.make_opts(lib.DTYPE_BF16, stream=0)
    chain = lib.workspace_bytes(lib.OP_GDN, B, H, F, L, d, d, lib.make_opts(lib.DTYPE_BF16, stream=0, segments=1))
    nch = (L + 47) // 48  # the tensor-core frame kernel keeps each 48-token chunk's Linv
    want = up(chain) + 3 * up(fr * d * d * 4) + up(fr * 7 * 4) + up(fr * nch * 48 * 48 * 4)
    assert lib.workspace_bytes(lib.OP_GDN_BWD, B, H, F, L, d, d, tc) == want
    # d_v > d_k: the residuals need their own rows (d_k's rows hold them otherwise)
    assert lib.workspace_bytes(lib.OP_GDN_BWD, B, H, F, L, 48, 112, tc) == \
        up(lib.workspace_bytes(lib.OP_GDN, B, H, F, L, 48, 112, lib.make_opts(lib.DTYPE_BF16, stream=0, segments=1))) + \
        up(fr * 48 * 48 * 4) + 2 * up(fr * 48 * 112 * 4) + up(fr * 7 * 4) + up(fr * nch * 48 * 48 * 4) + \
        up(fr * L * 112 * 4)
    f32 = lib.make_opts(lib.DTYPE_F32, stream=0)  # the fp32 recompute publishes fp32 states
    chain32 = 256 + up(fr * 4) + up(fr * d * d * 4)
    assert lib.workspace_bytes(lib.OP_GDN_BWD, B, H, F, L, d, d, f32) == up(chain32) + 3 * up(fr * d * d * 4) + \
        up(fr * 7 * 4)
    # the 3D RoPE: the same layout, then the table (time [F][dt/2], height [L/gw][dh/2],
    # width [gw][dh/2] cos/sin pairs)
    rope = dict(grid_w=40)
    dh = 2 * (d // 6)
    dt = d - 2 * dh
    table = up(8 * (F * (dt // 2) + (L // 40) * (dh // 2) + 40 * (dh // 2)))
    assert lib.workspace_bytes(lib.OP_GDN_BWD, B, H, F, L, d, d, lib.make_opts(lib.DTYPE_BF16, stream=0, rope=rope)) \
        == want + table
    assert lib.workspace_bytes(lib.OP_GDN_BWD, B, H, F, L, d, d, lib.make_opts(lib.DTYPE_F32, stream=0, rope=rope)) \
        == lib.workspace_bytes(lib.OP_GDN_BWD, B, H, F, L, d, d, f32) + table
    raw = lib._lib
    P = ctypes.c_void_p
    q, k, v, a, b, do = (P(0x1000000 * (i + 1)) for i in range(6))
    outs = [P(0x10000000 * (i + 1)) for i in range(6)]
    ws = P(0x70000000)
    o = lib.make_opts(lib.DTYPE_BF16, stream=0)
    o.workspace = 0x70000000
    o.workspace_bytes = 1 << 40
    call = lambda *args, sizes=(1, 2, 3, 16, 32, 32): raw.gdn_frame_bwd(*args, *sizes, ctypes.byref(o))
    assert call(q, k, v, a, b, None, None, None, *outs) == lib.ERR_INVALID_ARG            # null d_o
    assert call(q, k, v, a, b, None, do, None, None, *outs[1:]) == lib.ERR_INVALID_ARG    # null dq
    assert call(q, k, v, a, b, None, do, None, *outs, sizes=(1, 2, 3, 16, 128, 32)) == lib.ERR_UNSUPPORTED
    assert call(q, k, v, a, b, None, do, None, P(0x1000000 + 64), *outs[1:]) == lib.ERR_INVALID_ARG  # dq in q
    assert call(q, k, v, a, b, None, do, None, outs[0], outs[0], *outs[2:]) == lib.ERR_INVALID_ARG  # dq = dk
    assert call(P(0x1000004), k, v, a, b, None, do, None, *outs) == lib.ERR_INVALID_ARG  # misaligned
    o.rope_grid_w = 5
    assert call(q, k, v, a, b, None, do, None, *outs) == lib.ERR_INVALID_ARG              # L % grid_w != 0
    o.rope_grid_w, o.rope_frame_offset = 4, -1
    assert call(q, k, v, a, b, None, do, None, *outs) == lib.ERR_INVALID_ARG              # negative offset
    o.rope_grid_w, o.rope_frame_offset = 0, 0
    o.impl = lib.IMPL_SEQ
    assert call(q, k, v, a, b, None, do, None, *outs) == lib.ERR_INVALID_ARG              # no such recompute
    o.impl = lib.IMPL_AUTO
    assert raw.gdn_frame_bwd(q, k, v, a, b, None, do, None, *outs, 1, 2, 3, 16, 32, 32, None) == lib.ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():  # valid arguments: the device check comes last
        assert call(q, k, v, a, b, None, do, None, *outs) == lib.ERR_NO_DEVICE
        o.rope_grid_w = 4
        assert call(q, k, v, a, b, None, do, None, *outs) == lib.ERR_NO_DEVICE
        o.rope_grid_w = 0
    del ws
