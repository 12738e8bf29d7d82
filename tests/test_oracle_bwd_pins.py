"""Pins of the backward oracle (``oracle.gdn_bwd``) to things other than itself.

The backward is reverse-mode differentiation of the Gated DeltaNet frame
recurrence.  Each gradient is checked against
  * central finite differences of the FORWARD oracle (Richardson-extrapolated;
    inputs and steps are dyadic so that x +- h is exact in float32 and the
    forward runs in fp64 on exactly the perturbed values),
  * torch autograd through an independent fp64 per-token loop of the forward,
  * closed forms (no writes, alpha = 1), linearity in (do, dstate_out),
    additivity over groups of d_v columns, and the key-norm clamp,
and a Python copy of the algorithm with plausible mistakes planted in it shows
that the finite-difference pin fails each of them.
"""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")


def _dyadic(rng, shape, scale=1.0, bits=6):
    """Normal values rounded to multiples of 2^-bits (exact in float32)."""
    x = rng.standard_normal(shape) * scale
    return (np.round(x * 2 ** bits) / 2 ** bits).astype(np.float32)


def _case(rng, nh, F, L, dk, dv, logits=True):
    q = _dyadic(rng, (nh, F * L, dk))
    k = _dyadic(rng, (nh, F * L, dk))
    v = _dyadic(rng, (nh, F * L, dv))
    if logits:
        a = _dyadic(rng, (nh, F))
        b = _dyadic(rng, (nh, F * L))
    else:  # gate values in (0, 1), multiples of 2^-8
        a = (rng.integers(32, 250, (nh, F)) / 256.0).astype(np.float32)
        b = (rng.integers(8, 250, (nh, F * L)) / 256.0).astype(np.float32)
    s_in = rng.standard_normal((nh, dk, dv))
    d_o = _dyadic(rng, (nh, F * L, dv))
    ds_out = rng.standard_normal((nh, dk, dv))
    return dict(q=q, k=k, v=v, a=a, b=b, s_in=s_in, d_o=d_o, ds_out=ds_out)


def _loss(c, F, L, logits, **over):
    x = dict(c, **over)
    o, s = oracle.gdn(x["q"], x["k"], x["v"], x["a"], x["b"], F=F, L=L, gates_are_logits=logits,
                      state_in=x["s_in"], nthreads=1, rope=x.get("rope"))
    return float(np.sum(o * x["d_o"].astype(np.float64)) + np.sum(s * x["ds_out"]))


def _fd(c, name, F, L, logits, h, idx):
    """Richardson-extrapolated central difference of the loss in one element."""
    def d(step):
        xp = c[name].copy()
        xm = c[name].copy()
        xp[idx] += step
        xm[idx] -= step
        assert name == "s_in" or (float(xp[idx]) - float(c[name][idx]) == step)  # exact in float32
        return (_loss(c, F, L, logits, **{name: xp}) - _loss(c, F, L, logits, **{name: xm})) / (2 * step)
    return (4 * d(h / 2) - d(h)) / 3


GRAD = dict(q="dq", k="dk", v="dv", a="dalpha", b="dbeta", s_in="dstate_in")


def _check_fd(c, g, F, L, logits, names=GRAD, h=2.0 ** -10, rtol=1e-7):
    for name in names:
        ref = g[GRAD[name]]
        scale = max(np.abs(ref).max(), 1e-3)
        for idx in np.ndindex(c[name].shape):
            fd = _fd(c, name, F, L, logits, h, idx)
            assert abs(fd - ref[idx]) <= rtol * scale + 1e-9, (name, idx, fd, ref[idx])


def _bwd(c, F, L, logits, **kw):
    return oracle.gdn_bwd(c["q"], c["k"], c["v"], c["a"], c["b"], c["d_o"], F=F, L=L, gates_are_logits=logits,
                          state_in=c["s_in"], dstate_out=c["ds_out"], nthreads=1, rope=c.get("rope"), **kw)


@pytest.mark.parametrize("F,L,dk,dv,logits", [(3, 4, 4, 3, True), (2, 3, 3, 5, False), (1, 1, 2, 2, True),
                                               (4, 2, 3, 3, True)])
def test_bwd_matches_finite_differences(F, L, dk, dv, logits):
    rng = np.random.default_rng(100 + F * 10 + L)
    c = _case(rng, 1, F, L, dk, dv, logits)
    _check_fd(c, _bwd(c, F, L, logits), F, L, logits)


@pytest.mark.parametrize("F,L,d,gw,off", [(3, 4, 8, 2, 0), (2, 6, 12, 3, 5)])
def test_bwd_with_rope_matches_finite_differences(F, L, d, gw, off):
    """With the 3D RoPE on q and k: the gradients with respect to the unrotated
    q and k (and every other input) against central differences of the forward
    oracle with the same embedding."""
    rng = np.random.default_rng(200 + d)
    c = _case(rng, 1, F, L, d, 3)
    c["rope"] = dict(grid_w=gw, frame_offset=off, base=100.0)
    g = _bwd(c, F, L, True)
    _check_fd(c, g, F, L, True)
    c0 = dict(c)
    c0.pop("rope")
    g0 = _bwd(c0, F, L, True)
    assert np.abs(g["dk"] - g0["dk"]).max() > 1e-3  # the embedding changes the key gradients


def _torch_forward(c, F, L, logits, leaves):
    """Independent fp64 forward: the per-token loop written directly in torch."""
    q, k, v, a, b, S = (leaves[n] for n in ("q", "k", "v", "a", "b", "s_in"))
    d_o = torch.from_numpy(c["d_o"].astype(np.float64))
    ds = torch.from_numpy(c["ds_out"])
    loss = torch.zeros((), dtype=torch.float64)
    for h in range(q.shape[0]):
        St = S[h]
        for f in range(F):
            al = 1.0 / (1.0 + torch.exp(a[h, f])) if logits else a[h, f]
            St = al * St
            for t in range(f * L, (f + 1) * L):
                kh = k[h, t] / torch.clamp(torch.linalg.norm(k[h, t]), min=1e-6)
                be = torch.sigmoid(b[h, t]) if logits else b[h, t]
                St = St + be * torch.outer(kh, v[h, t] - St.T @ kh)
            for t in range(f * L, (f + 1) * L):
                loss = loss + torch.dot(St.T @ q[h, t], d_o[h, t])
        loss = loss + torch.sum(St * ds[h])
    return loss


@pytest.mark.parametrize("logits", [True, False])
def test_bwd_matches_torch_autograd(logits):
    rng = np.random.default_rng(7 + logits)
    F, L, dk, dv = 3, 5, 4, 3
    c = _case(rng, 2, F, L, dk, dv, logits)
    leaves = {n: torch.tensor(np.asarray(c[n], np.float64), requires_grad=True)
              for n in ("q", "k", "v", "a", "b", "s_in")}
    _torch_forward(c, F, L, logits, leaves).backward()
    g = _bwd(c, F, L, logits)
    for n, gn in GRAD.items():
        np.testing.assert_allclose(g[gn], leaves[n].grad.numpy(), rtol=1e-10, atol=1e-11, err_msg=n)


def test_bwd_key_norm_clamp_and_zero_gates():
    """A key with ||k|| < eps (khat = k / eps), a frame with alpha = 0 (the
    state is reset: nothing flows to the frames before it) and write strengths
    beta = 0, all with gate values."""
    rng = np.random.default_rng(21)
    F, L, dk, dv = 3, 3, 4, 3
    c = _case(rng, 1, F, L, dk, dv, logits=False)
    c["k"][0, 4] = np.array([1, 2, -1, 3], np.float32) * 2.0 ** -24  # norm 2.3e-7 < 1e-6
    c["a"][0, 1] = 0.0
    c["b"][0, 2] = 0.0
    c["b"][0, 7] = 0.0
    g = _bwd(c, F, L, False)
    # the clamp branch, by finite differences in the small key (steps of 2^-30)
    for i in range(dk):
        fd = _fd(c, "k", F, L, False, 2.0 ** -30, (0, 4, i))
        assert abs(fd - g["dk"][0, 4, i]) <= 1e-6 * max(abs(fd), 1.0), (i, fd, g["dk"][0, 4, i])
    # alpha_1 = 0: frame 0 and the start state receive nothing from frames 1, 2
    c2 = dict(c, d_o=c["d_o"].copy())
    c2["d_o"][0, :L] = 0.0
    g2 = _bwd(c2, F, L, False)
    assert np.all(g2["dstate_in"] == 0.0) and np.all(g2["dq"][0, :L] == 0.0)
    assert np.all(g2["dk"][0, :L] == 0.0) and np.all(g2["dv"][0, :L] == 0.0)
    # beta_t = 0: token t writes nothing, so dv_t = 0, but dbeta_t is defined
    assert np.all(g["dv"][0, 2] == 0.0) and np.all(g["dv"][0, 7] == 0.0)
    _check_fd(c, g, F, L, False, names=("q", "v", "a", "b", "s_in"), h=2.0 ** -12)


def test_bwd_closed_form_without_writes():
    """beta = 0, alpha = 1 (gate values): S = S_in throughout, so o_t = S_in^T q_t,
    and with H_f = dS_out + sum_{t in frames >= f} q_t do_t^T:
    dq_t = S_in do_t, dv = 0, dk = 0 (beta multiplies every key term),
    dbeta_t = -khat_t^T H_f (S_in^T khat_t - v_t), dalpha_f = <H_f, S_in>,
    dstate_in = H_0."""
    rng = np.random.default_rng(22)
    F, L, dk, dv = 3, 4, 3, 2
    c = _case(rng, 1, F, L, dk, dv, logits=False)
    c["a"][:] = 1.0
    c["b"][:] = 0.0
    g = _bwd(c, F, L, False)
    S = c["s_in"][0]
    q, k, v, d_o = (c[n][0].astype(np.float64) for n in ("q", "k", "v", "d_o"))
    np.testing.assert_allclose(g["dq"][0], d_o @ S.T, rtol=1e-12, atol=1e-12)
    assert np.all(g["dv"] == 0) and np.all(g["dk"] == 0)
    Hs = []
    for f in range(F):
        H = c["ds_out"][0].copy()
        for t in range(f * L, F * L):
            H += np.outer(q[t], d_o[t])
        Hs.append(H)
        np.testing.assert_allclose(g["dalpha"][0, f], np.sum(H * S), rtol=1e-12)
        for t in range(f * L, (f + 1) * L):
            kh = k[t] / np.linalg.norm(k[t])
            np.testing.assert_allclose(g["dbeta"][0, t], -kh @ H @ (S.T @ kh - v[t]), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(g["dstate_in"][0], Hs[0], rtol=1e-12)


def test_bwd_linear_in_upstream_gradients_and_head_subsets():
    rng = np.random.default_rng(23)
    F, L, dk, dv = 2, 3, 3, 3
    c = _case(rng, 3, F, L, dk, dv)
    c1 = dict(c, ds_out=np.zeros_like(c["ds_out"]))
    c2 = dict(c, d_o=np.zeros_like(c["d_o"]))
    g, g1, g2 = _bwd(c, F, L, True), _bwd(c1, F, L, True), _bwd(c2, F, L, True)
    for n in GRAD.values():
        np.testing.assert_allclose(g[n], g1[n] + g2[n], rtol=1e-11, atol=1e-12, err_msg=n)
    gs = _bwd(c, F, L, True, heads=[2, 0])
    for n in GRAD.values():
        np.testing.assert_array_equal(gs[n][[0, 2]], g[n][[0, 2]])
        assert np.isnan(gs[n][1]).all()



@pytest.mark.parametrize("rope", [None, dict(grid_w=2, frame_offset=1)])
def test_bwd_additive_over_value_columns(rope):
    """The recurrence never mixes d_v columns: column j of S evolves from column j
    of v alone, and o's column j reads only it.  So the loss splits into one
    term per column group, and the gradients of the whole problem are those of
    its column groups: dq, dk, dalpha and dbeta summed over the groups, dv and
    dstate_in put side by side."""
    rng = np.random.default_rng(31)
    F, L, dk, dv = 3, 4, 6, 5
    c = _case(rng, 2, F, L, dk, dv)
    c["rope"] = rope
    g = _bwd(c, F, L, True)
    parts = []
    for cols in (slice(0, 2), slice(2, 5)):
        ci = dict(c, v=np.ascontiguousarray(c["v"][..., cols]), d_o=np.ascontiguousarray(c["d_o"][..., cols]),
                  s_in=np.ascontiguousarray(c["s_in"][..., cols]), ds_out=np.ascontiguousarray(c["ds_out"][..., cols]))
        parts.append(_bwd(ci, F, L, True))
    for n in ("dq", "dk", "dalpha", "dbeta"):
        np.testing.assert_allclose(g[n], parts[0][n] + parts[1][n], rtol=1e-10, atol=1e-12, err_msg=n)
    for n in ("dv", "dstate_in"):
        np.testing.assert_allclose(g[n], np.concatenate([parts[0][n], parts[1][n]], axis=-1), rtol=1e-10,
                                   atol=1e-12, err_msg=n)


# ---------------------------------------------------------------- planted mistakes

def _py_bwd(c, F, L, mistake=None):
    """The oracle's algorithm in numpy (logit gates, one head), with a switch
    for one planted mistake."""
    q, k, v, d_o = (c[n][0].astype(np.float64) for n in ("q", "k", "v", "d_o"))
    a, b = c["a"][0].astype(np.float64), c["b"][0].astype(np.float64)
    al = 1 / (1 + np.exp(a))
    be = 1 / (1 + np.exp(-b))
    dk_, dv_ = q.shape[1], v.shape[1]
    S = c["s_in"][0].copy()
    Sprev = []
    for f in range(F):
        Sprev.append(S.copy())
        S = al[f] * S
        for t in range(f * L, (f + 1) * L):
            kh = k[t] / np.linalg.norm(k[t])
            S = S - be[t] * np.outer(kh, S.T @ kh - v[t])
    out = dict(dq=np.zeros((F * L, dk_)), dk=np.zeros((F * L, dk_)), dv=np.zeros((F * L, dv_)),
               dalpha=np.zeros(F), dbeta=np.zeros(F * L))
    H = c["ds_out"][0].copy()
    for f in reversed(range(F)):
        S = al[f] * Sprev[f]
        rs = {}
        for t in range(f * L, (f + 1) * L):
            kh = k[t] / np.linalg.norm(k[t])
            rs[t] = S.T @ kh - v[t]
            S = S - be[t] * np.outer(kh, rs[t])
        for t in range(f * L, (f + 1) * L):
            out["dq"][t] = (S.T if mistake == "dq_transposed" else S) @ d_o[t]
            H = H + np.outer(q[t], d_o[t])
        for t in reversed(range(f * L, (f + 1) * L)):
            nk = np.linalg.norm(k[t])
            kh = k[t] / nk
            r = rs[t]
            if mistake != "state_not_undone":
                S = S + be[t] * np.outer(kh, r)
            g = H.T @ kh
            out["dv"][t] = g if mistake == "dv_without_beta" else be[t] * g
            db = -(g @ r) if mistake != "dbeta_sign" else g @ r
            dkh = -be[t] * (H @ r + (0 if mistake == "dk_drop_state_term" else S @ g))
            H = H - be[t] * np.outer(kh, g)
            out["dk"][t] = dkh / nk if mistake == "dk_no_projection" else (dkh - kh * (kh @ dkh)) / nk
            out["dbeta"][t] = db * be[t] * (1 - be[t])
        Sd = al[f] * Sprev[f] if mistake == "dalpha_decayed_state" else Sprev[f]
        out["dalpha"][f] = np.sum(H * Sd) * (-al[f] * (1 - al[f]))
        H = (1.0 if mistake == "no_decay_in_carry" else al[f]) * H
    out["dstate_in"] = H
    return out


def test_fd_pin_catches_planted_mistakes():
    rng = np.random.default_rng(31)
    F, L, dk, dv = 2, 3, 3, 3
    c = _case(rng, 1, F, L, dk, dv)
    g = _bwd(c, F, L, True)
    ok = _py_bwd(c, F, L)
    for n in GRAD.values():
        np.testing.assert_allclose(ok[n], g[n][0], rtol=1e-10, atol=1e-12, err_msg=n)
    for m in ["dq_transposed", "dbeta_sign", "dk_drop_state_term", "dk_no_projection", "no_decay_in_carry",
              "state_not_undone", "dv_without_beta", "dalpha_decayed_state"]:
        bad = _py_bwd(c, F, L, m)
        wrong = {gn: bad[gn] for gn in GRAD.values()}
        with pytest.raises(AssertionError):
            _check_fd(c, {gn: wrong[gn][None] for gn in GRAD.values()}, F, L, True)
