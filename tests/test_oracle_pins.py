"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against a closed form, a hand-derived worked case,
an invariant of the recurrence, or an independent brute-force construction
(explicit dense matrix products, O(N^2) masked attention), chosen so that a
dropped term, a wrong sign or index, or a transposed operand in the oracle
fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def _rand_case(nh, F, L, dk, dv, rng, unit=True):
    q = rng.standard_normal((nh, F * L, dk)).astype(np.float32)
    k = rng.standard_normal((nh, F * L, dk)).astype(np.float32)
    if unit:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((nh, F * L, dv)).astype(np.float32)
    a = rng.standard_normal((nh, F)).astype(np.float32)
    b = rng.standard_normal((nh, F * L)).astype(np.float32)
    return q, k, v, a, b


# ---------------------------------------------------------------- gates

def test_gate_closed_forms():
    # exp(-softplus(a)) == 1/(1+e^a) == sigmoid(-a); sigmoid(b) == 1/(1+e^-b)
    for a in [-30.0, -5.0, -2.0, -0.5, 0.0, 0.3, 1.0, 4.0, 20.0]:
        assert oracle.gate_alpha(a) == pytest.approx(1.0 / (1.0 + np.exp(a)), rel=1e-14, abs=1e-300)
        assert oracle.gate_beta(a) == pytest.approx(1.0 / (1.0 + np.exp(-a)), rel=1e-14)
    assert oracle.gate_alpha(0.0) == 0.5 and oracle.gate_beta(0.0) == 0.5
    # alpha in (0,1], beta in (0,1): limits
    assert oracle.gate_alpha(-800.0) == 1.0
    assert oracle.gate_alpha(800.0) == 0.0


# ---------------------------------------------------------------- worked cases

def test_gdn_worked_2d_golden():
    g = json.load(open(os.path.join(GOLDEN, "gdn_worked_2d.json")))
    q, k, v = (np.array(g[x], np.float32)[None] for x in ("q", "k", "v"))
    al = np.array(g["alpha"], np.float32)[None]
    be = np.array(g["beta"], np.float32)[None]
    o, s = oracle.gdn(q, k, v, al, be, F=g["F"], L=g["L"], gates_are_logits=False)
    np.testing.assert_allclose(o[0], np.array(g["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(s[0], np.array(g["state_out"]), rtol=0, atol=1e-12)


def test_relu_la_worked_2d_golden():
    g = json.load(open(os.path.join(GOLDEN, "relu_la_worked_2d.json")))
    q, k, v = (np.array(g[x], np.float32)[None] for x in ("q", "k", "v"))
    o, kv, z = oracle.relu_la(q, k, v, F=g["F"], L=g["L"], eps=g["eps"])
    np.testing.assert_allclose(o[0], np.array(g["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(kv[0], np.array(g["kv_out"]), rtol=0, atol=0)
    np.testing.assert_allclose(z[0], np.array(g["z_out"]), rtol=0, atol=0)


# ---------------------------------------------------------------- brute force

def _bruteforce_gdn(q, k, v, alpha, beta, F, L, S0):
    """Independent construction: S_F as explicit products of dense factors.

    With M_t = I - beta_t khat_t khat_t^T and scalar decays alpha_f at frame
    starts, S after step n is  P(0..n) S0 + sum_t P(t+1..n) beta_t khat_t v_t^T,
    where P(i..n) is the ordered product (latest factor on the left) of every
    factor after position i.  Each frame's outputs use the state at its end.
    """
    dk, dv = k.shape[-1], v.shape[-1]
    ops = []  # sequence of ("decay", alpha) / ("tok", t)
    for f in range(F):
        ops.append(("decay", float(alpha[f])))
        for t in range(f * L, (f + 1) * L):
            ops.append(("tok", t))

    def factor(op):
        kind, x = op
        if kind == "decay":
            return x * np.eye(dk)
        kk = k[x].astype(np.float64)
        nrm = max(np.sqrt(kk @ kk), 1e-6)
        kh = kk / nrm
        return np.eye(dk) - float(beta[x]) * np.outer(kh, kh)

    def state_after(n):  # state after ops[0..n] inclusive
        P = np.eye(dk)
        for op in ops[: n + 1]:
            P = factor(op) @ P
        S = P @ S0
        for i in range(n + 1):
            kind, t = ops[i]
            if kind != "tok":
                continue
            Q = np.eye(dk)
            for op in ops[i + 1: n + 1]:
                Q = factor(op) @ Q
            kk = k[t].astype(np.float64)
            kh = kk / max(np.sqrt(kk @ kk), 1e-6)
            S = S + Q @ (float(beta[t]) * np.outer(kh, v[t].astype(np.float64)))
        return S

    o = np.zeros((F * L, dv))
    idx = -1
    for f in range(F):
        idx += 1 + L
        Sf = state_after(idx)
        for t in range(f * L, (f + 1) * L):
            o[t] = Sf.T @ q[t].astype(np.float64)
    return o, state_after(len(ops) - 1)


@pytest.mark.parametrize("F,L,dk,dv,unit", [(1, 1, 3, 2, True), (2, 3, 4, 3, True), (3, 4, 4, 4, False),
                                             (3, 2, 2, 4, True)])
def test_gdn_bruteforce_products(F, L, dk, dv, unit):
    rng = np.random.default_rng(F * 100 + L * 10 + dk)
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng, unit=unit)
    S0 = rng.standard_normal((dk, dv))
    al = np.array([oracle.gate_alpha(x) for x in a[0]], np.float32)
    be = np.array([oracle.gate_beta(x) for x in b[0]], np.float32)
    o, s = oracle.gdn(q, k, v, al[None], be[None], F=F, L=L, gates_are_logits=False, state_in=S0[None])
    o_ref, s_ref = _bruteforce_gdn(q[0], k[0], v[0], al, be, F, L, S0)
    np.testing.assert_allclose(o[0], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s[0], s_ref, rtol=0, atol=1e-12)
    # the same run through the logit path must agree with the value path
    o2, s2 = oracle.gdn(q, k, v, a, b, F=F, L=L, gates_are_logits=True, state_in=S0[None])
    np.testing.assert_allclose(o2[0], o_ref, rtol=0, atol=1e-6)


# ---------------------------------------------------------------- closed forms

def test_gdn_identity_gates_leave_state():
    # alpha = 1, beta = 0: S never changes and o_t = S0^T q_t
    rng = np.random.default_rng(1)
    F, L, dk, dv = 3, 5, 6, 4
    q, k, v, _, _ = _rand_case(2, F, L, dk, dv, rng)
    S0 = rng.standard_normal((2, dk, dv))
    o, s = oracle.gdn(q, k, v, np.ones((2, F), np.float32), np.zeros((2, F * L), np.float32),
                      F=F, L=L, gates_are_logits=False, state_in=S0)
    np.testing.assert_allclose(s, S0, rtol=0, atol=0)
    np.testing.assert_allclose(o, np.einsum("hnd,hde->hne", q.astype(np.float64), S0), rtol=0, atol=1e-12)


def test_gdn_single_token_orthonormal():
    # S0 = 0, one token with unit key: S = beta khat v^T; o = S^T q
    dk, dv = 5, 3
    for i in range(dk):
        k = np.zeros((1, 1, dk), np.float32)
        k[0, 0, i] = 1.0
        v = np.array([[[1.5, -2.0, 0.25]]], np.float32)
        q = np.arange(dk, dtype=np.float32).reshape(1, 1, dk)
        beta = 0.375
        o, s = oracle.gdn(q, k, v, np.ones((1, 1), np.float32), np.full((1, 1), beta, np.float32),
                          F=1, L=1, gates_are_logits=False)
        expect = beta * np.outer(k[0, 0], v[0, 0])
        np.testing.assert_allclose(s[0], expect, rtol=0, atol=1e-15)
        np.testing.assert_allclose(o[0, 0], expect.T @ q[0, 0], rtol=0, atol=1e-15)


def test_gdn_exact_recall_orthonormal_keys():
    # beta = 1 and L <= dk orthonormal keys: S^T khat_i = v_i for every key written
    rng = np.random.default_rng(7)
    dk, dv, L = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :L].T.astype(np.float32)[None]  # rows orthonormal (up to fp32 rounding)
    v = rng.standard_normal((1, L, dv)).astype(np.float32)
    q = rng.standard_normal((1, L, dk)).astype(np.float32)
    S0 = rng.standard_normal((1, dk, dv))
    o, s = oracle.gdn(q, k, v, np.ones((1, 1), np.float32), np.ones((1, L), np.float32),
                      F=1, L=L, gates_are_logits=False, state_in=S0)
    kh = k[0].astype(np.float64)
    kh /= np.linalg.norm(kh, axis=1, keepdims=True)
    np.testing.assert_allclose(kh @ s[0], v[0], rtol=0, atol=1e-6)  # limited by fp32 orthogonality of k
    # directions orthogonal to every key keep their original read-out
    P = np.eye(dk) - kh.T @ kh
    np.testing.assert_allclose(P @ s[0], P @ S0[0], rtol=0, atol=1e-6)


def test_gdn_zero_key_is_a_no_op():
    rng = np.random.default_rng(3)
    F, L, dk, dv = 2, 4, 4, 3
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng)
    o, s = oracle.gdn(q, k, v, a, b, F=F, L=L)
    k2 = k.copy()
    k2[0, 2] = 0.0
    k2[0, 5] = 0.0
    o2, s2 = oracle.gdn(q, k2, v, a, b, F=F, L=L)
    # compare against a run with those tokens removed (beta forced to 0)
    b3 = b.copy()
    b3[0, 2] = -1e4
    b3[0, 5] = -1e4
    o3, s3 = oracle.gdn(q, k, v, a, b3, F=F, L=L)
    np.testing.assert_allclose(s2, s3, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2, o3, rtol=0, atol=1e-12)
    assert not np.allclose(s, s2)


# ---------------------------------------------------------------- invariants

def test_gdn_key_scale_invariance():
    # khat is invariant to positive rescaling of k_t
    rng = np.random.default_rng(4)
    F, L, dk, dv = 2, 3, 5, 4
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng, unit=False)
    o, s = oracle.gdn(q, k, v, a, b, F=F, L=L)
    scale = np.array([0.5, 2.0, 8.0, 0.25, 4.0, 1.0], np.float32)[None, :, None]
    o2, s2 = oracle.gdn(q, k * scale, v, a, b, F=F, L=L)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, s, rtol=0, atol=1e-12)


def test_gdn_affine_in_state_and_linear_in_values():
    rng = np.random.default_rng(5)
    F, L, dk, dv = 3, 4, 5, 4
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng)
    S1 = rng.standard_normal((1, dk, dv))
    S2 = rng.standard_normal((1, dk, dv))
    run = lambda vv, S: oracle.gdn(q, k, vv, a, b, F=F, L=L, state_in=S)
    o0, s0 = run(v, None)
    oa, sa = run(v, S1)
    ob, sb = run(v, S2)
    oab, sab = run(v, S1 + S2)
    np.testing.assert_allclose(sab - s0, (sa - s0) + (sb - s0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(oab - o0, (oa - o0) + (ob - o0), rtol=0, atol=1e-12)
    # linear in v when S0 = 0 (v values kept exactly representable in fp32)
    v1 = np.round(rng.standard_normal(v.shape) * 64).astype(np.float32) / 64
    v2 = np.round(rng.standard_normal(v.shape) * 64).astype(np.float32) / 64
    o1, t1 = run(v1, None)
    o2, t2 = run(v2, None)
    o12, t12 = run(v1 + v2, None)
    np.testing.assert_allclose(t12, t1 + t2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o12, o1 + o2, rtol=0, atol=1e-12)


def test_gdn_column_permutation_equivariance_and_column_subsets():
    rng = np.random.default_rng(6)
    F, L, dk, dv = 2, 5, 6, 7
    q, k, v, a, b = _rand_case(2, F, L, dk, dv, rng)
    S0 = rng.standard_normal((2, dk, dv))
    o, s = oracle.gdn(q, k, v, a, b, F=F, L=L, state_in=S0)
    perm = rng.permutation(dv)
    o2, s2 = oracle.gdn(q, k, v[..., perm], a, b, F=F, L=L, state_in=S0[..., perm])
    np.testing.assert_array_equal(o2, o[..., perm])
    np.testing.assert_array_equal(s2, s[..., perm])
    # computing a subset of columns gives bit-identical values for those columns
    o3, s3 = oracle.gdn(q, k, v, a, b, F=F, L=L, state_in=S0, cols=(2, 5))
    np.testing.assert_array_equal(o3[..., 2:5], o[..., 2:5])
    np.testing.assert_array_equal(s3[..., 2:5], s[..., 2:5])
    assert np.isnan(o3[..., :2]).all()


def test_gdn_contraction():
    # each factor has spectral norm <= 1 (unit keys, beta in (0,1), alpha <= 1)
    rng = np.random.default_rng(8)
    F, L, dk, dv = 3, 6, 6, 5
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng)
    for _ in range(5):
        S1 = rng.standard_normal((1, dk, dv)) * 3
        S2 = rng.standard_normal((1, dk, dv)) * 3
        _, s1 = oracle.gdn(q, k, v, a, b, F=F, L=L, state_in=S1)
        _, s2 = oracle.gdn(q, k, v, a, b, F=F, L=L, state_in=S2)
        assert np.linalg.norm(s1[0] - s2[0], 2) <= np.linalg.norm(S1[0] - S2[0], 2) * (1 + 1e-12)


def test_gdn_readout_uses_end_of_frame_state_and_split_resume():
    rng = np.random.default_rng(9)
    F, L, dk, dv = 4, 3, 5, 4
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng)
    o, s = oracle.gdn(q, k, v, a, b, F=F, L=L)
    for f in range(F):
        n = (f + 1) * L
        _, sf = oracle.gdn(q[:, :n], k[:, :n], v[:, :n], a[:, :f + 1], b[:, :n], F=f + 1, L=L)
        np.testing.assert_allclose(o[0, f * L:n], q[0, f * L:n].astype(np.float64) @ sf[0], rtol=0, atol=1e-12)
    # resume from the state after 2 frames == one run over all frames
    _, s2 = oracle.gdn(q[:, :2 * L], k[:, :2 * L], v[:, :2 * L], a[:, :2], b[:, :2 * L], F=2, L=L)
    o_r, s_r = oracle.gdn(q[:, 2 * L:], k[:, 2 * L:], v[:, 2 * L:], a[:, 2:], b[:, 2 * L:], F=2, L=L,
                          state_in=s2)
    np.testing.assert_allclose(o_r, o[:, 2 * L:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_r, s, rtol=0, atol=1e-12)


def test_gdn_frame_map_composes_from_chunk_segments():
    """A frame's update is affine in the incoming state, S_out = A S_in + B, and
    the maps of consecutive runs of tokens compose: the frame decay belongs to
    the first run only.  This is the algebra that lets a frame be built in
    pieces (one per run of chunks) and chained; here each piece's map is taken
    from a short oracle run (A from state I with zero values, B from a zero
    state), and the composition must reproduce the whole-sequence states and
    read-outs."""
    F, L, dk, dv = 2, 10, 4, 3
    rng = np.random.default_rng(77)
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng, unit=False)
    al = np.array([oracle.gate_alpha(x) for x in a[0]], np.float64)
    be = np.array([oracle.gate_beta(x) for x in b[0]], np.float32)
    S0 = rng.standard_normal((dk, dv))
    o_ref, s_ref = oracle.gdn(q, k, v, al[None].astype(np.float32), be[None], F=F, L=L, gates_are_logits=False,
                              state_in=S0[None])
    for cuts in ([0, 10], [0, 3, 10], [0, 3, 6, 10], [0, 1, 2, 9, 10]):
        S = S0.copy()
        o = np.zeros((F * L, dv))
        for f in range(F):
            for s_i, (t0, t1) in enumerate(zip(cuts[:-1], cuts[1:])):
                sl = slice(f * L + t0, f * L + t1)
                n = t1 - t0
                decay = np.array([[al[f] if s_i == 0 else 1.0]], np.float32)
                zeros_v = np.zeros((1, n, dk), np.float32)
                _, A = oracle.gdn(q[:, sl], k[:, sl], zeros_v, decay, be[None, sl], F=1, L=n,
                                  gates_are_logits=False, state_in=np.eye(dk)[None], want_o=False)
                _, B = oracle.gdn(q[:, sl], k[:, sl], v[:, sl], decay, be[None, sl], F=1, L=n,
                                  gates_are_logits=False, state_in=np.zeros((1, dk, dv)), want_o=False)
                S = A[0] @ S + B[0]
            o[f * L:(f + 1) * L] = q[0, f * L:(f + 1) * L].astype(np.float64) @ S
        np.testing.assert_allclose(S, s_ref[0], rtol=0, atol=1e-10)
        np.testing.assert_allclose(o, o_ref[0], rtol=0, atol=1e-10)


def test_gdn_frames_are_block_causal():
    # changing a later frame's inputs never changes an earlier frame's outputs
    rng = np.random.default_rng(10)
    F, L, dk, dv = 3, 4, 4, 4
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng)
    o, _ = oracle.gdn(q, k, v, a, b, F=F, L=L)
    v2 = v.copy()
    v2[0, 2 * L:] += 1.0
    o2, _ = oracle.gdn(q, k, v2, a, b, F=F, L=L)
    np.testing.assert_array_equal(o2[0, :2 * L], o[0, :2 * L])
    assert not np.allclose(o2[0, 2 * L:], o[0, 2 * L:])
    # but a change inside the frame reaches every token of that frame (bidirectional within a frame)
    v3 = v.copy()
    v3[0, 2 * L + L - 1] += 1.0
    o3, _ = oracle.gdn(q, k, v3, a, b, F=F, L=L)
    assert (np.abs(o3[0, 2 * L:] - o[0, 2 * L:]).max(axis=1) > 0).all()


# ---------------------------------------------------------------- streaming (block cache, several steps per frame)

def _stream_calls(nframes, steps, L, dk, dv, seed):
    """Fresh inputs per call (one frame each), as value gates, for streaming pins."""
    rng = np.random.default_rng(seed)
    calls = []
    for _ in range(nframes * steps):
        q, k, v, a, b = _rand_case(1, 1, L, dk, dv, rng)
        calls.append(dict(q=q, k=k, v=v, a=a, b=b))
    return calls


def _feeder(calls):
    return lambda c: calls[c] if c < len(calls) else None


def test_gdn_stream_one_step_equals_whole_sequence():
    """With one step per frame, streaming is the whole-sequence recurrence over
    the same frames: every output and the final state are bit-identical."""
    F, L, dk, dv = 4, 5, 6, 4
    calls = _stream_calls(F, 1, L, dk, dv, 31)
    S0 = np.random.default_rng(3).standard_normal((1, dk, dv))
    outs, S, committed = oracle.gdn_stream(_feeder(calls), steps=1, L=L, state_in=S0)
    cat = {n: np.concatenate([c[n] for c in calls], axis=1) for n in "qkvab"}
    o_ref, s_ref = oracle.gdn(cat["q"], cat["k"], cat["v"], cat["a"], cat["b"], F=F, L=L, state_in=S0)
    np.testing.assert_array_equal(np.concatenate(outs, axis=1), o_ref)
    np.testing.assert_array_equal(S, s_ref)
    assert len(committed) == F


def test_gdn_stream_commits_only_the_last_step():
    """Steps 1..3 of a frame leave no trace: changing their inputs changes
    neither any committed state nor any last-step output; and the committed
    state after frame f is the whole-sequence state over the last-step inputs
    of frames 0..f."""
    nf, steps, L, dk, dv = 3, 4, 6, 5, 4
    calls = _stream_calls(nf, steps, L, dk, dv, 41)
    outs, S, committed = oracle.gdn_stream(_feeder(calls), steps=steps, L=L)
    rng = np.random.default_rng(5)
    changed = [dict(c) for c in calls]
    for c in range(len(calls)):
        if c % steps != steps - 1:
            changed[c] = {n: (x + rng.standard_normal(x.shape).astype(np.float32)) for n, x in calls[c].items()}
    outs2, S2, committed2 = oracle.gdn_stream(_feeder(changed), steps=steps, L=L)
    for f in range(nf):
        np.testing.assert_array_equal(committed2[f], committed[f])
        last = f * steps + steps - 1
        np.testing.assert_array_equal(outs2[last], outs[last])
        # a non-committing step's output does depend on its own inputs
        assert not np.array_equal(outs2[f * steps], outs[f * steps])
    for f in range(nf):
        lasts = [calls[g * steps + steps - 1] for g in range(f + 1)]
        cat = {n: np.concatenate([c[n] for c in lasts], axis=1) for n in "qkvab"}
        _, s_ref = oracle.gdn(cat["q"], cat["k"], cat["v"], cat["a"], cat["b"], F=f + 1, L=L)
        np.testing.assert_array_equal(committed[f], s_ref)


def test_gdn_stream_every_step_matches_bruteforce():
    """Each step's output, and each committed state, equals the brute-force
    dense-product result started from the state committed by the previous
    frame (an independent construction, not the oracle's own loop)."""
    nf, steps, L, dk, dv = 2, 3, 3, 4, 3
    calls = _stream_calls(nf, steps, L, dk, dv, 51)
    outs, S, committed = oracle.gdn_stream(_feeder(calls), steps=steps, L=L)
    S_prev = np.zeros((dk, dv))
    for f in range(nf):
        for s_i in range(steps):
            c = calls[f * steps + s_i]
            al = np.array([oracle.gate_alpha(x) for x in c["a"][0]], np.float64)  # gates from logits, in double
            be = np.array([oracle.gate_beta(x) for x in c["b"][0]], np.float64)
            o_b, s_b = _bruteforce_gdn(c["q"][0], c["k"][0], c["v"][0], al, be, 1, L, S_prev)
            np.testing.assert_allclose(outs[f * steps + s_i][0], o_b, rtol=0, atol=1e-12)
        np.testing.assert_allclose(committed[f][0], s_b, rtol=0, atol=1e-12)
        S_prev = s_b
    np.testing.assert_array_equal(S, committed[-1])


def test_gdn_stream_refuses_a_frame_cut_short():
    calls = _stream_calls(1, 4, 3, 4, 3, 61)[:3]  # three of a frame's four steps
    with pytest.raises(ValueError, match="inside a frame"):
        oracle.gdn_stream(_feeder(calls), steps=4, L=3)
    outs, S, committed = oracle.gdn_stream(_feeder([]), steps=4, L=3)
    assert outs == [] and S is None and committed == []


# ---------------------------------------------------------------- 3D RoPE

def _rope_complex(x, F, L, grid_w, frame_offset=0, base=1e4):
    """Independent construction: each rotated pair as a complex number times
    exp(i * angle), the parts laid out as time, height, width."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    dh = 2 * (d // 6)
    dt = d - 2 * dh
    t = np.arange(F * L)
    frame, tl = t // L + frame_offset, t % L
    out = np.empty_like(x)
    for (o, n), pos in zip([(0, dt), (dt, dh), (dt + dh, dh)], [frame, tl // grid_w, tl % grid_w]):
        z = x[..., o:o + n:2] + 1j * x[..., o + 1:o + n:2]
        z = z * np.exp(1j * np.outer(pos, base ** (-np.arange(0, n, 2) / n)))
        out[..., o:o + n:2], out[..., o + 1:o + n:2] = z.real, z.imag
    return out


@pytest.mark.parametrize("d,grid_w,off", [(12, 3, 0), (112, 40, 7), (32, 4, 100)])
def test_rope3d_matches_complex_rotation(d, grid_w, off):
    F, L = 3, 2 * grid_w
    x = np.random.default_rng(d).standard_normal((2, F * L, d)).astype(np.float32)
    got = oracle.rope3d(x, F=F, L=L, grid_w=grid_w, frame_offset=off)
    np.testing.assert_allclose(got, _rope_complex(x, F, L, grid_w, off), rtol=0, atol=1e-12)


def test_rope3d_invariants():
    """Rotations keep norms (per token and per part), position (0, 0, 0) is the
    identity, and the score of two rotated vectors depends only on their
    relative position: shifting both in time by the same amount leaves it."""
    d, grid_w, F, L = 24, 3, 4, 6
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, F * L, d)).astype(np.float32)
    k = rng.standard_normal((1, F * L, d)).astype(np.float32)
    rq = oracle.rope3d(q, F=F, L=L, grid_w=grid_w)
    np.testing.assert_allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(q.astype(np.float64), axis=-1),
                               rtol=1e-13)
    np.testing.assert_array_equal(rq[0, 0], q[0, 0].astype(np.float64))  # frame 0, row 0, column 0
    rk = oracle.rope3d(k, F=F, L=L, grid_w=grid_w)
    rq5 = oracle.rope3d(q, F=F, L=L, grid_w=grid_w, frame_offset=5)
    rk5 = oracle.rope3d(k, F=F, L=L, grid_w=grid_w, frame_offset=5)
    np.testing.assert_allclose(rq[0] @ rk[0].T, rq5[0] @ rk5[0].T, rtol=1e-10, atol=1e-10)
    # a vector that lives only in the height part ignores frame and column
    dh = 2 * (d // 6)
    dt = d - 2 * dh
    hv = np.zeros((1, F * L, d), np.float32)
    hv[..., dt:dt + dh] = 1.0
    r = oracle.rope3d(hv, F=F, L=L, grid_w=grid_w)
    rows = (np.arange(F * L) % L) // grid_w
    for i in range(F * L):
        j = np.where(rows == rows[i])[0][0]  # first token on the same row (another column or frame)
        np.testing.assert_allclose(r[0, i], r[0, j], rtol=0, atol=1e-14)


def test_gdn_with_rope_equals_gdn_on_rotated_inputs():
    """RoPE enters the recurrence only through q and k: the RoPE run equals a
    plain run fed q and k rotated by the independent complex construction."""
    F, L, d, dv, grid_w = 3, 6, 12, 5, 3
    q, k, v, a, b = _rand_case(2, F, L, d, dv, np.random.default_rng(21), unit=False)
    o_r, s_r = oracle.gdn(q, k, v, a, b, F=F, L=L, rope=dict(grid_w=grid_w, frame_offset=2))
    qr = _rope_complex(q, F, L, grid_w, 2).astype(np.float32)
    kr = _rope_complex(k, F, L, grid_w, 2).astype(np.float32)
    o_p, s_p = oracle.gdn(qr, kr, v, a, b, F=F, L=L)
    np.testing.assert_allclose(o_r, o_p, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(s_r, s_p, rtol=1e-5, atol=1e-6)
    o_n, _ = oracle.gdn(q, k, v, a, b, F=F, L=L)
    assert np.abs(o_n - o_r).max() > 1e-2  # and it does change the result


# ---------------------------------------------------------------- causal temporal conv with block cache

def _training_construction(blocks, w, bias):
    """The talk's training-time construction, through a library convolution: the
    blocks laid end to end along time with a zero token and then a copy of the
    previous block's last frame before every later block, one depthwise
    kernel-3 convolution (zero padding at both ends) over the whole sequence,
    and the inserted positions dropped."""
    import torch
    seq, keep = [], []
    for i, blk in enumerate(blocks):
        if i > 0:
            seq += [np.zeros_like(blk[:, :1]), blocks[i - 1][:, -1:]]
            keep += [False, False]
        seq.append(blk)
        keep += [True] * blk.shape[1]
    x = np.concatenate(seq, axis=1).astype(np.float64)           # [B, T, HW, C]
    B, T, HW, C = x.shape
    xt = torch.from_numpy(x).permute(0, 2, 3, 1).reshape(B * HW, C, T)
    wt = torch.from_numpy(np.asarray(w, np.float64)).reshape(C, 1, 3)
    bt = None if bias is None else torch.from_numpy(np.asarray(bias, np.float64))
    yt = torch.nn.functional.conv1d(xt, wt, bt, padding=1, groups=C)
    y = yt.reshape(B, HW, C, T).permute(0, 3, 1, 2).numpy()
    return y[:, np.array(keep)]


@pytest.mark.parametrize("with_bias", [False, True])
def test_temporal_conv_stream_equals_training_construction(with_bias):
    rng = np.random.default_rng(31)
    B, HW, C = 2, 5, 6
    blocks = [rng.standard_normal((B, F, HW, C)).astype(np.float32) for F in (3, 1, 4)]
    w = rng.standard_normal((C, 3)).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32) if with_bias else None
    outs, cache = [], None
    for blk in blocks:
        y, cache = oracle.temporal_conv(blk, w, bias=bias, cache_in=cache)
        outs.append(y)
        np.testing.assert_array_equal(cache, blk[:, -1].astype(np.float64))
    np.testing.assert_allclose(np.concatenate(outs, axis=1), _training_construction(blocks, w, bias),
                               rtol=1e-12, atol=1e-12)


def test_temporal_conv_impulse_and_block_boundaries():
    """An impulse at frame f of a block spreads to frames f-1, f, f+1 of the same
    block only (through the cache, to the first frame of the next block when f
    is the last frame; never back into the previous block)."""
    B, F, HW, C = 1, 4, 1, 3
    w = np.array([[1., 2., 3.], [4., 5., 6.], [7., 8., 9.]], np.float32)
    for f in range(F):
        x = np.zeros((B, F, HW, C), np.float32)
        x[0, f, 0, :] = 1.0
        y, cache = oracle.temporal_conv(x, w)
        expect = np.zeros((B, F, HW, C))
        expect[0, f, 0] = w[:, 1]
        if f > 0:
            expect[0, f - 1, 0] = w[:, 2]
        if f + 1 < F:
            expect[0, f + 1, 0] = w[:, 0]
        np.testing.assert_array_equal(y, expect)
        y2, _ = oracle.temporal_conv(np.zeros_like(x), w, cache_in=cache)
        np.testing.assert_array_equal(y2[0, 0, 0], w[:, 0] * (1.0 if f == F - 1 else 0.0))


# ---------------------------------------------------------------- windowed softmax attention

def _sdpa_window(q, k, v, F, L, W, scale=None):
    """The windowed layer through the library's attention primitive: one fp64
    scaled_dot_product_attention over the whole sequence with a boolean mask
    (key frame within [query frame - W + 1, query frame])."""
    import torch
    fr = np.arange(F * L) // L
    allowed = (fr[None, :] <= fr[:, None]) & (fr[None, :] >= fr[:, None] - W + 1)
    qt, kt, vt = (torch.from_numpy(np.asarray(x, np.float64)) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(allowed),
                                                           scale=scale)
    return out.numpy()


@pytest.mark.parametrize("F,L,W,dk,dv", [(5, 3, 2, 4, 3), (4, 6, 1, 8, 8), (3, 5, 4, 6, 2), (6, 2, 3, 5, 7)])
def test_softmax_window_equals_masked_library_attention(F, L, W, dk, dv):
    rng = np.random.default_rng(40 + F)
    q = rng.standard_normal((2, 3, F * L, dk)).astype(np.float32)
    k = rng.standard_normal((2, 3, F * L, dk)).astype(np.float32)
    v = rng.standard_normal((2, 3, F * L, dv)).astype(np.float32)
    o = oracle.softmax_window(q, k, v, F=F, L=L, W=W)
    np.testing.assert_allclose(o, _sdpa_window(q, k, v, F, L, W), rtol=1e-12, atol=1e-12)
    o2 = oracle.softmax_window(q, k, v, F=F, L=L, W=W, scale=0.3)
    np.testing.assert_allclose(o2, _sdpa_window(q, k, v, F, L, W, scale=0.3), rtol=1e-12, atol=1e-12)


def test_softmax_window_closed_forms():
    rng = np.random.default_rng(5)
    F, L, d = 4, 3, 4
    q = rng.standard_normal((1, 1, F * L, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, F * L, d)).astype(np.float32)
    # constant values: every output row is that value
    v = np.tile(np.array([1.5, -2.0, 0.25], np.float32), (1, 1, F * L, 1))
    np.testing.assert_allclose(oracle.softmax_window(q, k, v, F=F, L=L, W=2), v.astype(np.float64), rtol=1e-14)
    # zero queries: the plain mean of the window's values (frames f-W+1 .. f, clipped at 0)
    v = rng.standard_normal((1, 1, F * L, 3)).astype(np.float32)
    o = oracle.softmax_window(np.zeros_like(q), k, v, F=F, L=L, W=2)
    for f in range(F):
        lo = max(0, f - 1) * L
        np.testing.assert_allclose(o[0, 0, f * L:(f + 1) * L], np.tile(v[0, 0, lo:(f + 1) * L].astype(np.float64).mean(0), (L, 1)),
                                   rtol=1e-12, atol=1e-14)
    # one dominant key inside the window picks its value; the same key just outside the window is ignored
    qd = np.zeros((1, 1, F * L, d), np.float32)
    kd = np.zeros((1, 1, F * L, d), np.float32)
    qd[..., 0] = 1.0
    kd[0, 0, 4, 0] = 60.0  # frame 1, token 1
    o = oracle.softmax_window(qd, kd, v, F=F, L=L, W=2, scale=1.0)
    np.testing.assert_allclose(o[0, 0, 3 * 1:3 * 3], np.tile(v[0, 0, 4], (6, 1)), rtol=1e-12, atol=1e-12)  # frames 1, 2
    uniform = o[0, 0, 9:12]  # frame 3 sees frames 2, 3 only: no dominant key, zero scores
    np.testing.assert_allclose(uniform, np.tile(v[0, 0, 6:12].astype(np.float64).mean(0), (3, 1)), rtol=1e-12, atol=1e-14)
    # W >= F: block-causal attention over all earlier frames; W = 1: within the frame only
    v = rng.standard_normal((1, 1, F * L, 3)).astype(np.float32)
    full = oracle.softmax_window(q, k, v, F=F, L=L, W=F + 3)
    np.testing.assert_allclose(full, oracle.softmax_window(q, k, v, F=F, L=L, W=F), rtol=0, atol=0)
    own = oracle.softmax_window(q, k, v, F=F, L=L, W=1)
    for f in range(F):
        sl = slice(f * L, (f + 1) * L)
        np.testing.assert_allclose(own[0, 0, sl], oracle.softmax_window(q[:, :, sl], k[:, :, sl], v[:, :, sl], F=1,
                                                                         L=L, W=1)[0, 0], rtol=1e-14)


def test_softmax_window_frame_subset_and_permutation():
    rng = np.random.default_rng(6)
    F, L, d = 5, 4, 6
    q, k = (rng.standard_normal((1, 2, F * L, d)).astype(np.float32) for _ in range(2))
    v = rng.standard_normal((1, 2, F * L, 5)).astype(np.float32)
    full = oracle.softmax_window(q, k, v, F=F, L=L, W=3)
    part = oracle.softmax_window(q, k, v, F=F, L=L, W=3, frames=[1, 4])
    for f in range(F):
        sl = slice(f * L, (f + 1) * L)
        if f in (1, 4):
            np.testing.assert_array_equal(part[:, :, sl], full[:, :, sl])
        else:
            assert np.isnan(part[:, :, sl]).all()
    # permuting the tokens inside every frame permutes the outputs the same way
    perm = np.concatenate([f * L + rng.permutation(L) for f in range(F)])
    outp = oracle.softmax_window(q[:, :, perm], k[:, :, perm], v[:, :, perm], F=F, L=L, W=3)
    np.testing.assert_allclose(outp, full[:, :, perm], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- ReLU mode

def _quadratic_masked_attention(q, k, v, F, L, eps):
    """O(N^2) block-causal masked attention with ReLU features (independent route)."""
    N = F * L
    rq = np.maximum(q.astype(np.float64), 0)
    rk = np.maximum(k.astype(np.float64), 0)
    frame = np.arange(N) // L
    mask = frame[None, :] <= frame[:, None]  # key frame <= query frame
    A = (rq @ rk.T) * mask
    return (A @ v.astype(np.float64)) / (A.sum(axis=1, keepdims=True) + eps)


@pytest.mark.parametrize("F,L,dk,dv", [(1, 7, 4, 3), (4, 5, 6, 5), (8, 8, 8, 8)])
def test_relu_la_equals_quadratic_masked_attention(F, L, dk, dv):
    rng = np.random.default_rng(F * L)
    q = rng.standard_normal((1, F * L, dk)).astype(np.float32)
    k = rng.standard_normal((1, F * L, dk)).astype(np.float32)
    v = rng.standard_normal((1, F * L, dv)).astype(np.float32)
    o, kv, z = oracle.relu_la(q, k, v, F=F, L=L, eps=1e-6)
    ref = _quadratic_masked_attention(q[0], k[0], v[0], F, L, 1e-6)
    np.testing.assert_allclose(o[0], ref, rtol=1e-12, atol=1e-12)
    rk = np.maximum(k[0].astype(np.float64), 0)
    np.testing.assert_allclose(kv[0], rk.T @ v[0].astype(np.float64), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z[0], rk.sum(axis=0), rtol=1e-12, atol=1e-12)


def test_relu_la_state_carry_and_zero_query():
    rng = np.random.default_rng(11)
    F, L, dk, dv = 4, 3, 5, 4
    q = rng.standard_normal((2, F * L, dk)).astype(np.float32)
    k = rng.standard_normal((2, F * L, dk)).astype(np.float32)
    v = rng.standard_normal((2, F * L, dv)).astype(np.float32)
    q[0, 1] = -np.abs(q[0, 1])  # relu(q) == 0 -> o == 0
    o, kv, z = oracle.relu_la(q, k, v, F=F, L=L)
    assert np.all(o[0, 1] == 0.0)
    o1, kv1, z1 = oracle.relu_la(q[:, :2 * L], k[:, :2 * L], v[:, :2 * L], F=2, L=L)
    o2, kv2, z2 = oracle.relu_la(q[:, 2 * L:], k[:, 2 * L:], v[:, 2 * L:], F=2, L=L, kv_in=kv1, z_in=z1)
    np.testing.assert_allclose(o2, o[:, 2 * L:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(kv2, kv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z2, z, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes():
    """The brute-force pin distinguishes the correct rule from plausible wrong ones."""
    rng = np.random.default_rng(13)
    F, L, dk, dv = 2, 3, 4, 4
    q, k, v, a, b = _rand_case(1, F, L, dk, dv, rng)
    al = np.array([oracle.gate_alpha(x) for x in a[0]], np.float32)
    be = np.array([oracle.gate_beta(x) for x in b[0]], np.float32)
    S0 = rng.standard_normal((dk, dv))
    o_ref, s_ref = _bruteforce_gdn(q[0], k[0], v[0], al, be, F, L, S0)

    def variant(sign=1.0, transpose_read=False, per_token_read=False, decay_after=False):
        S = S0.copy()
        o = np.zeros((F * L, dv))
        for f in range(F):
            if not decay_after:
                S = al[f] * S
            for t in range(f * L, (f + 1) * L):
                kh = k[0, t].astype(np.float64)
                kh /= np.linalg.norm(kh)
                r = (S @ kh if transpose_read else S.T @ kh) - v[0, t]
                S = S - sign * be[t] * np.outer(kh, r)
                if per_token_read:
                    o[t] = S.T @ q[0, t]
            if decay_after:
                S = al[f] * S
            if not per_token_read:
                for t in range(f * L, (f + 1) * L):
                    o[t] = S.T @ q[0, t]
        return o, S

    o_ok, s_ok = variant()
    np.testing.assert_allclose(o_ok, o_ref, atol=1e-6)
    for kw in [dict(sign=-1.0), dict(transpose_read=True), dict(per_token_read=True), dict(decay_after=True)]:
        o_bad, s_bad = variant(**kw)
        assert np.abs(o_bad - o_ref).max() > 1e-3, kw
