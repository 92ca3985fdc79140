"""Pins for the fp64 oracle (CPU only).

The pages print no worked numeric example, so the oracle is pinned to things
other than itself: a hand-worked two-token example, closed forms of special
cases, reductions to the simpler published rules (linear attention, DeltaNet,
Gated DeltaNet), the erase-then-write recall property, a brute-force product of
dense transition matrices, a norm inequality, and equivalences that restate the
recurrence (continuation, packing, one-step chaining).  Each test names what a
plausible mistake in the oracle (dropped term, wrong sign or index, transposed
operand, decay after instead of before the prediction, scale applied twice)
would break.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(rng, N, T, H, dk, dv, unit_keys=True):
    q = rng.standard_normal((1, N * T, H, dk))
    k = rng.standard_normal((1, N * T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((1, N * T, H, dv))
    g = -np.log1p(np.exp(rng.standard_normal((1, N * T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, N * T, H))))
    h0 = 0.3 * rng.standard_normal((N, H, dk, dv))
    cu = np.arange(N + 1) * T
    return q, k, v, g, b, h0, cu


# --------------------------------------------------------------------------
# Hand-worked example (tests/golden/hand_worked_dk2_dv1.txt)
# --------------------------------------------------------------------------
def test_hand_worked_example():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "hand_worked_dk2_dv1.txt"))
            if ln.strip() and not ln.startswith("#")]
    h0 = np.array([float(x) for x in rows[0][1:]]).reshape(1, 1, 2, 1)
    toks = [list(map(float, r[1:])) for r in rows if r[0] == "tok"]
    hT_ref = np.array([float(x) for x in rows[-1][1:]]).reshape(1, 1, 2, 1)
    T = len(toks)
    g = np.zeros((1, T, 1, 2)); k = np.zeros((1, T, 1, 2)); v = np.zeros((1, T, 1, 1))
    b = np.zeros((1, T, 1)); q = np.zeros((1, T, 1, 2)); o_ref = np.zeros((1, T, 1, 1))
    for t, r in enumerate(toks):
        g[0, t, 0] = np.log(r[0:2]); k[0, t, 0] = r[2:4]; v[0, t, 0] = r[4:5]
        b[0, t, 0] = r[5]; q[0, t, 0] = r[6:8]; o_ref[0, t, 0] = r[8:9]
    out, hT = oracle.fwd(q, k, v, g, b, 1.0, h0=h0)
    np.testing.assert_allclose(out, o_ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(hT, hT_ref, rtol=0, atol=1e-14)
    # the same example through the decode step, token by token
    S = h0.reshape(1, 1, 2, 1)
    for t in range(T):
        o, S = oracle.step(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], S, 1.0)
        np.testing.assert_allclose(o, o_ref[:, t], rtol=0, atol=1e-14)
    np.testing.assert_allclose(S, hT_ref, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# P-brute: dense transition-matrix product
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dk,dv,T", [(4, 4, 24), (8, 8, 17), (8, 3, 12)])
def test_bruteforce_transition_product(dk, dv, T):
    """S_T = M_T..M_1 h0 + sum_t M_T..M_{t+1} beta_t k_t v_t^T with dense
    M_t = (I - beta_t k_t k_t^T) Diag(alpha_t); o_t = scale S_t^T q_t.

    Written as matrix products (no per-token "predict/correct" code), so a
    wrong operation order, a transposed state or a dropped term disagrees."""
    rng = np.random.default_rng(11)
    N, H, scale = 2, 3, 0.37
    q, k, v, g, b, h0, cu = _rand_inputs(rng, N, T, H, dk, dv, unit_keys=False)
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0, cu_seqlens=cu)
    for n in range(N):
        for h in range(H):
            ts = range(cu[n], cu[n + 1])
            Ms = []
            for t in ts:
                kt = k[0, t, h][:, None]
                Ms.append((np.eye(dk) - b[0, t, h] * kt @ kt.T) @ np.diag(np.exp(g[0, t, h])))
            for idx, t in enumerate(ts):
                # state after token idx, from scratch
                P = np.eye(dk)
                for M in Ms[:idx + 1]:
                    P = M @ P
                S = P @ h0[n, h]
                for s in range(idx + 1):
                    P = np.eye(dk)
                    for M in Ms[s + 1:idx + 1]:
                        P = M @ P
                    S = S + P @ (b[0, ts[s], h] * np.outer(k[0, ts[s], h], v[0, ts[s], h]))
                o = scale * S.T @ q[0, t, h]
                np.testing.assert_allclose(out[0, t, h], o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(hT[n, h], S, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P-GDN and P-DeltaNet: reductions to the predecessors
# --------------------------------------------------------------------------
def _gdn_reference(q, k, v, a, b, h0, scale):
    """Scalar-gate Gated DeltaNet, operator form S = a (I - b k k^T) S + b k v^T."""
    T = q.shape[0]
    S = h0.copy()
    outs = []
    for t in range(T):
        kt = k[t][:, None]
        S = a[t] * (np.eye(len(k[t])) - b[t] * kt @ kt.T) @ S + b[t] * kt @ v[t][None, :]
        outs.append(scale * S.T @ q[t])
    return np.array(outs), S


def test_reduces_to_gated_deltanet_with_uniform_gate():
    """alpha_t = a_t * ones: KDA equals Gated DeltaNet with scalar gate a_t."""
    rng = np.random.default_rng(5)
    T, H, dk, dv, scale = 40, 2, 8, 5, 0.5
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    a = np.exp(-np.log1p(np.exp(rng.standard_normal((T, H)))))
    g = np.repeat(np.log(a)[None, :, :, None], dk, axis=-1)
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    for h in range(H):
        o_ref, S_ref = _gdn_reference(q[0, :, h], k[0, :, h], v[0, :, h], a[:, h], b[0, :, h],
                                      h0[0, h], scale)
        np.testing.assert_allclose(out[0, :, h], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(hT[0, h], S_ref, rtol=0, atol=1e-12)


def test_reduces_to_deltanet_without_decay():
    """alpha = 1: the plain delta rule S = S - b k (k^T S) + b k v^T."""
    rng = np.random.default_rng(6)
    T, H, dk, dv, scale = 33, 1, 6, 6, 1.0
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    g[:] = 0.0
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    S = h0[0, 0].copy()
    for t in range(T):
        kt, vt, bt = k[0, t, 0], v[0, t, 0], b[0, t, 0]
        S = S - bt * np.outer(kt, kt @ S) + bt * np.outer(kt, vt)
        np.testing.assert_allclose(out[0, t, 0], scale * S.T @ q[0, t, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(hT[0, 0], S, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P-recall and P-orthonormal: erase-then-write semantics
# --------------------------------------------------------------------------
def test_exact_recall_of_current_key():
    """beta=1, unit k, q=k, scale=1: the read returns v_t exactly, for any h0
    and any per-channel decay (S_t^T k = vhat + (v - vhat)(k.k) = v)."""
    rng = np.random.default_rng(7)
    T, H, dk, dv = 50, 2, 16, 9
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    b[:] = 1.0
    out, _ = oracle.fwd(k, k, v, g, b, 1.0, h0=3.0 * h0)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-12)


def test_orthonormal_keys_store_and_overwrite():
    """alpha=1, beta=1, h0=0, orthonormal keys: querying k_j (with a beta=0
    read-only token) returns v_j; rewriting k_j with v' replaces it."""
    rng = np.random.default_rng(8)
    dk, dv, n = 8, 4, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T                       # n orthonormal keys
    vals = rng.standard_normal((n, dv))
    vnew = rng.standard_normal(dv)
    # tokens: write n keys, read all n, overwrite key 2, read key 2 and key 3
    K = list(keys) + list(keys) + [keys[2], keys[2], keys[3]]
    Q = list(keys) + list(keys) + [keys[2], keys[2], keys[3]]
    V = list(vals) + [np.zeros(dv)] * n + [vnew, np.zeros(dv), np.zeros(dv)]
    B = [1.0] * n + [0.0] * n + [1.0, 0.0, 0.0]
    T = len(K)
    q = np.array(Q)[None, :, None, :]; k = np.array(K)[None, :, None, :]
    v = np.array(V)[None, :, None, :]; b = np.array(B)[None, :, None]
    g = np.zeros((1, T, 1, dk))
    out, _ = oracle.fwd(q, k, v, g, b, 1.0)
    np.testing.assert_allclose(out[0, n:2 * n, 0], vals, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0, 2 * n, 0], vnew, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0, 2 * n + 1, 0], vnew, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0, 2 * n + 2, 0], vals[3], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P-linattn: linear attention with orthogonal keys, and to first order in beta
# --------------------------------------------------------------------------
def test_linear_attention_with_orthogonal_keys():
    """alpha=1, h0=0, mutually orthogonal keys (T <= dk): the erase term
    vanishes and o_t = scale * sum_{s<=t} beta_s (q_t . k_s) v_s, the plain
    outer-product accumulation of linear attention with beta-scaled values."""
    rng = np.random.default_rng(9)
    dk, dv, T, scale = 12, 5, 12, 0.29
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = (Qm.T * rng.uniform(0.5, 1.5, size=(dk, 1)))[None, :, None, :]   # orthogonal, not unit
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    b = rng.uniform(0.1, 0.9, size=(1, T, 1))
    g = np.zeros((1, T, 1, dk))
    out, _ = oracle.fwd(q, k, v, g, b, scale)
    S = np.zeros((dk, dv))
    for t in range(T):
        S = S + np.outer(k[0, t, 0], v[0, t, 0]) * b[0, t, 0]   # linear-attention write
        np.testing.assert_allclose(out[0, t, 0], scale * S.T @ q[0, t, 0], rtol=0, atol=1e-12)


def test_first_order_in_beta_is_linear_attention():
    """h0=0, alpha=1: [KDA(eps*beta)]/eps -> scale sum_s beta_s (q_t.k_s) v_s as eps -> 0."""
    rng = np.random.default_rng(10)
    T, H, dk, dv, scale = 30, 1, 8, 4, 0.7
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    g[:] = 0.0
    eps = 1e-7
    out, _ = oracle.fwd(q, k, v, g, eps * b, scale)
    lin = np.zeros((T, dv))
    for t in range(T):
        for s in range(t + 1):
            lin[t] += scale * b[0, s, 0] * (q[0, t, 0] @ k[0, s, 0]) * v[0, s, 0]
    np.testing.assert_allclose(out[0, :, 0] / eps, lin, rtol=0, atol=1e-5)


# --------------------------------------------------------------------------
# P-decay: beta = 0 closed form
# --------------------------------------------------------------------------
def test_beta_zero_closed_form():
    """beta=0: nothing is written, S_t = Diag(prod_{s<=t} alpha_s) h0, so
    o_t = scale (Diag(prod alpha) h0)^T q_t and hT = Diag(prod_all alpha) h0."""
    rng = np.random.default_rng(12)
    T, H, dk, dv, scale = 25, 2, 7, 3, 0.41
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    b[:] = 0.0
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    for h in range(H):
        cum = np.cumsum(g[0, :, h], axis=0)          # log of the running product
        for t in range(T):
            S = np.exp(cum[t])[:, None] * h0[0, h]
            np.testing.assert_allclose(out[0, t, h], scale * S.T @ q[0, t, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(hT[0, h], np.exp(cum[-1])[:, None] * h0[0, h], rtol=0,
                                   atol=1e-12)
    # alpha = 1 as well: every read is scale * h0^T q_t
    g[:] = 0.0
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    for h in range(H):
        np.testing.assert_allclose(out[0, :, h], scale * q[0, :, h] @ h0[0, h], rtol=0,
                                   atol=1e-12)


# --------------------------------------------------------------------------
# P-contract: the transition is non-expansive for unit keys and beta in [0, 2]
# --------------------------------------------------------------------------
def test_state_norm_non_increasing_without_writes():
    rng = np.random.default_rng(13)
    T, H, dk, dv = 60, 2, 16, 8
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    b = rng.uniform(0.0, 2.0, size=b.shape)
    v[:] = 0.0
    S = h0.copy()
    prev = np.linalg.norm(S.reshape(H, -1), axis=-1)
    for t in range(T):
        _, S = oracle.step(q[0, t][None], k[0, t][None], v[0, t][None], g[0, t][None],
                           b[0, t][None], S, 1.0)
        cur = np.linalg.norm(S.reshape(H, -1), axis=-1)
        assert np.all(cur <= prev + 1e-12)
        prev = cur
    # general bound with writes: ||S_t|| <= ||S_{t-1}|| + beta ||k|| ||v||
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    S = h0.copy()
    for t in range(T):
        before = np.linalg.norm(S.reshape(H, -1), axis=-1)
        _, S = oracle.step(q[0, t][None], k[0, t][None], v[0, t][None], g[0, t][None],
                           b[0, t][None], S, 1.0)
        after = np.linalg.norm(S.reshape(H, -1), axis=-1)
        bound = before + b[0, t] * np.linalg.norm(k[0, t], axis=-1) * np.linalg.norm(v[0, t], axis=-1)
        assert np.all(after <= bound + 1e-12)


# --------------------------------------------------------------------------
# P-split: continuation, packing, decode chaining
# --------------------------------------------------------------------------
@pytest.mark.parametrize("t1", [1, 16, 37, 64])
def test_continuation_equals_single_pass(t1):
    rng = np.random.default_rng(14)
    T, H, dk, dv, scale = 80, 2, 8, 6, 0.3
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    o1, h1 = oracle.fwd(q[:, :t1], k[:, :t1], v[:, :t1], g[:, :t1], b[:, :t1], scale, h0=h0)
    o2, h2 = oracle.fwd(q[:, t1:], k[:, t1:], v[:, t1:], g[:, t1:], b[:, t1:], scale, h0=h1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(h2, hT, rtol=0, atol=1e-12)


def test_packed_sequences_equal_separate_calls():
    rng = np.random.default_rng(15)
    lens = [1, 63, 64, 65, 0, 130]
    H, dk, dv, scale = 2, 8, 4, 0.5
    Tt = sum(lens)
    q, k, v, g, b, _, _ = _rand_inputs(rng, 1, Tt, H, dk, dv)
    h0 = rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0, cu_seqlens=cu)
    for n, L in enumerate(lens):
        s = slice(cu[n], cu[n + 1])
        if L == 0:
            np.testing.assert_array_equal(hT[n], h0[n])     # empty sequence: state passes through
            continue
        o, h = oracle.fwd(q[:, s], k[:, s], v[:, s], g[:, s], b[:, s], scale, h0=h0[n:n + 1])
        np.testing.assert_allclose(out[:, s], o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(hT[n], h[0], rtol=0, atol=1e-12)


def test_decode_steps_chain_to_forward():
    rng = np.random.default_rng(16)
    N, T, H, dk, dv, scale = 3, 20, 2, 8, 8, 0.35
    q = rng.standard_normal((N, T, H, dk)); k = rng.standard_normal((N, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, T, H, dv))
    g = -np.log1p(np.exp(rng.standard_normal((N, T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((N, T, H))))
    h0 = rng.standard_normal((N, H, dk, dv))
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    S = h0
    for t in range(T):
        o, S = oracle.step(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], S, scale)
        np.testing.assert_allclose(o, out[:, t], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, hT, rtol=0, atol=1e-12)


def test_scale_applied_once():
    """Output is linear in scale and the state does not depend on it."""
    rng = np.random.default_rng(17)
    q, k, v, g, b, h0, cu = _rand_inputs(rng, 1, 20, 1, 8, 4)
    o1, h1 = oracle.fwd(q, k, v, g, b, 1.0, h0=h0)
    o2, h2 = oracle.fwd(q, k, v, g, b, 0.125, h0=h0)
    np.testing.assert_allclose(o2, 0.125 * o1, rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(h1, h2)


def test_rel_l2_metric():
    a = np.array([3.0, 4.0])
    assert oracle.rel_l2(a, a) == 0.0
    assert math.isclose(oracle.rel_l2(np.array([3.0, 4.0 + 0.5]), a), 0.1, rel_tol=1e-15)


# --------------------------------------------------------------------------
# P-affine: segment maps (context parallelism) from the linearity of the step
# --------------------------------------------------------------------------
def test_segment_map_is_dense_transition_product():
    """oracle.segment_map gives M = M_T..M_1 and B = sum_t M_T..M_{t+1} b_t k_t v_t^T
    with the dense M_t = (I - b_t k_t k_t^T) Diag(alpha_t): a map built with the
    wrong start (not the identity), with the values left in, or transposed
    disagrees."""
    rng = np.random.default_rng(21)
    N, T, H, dk, dv = 2, 9, 2, 6, 4
    q, k, v, g, b, _, cu = _rand_inputs(rng, N, T, H, dk, dv, unit_keys=False)
    M, Bm = oracle.segment_map(q, k, v, g, b, cu_seqlens=cu)
    for n in range(N):
        for h in range(H):
            P = np.eye(dk)
            Bref = np.zeros((dk, dv))
            for t in range(cu[n], cu[n + 1]):
                kt = k[0, t, h][:, None]
                Mt = (np.eye(dk) - b[0, t, h] * kt @ kt.T) @ np.diag(np.exp(g[0, t, h]))
                P = Mt @ P
                Bref = Mt @ Bref + b[0, t, h] * np.outer(k[0, t, h], v[0, t, h])
            np.testing.assert_allclose(M[n, h], P, rtol=0, atol=1e-13)
            np.testing.assert_allclose(Bm[n, h], Bref, rtol=0, atol=1e-13)
    assert not np.allclose(M[0, 0], M[0, 0].T)        # not symmetric: a transpose would show


@pytest.mark.parametrize("cuts", [(0, 80), (17, 80), (64, 128), (1, 2, 79)])
def test_composed_segment_maps_reproduce_the_sequence(cuts):
    """Pieces [c_i, c_{i+1}) run from the composed entry states give the
    single-pass outputs and final state (what a context-parallel split returns)."""
    rng = np.random.default_rng(22)
    T, H, dk, dv, scale = 80, 2, 8, 6, 0.3
    q, k, v, g, b, h0, _ = _rand_inputs(rng, 1, T, H, dk, dv)
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
    bounds = sorted(set((0,) + tuple(cuts) + (T,)))
    sl = lambda x, a, c: x[:, a:c]
    pieces = list(zip(bounds[:-1], bounds[1:]))
    maps, offs = zip(*(oracle.segment_map(sl(q, a, c), sl(k, a, c), sl(v, a, c), sl(g, a, c),
                                          sl(b, a, c)) for a, c in pieces))
    outs = []
    for r, (a, c) in enumerate(pieces):
        X = oracle.compose(np.stack(maps[:r]), np.stack(offs[:r]), h0) if r else h0
        o, S = oracle.fwd(sl(q, a, c), sl(k, a, c), sl(v, a, c), sl(g, a, c), sl(b, a, c),
                          scale, h0=X)
        outs.append(o)
    np.testing.assert_allclose(np.concatenate(outs, axis=1), out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, hT, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.compose(np.stack(maps), np.stack(offs), h0), hT,
                               rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# P-grad: the backward pass (training)
# --------------------------------------------------------------------------
def _loss(q, k, v, g, b, h0, cu, scale, dout, dhT):
    out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0, cu_seqlens=cu)
    return float(np.sum(out * dout) + np.sum(hT * dhT))


def test_backward_matches_finite_differences():
    """Central differences of sum(dout*out) + sum(dhT*hT) for every input
    element; the second sequence crosses the oracle's 64-token replay block."""
    rng = np.random.default_rng(31)
    lens, H, dk, dv, scale = [4, 67], 1, 3, 2, 0.7
    T = sum(lens)
    q, k, v, g, b, _, _ = _rand_inputs(rng, 1, T, H, dk, dv)
    h0 = 0.5 * rng.standard_normal((2, H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    dout = rng.standard_normal((1, T, H, dv))
    dhT = rng.standard_normal((2, H, dk, dv))
    grads = oracle.bwd(q, k, v, g, b, scale, dout, h0=h0, dhT=dhT, cu_seqlens=cu)
    inputs = [q, k, v, g, b, h0]
    eps = 1e-6
    for x, gx in zip(inputs, grads):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + eps
            lp = _loss(*inputs, cu, scale, dout, dhT)
            x[idx] = old - eps
            lm = _loss(*inputs, cu, scale, dout, dhT)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(gx, fd, rtol=1e-6, atol=1e-7)


def test_backward_matches_autograd_of_a_plain_recurrence():
    """torch autograd (fp64) through a separately written dense-matrix form of
    the step, S_t = (I - b k k^T) Diag(alpha) S_{t-1} + b k v^T, o = scale S^T q."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(32)
    lens, H, dk, dv, scale = [150, 0, 70], 2, 8, 6, 0.35
    T = sum(lens)
    q, k, v, g, b, _, _ = _rand_inputs(rng, 1, T, H, dk, dv)
    h0 = 0.3 * rng.standard_normal((3, H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    dout = rng.standard_normal((1, T, H, dv))
    dhT = rng.standard_normal((3, H, dk, dv))
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, g, b, h0)]
    tq, tk, tv, tg, tb, th0 = ts
    loss = 0.0
    eye = torch.eye(dk, dtype=torch.float64)
    for n in range(3):
        for h in range(H):
            S = th0[n, h]
            for t in range(cu[n], cu[n + 1]):
                kt = tk[0, t, h][:, None]
                M = (eye - tb[0, t, h] * kt @ kt.T) @ torch.diag(torch.exp(tg[0, t, h]))
                S = M @ S + tb[0, t, h] * kt @ tv[0, t, h][None, :]
                o = scale * S.T @ tq[0, t, h]
                loss = loss + (o * torch.from_numpy(dout[0, t, h])).sum()
            loss = loss + (S * torch.from_numpy(dhT[n, h])).sum()
    loss.backward()
    grads = oracle.bwd(q, k, v, g, b, scale, dout, h0=h0, dhT=dhT, cu_seqlens=cu)
    for t, gx in zip(ts, grads):
        np.testing.assert_allclose(gx, t.grad.numpy(), rtol=1e-10, atol=1e-11)


def test_scalar_gate_gradient_is_the_channel_sum():
    """Gated DeltaNet: with one gate per (token, head) broadcast over the key
    channels, the gate's gradient (central differences of the loss in the
    scalar gate) equals the channel sum of oracle.bwd's per-channel gradient."""
    rng = np.random.default_rng(33)
    T, H, dk, dv, scale = 20, 1, 4, 3, 0.6
    q, k, v, _, b, h0, cu = _rand_inputs(rng, 1, T, H, dk, dv)
    la = -np.log1p(np.exp(rng.standard_normal((1, T, H))))
    dout = rng.standard_normal((1, T, H, dv))
    dhT = rng.standard_normal((1, H, dk, dv))
    g = lambda a: np.repeat(a[..., None], dk, axis=-1)
    grads = oracle.bwd(q, k, v, g(la), b, scale, dout, h0=h0, dhT=dhT)
    eps = 1e-6
    for t in range(T):
        lp, lm = la.copy(), la.copy()
        lp[0, t, 0] += eps
        lm[0, t, 0] -= eps
        fd = (_loss(q, k, v, g(lp), b, h0, None, scale, dout, dhT) -
              _loss(q, k, v, g(lm), b, h0, None, scale, dout, dhT)) / (2 * eps)
        np.testing.assert_allclose(grads[3][0, t, 0].sum(), fd, rtol=1e-6, atol=1e-7)
