"""fp64 check of the chunkwise equations the CUDA kernels implement (CPU only).

The pages say a chunkwise algorithm with diagonal-plus-low-rank structure
exists ("Kimi Linear acaba de superar a la atencion completa...", the section
on the chunk training algorithm and the DPLR transition) but print no
equations.  The chunk form below is derived by unrolling the per-token step of
"Kimi Delta Attention: la atencion lineal detras de Kimi K2 y Qwen3" (section
"Como funciona Kimi Delta Attention paso a paso"), and this file proves it
equals the token recurrence (the oracle) to fp64 rounding -- including the
16-token sub-chunk reference points used to keep every exponential factor in
range, the blocked inversion of (I + A), partial last chunks and h0 != 0.
It is written in numpy, shares nothing with the CUDA sources and imports only
the oracle.

Per chunk of C tokens (padded with g = 0, beta = 0, k = q = v = 0), with
G_i = sum_{j <= i} g_j (inclusive, restarting at the chunk):
  A_ij   = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}          (i > j)
  Aqk_ij = scale  sum_c q_ic k_jc e^{G_ic - G_jc}          (i >= j)
  T      = (I + A)^{-1}
  W      = T diag(beta) (K * e^G),   Ut = T diag(beta) V
  U      = Ut - W S,   O = scale (Q * e^G) S + Aqk U
  S'     = Diag(e^{G_last}) S + (K * e^{G_last - G})^T U
"""
import numpy as np
import pytest

import oracle

C, SC = 64, 16


def blocked_unit_lower_inverse(A, sc=SC):
    """(I + A)^{-1} for strictly lower A: invert the sc x sc diagonal blocks by
    forward substitution, then fill block (p, r) as
    -T_pp * sum_{r <= m < p} A_pm T_mr, block-row by block-row."""
    n = A.shape[0]
    nb = n // sc
    T = np.zeros_like(A)
    for p in range(nb):
        s = slice(p * sc, (p + 1) * sc)
        Ab = A[s, s]
        Tb = np.eye(sc)
        for i in range(sc):
            for c in range(i):
                Tb[i, c] = -sum(Ab[i, j] * Tb[j, c] for j in range(c, i))
        T[s, s] = Tb
    for p in range(1, nb):
        sp = slice(p * sc, (p + 1) * sc)
        for r in range(p - 1, -1, -1):
            sr = slice(r * sc, (r + 1) * sc)
            acc = np.zeros((sc, sc))
            for m in range(r, p):
                sm = slice(m * sc, (m + 1) * sc)
                acc += A[sp, sm] @ T[sm, sr]
            T[sp, sr] = -T[sp, sp] @ acc
    return T


def chunk_intra(qc, kc, vc, gc, bc, scale):
    """Intra-chunk quantities for one padded chunk (C rows)."""
    G = np.cumsum(gc, axis=0)
    f = (np.arange(C) // SC) * SC
    Kin = kc * np.exp(G - G[f])          # every factor <= 1
    Qin = qc * np.exp(G - G[f])
    Akk = np.zeros((C, C))
    Aqk = np.zeros((C, C))
    for p in range(C // SC):
        fp = p * SC
        n = fp + SC
        Kvar = kc[:n] * np.exp(G[fp] - G[:n])   # <= 1 before fp, >= 1 (<= 15 tokens) after
        rows = slice(fp, n)
        Akk[rows, :n] = Kin[rows] @ Kvar.T
        Aqk[rows, :n] = Qin[rows] @ Kvar.T
    A = np.tril(Akk, -1) * bc[:, None]
    Aqk = np.tril(Aqk, 0) * scale
    T = blocked_unit_lower_inverse(A)
    W = T @ (bc[:, None] * kc * np.exp(G))
    Ut = T @ (bc[:, None] * vc)
    QG = scale * qc * np.exp(G)
    KGl = kc * np.exp(G[-1] - G)
    return dict(G=G, A=A, T=T, W=W, Ut=Ut, Aqk=Aqk, QG=QG, KGl=KGl, gam=np.exp(G[-1]))


def chunk_forward(q, k, v, g, b, h0, scale):
    """One (sequence, head): q,k [L,dk], v [L,dv], g [L,dk], b [L]."""
    L, dk = k.shape
    dv = v.shape[1]
    S = h0.copy()
    out = np.zeros((L, dv))
    for s0 in range(0, L, C):
        n = min(C, L - s0)
        pad = lambda x: np.concatenate([x[s0:s0 + n], np.zeros((C - n,) + x.shape[1:])])
        I = chunk_intra(pad(q), pad(k), pad(v), pad(g), pad(b), scale)
        U = I["Ut"] - I["W"] @ S
        O = I["QG"] @ S + I["Aqk"] @ U
        S = I["gam"][:, None] * S + I["KGl"].T @ U
        out[s0:s0 + n] = O[:n]
    return out, S


def _inputs(rng, L, dk, dv, gate_shift=0.0):
    q = rng.standard_normal((L, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, dv))
    g = -np.log1p(np.exp(rng.standard_normal((L, dk)) + gate_shift))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    return q, k, v, g, b


@pytest.mark.parametrize("L", [1, 15, 64, 100, 193, 256])
def test_chunk_form_equals_token_recurrence(L):
    rng = np.random.default_rng(100 + L)
    dk, dv, scale = 16, 12, 0.25
    q, k, v, g, b = _inputs(rng, L, dk, dv)
    h0 = 0.5 * rng.standard_normal((dk, dv))
    out, hT = chunk_forward(q, k, v, g, b, h0, scale)
    o_ref, h_ref = oracle.fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                              g[None, :, None], b[None, :, None], scale, h0=h0[None, None])
    np.testing.assert_allclose(out, o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(hT, h_ref[0, 0], rtol=0, atol=1e-12)


def test_fast_decay_stays_finite_and_exact():
    """Mean per-token decay about e^-3.1 (gate shift +3): the sub-chunk
    references keep every factor finite; the result still matches."""
    rng = np.random.default_rng(3)
    L, dk, dv, scale = 160, 16, 8, 0.25
    q, k, v, g, b = _inputs(rng, L, dk, dv, gate_shift=3.0)
    out, hT = chunk_forward(q, k, v, g, b, np.zeros((dk, dv)), scale)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(hT))
    o_ref, h_ref = oracle.fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                              g[None, :, None], b[None, :, None], scale)
    np.testing.assert_allclose(out, o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(hT, h_ref[0, 0], rtol=0, atol=1e-12)


def test_blocked_inverse():
    rng = np.random.default_rng(4)
    A = np.tril(rng.standard_normal((C, C)) * 0.3, -1)
    T = blocked_unit_lower_inverse(A)
    np.testing.assert_allclose(T @ (np.eye(C) + A), np.eye(C), rtol=0, atol=1e-10)
    np.testing.assert_array_equal(np.triu(T, 1), 0.0)
    np.testing.assert_array_equal(np.diag(T), 1.0)


def test_chunk_is_one_affine_map():
    """Each chunk maps S -> M S + Bm with M = Diag(e^{G_last}) - KGl^T W and
    Bm = KGl^T Ut (the form a sequence-parallel scan would compose)."""
    rng = np.random.default_rng(5)
    dk, dv, scale = 8, 6, 0.3
    q, k, v, g, b = _inputs(rng, C, dk, dv)
    I = chunk_intra(q, k, v, g, b, scale)
    M = np.diag(I["gam"]) - I["KGl"].T @ I["W"]
    Bm = I["KGl"].T @ I["Ut"]
    S0 = rng.standard_normal((dk, dv))
    _, S1 = chunk_forward(q, k, v, g, b, S0, scale)
    np.testing.assert_allclose(M @ S0 + Bm, S1, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Backward of the chunk equations (what the backward kernels compute)
# --------------------------------------------------------------------------
def chunk_backward_one(qc, kc, vc, gc, bc, S, dO, dSn, scale):
    """Gradients of one padded chunk from its entry state S, the output
    gradient dO and the gradient dSn of its exit state.  Pairwise
    exponentials e^{G_ic - G_jc} (no sub-chunk references), as the fp32
    backward kernels take them.  Returns (dq, dk, dv, dg, db, dS)."""
    G = np.cumsum(gc, axis=0)
    Ex = np.exp(G[:, None, :] - G[None, :, :])                 # [i, j, c]
    Pkk = kc[:, None, :] * kc[None, :, :] * Ex                  # k_ic k_jc e^{..}
    Pqk = scale * qc[:, None, :] * kc[None, :, :] * Ex
    low = np.tril(np.ones((C, C)), -1)
    lowd = np.tril(np.ones((C, C)), 0)
    Ap = Pkk.sum(-1) * low                                     # A' (i > j)
    A = bc[:, None] * Ap
    Aqk = Pqk.sum(-1) * lowd
    T = np.linalg.inv(np.eye(C) + A)
    Tp = T * bc[None, :]                                       # T' = T diag(beta)
    KG = kc * np.exp(G)
    W = Tp @ KG
    R = vc - KG @ S
    E = Tp @ R
    Khat = kc * np.exp(G[-1] - G)
    QGs = scale * qc * np.exp(G)
    gam = np.exp(G[-1])
    # state side
    dE = Aqk.T @ dO + Khat @ dSn
    dS = QGs.T @ dO + gam[:, None] * dSn - W.T @ dE
    dR = Tp.T @ dE
    dv = dR.copy()
    dKG = -dR @ S.T
    dTp = dE @ R.T
    dQGs = dO @ S.T
    dAqk = (dO @ E.T) * lowd
    dKhat = E @ dSn.T
    dq = scale * np.exp(G) * dQGs
    dG = QGs * dQGs
    dk = np.exp(G[-1] - G) * dKhat
    dGl = (dKhat * Khat).sum(0) + gam * (S * dSn).sum(1)
    dG -= dKhat * Khat
    dk += np.exp(G) * dKG
    dG += KG * dKG
    # T' = T diag(beta), T = (I + A)^{-1}, A = diag(beta) A'
    dT = dTp * bc[None, :]
    db = (T * dTp).sum(0)
    dA = -(T.T @ dT @ T.T) * low
    db += (dA * Ap).sum(1)
    dAp = bc[:, None] * dA
    # pairwise products
    dk += np.einsum("ij,ijc->ic", dAp, kc[None, :, :] * Ex)
    dk += np.einsum("ij,ijc->jc", dAp, kc[:, None, :] * Ex)
    dG += np.einsum("ij,ijc->ic", dAp, Pkk) - np.einsum("ij,ijc->jc", dAp, Pkk)
    dq += np.einsum("ij,ijc->ic", dAqk, scale * kc[None, :, :] * Ex)
    dk += np.einsum("ij,ijc->jc", dAqk, scale * qc[:, None, :] * Ex)
    dG += np.einsum("ij,ijc->ic", dAqk, Pqk) - np.einsum("ij,ijc->jc", dAqk, Pqk)
    dG[-1] += dGl
    dg = np.cumsum(dG[::-1], axis=0)[::-1]                     # G = cumsum(g)
    return dq, dk, dv, dg, db, dS


def chunk_backward(q, k, v, g, b, h0, dout, dhT, scale):
    """One (sequence, head): forward walk for the entry states, then the
    chunks in reverse with the state gradient carried between them."""
    L, dk_ = k.shape
    dv_ = v.shape[1]
    starts = list(range(0, L, C))
    pad = lambda x, s0, n: np.concatenate([x[s0:s0 + n], np.zeros((C - n,) + x.shape[1:])])
    S = h0.copy()
    entry = []
    for s0 in starts:
        n = min(C, L - s0)
        I = chunk_intra(pad(q, s0, n), pad(k, s0, n), pad(v, s0, n), pad(g, s0, n),
                        pad(b, s0, n), scale)
        entry.append(S)
        U = I["Ut"] - I["W"] @ S
        S = I["gam"][:, None] * S + I["KGl"].T @ U
    grads = [np.zeros_like(x) for x in (q, k, v, g, b)]
    dS = dhT.copy()
    for ci in range(len(starts) - 1, -1, -1):
        s0 = starts[ci]
        n = min(C, L - s0)
        r = chunk_backward_one(pad(q, s0, n), pad(k, s0, n), pad(v, s0, n), pad(g, s0, n),
                               pad(b, s0, n), entry[ci], pad(dout, s0, n), dS, scale)
        for gx, part in zip(grads, r[:5]):
            gx[s0:s0 + n] = part[:n]
        dS = r[5]
    return (*grads, dS)


@pytest.mark.parametrize("L", [1, 64, 100, 193])
def test_chunk_backward_equals_oracle(L):
    rng = np.random.default_rng(40 + L)
    dk, dv, scale = 8, 6, 0.4
    q, k, v, g, b = _inputs(rng, L, dk, dv)
    h0 = 0.3 * rng.standard_normal((dk, dv))
    dout = rng.standard_normal((L, dv))
    dhT = rng.standard_normal((dk, dv))
    got = chunk_backward(q, k, v, g, b, h0, dout, dhT, scale)
    sh = lambda x: x[None, :, None]
    ref = oracle.bwd(sh(q), sh(k), sh(v), sh(g), b[None, :, None], scale, sh(dout),
                     h0=h0[None, None], dhT=dhT[None, None])
    ref = [r[0, :, 0] for r in ref[:5]] + [ref[5][0, 0]]
    for a, r in zip(got, ref):
        np.testing.assert_allclose(a, r, rtol=1e-9, atol=1e-10)


# --------------------------------------------------------------------------
# Exponent references of the fused tensor-core prep (what it multiplies out)
# --------------------------------------------------------------------------
# The pairwise factor e^{G_ic - G_jc} of A and Aqk becomes a matrix product once
# it is split as e^{G_ic} e^{-G_jc}.  The fused prep takes that split -- the row
# operands are then the image tiles K e^G and Q e^G themselves -- whenever every
# |G_tc| of the chunk stays within RANGE_LOG2 (log2 units; the margin below the fp32
# exponent range keeps the factors <= 1 of small key components normal).
# Otherwise it takes the lower triangle level by level: at level l the chunk is
# cut into blocks of 2s rows (s = 32, 16, ..., 1); a pair i > j belongs to the
# level where i is in the upper half of a block and j in its lower half, and both
# factors are referenced to the first row f of that upper half, so
# e^{G_i - G_f} <= 1 and e^{G_f - G_j} <= 1 for every channel, at any decay rate.
# One product per level covers every block (entries across blocks are not used),
# and a last product without exponents gives the diagonal of Aqk.
# Between the two, a chunk whose every |G_tc - G_31,c| stays within RANGE_LOG2
# (G_31 = the channel's decay over the first 32 tokens) is split as
# e^{G_ic - G_31,c} e^{G_31,c - G_jc}: still one product, for chunks decaying by up to
# twice the range; its row operands differ from the image tiles, which the prep then
# writes again at the chunk start.
RANGE_LOG2 = 100.0


def _pairwise(qc, kc, gc):
    G = np.cumsum(gc, axis=0)
    E = np.exp(G[:, None, :] - G[None, :, :])
    Akk = np.einsum("ic,jc,ijc->ij", kc, kc, E)
    Aqk = np.einsum("ic,jc,ijc->ij", qc, kc, E)
    return np.tril(Akk, -1), np.tril(Aqk, 0)


def _fast_needs_fallback(gc):
    G = np.cumsum(gc, axis=0)
    return np.abs(G).max() / np.log(2.0) > RANGE_LOG2


def _reference_choice(gc):
    """Which form the fused prep takes for one chunk: 'start', 'mid' or 'levels'."""
    G = np.cumsum(gc, axis=0) / np.log(2.0)
    if np.abs(G).max() <= RANGE_LOG2:
        return "start"
    if np.abs(G - G[min(31, len(G) - 1)]).max() <= RANGE_LOG2:
        return "mid"
    return "levels"


def _mid_reference(qc, kc, gc):
    """The mid-chunk split: A (strictly lower), Aqk (lower) and every factor's exponent."""
    G = np.cumsum(gc, axis=0)
    x = G - G[min(31, len(G) - 1)]
    KG, QG, Kn = kc * np.exp(x), qc * np.exp(x), kc * np.exp(-x)
    return np.tril(KG @ Kn.T, -1), np.tril(QG @ Kn.T, 0), x


def _single_reference(qc, kc, gc, dtype=np.float64):
    G = np.cumsum(gc, axis=0).astype(dtype)
    KG, QG, Kn = kc * np.exp(G), qc * np.exp(G), kc * np.exp(-G)
    return np.tril(KG @ Kn.T, -1), np.tril(QG @ Kn.T, 0), (KG, QG, Kn)


def _level_passes(qc, kc, gc, dtype=np.float64):
    """The fallback: returns A (strictly lower), Aqk (lower) and the exponents
    of every factor used."""
    G = np.cumsum(gc, axis=0)
    t = np.arange(C)
    Akk = np.zeros((C, C))
    Aqk = np.zeros((C, C))
    exps = []
    s = C // 2
    while s >= 1:
        upper = (t % (2 * s)) >= s
        f = (t // (2 * s)) * 2 * s + s                       # first row of the block's upper half
        x = (G - G[f]).astype(dtype)
        Kin = np.where(upper[:, None], kc * np.exp(x), 0.0)
        Qin = np.where(upper[:, None], qc * np.exp(x), 0.0)
        Kd = np.where(upper[:, None], 0.0, kc * np.exp(-x))
        Dk, Dq = Kin @ Kd.T, Qin @ Kd.T
        pair = upper[:, None] & ~upper[None, :] & ((t // (2 * s))[:, None] == (t // (2 * s))[None, :])
        Akk[pair] = Dk[pair]
        Aqk[pair] = Dq[pair]
        exps += [x[upper], -x[~upper]]
        s //= 2
    Aqk[t, t] = np.einsum("ic,ic->i", qc, kc)                # diagonal: no exponent
    return np.tril(Akk, -1), Aqk, exps


@pytest.mark.parametrize("shift", [-2.0, 0.0])
def test_single_reference_reproduces_pairs(shift):
    """The workload's gate distributions stay inside the e^{+-G} range (a chunk
    of the e^-0.8-per-token workloads decays by about 74 log2 units on average; a
    channel exceeds 100 about once in 20,000, so about one chunk-head in 170 takes
    the mid-chunk split instead) and the factored products equal the pairwise
    sums; the row operands are the image tiles K e^G and Q e^G."""
    rng = np.random.default_rng(50)
    q, k, v, g, b = _inputs(rng, C, 128, 4, gate_shift=shift)
    assert not _fast_needs_fallback(g)
    A_ref, Aqk_ref = _pairwise(q, k, g)
    A, Aqk, _ = _single_reference(q, k, g)
    np.testing.assert_allclose(A, A_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Aqk, Aqk_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shift", [8.0, 40.0])
def test_level_fallback_under_fast_decay(shift):
    """About 8 (and 40) nats of decay per token: the e^{-G} factors leave the
    fp32 range, so the prep must switch; every factor of the level passes is
    <= 1, and their products still equal the pairwise sums."""
    rng = np.random.default_rng(51)
    q, k, v, g, b = _inputs(rng, C, 128, 4, gate_shift=shift)
    assert _fast_needs_fallback(g)
    with np.errstate(over="ignore"):
        _, _, f32 = _single_reference(q, k, g, dtype=np.float32)
    assert not all(np.all(np.isfinite(f)) for f in f32)
    with np.errstate(under="ignore"):
        A_ref, Aqk_ref = _pairwise(q, k, g)
        A, Aqk, exps = _level_passes(q, k, g)
    assert all(np.all(x <= 0.0) for x in exps)
    np.testing.assert_allclose(A, A_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Aqk, Aqk_ref, rtol=0, atol=1e-12)


def test_level_fallback_slow_decay():
    """The level passes are exact at slow decay too, and cover each pair once."""
    rng = np.random.default_rng(52)
    q, k, v, g, b = _inputs(rng, C, 32, 4, gate_shift=-4.0)
    A_ref, Aqk_ref = _pairwise(q, k, g)
    A, Aqk, _ = _level_passes(q, k, g)
    np.testing.assert_allclose(A, A_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Aqk, Aqk_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shift", [0.3, 0.8])
def test_mid_reference_reproduces_pairs(shift):
    """About e^-1.0 and e^-1.3 of decay per token: a chunk decays past the
    chunk-start split's range but every factor of the mid-chunk split stays within
    2^+-100, and its products equal the pairwise sums (ragged chunk included)."""
    rng = np.random.default_rng(53)
    for L in (C, 44):
        q, k, v, g, b = _inputs(rng, L, 128, 4, gate_shift=shift)
        if L == C:
            assert _reference_choice(g) == "mid"
        if _reference_choice(g) == "levels":
            continue
        A_ref, Aqk_ref = _pairwise(q, k, g)
        A, Aqk, x = _mid_reference(q, k, g)
        assert np.abs(x).max() / np.log(2.0) <= RANGE_LOG2
        np.testing.assert_allclose(A, A_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Aqk, Aqk_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shift", [-2.0, 0.0])
def test_workload_gates_never_need_the_level_passes(shift):
    """At both workloads' gate distributions (log_alpha = -softplus(N(0, 1) + shift),
    per channel and token), 4000 chunk-heads of 128 channels all take one of the two
    single-product splits; at shift 0 some take the mid-chunk one."""
    rng = np.random.default_rng(54)
    x = rng.standard_normal((4000, C, 128)) + shift
    G = np.cumsum(np.log1p(np.exp(x)), axis=1) / np.log(2.0)     # |G| in log2 units
    start = np.abs(G).max(axis=(1, 2)) <= RANGE_LOG2
    mid = np.abs(G - G[:, 31:32, :]).max(axis=(1, 2)) <= RANGE_LOG2
    assert np.all(start | mid)
    if shift == 0.0:
        assert not np.all(start)
    else:
        assert np.all(start)
