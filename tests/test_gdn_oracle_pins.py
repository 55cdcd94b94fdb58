"""Pins of the Gated DeltaNet oracle (oracle.orc_gdn_chunk) to results fixed by
the mathematics of the gated delta rule, independent of its token loop.

The block is the GDN linear attention of SANA-Streaming (section "hybrid
diffusion transformer"); the recurrence is the published gated delta rule
(Yang, Kautz and Hatamizadeh, "Gated Delta Networks", ICLR 2025) with
L2-normalised queries and keys:
    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = scale S_t q_t.
"""
import numpy as np
import pytest

import oracle as O
from inputgen import fill_gates_host
from inputgen.workloads import Workload

RNG = np.random.default_rng(7)


def _unit(x):
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return np.where(n > 0, x / np.where(n > 0, n, 1), 0)


def _rand(T, H, D, g_scale=0.3):
    q = RNG.standard_normal((T, H, D))
    k = RNG.standard_normal((T, H, D))
    v = RNG.standard_normal((T, H, D))
    g = -g_scale * RNG.random((T, H))
    beta = RNG.random((T, H))
    return q, k, v, g, beta


def test_product_form_random():
    """Transition-matrix form, built with matrix products: with
    A_t = a_t (I - b_t k_t k_t^T), S_t = S_0 A_1...A_t + sum_i b_i v_i k_i^T A_{i+1}...A_t."""
    T, H, D = 23, 2, 6
    q, k, v, g, beta = _rand(T, H, D)
    S0 = RNG.standard_normal((H, D, D))
    state = S0.copy()
    scale = 0.7
    out = O.gdn_chunk(scale, state, q, k, v, g, beta)
    kh, qh = _unit(k), _unit(q)
    for h in range(H):
        A = [np.exp(g[t, h]) * (np.eye(D) - beta[t, h] * np.outer(kh[t, h], kh[t, h]))
             for t in range(T)]
        for t in range(T):
            St = S0[h].copy()
            for s in range(t + 1):
                St = St @ A[s]
            for i in range(t + 1):
                W = beta[i, h] * np.outer(v[i, h], kh[i, h])
                for s in range(i + 1, t + 1):
                    W = W @ A[s]
                St = St + W
            np.testing.assert_allclose(out[t, h], scale * St @ qh[t, h], atol=1e-11, rtol=0)
            if t == T - 1:
                np.testing.assert_allclose(state[h], St, atol=1e-11, rtol=0)


def test_orthonormal_keys_is_gated_linear_attention():
    """Fresh orthonormal keys from a zero state: the erase term vanishes, so
    o_t = scale sum_{i<=t} exp(g_{i+1}+...+g_t) b_i v_i (k_i . q_t)."""
    D, H = 16, 1
    T = D
    basis, _ = np.linalg.qr(RNG.standard_normal((D, D)))
    k = (basis.T * RNG.uniform(0.5, 3.0, size=(D, 1)))[:, None, :]   # rows: scaled basis vectors
    q = RNG.standard_normal((T, H, D))
    v = RNG.standard_normal((T, H, D))
    g = -0.4 * RNG.random((T, H))
    beta = RNG.random((T, H))
    state = np.zeros((H, D, D))
    out = O.gdn_chunk(1.0, state, q, k, v, g, beta)
    kh, qh = _unit(k[:, 0]), _unit(q[:, 0])
    for t in range(T):
        ref = np.zeros(D)
        for i in range(t + 1):
            decay = np.exp(g[i + 1:t + 1, 0].sum())
            ref += decay * beta[i, 0] * v[i, 0] * (kh[i] @ qh[t])
        np.testing.assert_allclose(out[t, 0], ref, atol=1e-12, rtol=0)


def test_repeated_key_overwrites():
    """beta = 1, no decay: writing v1 then v2 under the same key leaves
    S = v2 k^T (the delta rule replaces; plain linear attention would add)."""
    D = 8
    k1 = RNG.standard_normal(D)
    v1, v2 = RNG.standard_normal(D), RNG.standard_normal(D)
    k = np.stack([k1, 2.5 * k1])[:, None, :]
    v = np.stack([v1, v2])[:, None, :]
    q = np.stack([k1, k1])[:, None, :]
    g = np.zeros((2, 1))
    beta = np.ones((2, 1))
    state = np.zeros((1, D, D))
    out = O.gdn_chunk(1.0, state, q, k, v, g, beta)
    kh = k1 / np.linalg.norm(k1)
    np.testing.assert_allclose(out[0, 0], v1, atol=1e-13)
    np.testing.assert_allclose(out[1, 0], v2, atol=1e-13)
    np.testing.assert_allclose(state[0], np.outer(v2, kh), atol=1e-13)


def test_zero_beta_is_pure_decay():
    T, H, D = 9, 2, 5
    q, k, v, g, _ = _rand(T, H, D)
    beta = np.zeros((T, H))
    S0 = RNG.standard_normal((H, D, D))
    state = S0.copy()
    out = O.gdn_chunk(0.5, state, q, k, v, g, beta)
    qh = _unit(q)
    for h in range(H):
        for t in range(T):
            ref = 0.5 * np.exp(g[:t + 1, h].sum()) * S0[h] @ qh[t, h]
            np.testing.assert_allclose(out[t, h], ref, atol=1e-13, rtol=0)
        np.testing.assert_allclose(state[h], np.exp(g[:, h].sum()) * S0[h], atol=1e-13)


def test_chunk_split_is_exact():
    """Carrying the state across calls equals one call over all tokens, bit for bit."""
    T, H, D = 30, 3, 8
    q, k, v, g, beta = _rand(T, H, D)
    s1 = np.zeros((H, D, D))
    o1 = O.gdn_chunk(0.3, s1, q, k, v, g, beta)
    s2 = np.zeros((H, D, D))
    parts = [O.gdn_chunk(0.3, s2, q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b])
             for a, b in ((0, 7), (7, 8), (8, 30))]
    assert np.array_equal(np.concatenate(parts), o1)
    assert np.array_equal(s1, s2)


def test_normalisation_and_zero_vectors():
    T, H, D = 12, 1, 6
    q, k, v, g, beta = _rand(T, H, D)
    s_a = np.zeros((H, D, D))
    o_a = O.gdn_chunk(1.0, s_a, q, k, v, g, beta)
    s_b = np.zeros((H, D, D))
    c = RNG.uniform(0.1, 9.0, size=(T, H, 1))
    o_b = O.gdn_chunk(1.0, s_b, q * c[::-1], k * c, v, g, beta)
    np.testing.assert_allclose(o_b, o_a, atol=1e-12)
    np.testing.assert_allclose(s_b, s_a, atol=1e-12)
    # a zero key writes nothing (only the decay acts); a zero query reads zero
    k0, q0 = k.copy(), q.copy()
    k0[5] = 0.0
    q0[5] = 0.0
    s_c = np.zeros((H, D, D))
    o_c = O.gdn_chunk(1.0, s_c, q0, k0, v, g, beta)
    s_ref = np.zeros((H, D, D))
    O.gdn_chunk(1.0, s_ref, q[:5], k[:5], v[:5], g[:5], beta[:5])
    s_ref *= np.exp(g[5, 0])
    s_after = np.zeros((H, D, D))
    O.gdn_chunk(1.0, s_after, q0[:6], k0[:6], v[:6], g[:6], beta[:6])
    np.testing.assert_allclose(s_after, s_ref, atol=1e-14)
    assert np.all(o_c[5] == 0.0)


def test_rotation_equivariance():
    """Rotating every query and key by an orthogonal M leaves the outputs
    unchanged and maps the state to S M^T (catches a transposed state)."""
    T, H, D = 15, 2, 7
    q, k, v, g, beta = _rand(T, H, D)
    M, _ = np.linalg.qr(RNG.standard_normal((D, D)))
    S0 = RNG.standard_normal((H, D, D))
    s_a = S0.copy()
    o_a = O.gdn_chunk(1.1, s_a, q, k, v, g, beta)
    s_b = S0 @ M.T
    o_b = O.gdn_chunk(1.1, s_b, q @ M.T, k @ M.T, v, g, beta)
    np.testing.assert_allclose(o_b, o_a, atol=1e-12)
    np.testing.assert_allclose(s_b, s_a @ M.T, atol=1e-12)


def test_generated_gates_and_stream_carry():
    w = Workload("gdn_tiny", B=1, H=2, D=16, fh=2, fw=3, C=2, S=1, W=2, n_chunks=3,
                 dtype="f32", rope_dims=(8, 4, 4))
    g, beta = fill_gates_host(w, 0, 3, 0.25)
    assert g.shape == beta.shape == (w.Lc, w.H)
    assert np.all(g < 0) and np.all(g > -0.25) and np.all(beta > 0) and np.all(beta < 1)
    g2, _ = fill_gates_host(w, 0, 3, 0.25)
    assert np.array_equal(g, g2)
    g3, _ = fill_gates_host(w, 1, 3, 0.25)
    assert not np.array_equal(g, g3)
    out2, st2 = O.gdn_stream(w, 0, 2, 0.25, 0.5)
    _, st1 = O.gdn_stream(w, 0, 1, 0.25, 0.5)
    out2b, st2b = O.gdn_stream(w, 0, 2, 0.25, 0.5, state=st1, c0=2)
    assert np.array_equal(out2, out2b) and np.array_equal(st2, st2b)
    o_h1, _ = O.gdn_stream(w, 0, 2, 0.25, 0.5, heads=[1])
    assert np.array_equal(o_h1[:, 0], out2[:, 1])


@pytest.mark.parametrize("bad", ["H", "state"])
def test_bad_arguments(bad):
    L = O.lib()
    st = np.zeros((1, 4, 4))
    x = np.zeros((1, 1, 4))
    gg = np.zeros((1, 1))
    H = 0 if bad == "H" else 1
    sp = None if bad == "state" else st.ctypes.data
    rc = L.orc_gdn_chunk(H, 4, 1, 1.0, sp, x.ctypes.data, x.ctypes.data, x.ctypes.data,
                         gg.ctypes.data, gg.ctypes.data, x.ctypes.data)
    assert rc == -1


def _tri_inv_blocked(L):
    """(I + L)^-1 for strictly lower-triangular L (64 x 64): 16 x 16 diagonal
    blocks by forward substitution, then two merges with
    [A 0; C B]^-1 = [A^-1 0; -B^-1 C A^-1  B^-1]."""
    n = L.shape[0]
    T = np.zeros_like(L)
    for b0 in range(0, n, 16):
        for j in range(16):
            x = np.zeros(16)
            x[j] = 1.0
            for t in range(j + 1, 16):
                x[t] = -L[b0 + t, b0:b0 + t] @ x[:t]
            T[b0:b0 + 16, b0 + j] = x
    for w in (16, 32):
        for b0 in range(0, n, 2 * w):
            T11 = T[b0:b0 + w, b0:b0 + w]
            T22 = T[b0 + w:b0 + 2 * w, b0 + w:b0 + 2 * w]
            T[b0 + w:b0 + 2 * w, b0:b0 + w] = -T22 @ (L[b0 + w:b0 + 2 * w, b0:b0 + w] @ T11)
    return T


def _chunkwise(scale, S, q, k, v, g, beta, ct=64):
    """The chunkwise (WY) form of the gated delta rule on sub-chunks of ct
    tokens, one head: (I + L) U = diag(beta)(V - diag(e^G) K S^T), outputs and
    end state by triangular products. Ragged tail rows are zero."""
    Tn, D = q.shape
    out = np.zeros_like(q)
    for t0 in range(0, Tn, ct):
        n = min(ct, Tn - t0)
        K = np.zeros((ct, D)); Q = np.zeros((ct, D)); V = np.zeros((ct, S.shape[0]))
        gg = np.zeros(ct); bb = np.zeros(ct)
        K[:n], Q[:n], V[:n] = _unit(k[t0:t0 + n]), _unit(q[t0:t0 + n]), v[t0:t0 + n]
        gg[:n], bb[:n] = g[t0:t0 + n], beta[t0:t0 + n]
        G = np.cumsum(gg)
        E = np.exp(G[:, None] - G[None, :])
        L = np.tril(bb[:, None] * E * (K @ K.T), -1)
        P = np.tril(scale * E * (Q @ K.T), 0)
        U = _tri_inv_blocked(L) @ (bb[:, None] * (V - np.exp(G)[:, None] * (K @ S.T)))
        out[t0:t0 + n] = (scale * np.exp(G)[:, None] * (Q @ S.T) + P @ U)[:n]
        S = np.exp(G[-1]) * S + (U * np.exp(G[-1] - G)[:, None]).T @ K
    return out, S


@pytest.mark.parametrize("T,D,g_scale", [(150, 16, 0.3), (64, 32, 0.01), (200, 8, 2.0),
                                         (130, 64, 0.002)])
def test_chunkwise_form_equals_recurrence(T, D, g_scale):
    """The algebra the GPU kernel runs (chunkwise WY form with a blocked
    triangular inverse, ragged last sub-chunk) reproduces the token-by-token
    recurrence of the oracle."""
    q, k, v, g, beta = _rand(T, 1, D, g_scale)
    S0 = 0.3 * RNG.standard_normal((1, D, D))
    st = S0.copy()
    ref = O.gdn_chunk(0.5, st, q, k, v, g, beta)
    o, S = _chunkwise(0.5, S0[0].copy(), q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0])
    np.testing.assert_allclose(o, ref[:, 0], atol=1e-12, rtol=0)
    np.testing.assert_allclose(S, st[0], atol=1e-12, rtol=0)
