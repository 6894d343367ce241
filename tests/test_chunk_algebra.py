"""The chunked form the tensor-core kernel evaluates, written out in fp64 numpy from the
derivation in its header, reaches the plain recurrence of the oracle exactly (up to fp64
rounding): per 64-token chunk with start state S_0, decay products g, the scaled operands
KKd, Rd, Bi, Ki, the masked Grams M_ab, M_kb, Q_b, Q_k, A = (I + M_ab)^-1 and
    [S_C^T; Y] = [P; R~] S_0^T + [K~; Q~] V,
    P = diag(gC)(I - Bi^T A KKd), R~ = Rd - Q_b A KKd,
    K~ = diag(gC)(Ki^T - Bi^T A M_kb), Q~ = Q_k - Q_b A M_kb.
CPU only: this checks the algebra, the GPU parity tests check the kernel."""
import numpy as np
import pytest

from oracle import reference


def _chunk(S0, r, w, k, v, kk, a):
    """One chunk of L tokens for one head: returns (Y [L, N], S_C [N, N])."""
    L, N = r.shape
    g = np.cumprod(w, axis=0)                                   # g_t = prod_{s<=t} w_s
    g_prev = np.vstack([np.ones((1, N)), g[:-1]])               # g_{t-1}
    gC = g[-1]
    b = kk * a
    KKd, Rd, Bi, Ki = kk * g_prev, r * g, b / g, k / g
    M_ab = np.tril(KKd @ Bi.T, -1)
    M_kb = np.tril(KKd @ Ki.T, -1)
    Q_b = np.tril(Rd @ Bi.T)
    Q_k = np.tril(Rd @ Ki.T)
    A = np.linalg.inv(np.eye(L) + M_ab)
    P = gC[:, None] * (np.eye(N) - Bi.T @ A @ KKd)
    Rt = Rd - Q_b @ A @ KKd
    Kt = gC[:, None] * (Ki.T - Bi.T @ A @ M_kb)
    Qt = Q_k - Q_b @ A @ M_kb
    SCt = P @ S0.T + Kt @ v
    Y = Rt @ S0.T + Qt @ v
    return Y, SCt.T


@pytest.mark.parametrize("T", [1, 7, 64, 150, 257])
def test_chunked_form_reaches_the_recurrence(T):
    rng = np.random.default_rng(60 + T)
    B, H, N, C = 1, 2, 16, 64
    r, k, v = (rng.standard_normal((B, T, H, N)) for _ in range(3))
    w = rng.uniform(0.55, 1.0, (B, T, H, N))
    a = rng.uniform(0.0, 1.0, (B, T, H, N))
    kk = rng.standard_normal((B, T, H, N))
    kk /= np.linalg.norm(kk, axis=-1, keepdims=True)
    S0 = rng.standard_normal((B, H, N, N))
    y_ref, S_ref, _ = reference.wkv7_recurrence(r, w, k, v, kk, a, S0)
    for h in range(H):
        S = S0[0, h]
        ys = []
        for c0 in range(0, T, C):
            sl = slice(c0, min(T, c0 + C))
            Y, S = _chunk(S, *(x[0, sl, h] for x in (r, w, k, v, kk, a)))
            ys.append(Y)
        np.testing.assert_allclose(np.vstack(ys), y_ref[0, :, h], rtol=0, atol=1e-9)
        np.testing.assert_allclose(S, S_ref[0, h], rtol=0, atol=1e-9)


def test_removed_values_solve_the_unit_triangular_system():
    """U = A(-KKd S_0^T - M_kb V) holds the removed values u_t = -S_{t-1} kk_t."""
    rng = np.random.default_rng(70)
    L, N = 20, 8
    r, k, v = (rng.standard_normal((L, N)) for _ in range(3))
    w = rng.uniform(0.55, 1.0, (L, N))
    a = rng.uniform(0.0, 1.0, (L, N))
    kk = rng.standard_normal((L, N))
    kk /= np.linalg.norm(kk, axis=-1, keepdims=True)
    S0 = rng.standard_normal((N, N))
    g = np.cumprod(w, axis=0)
    g_prev = np.vstack([np.ones((1, N)), g[:-1]])
    KKd, Ki, Bi = kk * g_prev, k / g, kk * a / g
    M_ab, M_kb = np.tril(KKd @ Bi.T, -1), np.tril(KKd @ Ki.T, -1)
    U = np.linalg.solve(np.eye(L) + M_ab, -KKd @ S0.T - M_kb @ v)
    _, _, snaps = reference.wkv7_recurrence(*(x[None, :, None] for x in (r, w, k, v, kk, a)), S0[None, None],
                                            snap_every=1)
    states = np.concatenate([S0[None], snaps[0, :, 0]], axis=0)     # S_0 .. S_L
    u_ref = -np.einsum("tij,tj->ti", states[:-1], kk)
    np.testing.assert_allclose(U, u_ref, rtol=0, atol=1e-10)
