"""fp64 restatements of the chunked (UT/WY) form of the delta rule, used to pin
the token-by-token oracle to an independent derivation.

Both functions are derived here from the recurrence, not taken from any
listing; they share no code with the oracle or with the CUDA library.

Ungated form ("DeltaNet, or Parallelizing Linear Transformers with Delta
Rule" section of "22580: from GPT-2 to Kimi K3, explained", Householder
reparameterisation and chunk-wise parallel form): inside a chunk of C tokens
the deltas satisfy (I + tril_-1(diag(beta) K K^T)) D = diag(beta)(V - K S0),
so with X = (I + tril_-1(diag(beta) K K^T))^-1, W = X diag(beta) K and
U = X diag(beta) V one gets D = U - W S0, O = Q S0 + tril(Q K^T) D and
S1 = S0 + K^T D.

Gated (per-channel) form, derived for the KDA step
S_t = (I - b k k^T) Diag(a_t) S_{t-1} + b k v^T: with g_r the within-chunk
cumulative sum of log_alpha (per key channel),
    M_kk[r, j] = sum_c k_rc k_jc exp(g_rc - g_jc)   (j < r)
    M_qk[r, j] = sum_c q_rc k_jc exp(g_rc - g_jc)   (j <= r)
    X = (I + diag(beta) M_kk)^-1,  W = X diag(beta) (K * exp(g)),
    U = X diag(beta) V,
    D = U - W S0,  O = (Q * exp(g)) S0 + M_qk D,
    S1 = Diag(exp(g_last)) S0 + (K * exp(g_last - g))^T D.
The Gram matrices are evaluated through the same sub-chunk factorisation the
GPU kernel uses (left factor x_r exp(g_r - m_a), right factor
k_j exp(m_a - g_j), with m_a the midpoint of sub-chunk a's cumulative gate),
so the factorisation itself is pinned in fp64 before any kernel exists.
"""
import numpy as np


def chunk_delta_ungated(q, k, v, beta, C, S0=None):
    """One head, alpha == 1. q, k: [T, dk]; v: [T, dv]; beta: [T]."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.astype(np.float64).copy()
    O = np.zeros((T, dv))
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        Q, K, V, b = q[sl], k[sl], v[sl], beta[sl]
        L = K.shape[0]
        N = np.tril(b[:, None] * (K @ K.T), -1)
        X = np.linalg.inv(np.eye(L) + N)
        W = X @ (b[:, None] * K)
        U = X @ (b[:, None] * V)
        D = U - W @ S
        O[sl] = Q @ S + np.tril(Q @ K.T) @ D
        S = S + K.T @ D
    return O, S


def _gram_subchunk(x, k, g, sub):
    """sum_c x_rc k_jc exp(g_rc - g_jc) for j <= r, via sub-chunk references.

    Diagonal sub-blocks use the sub-chunk's own midpoint m_a on both sides;
    an off-diagonal block (row sub-chunk a > column sub-chunk b) uses m_a, the
    row sub-chunk's midpoint, which lies after every column position, so the
    right factor exp(m_a - g_j) is at most 1. Entries with j > r are zero.
    """
    L = k.shape[0]
    out = np.zeros((L, L))
    n_sub = (L + sub - 1) // sub
    mids = []
    for a in range(n_sub):
        s, e = a * sub, min(L, (a + 1) * sub) - 1
        mids.append(0.5 * (g[s] + g[e]))
    for r in range(L):
        a = r // sub
        left = x[r] * np.exp(g[r] - mids[a])
        for j in range(r + 1):
            right = k[j] * np.exp(mids[a] - g[j])
            out[r, j] = left @ right
    return out


def chunk_kda_gated(q, k, v, log_alpha, beta, C, S0=None, sub=16):
    """One head, per-channel gate. q, k, log_alpha: [T, dk]; v: [T, dv];
    beta: [T]. Returns (O [T, dv], final S [dk, dv])."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.astype(np.float64).copy()
    O = np.zeros((T, dv))
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        Q, K, V, b, lam = q[sl], k[sl], v[sl], beta[sl], log_alpha[sl]
        L = K.shape[0]
        g = np.cumsum(lam, axis=0)
        Mkk = np.tril(_gram_subchunk(K, K, g, sub), -1)
        Mqk = _gram_subchunk(Q, K, g, sub)
        X = np.linalg.inv(np.eye(L) + b[:, None] * Mkk)
        W = X @ (b[:, None] * (K * np.exp(g)))
        U = X @ (b[:, None] * V)
        D = U - W @ S
        O[sl] = (Q * np.exp(g)) @ S + Mqk @ D
        S = np.exp(g[-1])[:, None] * S + (K * np.exp(g[-1] - g)).T @ D
    return O, S


def block_unit_lower_inverse(N, blk=16):
    """(I + N)^-1 for strictly lower-triangular N by block forward
    substitution: invert each diagonal block by substitution, then
    X_ab = -X_aa sum_{b <= c < a} N_ac X_cb, row block by row block."""
    L = N.shape[0]
    nb = (L + blk - 1) // blk
    X = np.zeros((L, L))
    sl = [slice(i * blk, min(L, (i + 1) * blk)) for i in range(nb)]
    for a in range(nb):
        A = np.eye(sl[a].stop - sl[a].start) + N[sl[a], sl[a]]
        Xa = np.zeros_like(A)
        n = A.shape[0]
        for col in range(n):  # forward substitution, one column at a time
            e = np.zeros(n)
            e[col] = 1.0
            x = np.zeros(n)
            for r in range(n):
                x[r] = e[r] - A[r, :r] @ x[:r]
            Xa[:, col] = x
        X[sl[a], sl[a]] = Xa
        for bb in range(a):
            acc = np.zeros((sl[a].stop - sl[a].start, sl[bb].stop - sl[bb].start))
            for c in range(bb, a):
                acc += N[sl[a], sl[c]] @ X[sl[c], sl[bb]]
            X[sl[a], sl[bb]] = -Xa @ acc
    return X
