"""Naive chunkwise form of the KDA recurrence, fp64 NumPy -- TEST INFRASTRUCTURE ONLY.

A second witness for the oracle.  It restates the token recurrence of "Kimi K3:
Architecture, Training, and Million-Token Agentic RL" (sections 3.1-3.2) as
whole-chunk matrix products, the form that section 3.3 says chunked prefill
uses (tokens inside a chunk become matrix operations, the state crosses only
chunk boundaries: (X_[c], S_in[c]) -> (Y_[c], S_out[c]), S_in[c+1] = S_out[c]).
The note defers the derivation to a companion note that is not available, so
it is derived here from the recurrence itself:

Inside one chunk of tokens r = 1..C with incoming state S0, let
G_r = g_1 + ... + g_r (per key channel; inclusive, because alpha_r decays the
state before token r edits it).  Unrolling the edit-order step gives

  S_r      = Diag(e^{G_r}) S0 + sum_{s<=r} Diag(e^{G_r - G_s}) k_s d_s^T
  d_r      = beta_r (v_r - Sbar_r^T k_r)
           = beta_r (v_r - S0^T (k_r e^{G_r})
                      - sum_{s<r} <k_r e^{G_r}, k_s e^{-G_s}> d_s)

so with Kt = K*e^{G}, Kh = K*e^{-G}, Qt = Q*e^{G} (row r scaled by e^{G_r}):

  (I + A) D = Diag(beta) (V - Kt S0),   A = strictly_lower(Diag(beta) Kt Kh^T)
  D        = U - W S0,  U = T Diag(beta) V,  W = T Diag(beta) Kt,  T = (I + A)^-1
  O        = Qt S0 + lower_incl_diag(Qt Kh^T) D          (read after write)
  S_out    = Diag(e^{G_C}) S0 + (K * e^{G_C - G})^T D

Library primitives used: matrix products and ``np.linalg.inv``.  In fp64 the
e^{-G} factors stay finite for chunks up to about 140 tokens (G >= -5 per token).

With an unbounded gate (the negative Softplus of the earlier Kimi Linear design,
which the pages contrast with K3's lower bound) e^{-G} overflows inside a chunk.
``chunk_step_pairwise`` is then the position-pair form: every A and P entry takes
its decay e^{G_r - G_s} (s <= r, never above 1) as one exponent per pair and key
channel, and every other factor (e^{G}, e^{G_C - G}) is at most 1 -- the same
unrolled recurrence, with no reciprocal decay anywhere.
"""
from __future__ import annotations

import numpy as np

G_MIN = -5.0


def _gate(z: np.ndarray, A: np.ndarray, kind: str = "bounded") -> np.ndarray:
    """g = g_min * sigmoid(exp(A) * z), section 3.3 gate equation (one head);
    kind="softplus": g = -log(1 + exp(exp(A) * z))."""
    x = np.exp(A) * z
    if kind == "softplus":
        return -np.logaddexp(0.0, x)
    return G_MIN / (1.0 + np.exp(-x))


def chunk_step_pairwise(q, k, v, g, beta, S0):
    """``chunk_step`` with the intra-chunk decays taken pair by pair.

    A[r,s] = beta_r sum_c k_rc k_sc e^{G_rc - G_sc} (s < r) and
    P[r,s] = sum_c q_rc k_sc e^{G_rc - G_sc} (s <= r); the rest as in chunk_step.
    """
    C = q.shape[0]
    G = np.cumsum(g, axis=0)
    lower = np.tril(np.ones((C, C), dtype=bool))          # s <= r
    expo = np.where(lower[:, :, None], G[:, None, :] - G[None, :, :], -np.inf)
    E = np.exp(expo)                                      # [r, s, c], entries in [0, 1]
    A = np.tril(beta[:, None] * np.einsum("rc,sc,rsc->rs", k, k, E), -1)
    P = np.einsum("rc,sc,rsc->rs", q, k, E)
    Kt, Qt = k * np.exp(G), q * np.exp(G)
    Tinv = np.linalg.inv(np.eye(C) + A)
    W = Tinv @ (beta[:, None] * Kt)
    U = Tinv @ (beta[:, None] * v)
    D = U - W @ S0
    O = Qt @ S0 + P @ D
    S_out = np.exp(G[-1])[:, None] * S0 + (k * np.exp(G[-1] - G)).T @ D
    return O, S_out


def chunk_step(q, k, v, g, beta, S0):
    """One chunk for one head: q, k, g [C,dk]; v [C,dv]; beta [C]; S0 [dk,dv].

    Returns ``(O [C,dv], S_out [dk,dv])``.
    """
    C = q.shape[0]
    G = np.cumsum(g, axis=0)
    Kt, Kh, Qt = k * np.exp(G), k * np.exp(-G), q * np.exp(G)
    A = np.tril(beta[:, None] * (Kt @ Kh.T), -1)
    Tinv = np.linalg.inv(np.eye(C) + A)
    W = Tinv @ (beta[:, None] * Kt)
    U = Tinv @ (beta[:, None] * v)
    D = U - W @ S0
    O = Qt @ S0 + np.tril(Qt @ Kh.T) @ D
    S_out = np.exp(G[-1])[:, None] * S0 + (k * np.exp(G[-1] - G)).T @ D
    return O, S_out


def prefill(q, k, v, z, A, beta, cu_seqlens, initial_state=None, chunk: int = 16,
            gate: str = "bounded", pairwise: bool = False):
    """Chunkwise prefill with chunks aligned to each sequence start.

    Same shapes and result as ``oracle.prefill``; every argument is a float64
    (or int for cu_seqlens) NumPy array.  ``pairwise`` uses chunk_step_pairwise.
    """
    q, k, v, z, A, beta = (np.asarray(t, dtype=np.float64) for t in (q, k, v, z, A, beta))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, H, dk = q.shape
    dv = v.shape[2]
    n = cu.shape[0] - 1
    o = np.zeros((T, H, dv))
    sf = np.zeros((n, H, dk, dv))
    for i in range(n):
        for h in range(H):
            S = (np.zeros((dk, dv)) if initial_state is None
                 else np.asarray(initial_state[i, h], dtype=np.float64).copy())
            for c0 in range(int(cu[i]), int(cu[i + 1]), chunk):
                c1 = min(c0 + chunk, int(cu[i + 1]))
                g = _gate(z[c0:c1, h], A[h], gate)
                step = chunk_step_pairwise if pairwise else chunk_step
                O, S = step(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], g, beta[c0:c1, h], S)
                o[c0:c1, h] = O
            sf[i, h] = S
    return o, sf


def chunk_intermediates(q, k, v, g, beta, S0):
    """The stage values of ``chunk_step`` for one chunk of one head: G [C,dk], the
    strictly lower A [C,C], W = T Diag(beta) Kt [C,dk], U = T Diag(beta) V [C,dv],
    D = U - W S0 [C,dv] (the state-independent part of the update), O, S_out."""
    C = q.shape[0]
    G = np.cumsum(g, axis=0)
    Kt, Kh, Qt = k * np.exp(G), k * np.exp(-G), q * np.exp(G)
    A = np.tril(beta[:, None] * (Kt @ Kh.T), -1)
    Tinv = np.linalg.inv(np.eye(C) + A)
    W = Tinv @ (beta[:, None] * Kt)
    U = Tinv @ (beta[:, None] * v)
    D = U - W @ S0
    O = Qt @ S0 + np.tril(Qt @ Kh.T) @ D
    S_out = np.exp(G[-1])[:, None] * S0 + (k * np.exp(G[-1] - G)).T @ D
    return dict(G=G, A=A, W=W, U=U, D=D, O=O, S_out=S_out)


def prefill_intermediates(q, k, v, z, A, beta, cu_seqlens, initial_state=None, chunk: int = 64):
    """Per-token stage values over packed sequences, chunks aligned to each
    sequence start: G, W [T,H,dk]; U, D [T,H,dv]; plus o and the final states."""
    q, k, v, z, A, beta = (np.asarray(t, dtype=np.float64) for t in (q, k, v, z, A, beta))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, H, dk = q.shape
    dv = v.shape[2]
    n = cu.shape[0] - 1
    out = dict(G=np.zeros((T, H, dk)), W=np.zeros((T, H, dk)), U=np.zeros((T, H, dv)),
               D=np.zeros((T, H, dv)), o=np.zeros((T, H, dv)), final_state=np.zeros((n, H, dk, dv)))
    for i in range(n):
        for h in range(H):
            S = (np.zeros((dk, dv)) if initial_state is None
                 else np.asarray(initial_state[i, h], dtype=np.float64).copy())
            for c0 in range(int(cu[i]), int(cu[i + 1]), chunk):
                c1 = min(c0 + chunk, int(cu[i + 1]))
                r = chunk_intermediates(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], _gate(z[c0:c1, h], A[h]),
                                        beta[c0:c1, h], S)
                for key in ("G", "W", "U", "D"):
                    out[key][c0:c1, h] = r[key]
                out["o"][c0:c1, h] = r["O"]
                S = r["S_out"]
            out["final_state"][i, h] = S
    return out
