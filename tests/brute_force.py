"""Brute-force O(T^2) parallel form of one KDA unit, in numpy fp64.

This is the chunkwise output equation of "Kimi K3 · Lesson 3 of 14" (the CHUNKWISE diagram:
O = (Gamma (.) Q) S + A V~) taken with a single chunk that spans the whole sequence, evaluated
with exp(b_i - b_j) formed directly (no tiling, no 1/Gamma rescale).  It is a different algorithm
from the token-by-token recurrence of the oracle, so agreement between the two pins both.

Derivation (per unit, state S0 incoming, b_t = sum_{s<=t} g_s per key channel):
  unrolling the recurrence gives S_t = Diag(e^{b_t}) S0 + sum_{j<=t} Diag(e^{b_t - b_j}) k_j u_j^T
  with u_t = beta_t (v_t - (Diag(e^{g_t}) S_{t-1})^T k_t).  Substituting S_{t-1} shows
  (I + L) U = diag(beta) (V - K^ S0),   L_tj = beta_t sum_c k_tc k_jc e^{b_tc - b_jc} (j < t),
  and o_t = S_t^T q_t = S0^T (e^{b_t} (.) q_t) + sum_{j<=t} (sum_c q_tc k_jc e^{b_tc - b_jc}) u_j.
"""
import numpy as np


def parallel_form(q, k, v, g, beta, gate=None, S0=None, scale=1.0):
    q = np.asarray(q, np.float64) * scale
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    T, d_k = q.shape
    d_v = v.shape[1]
    S0 = np.zeros((d_k, d_v)) if S0 is None else np.asarray(S0, np.float64)
    b = np.cumsum(g, axis=0)                                  # [T, d_k]
    diff = b[:, None, :] - b[None, :, :]                      # [t, j, c] = b_t - b_j
    causal = np.tril(np.ones((T, T), dtype=bool))             # j <= t
    decay = np.where(causal[:, :, None], np.exp(np.where(causal[:, :, None], diff, 0.0)), 0.0)
    Gkk = np.einsum("tc,jc,tjc->tj", k, k, decay)
    Gqk = np.einsum("tc,jc,tjc->tj", q, k, decay)
    L = beta[:, None] * np.tril(Gkk, -1)
    Khat = k * np.exp(b)
    rhs = beta[:, None] * (v - Khat @ S0)
    U = np.linalg.solve(np.eye(T) + L, rhs)
    O = (q * np.exp(b)) @ S0 + Gqk @ U                        # Gqk already causal (incl. diagonal)
    Kbar = k * np.exp(b[-1][None, :] - b)                     # decay from token j to the end
    S_T = np.exp(b[-1])[:, None] * S0 + Kbar.T @ U
    if gate is not None:
        O = O / (1.0 + np.exp(-np.asarray(gate, np.float64)))
    return O, S_T
