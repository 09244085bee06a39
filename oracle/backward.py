"""fp64 oracle of the backward pass (gradients) of the KDA recurrence, one (sequence, head) unit.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the test suite and the reference arm of
``bench.py`` may import it; the library never does, and they share no code.

The pages describe only the forward recurrence ("Review A · Sequence and depth", Free recall: fade,
erase, write, read; "Kimi K3 · Lesson 3 of 14", eq. 5 passage: g = -5 sigmoid(e^A a); the sigmoid
output gate).  Its gradient is the plain reverse-mode derivative of that token-by-token recurrence:
the forward pass is run and every state kept, then the steps are undone in reverse order, each by
the chain rule (pure Python loop over tokens, numpy for the per-token vectors and matrices).

Forward, per token t (S is d_k x d_v, rows = key channels):
  x = e^A a_t,  g = -5 sigmoid(x),  alpha = e^g
  S' = Diag(alpha) S_{t-1};  u = beta_t (v_t - S'^T k_t);  S_t = S' + k_t u^T
  o = S_t^T (scale q_t);  out_t = sigmoid(gate_t) * o
Backward, given dout_t for every t and dS_T for the final state: the transposes of those steps.
"""
from __future__ import annotations

import numpy as np


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def recurrence_bwd(q, k, v, a, beta, A_log: float, dout, gate=None, S0=None, dS_T=None, scale: float = 1.0):
    """Returns a dict of fp64 gradients: dq, dk, dv, da [T, d], dbeta [T], dgate [T, d_v] (or None),
    dA_log (scalar), dS0 [d_k, d_v]."""
    q, k, v, a, dout = (np.asarray(x, np.float64) for x in (q, k, v, a, dout))
    beta = np.asarray(beta, np.float64)
    T, d_k = q.shape
    d_v = v.shape[1]
    eA = np.exp(A_log)
    S = np.zeros((d_k, d_v)) if S0 is None else np.array(S0, np.float64)
    states, alphas, us, os_ = [S.copy()], [], [], []
    for t in range(T):                                   # forward, keeping every state
        alpha = np.exp(-5.0 * _sig(eA * a[t]))
        Sp = alpha[:, None] * S
        u = beta[t] * (v[t] - Sp.T @ k[t])
        S = Sp + np.outer(k[t], u)
        alphas.append(alpha)
        us.append(u)
        os_.append(S.T @ (scale * q[t]))
        states.append(S.copy())
    dq, dk, dv, da = (np.zeros_like(x) for x in (q, k, v, a))
    dbeta = np.zeros(T)
    dgate = None if gate is None else np.zeros((T, d_v))
    dA_log = 0.0
    dS = np.zeros((d_k, d_v)) if dS_T is None else np.array(dS_T, np.float64)
    for t in range(T - 1, -1, -1):                       # reverse
        S_prev, S_t, alpha, u, o = states[t], states[t + 1], alphas[t], us[t], os_[t]
        if gate is not None:
            sg = _sig(np.asarray(gate[t], np.float64))
            dgate[t] = dout[t] * o * sg * (1.0 - sg)
            do = dout[t] * sg
        else:
            do = dout[t]
        # o = S_t^T (scale q)
        dq[t] = scale * (S_t @ do)
        dS = dS + np.outer(scale * q[t], do)
        # S_t = S' + k u^T
        du = dS.T @ k[t]
        dk[t] = dS @ u
        dSp = dS.copy()
        # u = beta (v - S'^T k)
        Sp = alpha[:, None] * S_prev
        r = Sp.T @ k[t]
        dbeta[t] = du @ (v[t] - r)
        dv[t] = beta[t] * du
        dr = -beta[t] * du
        dSp += np.outer(k[t], dr)
        dk[t] += Sp @ dr
        # S' = Diag(alpha) S_prev
        dalpha = (dSp * S_prev).sum(axis=1)
        dS = alpha[:, None] * dSp
        # alpha = e^g, g = -5 sigmoid(x), x = e^A a
        dg = dalpha * alpha
        x = eA * a[t]
        sx = _sig(x)
        dx = dg * (-5.0) * sx * (1.0 - sx)
        da[t] = dx * eA
        dA_log += float(dx @ x)
    return dict(dq=dq, dk=dk, dv=dv, da=da, dbeta=dbeta, dgate=dgate, dA_log=dA_log, dS0=dS)
