"""Pins of the oracle's backward pass (oracle/backward.py) against central finite differences of the
forward oracle (the C recurrence), which shares no code with it.  The scalar checked is
L = sum(dout * out) + sum(dS_T * S_T), so every gradient is a directional derivative of L."""
import numpy as np
import pytest

import oracle
from oracle.backward import recurrence_bwd


def _inputs(seed, T=6, d_k=4, d_v=3, gate=True, S0=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, d_k)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = r.standard_normal((T, d_k)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    return dict(q=q, k=k, v=r.standard_normal((T, d_v)), a=r.standard_normal((T, d_k)),
                beta=1 / (1 + np.exp(-r.standard_normal(T))), A_log=0.3,
                gate=r.standard_normal((T, d_v)) if gate else None,
                S0=0.5 * r.standard_normal((d_k, d_v)) if S0 else None,
                dout=r.standard_normal((T, d_v)), dS_T=r.standard_normal((d_k, d_v)), scale=0.8)


def _loss(x):
    g = oracle.gate_log_decay(x["a"], x["A_log"])
    out, S = oracle.recurrence_g(x["q"], x["k"], x["v"], g, x["beta"], gate=x["gate"], S0=x["S0"],
                                 scale=x["scale"])
    return float((x["dout"] * out).sum() + (x["dS_T"] * S).sum())


def _fd(x, key, eps=1e-6):
    base = x[key]
    if np.isscalar(base) or np.ndim(base) == 0:
        xp, xm = dict(x), dict(x)
        xp[key], xm[key] = base + eps, base - eps
        return (_loss(xp) - _loss(xm)) / (2 * eps)
    grad = np.zeros_like(base, dtype=np.float64)
    for idx in np.ndindex(base.shape):
        xp, xm = dict(x), dict(x)
        xp[key], xm[key] = base.copy(), base.copy()
        xp[key][idx] += eps
        xm[key][idx] -= eps
        grad[idx] = (_loss(xp) - _loss(xm)) / (2 * eps)
    return grad


@pytest.mark.parametrize("seed,gate,S0", [(0, True, True), (1, False, True), (2, True, False)])
def test_gradients_match_finite_differences(seed, gate, S0):
    x = _inputs(seed, gate=gate, S0=S0)
    g = recurrence_bwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"], x["dout"], gate=x["gate"],
                       S0=x["S0"], dS_T=x["dS_T"], scale=x["scale"])
    pairs = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("a", "da"), ("beta", "dbeta"), ("A_log", "dA_log")]
    if gate:
        pairs.append(("gate", "dgate"))
    if S0:
        pairs.append(("S0", "dS0"))
    for key, gkey in pairs:
        fd = _fd(x, key)
        assert np.allclose(g[gkey], fd, rtol=1e-5, atol=1e-7), f"{gkey}: max err {np.abs(g[gkey] - fd).max():.2e}"


def test_zero_upstream_gradient_gives_zero():
    x = _inputs(3)
    g = recurrence_bwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"], np.zeros_like(x["dout"]),
                       gate=x["gate"], S0=x["S0"], dS_T=None)
    for key in ("dq", "dk", "dv", "da", "dbeta", "dgate", "dS0"):
        assert np.all(g[key] == 0.0)
