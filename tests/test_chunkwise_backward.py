"""The chunkwise form of the backward (tests/chunkwise_backward.py) against the oracle's
token-by-token reverse-mode derivative (oracle/backward.py): the same gradients to rounding, for
several chunks with a ragged last one, with and without gate, initial state and final-state
gradient, and with chunk sizes that do or do not divide the sequence."""
import numpy as np
import pytest

from chunkwise_backward import chunkwise_bwd
from oracle.backward import recurrence_bwd


def _unit(seed, T, d_k=8, d_v=6, gate=True, S0=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, d_k)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = r.standard_normal((T, d_k)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    return dict(q=q, k=k, v=r.standard_normal((T, d_v)), a=r.standard_normal((T, d_k)),
                beta=1 / (1 + np.exp(-r.standard_normal(T))), A_log=0.2,
                dout=r.standard_normal((T, d_v)), gate=r.standard_normal((T, d_v)) if gate else None,
                S0=0.3 * r.standard_normal((d_k, d_v)) if S0 else None,
                dS_T=r.standard_normal((d_k, d_v)) if S0 else None)


@pytest.mark.parametrize("seed,T,C,gate,S0", [(0, 150, 64, True, True), (1, 64, 16, False, True),
                                             (2, 37, 16, True, False), (3, 100, 32, False, False)])
def test_chunkwise_gradients_match_the_token_level_oracle(seed, T, C, gate, S0):
    x = _unit(seed, T, gate=gate, S0=S0)
    args = (x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"], x["dout"])
    kw = dict(gate=x["gate"], S0=x["S0"], dS_T=x["dS_T"], scale=0.7)
    ref = recurrence_bwd(*args, **kw)
    got = chunkwise_bwd(*args, C=C, **kw)
    for key in ("dq", "dk", "dv", "da", "dbeta", "dgate", "dS0"):
        if ref[key] is None:
            assert got[key] is None
            continue
        err = np.abs(got[key] - ref[key]).max() / max(np.abs(ref[key]).max(), 1e-30)
        assert err <= 1e-9, f"{key}: relative max error {err:.2e}"
    assert abs(got["dA_log"] - ref["dA_log"]) <= 1e-9 * max(abs(ref["dA_log"]), 1.0)


@pytest.mark.parametrize("seed,T,C", [(4, 150, 64), (5, 40, 16)])
def test_overflow_free_pairwise_form_gives_the_same_gradients(seed, T, C):
    # the form a kernel would use (no 1/e^b outside a pair e^{b_i - b_j}, i >= j) against the direct one
    x = _unit(seed, T)
    args = (x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"], x["dout"])
    kw = dict(gate=x["gate"], S0=x["S0"], dS_T=x["dS_T"], scale=0.7, C=C)
    direct = chunkwise_bwd(*args, **kw)
    pair = chunkwise_bwd(*args, pairwise=True, **kw)
    for key in ("dq", "dk", "da", "dbeta", "dS0"):
        err = np.abs(pair[key] - direct[key]).max() / max(np.abs(direct[key]).max(), 1e-30)
        assert err <= 1e-10, f"{key}: relative max error {err:.2e}"
