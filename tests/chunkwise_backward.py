"""The gradients of one KDA unit in chunkwise form, numpy fp64 (a design check, not the library).

The prefill's chunkwise algebra ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram: per chunk,
O = (Gamma (.) Q) S + A V~, the state passed from chunk to chunk), per chunk of C tokens with
incoming state S0, b_r the chunk-local running sum of g, Gamma = e^b, Gamma_C its last row:
  Q^ = Gamma (.) scale q, K^ = Gamma (.) k, K~ = k / Gamma, K- = (Gamma_C / Gamma) (.) k
  L = strict_lower(diag(beta) K^ K~^T),  A = lower_incl(Q^ K~^T),  T' = (I + L)^-1 diag(beta)
  W = T' K^,  U~ = T' V,  U = U~ - W S0,  O = Q^ S0 + A U,  S_C = Diag(Gamma_C) S0 + K-^T U
is differentiated step by step, chunk by chunk in reverse: the state gradient is the only thing
carried between chunks (dS0 = Q^T dO + Diag(Gamma_C) dS_C - W^T dU, dU = A^T dO + K- dS_C); the
rest is chunk-local products, the derivative of the inverse (dL = -X^T dX X^T on the strict lower
triangle, X = (I + L)^-1), and a reverse running sum that takes the gradient of b to that of g.
Agreement with the token-by-token reverse-mode oracle (oracle/backward.py) to rounding checks the
algebra a chunkwise backward kernel would follow.  The forward here forms e^b and 1/e^b directly
(fp64, moderate decays); with pairwise=True the key and query gradients are formed as a kernel
would, every 1/e^b inside a pair e^{b_i - b_j} with i >= j (at most 1, so nothing overflows).
"""
import numpy as np


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def chunkwise_bwd(q, k, v, a, beta, A_log, dout, gate=None, S0=None, dS_T=None, scale=1.0, C=64, pairwise=False):
    """pairwise: form dq, dk and the gradient of b without any 1/e^b on its own, every such factor
    inside a pair E_ijc = e^{b_ic - b_jc} with i >= j (so E <= 1), as a kernel would."""
    q, k, v, a, dout = (np.asarray(x, np.float64) for x in (q, k, v, a, dout))
    beta = np.asarray(beta, np.float64)
    T, d_k = q.shape
    d_v = v.shape[1]
    eA = np.exp(A_log)
    x = eA * a
    g = -5.0 * _sig(x)
    S = np.zeros((d_k, d_v)) if S0 is None else np.array(S0, np.float64)

    # forward, chunk by chunk, keeping each chunk's operands and incoming state
    chunks = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        qc, kc, vc, bc = scale * q[sl], k[sl], v[sl], beta[sl]
        n = len(qc)
        b = np.cumsum(g[sl], axis=0)
        G = np.exp(b)
        GC = G[-1]
        Qh, Kh, Kt, Kb = qc * G, kc * G, kc / G, kc * (GC / G)
        M = Kh @ Kt.T
        L = bc[:, None] * np.tril(M, -1)
        A = np.tril(Qh @ Kt.T)
        X = np.linalg.inv(np.eye(n) + L)
        Tp = X * bc[None, :]
        W, Ut = Tp @ Kh, Tp @ vc
        U = Ut - W @ S
        O = Qh @ S + A @ U
        chunks.append(dict(sl=sl, vc=vc, bc=bc, b=b, G=G, GC=GC, Qh=Qh, Kh=Kh, Kt=Kt, Kb=Kb, M=M, A=A, X=X,
                           Tp=Tp, W=W, U=U, S0=S, O=O))
        S = GC[:, None] * S + Kb.T @ U

    O_all = np.concatenate([c["O"] for c in chunks]) if chunks else np.zeros((0, d_v))
    if gate is not None:
        sg = _sig(np.asarray(gate, np.float64))
        dgate = dout * O_all * sg * (1.0 - sg)
        dO_all = dout * sg
    else:
        dgate, dO_all = None, dout
    dq, dk, dv, dg = (np.zeros_like(t) for t in (q, k, v, g))
    dbeta = np.zeros(T)
    dS = np.zeros((d_k, d_v)) if dS_T is None else np.array(dS_T, np.float64)
    for c in reversed(chunks):
        sl, vc, bc, G, GC = c["sl"], c["vc"], c["bc"], c["G"], c["GC"]
        Qh, Kh, Kt, Kb, M, A, X, Tp, W, U, S0c = (c[key] for key in ("Qh", "Kh", "Kt", "Kb", "M", "A", "X", "Tp",
                                                                     "W", "U", "S0"))
        dO = dO_all[sl]
        # the state pass and the outputs
        dU = A.T @ dO + Kb @ dS
        dS0 = Qh.T @ dO + GC[:, None] * dS - W.T @ dU
        dQh = dO @ S0c.T
        dA = np.tril(dO @ U.T)
        dQh += dA @ Kt
        dKt = dA.T @ Qh
        dKb = U @ dS.T
        dGC = (dS * S0c).sum(axis=1)
        # U = U~ - W S0, W = T' K^, U~ = T' V, T' = X diag(beta), X = (I + L)^-1
        dW = -dU @ S0c.T
        dTp = dW @ Kh.T + dU @ vc.T
        dKh = Tp.T @ dW
        dv[sl] = Tp.T @ dU
        dX = dTp * bc[None, :]
        dbeta[sl] = (dTp * X).sum(axis=0)
        dL = np.tril(-X.T @ dX @ X.T, -1)
        # L = strict_lower(diag(beta) K^ K~^T)
        dbeta[sl] += (dL * M).sum(axis=1)
        dMm = bc[:, None] * dL
        dKh += dMm @ Kt
        dKt += dMm.T @ Kh
        # back to q, k and the running sum b of g
        if not pairwise:
            dq[sl] = scale * G * dQh
            db = dQh * Qh + dKh * Kh - dKt * Kt - dKb * Kb
            dk[sl] = G * dKh + dKt / G + (GC / G) * dKb
            db[-1] += (dKb * Kb).sum(axis=0) + dGC * GC
        else:
            kc, sq, b = k[sl], scale * q[sl], c["b"]
            n = len(b)
            incl = np.tril(np.ones((n, n), dtype=bool))
            E = np.where(incl[:, :, None], np.exp(np.where(incl[:, :, None], b[:, None, :] - b[None, :, :], 0.0)), 0.0)
            dAl, dMl = np.tril(dA), np.tril(dMm, -1)
            dq[sl] = scale * (G * (dO @ S0c.T) + np.einsum("ij,jc,ijc->ic", dAl, kc, E))
            P = G * (Tp.T @ dW) + np.einsum("ij,jc,ijc->ic", dMl, kc, E)
            Qs = np.einsum("ij,ic,ijc->jc", dAl, sq, E) + np.einsum("ij,ic,ijc->jc", dMl, kc, E)
            R = (GC / G) * dKb
            dk[sl] = P + Qs + R
            db = dq[sl] * q[sl] + (P - Qs - R) * kc
            db[-1] += (R * kc).sum(axis=0) + dGC * GC
        dg[sl] = np.cumsum(db[::-1], axis=0)[::-1]
        dS = dS0
    sx = _sig(x)
    dx = dg * (-5.0) * sx * (1.0 - sx)
    return dict(dq=dq, dk=dk, dv=dv, da=dx * eA, dbeta=dbeta, dgate=dgate, dA_log=float((dx * x).sum()), dS0=dS)
