"""fp64 oracle of the KDA module pieces around the recurrence: short convolution and pre-gate
normalisation with the output gate.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the test suite and the reference arm of
``bench.py`` may import it; the library never does, and they share no code.

The pages name these pieces without giving their form ("K3 Architecture Illustrated", FIG 21: the
actual KDA module also includes short convolution, normalisation and output gating; §"Why can K3's
MLA use NoPE?": short convolution depends on input order).  The definitions below are the
plainest readings, written out element by element (pure Python loops over tokens; numpy only for
the per-row vectors):

  short convolution  y_t[h][c] = sum_{j < W} w[h][c][j] * x_{t-(W-1)+j}[h][c], with x = 0 before the
                     start of the token's own sequence; optionally y_t[h] / sqrt(|y_t[h]|^2 + 1e-12)
  norm + gate        out_t[h][c] = sigmoid(gate_t[h][c]) * o_t[h][c] / sqrt(mean_c o_t[h]^2 + eps) * w[c]
"""
from __future__ import annotations

import numpy as np


def short_conv(x, w, cu_seqlens, l2norm: bool = False) -> np.ndarray:
    """x [T, H, d], w [H, d, W], cu_seqlens [N + 1] -> y [T, H, d] (fp64)."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    T, H, d = x.shape
    W = w.shape[-1]
    cu = [int(c) for c in cu_seqlens]
    y = np.zeros((T, H, d))
    for n in range(len(cu) - 1):
        start, end = cu[n], cu[n + 1]
        for t in range(start, end):
            acc = np.zeros((H, d))
            for j in range(W):
                src = t - (W - 1) + j
                if src >= start:
                    acc += w[:, :, j] * x[src]
            if l2norm:
                acc = acc / np.sqrt((acc * acc).sum(axis=-1, keepdims=True) + 1e-12)
            y[t] = acc
    return y


def output_norm_gate(o, gate, w, eps: float = 1e-6) -> np.ndarray:
    """o [T, H, d_v], gate [T, H, d_v] or None, w [d_v] -> out [T, H, d_v] (fp64)."""
    o = np.asarray(o, np.float64)
    w = np.asarray(w, np.float64)
    out = np.zeros_like(o)
    for t in range(o.shape[0]):
        for h in range(o.shape[1]):
            row = o[t, h]
            y = row / np.sqrt(np.mean(row * row) + eps) * w
            if gate is not None:
                y = y / (1.0 + np.exp(-np.asarray(gate[t, h], np.float64)))
            out[t, h] = y
    return out
