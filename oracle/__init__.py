"""fp64 CPU oracle of the KDA gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY.  This package is the reference that the CUDA path is checked against.
Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  The library path (``kda_chunkwise_b200``) never imports, links or calls anything
here, and the two share no code.

The arithmetic lives in ``kda_oracle.c`` (plain C, double precision, token by token); this module
only compiles it with gcc and marshals numpy arrays to it.

Definition (per sequence n, head h; state S is d_k x d_v, row = key channel):
  g_t = -5 * sigmoid(exp(A_h) * a_t)                   "Kimi K3 · Lesson 3 of 14", eq. 5 passage
  S <- Diag(exp(g_t)) S ; r = S^T k_t                  "Review A · Sequence and depth", Free recall
  S <- S + beta_t k_t (v_t - r)^T                      "K3 Architecture Illustrated", FIG 21
  o_t = S^T (scale q_t) ; out_t = sigmoid(gate_t) * o_t "Kimi K3 · Lesson 3 of 14", output gate
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

G_MIN = -5.0  # fixed floor of the log-decay ("Kimi K3 · Lesson 3 of 14", eq. 5 passage)


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into libkda_oracle.so with gcc (fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-march=native", "-fno-fast-math", "-ffp-contract=off",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.kda_oracle_gate.argtypes = [i64, dp, ctypes.c_double, dp]
        lib.kda_oracle_gate.restype = None
        lib.kda_oracle_unit_g.argtypes = [i64, ctypes.c_int, ctypes.c_int,
                                          dp, i64, dp, i64, dp, i64, dp, i64, dp, i64, dp, i64,
                                          ctypes.c_double, dp, dp, i64, dp, dp, dp]
        lib.kda_oracle_unit_g.restype = None
        lib.kda_oracle_fwd.argtypes = [i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int64), dp, dp, dp, dp, dp, dp, dp,
                                       ctypes.c_double, dp, dp, dp, ctypes.c_int]
        lib.kda_oracle_fwd.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gate_log_decay(a, A_log: float) -> np.ndarray:
    """g = -5 * sigmoid(exp(A_log) * a), elementwise, fp64."""
    a = _f64(a)
    g = np.empty_like(a)
    _load().kda_oracle_gate(a.size, _ptr(a), float(A_log), _ptr(g))
    return g


def recurrence_g(q, k, v, g, beta, gate=None, S0=None, scale: float = 1.0):
    """One (sequence, head) unit with the log-decay g given directly.

    q, k, g: [T, d_k]; v, gate: [T, d_v]; beta: [T]; S0: [d_k, d_v] or None.
    Returns (out [T, d_v], S_final [d_k, d_v]) in fp64.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    gate, S0 = _f64(gate), _f64(S0)
    T, d_k = q.shape
    d_v = v.shape[1]
    out = np.zeros((T, d_v))
    S_final = np.zeros((d_k, d_v))
    S = np.zeros((d_k, d_v))
    r = np.zeros(d_v)
    _load().kda_oracle_unit_g(T, d_k, d_v, _ptr(q), d_k, _ptr(k), d_k, _ptr(v), d_v, _ptr(g), d_k,
                              _ptr(beta), 1, _ptr(gate), d_v, float(scale), _ptr(S0),
                              _ptr(out), d_v, _ptr(S_final), _ptr(S), _ptr(r))
    return out, S_final


def kda_fwd(q, k, v, a, beta, A_log, cu_seqlens, gate=None, S0=None, scale: float = 1.0,
            n_threads: int | None = None):
    """All (sequence, head) units of a packed batch, token-major, as the library takes them.

    q, k, a: [T_total, H, d_k]; v, gate: [T_total, H, d_v]; beta: [T_total, H]; A_log: [H];
    cu_seqlens: [num_seqs + 1]; S0: [num_seqs, H, d_k, d_v] or None.
    Returns (out [T_total, H, d_v], S_final [num_seqs, H, d_k, d_v]) in fp64.
    Inputs of any float dtype are widened exactly to fp64 first (bf16 -> fp64 is exact).
    """
    q, k, v, a, beta, A_log = map(_f64, (q, k, v, a, beta, A_log))
    gate, S0 = _f64(gate), _f64(S0)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    num_seqs = cu.size - 1
    out = np.zeros((T_total, H, d_v))
    S_final = np.zeros((num_seqs, H, d_k, d_v))
    if n_threads is None:
        n_threads = len(os.sched_getaffinity(0))
    rc = _load().kda_oracle_fwd(T_total, H, d_k, d_v, num_seqs,
                                cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate),
                                _ptr(A_log), float(scale), _ptr(S0), _ptr(out), _ptr(S_final),
                                int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle kda_oracle_fwd failed with status {rc}")
    return out, S_final
