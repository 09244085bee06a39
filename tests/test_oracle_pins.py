"""Pins for the fp64 oracle: closed forms, page-printed values, invariants and an independent
brute-force parallel form.  CPU only.

Each test names the passage it follows.  A plausible mistake in the oracle (dropped fade, erase
before fade, read before the write, wrong sign of the delta, transposed state, a gate applied
twice, a wrong g mapping) fails at least one of them:
  - dropped or misplaced fade, wrong g mapping  -> test_fade_closed_form, test_gate_*,
    test_matches_parallel_form
  - wrong erase/write sign or order             -> test_worked_example, test_orthonormal_retrieval,
    test_reflection_invariant, test_matches_parallel_form
  - read before write                           -> test_worked_example (reads 1, not 3)
  - transposed state / swapped d_k, d_v         -> test_identity_at_beta0 (d_k != d_v)
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from brute_force import parallel_form

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")))
BF16_MAX = float(np.ldexp(np.float64(0xFF) / 128.0, 127))  # (2 - 2^-7) * 2^127, the bf16 format


def rng(seed):
    return np.random.default_rng(seed)


def unit_vectors(r, T, d):
    x = r.standard_normal((T, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


# ---- decay mapping ("Kimi K3 · Lesson 3 of 14", eq. 5 passage) -------------------------------

def test_gate_range_and_endpoints():
    r = rng(0)
    a = np.concatenate([r.standard_normal(10000) * 4.0, [0.0, 40.0, 100.0, -40.0, -100.0]])
    for A_log in (0.0, -1.0, 0.7):
        g = oracle.gate_log_decay(a, A_log)
        assert np.all(g <= 0.0) and np.all(g >= GOLDEN["decay_floor"]["g_min"])
    g = oracle.gate_log_decay(np.array([0.0, 40.0, 100.0, -40.0, -100.0]), 0.0)
    assert g[0] == -2.5                      # sigmoid(0) = 1/2 exactly
    assert g[1] == -5.0 and g[2] == -5.0     # saturates to the floor in fp64
    assert abs(g[3]) < 1e-16 and abs(g[4]) < 1e-16
    # the per-head log-scale multiplies the logit: g(A, a) = g(0, e^A a)
    a = r.standard_normal(100)
    np.testing.assert_array_equal(oracle.gate_log_decay(a, math.log(2.0)),
                                  oracle.gate_log_decay(2.0 * a, 0.0))


def test_gate_closed_form_values():
    # -5 * sigmoid(x) = -5 / (1 + e^-x): e.g. x = ln 3 gives -5 * 3/4
    g = oracle.gate_log_decay(np.array([math.log(3.0), -math.log(3.0)]), 0.0)
    np.testing.assert_allclose(g, [-3.75, -1.25], rtol=1e-15)


def test_tile_bound_and_bf16_margin():
    tb, bm = GOLDEN["tile_bound"], GOLDEN["bf16_margin"]
    gmin = GOLDEN["decay_floor"]["g_min"]
    # worst case: every token of a tile at the floor
    a = np.full(tb["tile_tokens"], 1000.0)
    tile_sum = -np.sum(oracle.gate_log_decay(a, 0.0))
    assert tile_sum == tb["max_accumulated_log_decay"] == -gmin * tb["tile_tokens"]
    # random saturated inputs never exceed it
    g = oracle.gate_log_decay(rng(1).standard_normal(16 * 4096) + 8.0, 0.0).reshape(-1, 16)
    assert np.all(-g.sum(axis=1) <= tb["max_accumulated_log_decay"])
    e80 = math.exp(tb["max_accumulated_log_decay"])
    assert abs(e80 / tb["max_reciprocal_printed"] - 1) < tb["max_reciprocal_printed_rel_precision"]
    assert abs(BF16_MAX / bm["bf16_max_printed"] - 1) < bm["bf16_max_printed_rel_precision"]
    overflow = math.log(BF16_MAX)
    assert abs(overflow - bm["overflow_log_decay_printed"]) < bm["overflow_log_decay_printed_abs_precision"]
    assert e80 < BF16_MAX and tb["max_accumulated_log_decay"] < overflow
    assert math.exp(-80.0) > np.finfo(np.float32).tiny   # e^-80 is a normal fp32/bf16 number
    for case in bm["breaking_cases"]:
        assert -case["g_floor"] * case["tile_tokens"] > overflow


# ---- erase/write ("K3 Architecture Illustrated", FIG 21; "Review A", Free recall) ------------

def test_worked_example():
    ex = GOLDEN["delta_overwrite_example"]
    S0 = np.array([[ex["old_value"]]])
    k = np.array([[ex["key"]]])
    out, S = oracle.recurrence_g(q=k, k=k, v=np.array([[ex["new_value"]]]),
                                 g=np.array([[math.log(ex["alpha"])]]),
                                 beta=np.array([ex["beta"]]), S0=S0)
    assert S[0, 0] == ex["retrieved_after"]
    assert out[0, 0] == ex["retrieved_after"]     # the read sees the token's own write


def test_orthonormal_retrieval():
    r = rng(2)
    d = 16
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    keys = Qm.T                                    # rows are orthonormal
    vals = r.standard_normal((d, 12)) + np.arange(d)[:, None]
    S0 = r.standard_normal((d, 12))
    # write all d keys (alpha = 1, beta = 1), then read each key with beta = 0
    k = np.concatenate([keys, keys])
    v = np.concatenate([vals, np.zeros_like(vals)])
    beta = np.concatenate([np.ones(d), np.zeros(d)])
    out, S = oracle.recurrence_g(q=k, k=k, v=v, g=np.zeros((2 * d, d)), beta=beta, S0=S0)
    np.testing.assert_allclose(out[d:], vals, rtol=0, atol=1e-13 * np.abs(vals).max())
    np.testing.assert_allclose(keys @ S, vals, rtol=0, atol=1e-13 * np.abs(vals).max())


def test_identity_at_beta0():
    r = rng(3)
    T, dk, dv = 37, 8, 5
    q = r.standard_normal((T, dk))
    S0 = r.standard_normal((dk, dv))
    out, S = oracle.recurrence_g(q=q, k=r.standard_normal((T, dk)), v=r.standard_normal((T, dv)),
                                 g=np.zeros((T, dk)), beta=np.zeros(T), S0=S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(out, q @ S0, rtol=1e-14, atol=1e-14)


def test_reflection_invariant():
    # I - 2 k k^T is a reflection for a unit k ("K3 Architecture Illustrated", PaTH/KDA passage)
    r = rng(4)
    T, dk, dv = 50, 12, 7
    k = unit_vectors(r, T, dk)
    S0 = r.standard_normal((dk, dv))
    _, S = oracle.recurrence_g(q=k, k=k, v=np.zeros((T, dv)), g=np.zeros((T, dk)),
                               beta=np.full(T, 2.0), S0=S0)
    assert abs(np.linalg.norm(S) / np.linalg.norm(S0) - 1.0) < 1e-13
    # and with beta = 1 it is a projection: the state loses its component along k
    _, S1 = oracle.recurrence_g(q=k[:1], k=k[:1], v=np.zeros((1, dv)), g=np.zeros((1, dk)),
                                beta=np.ones(1), S0=S0)
    np.testing.assert_allclose(k[0] @ S1, 0.0, atol=1e-14)


def test_fade_closed_form():
    r = rng(5)
    T, dk, dv = 40, 6, 9
    g = oracle.gate_log_decay(r.standard_normal((T, dk)), 0.3)
    S0 = r.standard_normal((dk, dv))
    _, S = oracle.recurrence_g(q=r.standard_normal((T, dk)), k=r.standard_normal((T, dk)),
                               v=r.standard_normal((T, dv)), g=g, beta=np.zeros(T), S0=S0)
    np.testing.assert_allclose(S, np.exp(g.sum(axis=0))[:, None] * S0, rtol=1e-13)


def test_output_gate():
    r = rng(6)
    T, dk, dv = 20, 8, 8
    args = dict(q=unit_vectors(r, T, dk), k=unit_vectors(r, T, dk), v=r.standard_normal((T, dv)),
                g=oracle.gate_log_decay(r.standard_normal((T, dk)), 0.0),
                beta=1 / (1 + np.exp(-r.standard_normal(T))), S0=r.standard_normal((dk, dv)))
    gate = r.standard_normal((T, dv))
    o_plain, S_plain = oracle.recurrence_g(**args)
    o_gated, S_gated = oracle.recurrence_g(gate=gate, **args)
    np.testing.assert_array_equal(S_plain, S_gated)          # the gate never touches the state
    np.testing.assert_allclose(o_gated, o_plain / (1 + np.exp(-gate)), rtol=1e-15)
    o_open, _ = oracle.recurrence_g(gate=np.full((T, dv), 40.0), **args)
    np.testing.assert_array_equal(o_open, o_plain)          # sigmoid(40) == 1 in fp64


# ---- chunkwise algebra ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram) -----------------------

@pytest.mark.parametrize("T,dk,dv,a_mean,seed", [
    (1, 4, 3, 0.0, 0), (7, 8, 8, 0.0, 1), (16, 16, 12, 0.0, 2), (17, 5, 16, 0.0, 3),
    (64, 16, 16, 0.0, 4), (64, 16, 16, 8.0, 5), (64, 16, 16, -8.0, 6), (48, 9, 7, 3.0, 7)])
def test_matches_parallel_form(T, dk, dv, a_mean, seed):
    r = rng(seed)
    q, k = unit_vectors(r, T, dk), unit_vectors(r, T, dk)
    v = r.standard_normal((T, dv))
    g = oracle.gate_log_decay(r.standard_normal((T, dk)) + a_mean, r.uniform(-1, 1))
    beta = 1 / (1 + np.exp(-r.standard_normal(T)))
    gate = r.standard_normal((T, dv))
    S0 = 0.3 * r.standard_normal((dk, dv))
    o_ref, S_ref = parallel_form(q, k, v, g, beta, gate=gate, S0=S0, scale=0.7)
    o, S = oracle.recurrence_g(q, k, v, g, beta, gate=gate, S0=S0, scale=0.7)
    scale_o = max(np.abs(o_ref).max(), 1e-300)
    assert np.abs(o - o_ref).max() <= 1e-10 * scale_o
    assert np.abs(S - S_ref).max() <= 1e-10 * max(np.abs(S_ref).max(), 1e-300)


def test_state_handoff_exact():
    r = rng(8)
    T1, T2, dk, dv = 23, 41, 8, 6
    T = T1 + T2
    q, k = unit_vectors(r, T, dk), unit_vectors(r, T, dk)
    v, gate = r.standard_normal((T, dv)), r.standard_normal((T, dv))
    g = oracle.gate_log_decay(r.standard_normal((T, dk)), 0.0)
    beta = r.uniform(0, 1, T)
    S0 = r.standard_normal((dk, dv))
    o, S = oracle.recurrence_g(q, k, v, g, beta, gate=gate, S0=S0)
    o1, S1 = oracle.recurrence_g(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], gate=gate[:T1], S0=S0)
    o2, S2 = oracle.recurrence_g(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], gate=gate[T1:], S0=S1)
    np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
    np.testing.assert_array_equal(S2, S)
    # one token at a time (the decode step) is the same computation
    Sd = S0
    for t in range(T):
        ot, Sd = oracle.recurrence_g(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1],
                                     beta[t:t + 1], gate=gate[t:t + 1], S0=Sd)
        np.testing.assert_array_equal(ot[0], o[t])
    np.testing.assert_array_equal(Sd, S)


def _packed_case(seed, lens, H, dk, dv, with_state=True, with_gate=True):
    r = rng(seed)
    T = sum(lens)
    q = unit_vectors(r, T * H, dk).reshape(T, H, dk)
    k = unit_vectors(r, T * H, dk).reshape(T, H, dk)
    v = r.standard_normal((T, H, dv))
    a = r.standard_normal((T, H, dk))
    beta = r.uniform(0, 1, (T, H))
    gate = r.standard_normal((T, H, dv)) if with_gate else None
    A_log = r.uniform(-1, 1, H)
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = r.standard_normal((len(lens), H, dk, dv)) * 0.1 if with_state else None
    return q, k, v, a, beta, gate, A_log, cu, S0


def test_packed_driver_matches_units():
    lens = [5, 0, 17, 1, 33]
    H, dk, dv = 3, 8, 4
    q, k, v, a, beta, gate, A_log, cu, S0 = _packed_case(9, lens, H, dk, dv)
    out, SF = oracle.kda_fwd(q, k, v, a, beta, A_log, cu, gate=gate, S0=S0, scale=0.5, n_threads=3)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        for h in range(H):
            g = oracle.gate_log_decay(a[s:e, h], A_log[h])
            o, S = oracle.recurrence_g(q[s:e, h], k[s:e, h], v[s:e, h], g, beta[s:e, h],
                                       gate=gate[s:e, h], S0=S0[n, h], scale=0.5)
            np.testing.assert_array_equal(out[s:e, h], o)
            np.testing.assert_array_equal(SF[n, h], S)
    # a zero-length sequence hands its initial state straight through
    np.testing.assert_array_equal(SF[1], S0[1])
    # thread count does not change a bit
    out1, SF1 = oracle.kda_fwd(q, k, v, a, beta, A_log, cu, gate=gate, S0=S0, scale=0.5, n_threads=1)
    np.testing.assert_array_equal(out1, out)
    np.testing.assert_array_equal(SF1, SF)


def test_packed_driver_defaults():
    lens = [9, 4]
    q, k, v, a, beta, _, A_log, cu, _ = _packed_case(10, lens, 2, 4, 4, with_state=False,
                                                      with_gate=False)
    out, SF = oracle.kda_fwd(q, k, v, a, beta, A_log, cu)
    zero = np.zeros((2, 2, 4, 4))
    out2, SF2 = oracle.kda_fwd(q, k, v, a, beta, A_log, cu, S0=zero,
                               gate=np.full(v.shape, 40.0))
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(SF, SF2)


def test_packed_driver_rejects_bad_cu_seqlens():
    q, k, v, a, beta, _, A_log, cu, _ = _packed_case(11, [3, 3], 1, 4, 4, with_state=False)
    with pytest.raises(ValueError):
        oracle.kda_fwd(q, k, v, a, beta, A_log, np.array([0, 4, 3]))
