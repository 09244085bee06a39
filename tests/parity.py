"""Helpers shared by the parity tests: run the fp64 oracle on selected (sequence, head) units of a
batch that lives on the GPU, and compare unit by unit.

Tolerances (fixed for every workload, unit by unit):
  relative L2 error of a unit's outputs      <= 5e-3
  relative L2 error of a unit's final state  <= 5e-3
  max |error| of a unit's outputs            <= 2e-2 * rms(oracle outputs of the unit)
The max-|error| bound is applied as stated to fp32-stored outputs.  For bf16-stored outputs the
format's own rounding is added element by element: round-to-nearest bf16 (8 significant bits)
moves a value x by at most 2^-8 |x|, so there the bound is |err_i| <= 2e-2 * rms + 2^-8 |ref_i|.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle

REL_L2_TOL = 5e-3
MAX_ABS_FRAC = 2e-2
BF16_HALF_ULP_REL = 2.0 ** -8


def host(t):
    """Exact host copy (bf16 and fp32 widen exactly to fp64)."""
    return None if t is None else t.detach().to("cpu").to(torch.float64).numpy()


def oracle_unit(unit, scale=1.0):
    g = oracle.gate_log_decay(unit["a"], unit["A_log"])
    return oracle.recurrence_g(unit["q"], unit["k"], unit["v"], g, unit["beta"], gate=unit["gate"],
                               S0=unit["S0"], scale=scale)


def gather_unit(inp, n, h, t_end=None):
    """Host fp64 slices of unit (sequence n, head h); optionally only its first t_end tokens."""
    cu = inp["cu_seqlens"].cpu().tolist()
    s, e = cu[n], cu[n + 1]
    if t_end is not None:
        e = min(e, s + t_end)
    sl = slice(s, e)
    gate = inp.get("gate")
    S0 = inp.get("initial_state")
    return dict(q=host(inp["q"][sl, h]), k=host(inp["k"][sl, h]), v=host(inp["v"][sl, h]),
                a=host(inp["a"][sl, h]), beta=host(inp["beta"][sl, h]),
                gate=None if gate is None else host(gate[sl, h]),
                A_log=float(inp["A_log"][h]), S0=None if S0 is None else host(S0[n, h]),
                span=(s, e))


def run_oracle_units(units, scale=1.0, threads=None):
    threads = threads or max(1, len(os.sched_getaffinity(0)))
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda u: oracle_unit(u, scale), units))


def unit_errors(out_gpu, out_ref, S_gpu=None, S_ref=None, out_bf16=False):
    out_gpu = np.asarray(out_gpu, np.float64)
    d = out_gpu - out_ref
    ref_norm = np.linalg.norm(out_ref)
    fmt = BF16_HALF_ULP_REL if out_bf16 else 0.0
    res = dict(out_rel_l2=float(np.linalg.norm(d) / ref_norm) if ref_norm > 0 else 0.0,
               out_max_abs=float(np.abs(d).max()) if d.size else 0.0,
               out_max_excess=float((np.abs(d) - fmt * np.abs(out_ref)).max()) if d.size else 0.0,
               out_rms=float(np.sqrt(np.mean(out_ref ** 2))) if out_ref.size else 0.0)
    if S_gpu is not None:
        S_gpu = np.asarray(S_gpu, np.float64)
        sn = np.linalg.norm(S_ref)
        res["state_rel_l2"] = float(np.linalg.norm(S_gpu - S_ref) / sn) if sn > 0 else \
            float(np.abs(S_gpu).max())
    return res


def assert_unit_ok(err, label=""):
    assert err["out_rel_l2"] <= REL_L2_TOL, f"{label} output rel L2 {err['out_rel_l2']:.3e}"
    assert err["out_max_excess"] <= MAX_ABS_FRAC * err["out_rms"] + 1e-30, \
        f"{label} output max|err| {err['out_max_abs']:.3e} (beyond output rounding " \
        f"{err['out_max_excess']:.3e}) vs rms {err['out_rms']:.3e}"
    if "state_rel_l2" in err:
        assert err["state_rel_l2"] <= REL_L2_TOL, f"{label} state rel L2 {err['state_rel_l2']:.3e}"


def check_units(inp, out, final_state, units, scale=1.0, t_end=None, batch=16):
    """Oracle-check the listed (n, h) units of a GPU run, `batch` units at a time (the fp64 host
    copies of long units are large); returns the worst errors seen."""
    worst = dict(out_rel_l2=0.0, state_rel_l2=0.0, out_max_abs_frac=0.0)
    for b0 in range(0, len(units), batch):
        part = units[b0:b0 + batch]
        data = [gather_unit(inp, n, h, t_end) for n, h in part]
        refs = run_oracle_units(data, scale)
        for (n, h), u, (o_ref, S_ref) in zip(part, data, refs):
            s, e = u["span"]
            o_gpu = host(out[s:e, h])
            S_gpu = host(final_state[n, h]) if (final_state is not None and t_end is None) else None
            err = unit_errors(o_gpu, o_ref, S_gpu, S_ref if S_gpu is not None else None,
                              out_bf16=out.dtype == torch.bfloat16)
            assert_unit_ok(err, f"unit (n={n}, h={h})")
            worst["out_rel_l2"] = max(worst["out_rel_l2"], err["out_rel_l2"])
            worst["state_rel_l2"] = max(worst["state_rel_l2"], err.get("state_rel_l2", 0.0))
            if err["out_rms"] > 0:
                worst["out_max_abs_frac"] = max(worst["out_max_abs_frac"],
                                                err["out_max_abs"] / err["out_rms"])
        del data, refs
    return worst
