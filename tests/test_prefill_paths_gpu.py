"""GPU parity of both prefill kernels, each forced in turn, against the fp64 oracle.

kda_chunk_fwd runs one of two kernels for d_k = d_v = 128 (kda_set_prefill_path): the cluster
kernel (a unit's chunks spread over four CTAs, chunk records in the workspace) or the per-unit
kernel (one CTA per (sequence, head), everything on chip).  Both compute the chunkwise form of the
recurrence; each must meet the tolerances of tests/parity.py on its own, on ragged lengths (partial
tiles and chunks, empty sequences), saturated and no-fade decay, decay logits far past saturation,
with and without gate and initial state, in both output formats.
"""
import pytest
import torch

import kda_inputs as KI
from parity import check_units

pytestmark = pytest.mark.gpu

F32, BF16 = torch.float32, torch.bfloat16
PATHS = (1, 2)


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    yield m
    m.kda_set_prefill_path(0)


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run(kda, inp, path, **kw):
    kda.kda_set_prefill_path(path)
    try:
        out, S = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"],
                                   inp["cu_seqlens"], gate=inp["gate"], initial_state=inp["initial_state"], **kw)
        kda.kda_sync_check()
    finally:
        kda.kda_set_prefill_path(0)
    return out, S


def all_units(w):
    return [(n, h) for n in range(w.num_seqs) for h in range(w.H)]


RAGGED = (1, 15, 16, 17, 63, 64, 65, 130, 0, 200, 257)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("with_gate,with_state,out_dtype", [(True, True, F32), (False, False, BF16), (True, False, F32)])
def test_ragged(kda, path, with_gate, with_state, out_dtype):
    w = KI.Workload("ragged", RAGGED, 3, 128, 128, A_log="uniform", gate=with_gate,
                    init_state="normal_0.02" if with_state else "none", seed=11)
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, path, scale=0.5, out_dtype=out_dtype)
    check_units(inp, out, S, all_units(w), scale=0.5)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("a_mean,seed", [(8.0, 0), (-8.0, 1)])
def test_saturated_and_nofade(kda, path, a_mean, seed):
    w = KI.SATURATED.replace(name="sat_small", seqlens=(700, 129, 64), H=3, a_mean=a_mean, seed=seed)
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, path, out_dtype=F32)
    check_units(inp, out, S, all_units(w))


@pytest.mark.parametrize("path", PATHS)
def test_extreme_decay_logits(kda, path):
    w = KI.Workload("extreme", (160, 97, 300), 2, 128, 128, a_mean=0.0, a_std=60.0, seed=5,
                    init_state="normal_0.02")
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, path, out_dtype=F32)
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    check_units(inp, out, S, all_units(w))


def test_paths_agree_and_per_unit_path_needs_no_workspace(kda):
    w = KI.Workload("agree", (512, 200, 1000, 64), 4, 128, 128, A_log="uniform", init_state="normal_0.02", seed=12)
    inp = KI.make_inputs(w, "cuda")
    out1, S1 = run(kda, inp, 1, out_dtype=F32)
    kda.kda_set_prefill_path(2)
    try:
        assert kda.kda_chunk_fwd_workspace_size(w.total_tokens, w.num_seqs, 1000, w.H, 128, 128) == 0
        assert kda.kda_prefill_path(w.num_seqs * w.H, 128, 128) == 2
        assert kda.kda_prefill_path(w.num_seqs * w.H, 64, 64) == 1
    finally:
        kda.kda_set_prefill_path(0)
    out2, S2 = run(kda, inp, 2, out_dtype=F32, workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
    rel = (out1 - out2).norm() / out1.norm()
    rels = (S1 - S2).norm() / S1.norm()
    assert rel < 2e-3 and rels < 2e-3


def test_per_unit_path_is_deterministic(kda):
    w = KI.Workload("det", (300, 77), 3, 128, 128, A_log="uniform", init_state="normal_0.02", seed=13)
    inp = KI.make_inputs(w, "cuda")
    a = run(kda, inp, 2)
    b = run(kda, inp, 2)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("path", PATHS)
def test_state_beyond_fp16_range_is_reported(kda, path):
    # the state and the values reach the tensor cores as fp16: an initial state of 1e6 (beyond
    # +-65504) cannot be represented; the call must end with KDA_ERR_RANGE, not with silent infs
    w = KI.Workload("range", (100, 70), 2, 128, 128, init_state="normal_0.02", seed=14)
    inp = KI.make_inputs(w, "cuda")
    S0 = torch.full_like(inp["initial_state"], 1e6)
    kda.kda_set_prefill_path(path)
    try:
        kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                          gate=inp["gate"], initial_state=S0)
        with pytest.raises(kda.KDAError) as ei:
            kda.kda_sync_check()
        assert ei.value.status == kda.KDA_ERR_RANGE
        # the error word is cleared: an in-range call afterwards is clean
        kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                          gate=inp["gate"], initial_state=inp["initial_state"])
        kda.kda_sync_check()
    finally:
        kda.kda_set_prefill_path(0)
