"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, unit by unit.

Tolerances (tests/parity.py): per (sequence, head) unit, relative L2 error of outputs and of the
final state <= 5e-3, and max |error| of outputs <= 2e-2 * rms(oracle outputs).
Small cases check every unit; the full-size workloads check sampled units, each from its first
token (the oracle must run a unit from the start to reach any of its outputs).
"""
import numpy as np
import pytest
import torch

import kda_inputs as KI
from parity import check_units, host, oracle_unit, unit_errors, assert_unit_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    return m


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run(kda, inp, **kw):
    return kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"],
                             inp["cu_seqlens"], gate=inp["gate"],
                             initial_state=inp["initial_state"], **kw)


def all_units(w):
    return [(n, h) for n in range(w.num_seqs) for h in range(w.H)]


def sampled_units(w, count, seed=0):
    r = np.random.default_rng(seed)
    units = all_units(w)
    idx = r.choice(len(units), size=min(count, len(units)), replace=False)
    return [units[i] for i in sorted(idx)]


F32, BF16 = torch.float32, torch.bfloat16


@pytest.mark.parametrize("out_dtype", [F32, BF16])
def test_pr1_reference_workload(kda, out_dtype):
    w = KI.PR1_REF
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, out_dtype=out_dtype)
    kda.kda_sync_check()
    worst = check_units(inp, out, S, all_units(w))
    assert worst["out_rel_l2"] < 5e-3


RAGGED = (1, 15, 16, 17, 63, 64, 65, 130, 0, 200)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("with_gate,with_state,out_dtype", [(True, True, F32), (False, False, BF16)])
def test_ragged_varlen(kda, dk, dv, with_gate, with_state, out_dtype):
    w = KI.Workload("ragged", RAGGED, 3, dk, dv, A_log="uniform", gate=with_gate,
                    init_state="normal_0.02" if with_state else "none", seed=3)
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, scale=0.5, out_dtype=out_dtype)
    kda.kda_sync_check()
    check_units(inp, out, S, all_units(w), scale=0.5)


@pytest.mark.parametrize("a_mean,seed", [(8.0, 0), (-8.0, 1)])
def test_saturated_and_nofade_small(kda, a_mean, seed):
    w = KI.SATURATED.replace(name="sat_small", seqlens=(300, 129), H=4, a_mean=a_mean, seed=seed)
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, out_dtype=F32)
    kda.kda_sync_check()
    check_units(inp, out, S, all_units(w))


def test_extreme_decay_logits(kda):
    # a far beyond saturation on both sides: g is exactly -5 (1/Gamma = e^80 per tile) or 0
    w = KI.Workload("extreme", (160, 97), 2, 128, 128, a_mean=0.0, a_std=60.0, seed=5,
                    init_state="normal_0.02")
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, out_dtype=F32)
    kda.kda_sync_check()
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    check_units(inp, out, S, all_units(w))


def test_small_workspace_gives_identical_bits(kda):
    w = KI.Workload("windows", (700, 64, 333), 2, 128, 128, A_log="uniform",
                    init_state="normal_0.02", seed=7)
    inp = KI.make_inputs(w, "cuda")
    out_big, S_big = run(kda, inp)
    T, N = w.total_tokens, w.num_seqs
    mn = kda.kda_chunk_fwd_workspace_min(T, N, 700, w.H, 128, 128)
    ws = torch.empty(mn, dtype=torch.uint8, device="cuda")
    out_small, S_small = run(kda, inp, workspace=ws, max_seqlen=700)
    kda.kda_sync_check()
    assert torch.equal(out_big, out_small) and torch.equal(S_big, S_small)


def test_final_state_options(kda):
    w = KI.Workload("states", (100, 37), 2, 64, 64, init_state="normal_0.02", seed=8)
    inp = KI.make_inputs(w, "cuda")
    out_ref, S_ref = run(kda, inp)
    out_none, S_none = run(kda, inp, output_final_state=False)
    assert S_none is None and torch.equal(out_none, out_ref)
    S_alias = inp["initial_state"].clone()
    out_alias, S_out = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"],
                                         inp["A_log"], inp["cu_seqlens"], gate=inp["gate"],
                                         initial_state=S_alias, final_state=S_alias)
    kda.kda_sync_check()
    assert S_out.data_ptr() == S_alias.data_ptr()
    assert torch.equal(out_alias, out_ref) and torch.equal(S_alias, S_ref)


def test_chunk_continuation(kda):
    # fwd(T1) then fwd(T2 from S_T1) equals fwd(T1 + T2) (state hand-off between calls)
    w = KI.Workload("cont", (260,), 2, 128, 128, init_state="normal_0.02", seed=9)
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, out_dtype=F32)
    T1 = 131
    cu1 = torch.tensor([0, T1], dtype=torch.int32, device="cuda")
    cu2 = torch.tensor([0, 260 - T1], dtype=torch.int32, device="cuda")
    sl1, sl2 = slice(0, T1), slice(T1, 260)
    o1, S1 = kda.kda_chunk_fwd(*(inp[x][sl1].contiguous() for x in "qkva"), inp["beta"][sl1].contiguous(),
                               inp["A_log"], cu1, gate=inp["gate"][sl1].contiguous(),
                               initial_state=inp["initial_state"], out_dtype=F32)
    o2, S2 = kda.kda_chunk_fwd(*(inp[x][sl2].contiguous() for x in "qkva"), inp["beta"][sl2].contiguous(),
                               inp["A_log"], cu2, gate=inp["gate"][sl2].contiguous(), initial_state=S1,
                               out_dtype=F32)
    kda.kda_sync_check()
    # a split that is not chunk-aligned moves the chunk boundaries: the two runs agree to the
    # path's own rounding (tensor-core operands), and each agrees with the oracle
    both = torch.cat([o1, o2])
    assert (both - out).norm() / out.norm() < 2e-3
    assert (S2 - S).norm() / S.norm() < 2e-3
    check_units(inp, torch.cat([o1, o2]), S2, all_units(w))


def test_zero_length_batch_copies_state(kda):
    H, d = 2, 64
    S0 = torch.randn(3, H, d, d, device="cuda")
    e = torch.empty((0, H, d), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    out, S = kda.kda_chunk_fwd(e, e, e, e, torch.empty((0, H), device="cuda"),
                               torch.zeros(H, device="cuda"), cu, initial_state=S0)
    kda.kda_sync_check()
    assert out.shape == (0, H, d) and torch.equal(S, S0)


def test_device_reports_bad_seqlens(kda):
    w = KI.Workload("bad", (40, 100), 2, 64, 64, seed=10)
    inp = KI.make_inputs(w, "cuda")
    # max_seqlen smaller than a sequence (100 tokens = 2 chunks, 50 allows 1)
    with pytest.raises(kda.KDAError):
        run(kda, inp, max_seqlen=50)
        kda.kda_sync_check()
    kda.kda_sync_check()  # the error word was cleared
    # last offset beyond total_tokens (kernels clamp it, the error word reports it)
    bad = dict(inp, cu_seqlens=torch.tensor([0, 40, 150], dtype=torch.int32, device="cuda"))
    with pytest.raises(kda.KDAError):
        run(kda, bad, max_seqlen=100)
        kda.kda_sync_check()
    kda.kda_sync_check()


def test_bounded_wait_gives_up_and_context_survives(kda):
    """Failure injection on the host side of the boundary: chunk 0 of every unit is never
    published, so the consumers' waits (and, past the ring's 2G slots, the producers' waits) can
    only end by their bound, here 20 ms.  The launch must end, kda_sync_check must report
    KDA_ERR_TIMEOUT, and the next call on the same context must be correct."""
    w = KI.Workload("stall", (1100, 130), 2, 64, 128, seed=11)
    inp = KI.make_inputs(w, "cuda")
    kda.kda_inject_stall(True, 20_000_000)
    try:
        run(kda, inp, max_seqlen=1100)
        with pytest.raises(kda.KDAError) as err:
            kda.kda_sync_check()
        assert err.value.status == 4   # KDA_ERR_TIMEOUT
    finally:
        kda.kda_inject_stall(False)
    kda.kda_sync_check()
    out, S = run(kda, inp, max_seqlen=1100)
    kda.kda_sync_check()
    check_units(inp, out, S, all_units(w))


# ---- decode ------------------------------------------------------------------------------------

def decode_run(kda, inp, steps, scale=1.0, out_dtype=BF16):
    state = inp["state"].clone()
    outs = []
    for t in range(steps):
        outs.append(kda.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["a"][t],
                                        inp["beta"][t], inp["A_log"], state, gate=inp["gate"][t],
                                        scale=scale, out_dtype=out_dtype))
    kda.kda_sync_check()
    return torch.stack(outs), state


def decode_unit(inp, n, h, steps):
    return dict(q=host(inp["q"][:steps, n, h]), k=host(inp["k"][:steps, n, h]),
                v=host(inp["v"][:steps, n, h]), a=host(inp["a"][:steps, n, h]),
                beta=host(inp["beta"][:steps, n, h]), gate=host(inp["gate"][:steps, n, h]),
                A_log=float(inp["A_log"][h]), S0=host(inp["state"][n, h]))


@pytest.mark.parametrize("dk,dv,out_dtype", [(64, 64, F32), (128, 128, F32), (64, 128, F32),
                                             (128, 64, F32), (128, 128, BF16)])
def test_decode_matches_oracle(kda, dk, dv, out_dtype):
    w = KI.DecodeWorkload(N=5, H=3, d_k=dk, d_v=dv, steps=7, seed=2)
    inp = KI.make_decode_inputs(w, "cuda")
    outs, state = decode_run(kda, inp, w.steps, scale=0.8, out_dtype=out_dtype)
    for n in range(w.N):
        for h in range(w.H):
            o_ref, S_ref = oracle_unit(decode_unit(inp, n, h, w.steps), scale=0.8)
            err = unit_errors(host(outs[:, n, h]), o_ref, host(state[n, h]), S_ref,
                              out_bf16=out_dtype == BF16)
            assert_unit_ok(err, f"decode unit ({n},{h})")


def test_prefill_equals_decode_steps(kda):
    # T decode steps from S0 and one prefill of the same T tokens agree (GPU self-consistency)
    w = KI.DecodeWorkload(N=3, H=2, d_k=128, d_v=128, steps=150, seed=4)
    inp = KI.make_decode_inputs(w, "cuda")
    outs, state = decode_run(kda, inp, w.steps, out_dtype=F32)
    N, H, T = w.N, w.H, w.steps
    pack = lambda x: x.transpose(0, 1).reshape(N * T, *x.shape[2:]).contiguous()
    cu = torch.arange(0, (N + 1) * T, T, dtype=torch.int32, device="cuda")
    out_p, S_p = kda.kda_chunk_fwd(pack(inp["q"]), pack(inp["k"]), pack(inp["v"]), pack(inp["a"]),
                                   pack(inp["beta"]), inp["A_log"], cu, gate=pack(inp["gate"]),
                                   initial_state=inp["state"], out_dtype=F32)
    kda.kda_sync_check()
    dec = pack(outs)
    assert (out_p - dec).norm() / dec.norm() < 2e-3
    assert (S_p - state).norm() / state.norm() < 2e-3


# ---- full-size workloads ---------------------------------------------------------------------------
# Outputs are stored in fp32 so that the max-|error| bound applies exactly as stated (2e-2 x rms of
# the oracle's outputs, per unit), with no allowance for the bf16 output format.  Each test prints
# its worst errors over the units it checks.

def _report(name, worst):
    print(f"\n[full-size parity] {name}: worst out rel L2 {worst['out_rel_l2']:.2e}, "
          f"state rel L2 {worst['state_rel_l2']:.2e}, max|err|/rms {worst['out_max_abs_frac']:.2e}")


@pytest.mark.parametrize("name,count,path", [
    ("prefill_B1_H32_T8192_d128", 32, 0),      # 32 units: the cluster kernel
    ("prefill_B1_H32_T8192_d128", 32, 2),      # the per-unit kernel forced
    ("saturated_B2_H32_T16384_d128", 16, 0),   # 64 units: the cluster kernel
    ("saturated_B2_H32_T16384_d128", 16, 2),   # the per-unit kernel forced
    ("nofade_B2_H32_T16384_d128", 16, 0),
    ("nofade_B2_H32_T16384_d128", 16, 2),
])
def test_full_size_prefill(kda, name, count, path):
    w = KI.WORKLOADS[name]
    inp = KI.make_inputs(w, "cuda")
    kda.kda_set_prefill_path(path)
    try:
        out, S = run(kda, inp, out_dtype=F32)
        kda.kda_sync_check()
    finally:
        kda.kda_set_prefill_path(0)
    assert torch.isfinite(S).all()
    _report(f"{name} path {path}", check_units(inp, out, S, sampled_units(w, count)))


def test_full_size_varlen(kda):
    w = KI.VARLEN
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, out_dtype=F32)
    kda.kda_sync_check()
    lens = np.array(w.seqlens)
    # the longest and the shortest sequence, plus random ones
    units = [(int(lens.argmax()), 0), (int(lens.argmin()), w.H - 1)] + sampled_units(w, 14, seed=1)
    _report(w.name, check_units(inp, out, S, units))
    del inp, out, S


def test_full_size_long_prefill(kda):
    # every head of the 1 M-token sequence, eight at a time (fp64 copies of 1 M tokens x 128 channels)
    w = KI.LONG_1M
    inp = KI.make_inputs(w, "cuda")
    out, S = run(kda, inp, out_dtype=F32)
    kda.kda_sync_check()
    assert torch.isfinite(S).all()
    _report(w.name, check_units(inp, out, S, [(0, h) for h in range(w.H)], batch=8))


def test_full_size_decode(kda):
    w = KI.DECODE
    inp = KI.make_decode_inputs(w, "cuda")
    outs, state = decode_run(kda, inp, w.steps, out_dtype=F32)
    r = np.random.default_rng(0)
    worst = 0.0
    for _ in range(16):
        n, h = int(r.integers(w.N)), int(r.integers(w.H))
        o_ref, S_ref = oracle_unit(decode_unit(inp, n, h, w.steps))
        err = unit_errors(host(outs[:, n, h]), o_ref, host(state[n, h]), S_ref)
        assert_unit_ok(err, f"decode unit ({n},{h})")
        worst = max(worst, err["out_max_abs"] / max(err["out_rms"], 1e-30))
    print(f"\n[full-size parity] {w.name}: worst max|err|/rms {worst:.2e}")
