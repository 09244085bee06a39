"""GPU parity of multi-token decode with rollback (kda_decode_verify + kda_decode_commit).

The oracle is the token-by-token recurrence: verify's outputs for tokens 1..K must match it run
over those K tokens from the starting state, and after commit each state must match it run over
the sequence's accepted prefix only.  Tolerances as everywhere (tests/parity.py).
"""
import dataclasses

import numpy as np
import pytest
import torch

import kda_inputs as KI
from parity import assert_unit_ok, host, oracle_unit, unit_errors

pytestmark = pytest.mark.gpu

F32, BF16 = torch.float32, torch.bfloat16


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    return m


def spec_unit(inp, r, n, h, upto):
    sl = slice(0, upto)
    return dict(q=host(inp["q"][r, n, sl, h]), k=host(inp["k"][r, n, sl, h]), v=host(inp["v"][r, n, sl, h]),
                a=host(inp["a"][r, n, sl, h]), beta=host(inp["beta"][r, n, sl, h]),
                gate=host(inp["gate"][r, n, sl, h]), A_log=float(inp["A_log"][h]), S0=None)


def verify(kda, inp, r, state, out_dtype=F32, scale=1.0):
    return kda.kda_decode_verify(inp["q"][r], inp["k"][r], inp["v"][r], inp["a"][r], inp["beta"][r],
                                 inp["A_log"], state, gate=inp["gate"][r], scale=scale, out_dtype=out_dtype)


@pytest.mark.parametrize("dk,dv,K", [(64, 64, 4), (128, 128, 4), (64, 128, 1), (128, 64, 7), (128, 128, 16)])
def test_verify_and_commit_match_oracle(kda, dk, dv, K):
    w = dataclasses.replace(KI.SPEC, N=4, H=3, d_k=dk, d_v=dv, K=K, rounds=1, seed=3)
    inp = KI.make_spec_inputs(w, "cuda")
    # every acceptance length appears: 0, K and values between
    acc = torch.tensor([0, K, min(1, K), K // 2], dtype=torch.int32, device="cuda")
    state = inp["state"].clone()
    out, u = verify(kda, inp, 0, state, scale=0.9)
    kda.kda_sync_check()
    assert torch.equal(state, inp["state"]), "verify must not write the state"
    kda.kda_decode_commit(inp["k"][0], inp["a"][0], inp["A_log"], acc, u, state)
    kda.kda_sync_check()
    for n in range(w.N):
        j = int(acc[n])
        for h in range(w.H):
            unit = spec_unit(inp, 0, n, h, K)
            unit["S0"] = host(inp["state"][n, h])
            o_ref, _ = oracle_unit(unit, scale=0.9)
            err = unit_errors(host(out[n, :, h]), o_ref)
            assert_unit_ok(err, f"verify outputs ({n},{h})")
            if j == 0:
                assert torch.equal(state[n, h], inp["state"][n, h])
                continue
            pref = spec_unit(inp, 0, n, h, j)
            pref["S0"] = host(inp["state"][n, h])
            o_j, S_j = oracle_unit(pref, scale=0.9)
            e2 = unit_errors(host(out[n, :j, h]), o_j, host(state[n, h]), S_j)
            assert_unit_ok(e2, f"committed state ({n},{h}) after {j} tokens")


def test_rounds_follow_the_accepted_sequence(kda):
    # several verify/commit rounds equal the recurrence over the concatenated accepted prefixes
    w = dataclasses.replace(KI.SPEC, N=3, H=2, d_k=128, d_v=128, K=4, rounds=5, seed=4)
    inp = KI.make_spec_inputs(w, "cuda")
    state = inp["state"].clone()
    for r in range(w.rounds):
        _, u = verify(kda, inp, r, state)
        kda.kda_decode_commit(inp["k"][r], inp["a"][r], inp["A_log"], inp["accepted"][r], u, state)
    kda.kda_sync_check()
    acc = inp["accepted"].cpu().numpy()
    for n in range(w.N):
        for h in range(w.H):
            cat = {key: [] for key in ("q", "k", "v", "a", "beta", "gate")}
            for r in range(w.rounds):
                part = spec_unit(inp, r, n, h, int(acc[r, n]))
                for key in cat:
                    cat[key].append(part[key])
            unit = {key: np.concatenate(val) for key, val in cat.items()}
            unit.update(A_log=float(inp["A_log"][h]), S0=host(inp["state"][n, h]))
            if unit["q"].shape[0] == 0:
                assert torch.equal(state[n, h], inp["state"][n, h])
                continue
            _, S_ref = oracle_unit(unit)
            sn = np.linalg.norm(S_ref)
            assert np.linalg.norm(host(state[n, h]) - S_ref) / sn <= 5e-3


def test_commit_all_equals_decode_steps_bitwise(kda):
    # verify K tokens + commit K runs the same arithmetic, in the same order, as K decode steps
    w = dataclasses.replace(KI.SPEC, N=6, H=4, d_k=128, d_v=128, K=5, rounds=1, seed=5)
    inp = KI.make_spec_inputs(w, "cuda")
    s_spec = inp["state"].clone()
    out, u = verify(kda, inp, 0, s_spec, out_dtype=F32)
    kda.kda_decode_commit(inp["k"][0], inp["a"][0], inp["A_log"],
                          torch.full((w.N,), w.K, dtype=torch.int32, device="cuda"), u, s_spec)
    s_dec = inp["state"].clone()
    outs = []
    for t in range(w.K):
        tok = {key: inp[key][0, :, t].contiguous() for key in ("q", "k", "v", "a", "beta", "gate")}
        outs.append(kda.kda_decode_step(tok["q"], tok["k"], tok["v"], tok["a"], tok["beta"], inp["A_log"],
                                        s_dec, gate=tok["gate"], out_dtype=F32))
    kda.kda_sync_check()
    assert torch.equal(s_spec, s_dec)
    assert torch.equal(out, torch.stack(outs, dim=1))


def test_bad_accepted_count_is_reported_and_clamped(kda):
    w = dataclasses.replace(KI.SPEC, N=2, H=2, d_k=64, d_v=64, K=3, rounds=1, seed=6)
    inp = KI.make_spec_inputs(w, "cuda")
    state = inp["state"].clone()
    _, u = verify(kda, inp, 0, state)
    bad = torch.tensor([-1, 9], dtype=torch.int32, device="cuda")
    kda.kda_decode_commit(inp["k"][0], inp["a"][0], inp["A_log"], bad, u, state)
    with pytest.raises(kda.KDAError):
        kda.kda_sync_check()
    kda.kda_sync_check()   # cleared
    assert torch.equal(state[0], inp["state"][0])        # -1 -> 0 accepted
    ref = inp["state"].clone()
    kda.kda_decode_commit(inp["k"][0], inp["a"][0], inp["A_log"],
                          torch.tensor([0, 3], dtype=torch.int32, device="cuda"), u, ref)
    kda.kda_sync_check()
    assert torch.equal(state[1], ref[1])                  # 9 -> K accepted


def test_full_size_verify_commit_sampled(kda):
    # the decode configuration's shapes (256 sequences x 64 heads, 128 x 128 states), K = 4
    w = dataclasses.replace(KI.SPEC, rounds=1)
    inp = KI.make_spec_inputs(w, "cuda")
    state = inp["state"].clone()
    out, u = verify(kda, inp, 0, state, out_dtype=BF16)
    kda.kda_decode_commit(inp["k"][0], inp["a"][0], inp["A_log"], inp["accepted"][0], u, state)
    kda.kda_sync_check()
    acc = inp["accepted"][0].cpu().numpy()
    rng = np.random.default_rng(0)
    for idx in rng.choice(w.N * w.H, size=6, replace=False):
        n, h = divmod(int(idx), w.H)
        unit = spec_unit(inp, 0, n, h, w.K)
        unit["S0"] = host(inp["state"][n, h])
        o_ref, _ = oracle_unit(unit)
        assert_unit_ok(unit_errors(host(out[n, :, h]), o_ref, out_bf16=True), f"verify ({n},{h})")
        j = int(acc[n])
        if j == 0:
            assert torch.equal(state[n, h], inp["state"][n, h])
            continue
        pref = spec_unit(inp, 0, n, h, j)
        pref["S0"] = host(inp["state"][n, h])
        _, S_j = oracle_unit(pref)
        assert np.linalg.norm(host(state[n, h]) - S_j) / np.linalg.norm(S_j) <= 5e-3
