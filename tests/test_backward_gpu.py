"""GPU parity of the backward pass (kda_chunk_bwd) against the oracle's reverse-mode derivative of
the token-by-token recurrence (oracle/backward.py, itself pinned by finite differences).

Tolerances as for the forward outputs, applied to every gradient of every (sequence, head) unit:
relative L2 error <= 5e-3 and max |error| <= 2e-2 * rms(oracle gradient)."""
import numpy as np
import pytest
import torch

import kda_inputs as KI
from oracle.backward import recurrence_bwd
from parity import host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    return m


def _close(got, ref, label):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    nrm = np.linalg.norm(ref)
    if nrm == 0:
        assert np.abs(got).max() <= 1e-6, label
        return
    rel = np.linalg.norm(got - ref) / nrm
    rms = np.sqrt(np.mean(ref ** 2))
    assert rel <= 5e-3, f"{label}: rel L2 {rel:.2e}"
    assert np.abs(got - ref).max() <= 2e-2 * rms + 1e-30, f"{label}: max err {np.abs(got - ref).max():.2e} rms {rms:.2e}"


def _check(kda, inp, dout, dST, g, units, scale=1.0):
    cu = inp["cu_seqlens"].cpu().tolist()
    dA_ref = {}
    for n, h in units:
        s, e = cu[n], cu[n + 1]
        gate = inp["gate"]
        S0 = inp["initial_state"]
        ref = recurrence_bwd(host(inp["q"][s:e, h]), host(inp["k"][s:e, h]), host(inp["v"][s:e, h]),
                             host(inp["a"][s:e, h]), host(inp["beta"][s:e, h]), float(inp["A_log"][h]),
                             host(dout[s:e, h]), gate=None if gate is None else host(gate[s:e, h]),
                             S0=None if S0 is None else host(S0[n, h]),
                             dS_T=None if dST is None else host(dST[n, h]), scale=scale)
        lab = f"unit ({n},{h})"
        if e > s:
            for key in ("dq", "dk", "dv", "da"):
                _close(host(g[key][s:e, h]), ref[key], f"{lab} {key}")
            _close(host(g["dbeta"][s:e, h]), ref["dbeta"], f"{lab} dbeta")
            if gate is not None:
                _close(host(g["dgate"][s:e, h]), ref["dgate"], f"{lab} dgate")
        if S0 is not None:
            _close(host(g["dinitial_state"][n, h]), ref["dS0"], f"{lab} dS0")
        dA_ref[h] = dA_ref.get(h, 0.0) + ref["dA_log"]
    return dA_ref


@pytest.mark.parametrize("chunkwise", [False, True])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("with_gate,with_state", [(True, True), (False, False)])
def test_backward_matches_oracle(kda, dk, dv, with_gate, with_state, chunkwise):
    w = KI.Workload("bwd", (70, 1, 130, 0, 64), 2, dk, dv, A_log="uniform", gate=with_gate,
                    init_state="normal_0.02" if with_state else "none", seed=31)
    inp = KI.make_inputs(w, "cuda")
    g_ = torch.Generator(device="cuda").manual_seed(32)
    dout = torch.randn((w.total_tokens, w.H, dv), generator=g_, device="cuda")
    dST = torch.randn((w.num_seqs, w.H, dk, dv), generator=g_, device="cuda") if with_state else None
    g = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                          dout, gate=inp["gate"], initial_state=inp["initial_state"], dfinal_state=dST,
                          scale=0.9, chunkwise=chunkwise)
    kda.kda_sync_check()
    units = [(n, h) for n in range(w.num_seqs) for h in range(w.H)]
    dA_ref = _check(kda, inp, dout, dST, g, units, scale=0.9)
    for h, ref in dA_ref.items():   # dA_log sums over every sequence
        assert abs(float(g["dA_log"][h]) - ref) <= 5e-3 * max(abs(ref), 1e-6), f"dA_log[{h}]"


@pytest.mark.parametrize("chunkwise", [False, True])
def test_backward_full_size_sampled(kda, chunkwise):
    # the prefill workload (B=1, H=32, T=8192, d=128), three heads checked over all 8192 tokens
    w = KI.WORKLOADS["prefill_B1_H32_T8192_d128"]
    inp = KI.make_inputs(w, "cuda")
    g_ = torch.Generator(device="cuda").manual_seed(33)
    dout = torch.randn((w.total_tokens, w.H, w.d_v), generator=g_, device="cuda") * 0.1
    dST = torch.randn((w.num_seqs, w.H, w.d_k, w.d_v), generator=g_, device="cuda") * 0.1
    g = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                          dout, gate=inp["gate"], initial_state=inp["initial_state"], dfinal_state=dST,
                          chunkwise=chunkwise)
    kda.kda_sync_check()
    dA_ref = _check(kda, inp, dout, dST, g, [(0, 0), (0, 13), (0, 31)])
    for h, ref in dA_ref.items():
        assert abs(float(g["dA_log"][h]) - ref) <= 5e-3 * max(abs(ref), 1e-6), f"dA_log[{h}]"


@pytest.mark.parametrize("chunkwise", [False, True])
@pytest.mark.parametrize("a_mean,beta_lo", [(8.0, 0.9), (-8.0, 0.9)])
def test_backward_saturated_and_nofade(kda, chunkwise, a_mean, beta_lo):
    # a ~ N(8, 1): g = -5 in nearly every channel, a chunk decays by up to e^-320 (the pairwise form
    # must keep every 1/e^b inside an e^{b_i - b_j}, i >= j); a ~ N(-8, 1): almost no fade.
    w = KI.Workload("bwd_sat", (70, 130, 17), 2, 128, 128, a_mean=a_mean, beta="uniform_0.9_1" if beta_lo else "sigmoid_normal",
                    gate=True, init_state="normal_0.02", seed=34)
    inp = KI.make_inputs(w, "cuda")
    g_ = torch.Generator(device="cuda").manual_seed(35)
    dout = torch.randn((w.total_tokens, w.H, 128), generator=g_, device="cuda")
    dST = torch.randn((w.num_seqs, w.H, 128, 128), generator=g_, device="cuda")
    g = kda.kda_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"], inp["cu_seqlens"],
                          dout, gate=inp["gate"], initial_state=inp["initial_state"], dfinal_state=dST,
                          chunkwise=chunkwise)
    kda.kda_sync_check()
    units = [(n, h) for n in range(w.num_seqs) for h in range(w.H)]
    dA_ref = _check(kda, inp, dout, dST, g, units)
    for h, ref in dA_ref.items():
        assert abs(float(g["dA_log"][h]) - ref) <= 5e-3 * max(abs(ref), 1e-6), f"dA_log[{h}]"


@pytest.mark.parametrize("chunkwise", [False, True])
def test_backward_malformed_seqlens_stay_in_workspace(kda, chunkwise):
    # cu_seqlens = [0, T, 0, T]: every offset in range but not monotone, so the spans add up to twice
    # the tokens; the kernels must flag it and write nothing past the workspace they were given.
    T, H = 640, 2
    w = KI.Workload("bwd_bad", (T, 0, T), H, 128, 128, seed=36)
    inp = KI.make_inputs(w, "cuda")
    cu = torch.tensor([0, T, 0, T], dtype=torch.int32, device="cuda")
    q, k, v, a = (inp[x][:T] for x in ("q", "k", "v", "a"))
    beta = inp["beta"][:T]
    dout = torch.randn((T, H, 128), device="cuda")
    size = (kda.kda_chunk_bwd_chunkwise_workspace_size if chunkwise else kda.kda_chunk_bwd_workspace_size)(T, 3, H, 128, 128)
    guard = 1 << 20
    buf = torch.full((size + guard,), 0x5A, dtype=torch.uint8, device="cuda")
    with pytest.raises(kda.KDAError):
        kda.kda_chunk_bwd(q, k, v, a, beta, inp["A_log"], cu, dout, workspace=buf[:size], chunkwise=chunkwise)
        kda.kda_sync_check()
    torch.cuda.synchronize()
    assert bool((buf[size:] == 0x5A).all()), "a kernel wrote past its workspace"
