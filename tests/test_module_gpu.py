"""GPU parity of the module pieces around the recurrence (kda_short_conv, kda_output_norm_gate)
against the oracle's plain definitions (oracle/module.py), and of the chain
convolution -> chunkwise recurrence -> normalisation + gate against the oracle's chain."""
import numpy as np
import pytest
import torch

import kda_inputs as KI
from oracle import module as M
from parity import assert_unit_ok, check_units, host, oracle_unit, unit_errors

pytestmark = pytest.mark.gpu
BF16_REL = 2.0 ** -8     # one rounding of the bf16 result


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    return m


def _cu(lengths):
    return torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")


def _bf16_close(gpu, ref, label):
    gpu = host(gpu)
    err = np.abs(gpu - ref)
    bound = BF16_REL * np.abs(ref) + 1e-5 * (np.abs(ref).max() + 1e-30)
    worst = float((err - bound).max()) if err.size else 0.0
    assert worst <= 0.0, f"{label}: max excess {worst:.3e}"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("l2norm", [False, True])
def test_short_conv_matches_oracle(kda, d, W, l2norm):
    lengths = [1, 2, 3, 31, 33, 0, 70, 5]   # shorter than the window, across runs of 32, empty
    T, H = sum(lengths), 3
    g = torch.Generator(device="cuda").manual_seed(d * 10 + W)
    x = torch.randn((T, H, d), generator=g, device="cuda").to(torch.bfloat16)
    w = torch.randn((H, d, W), generator=g, device="cuda") * 0.5
    cu = _cu(lengths)
    y = kda.kda_short_conv(x, w, cu, l2norm=l2norm)
    kda.kda_sync_check()
    ref = M.short_conv(host(x), host(w), cu.cpu().numpy(), l2norm=l2norm)
    _bf16_close(y, ref, f"short conv d={d} W={W} l2norm={l2norm}")


def test_short_conv_full_size_sampled(kda):
    # the prefill workload's shapes (8192 tokens x 32 heads x 128), two sequences, checked on a
    # sample of heads over all tokens
    lengths = [3000, 5192]
    T, H, d, W = sum(lengths), 32, 128, 4
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn((T, H, d), generator=g, device="cuda").to(torch.bfloat16)
    w = torch.randn((H, d, W), generator=g, device="cuda") * 0.5
    cu = _cu(lengths)
    y = kda.kda_short_conv(x, w, cu, l2norm=True)
    kda.kda_sync_check()
    for h in (0, 17, 31):
        ref = M.short_conv(host(x[:, h:h + 1]), host(w[h:h + 1]), cu.cpu().numpy(), l2norm=True)
        _bf16_close(y[:, h:h + 1], ref, f"full-size short conv head {h}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("with_gate,out_dtype", [(True, torch.bfloat16), (False, torch.float32),
                                                 (True, torch.float32)])
def test_norm_gate_matches_oracle(kda, d, with_gate, out_dtype):
    T, H = 300, 4
    g = torch.Generator(device="cuda").manual_seed(d + int(with_gate))
    o = torch.randn((T, H, d), generator=g, device="cuda") * 3.0
    gate = torch.randn((T, H, d), generator=g, device="cuda").to(torch.bfloat16) if with_gate else None
    w = torch.rand((d,), generator=g, device="cuda") + 0.5
    out = kda.kda_output_norm_gate(o, gate, w, eps=1e-6, out_dtype=out_dtype)
    kda.kda_sync_check()
    ref = M.output_norm_gate(host(o), None if gate is None else host(gate), host(w), eps=1e-6)
    if out_dtype == torch.bfloat16:
        _bf16_close(out, ref, f"norm gate d={d}")
    else:
        assert np.abs(host(out) - ref).max() <= 1e-4 * np.abs(ref).max()


def test_convolution_recurrence_norm_chain(kda):
    # raw q, k, v -> short convolution (q, k L2-normalised) -> chunkwise recurrence (no gate, fp32
    # output) -> pre-gate normalisation + gate; every stage against the oracle on the GPU's inputs
    w_ = KI.Workload("chain", (200, 65, 129), 2, 64, 64, seed=12)
    inp = KI.make_inputs(w_, "cuda")
    cu = inp["cu_seqlens"]
    g = torch.Generator(device="cuda").manual_seed(13)
    raw = {key: torch.randn(inp[key].shape, generator=g, device="cuda").to(torch.bfloat16)
           for key in ("q", "k", "v")}
    cw = {key: torch.randn((w_.H, 64, 4), generator=g, device="cuda") * 0.5 for key in ("q", "k", "v")}
    conv = {key: kda.kda_short_conv(raw[key], cw[key], cu, l2norm=key != "v") for key in ("q", "k", "v")}
    kda.kda_sync_check()
    for key in ("q", "k", "v"):
        ref = M.short_conv(host(raw[key]), host(cw[key]), cu.cpu().numpy(), l2norm=key != "v")
        _bf16_close(conv[key], ref, f"chain conv {key}")
    chain = dict(inp, q=conv["q"], k=conv["k"], v=conv["v"], gate=None)
    o, S = kda.kda_chunk_fwd(chain["q"], chain["k"], chain["v"], chain["a"], chain["beta"], chain["A_log"],
                             cu, gate=None, initial_state=chain["initial_state"], out_dtype=torch.float32)
    nw = torch.rand((64,), generator=g, device="cuda") + 0.5
    out = kda.kda_output_norm_gate(o, inp["gate"], nw, eps=1e-6, out_dtype=torch.float32)
    kda.kda_sync_check()
    check_units(chain, o, S, [(n, h) for n in range(w_.num_seqs) for h in range(w_.H)])
    cuh = cu.cpu().tolist()
    for n in range(w_.num_seqs):
        s, e = cuh[n], cuh[n + 1]
        for h in range(w_.H):
            unit = dict(q=host(conv["q"][s:e, h]), k=host(conv["k"][s:e, h]), v=host(conv["v"][s:e, h]),
                        a=host(inp["a"][s:e, h]), beta=host(inp["beta"][s:e, h]), gate=None,
                        A_log=float(inp["A_log"][h]),
                        S0=None if inp["initial_state"] is None else host(inp["initial_state"][n, h]))
            o_ref, _ = oracle_unit(unit)
            ref = M.output_norm_gate(o_ref[:, None, :], host(inp["gate"][s:e, h:h + 1]), host(nw))[:, 0]
            assert_unit_ok(unit_errors(host(out[s:e, h]), ref), f"chain output ({n},{h})")


def test_short_conv_reports_bad_offsets(kda):
    x = torch.zeros((40, 2, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((2, 64, 4), device="cuda")
    bad = torch.tensor([0, 10, 30], dtype=torch.int32, device="cuda")   # ends before the 40 tokens
    kda.kda_short_conv(x, w, bad)
    with pytest.raises(kda.KDAError):
        kda.kda_sync_check()
    kda.kda_sync_check()
