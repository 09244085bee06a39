"""kda_chunk_fwd_host (inputs and outputs in host memory, pieces overlapped with their copies)
against kda_chunk_fwd on the same inputs: a cut inside a sequence falls on a 64-token chunk boundary
and the state crosses it in fp32 on the device, so the results must be the same bits.  The ragged
case has empty sequences, one-token sequences, sequences shorter and longer than a piece, and piece
sizes that are not multiples of the chunk."""
import pytest
import torch

import kda_inputs as KI

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import kda_chunkwise_b200 as m
    return m


def _host(t):
    return None if t is None else t.cpu().pin_memory()


def _compare(kda, inp, out_dtype, piece):
    ref, S_ref = kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"],
                                   inp["cu_seqlens"], gate=inp["gate"], initial_state=inp["initial_state"],
                                   out_dtype=out_dtype)
    h = {key: _host(inp[key]) for key in ("q", "k", "v", "a", "beta", "gate", "initial_state", "A_log", "cu_seqlens")}
    out, S = kda.kda_chunk_fwd_host(h["q"], h["k"], h["v"], h["a"], h["beta"], h["A_log"], h["cu_seqlens"],
                                    gate=h["gate"], initial_state=h["initial_state"], out_dtype=out_dtype,
                                    piece_tokens=piece)
    torch.cuda.synchronize()
    kda.kda_sync_check()
    assert torch.equal(out, ref.cpu()), f"piece {piece}: outputs differ"
    assert torch.equal(S, S_ref.cpu()), f"piece {piece}: final states differ"


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("piece", [64, 100, 256, 5000])
def test_host_prefill_matches_device_prefill(kda, dk, dv, piece):
    w = KI.Workload("host", (300, 1, 0, 700, 0, 30, 129), 3, dk, dv, A_log="uniform",
                    init_state="normal_0.02", seed=41)
    _compare(kda, KI.make_inputs(w, "cuda"), torch.float32, piece)


def test_host_prefill_without_gate_or_state(kda):
    w = KI.Workload("host2", (513, 64, 2), 2, 128, 128, gate=False, seed=42)
    _compare(kda, KI.make_inputs(w, "cuda"), torch.bfloat16, 128)


def test_host_prefill_full_size(kda):
    # the prefill workload (B=1, H=32, T=8192, d=128) with the default pieces, as the bench runs it
    _compare(kda, KI.make_inputs(KI.WORKLOADS["prefill_B1_H32_T8192_d128"], "cuda"), torch.bfloat16, 0)
